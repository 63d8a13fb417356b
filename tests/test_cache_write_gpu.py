"""GPU parity of the cache write (mla_write_kv) against the fp64 cache-write oracle.

Every new row is compared value by value (bf16: within half a bf16 ulp of the
exact value plus fp32 accumulation; e4m3: within half an e4m3 ulp of the exact
value, scale within fp32 rounding, codes equal but for values on a rounding
boundary); every other row of the cache must be left bit-identical.  The
written cache is then decoded and compared with the oracle's decode of the
oracle-written cache.
"""

import numpy as np
import pytest
import torch

from oracle import cache_write as cw
from oracle import mla_oracle as om

pytestmark = pytest.mark.gpu


def _inputs(B, s_q, d_h, lens, kv_dtype, num_pages=None, seed=21):
    g = torch.Generator().manual_seed(seed)
    max_pages = max((L + 63) // 64 for L in lens)
    num_pages = num_pages or B * max_pages + 3
    perm = torch.randperm(num_pages, generator=g)[:B * max_pages].reshape(B, max_pages).to(torch.int32)
    h = torch.randn(B, s_q, d_h, generator=g).to(torch.bfloat16)
    w = (torch.randn(576, d_h, generator=g) / d_h ** 0.5).to(torch.bfloat16)
    if kv_dtype == "bf16":
        kv = torch.randn(num_pages, 64, 576, generator=g).to(torch.bfloat16)
        scale = None
    else:
        kv = torch.randn(num_pages, 64, 576, generator=g).clamp(-448, 448).to(torch.float8_e4m3fn)
        scale = torch.rand(num_pages, 64, generator=g) + 0.5
    return h, w, kv, scale, perm, torch.tensor(lens, dtype=torch.int32)


def _run(cuda_lib, h, w, kv, scale, bt, sl, rope_base=10000.0):
    import head_latent_attention_06_b200 as mla
    dev = "cuda"
    h_d, w_d, kv_d = h.to(dev), w.to(dev), kv.to(dev)
    sc_d = None if scale is None else scale.to(dev)
    bt_d, sl_d = bt.to(dev), sl.to(dev)
    a = mla.make_write_kv_args(h=h_d, w_dkv=w_d, kv_cache=kv_d, kv_scale=sc_d, block_table=bt_d,
                               seq_lens=sl_d, rope_base=rope_base)
    ws = mla.alloc_workspace(a)
    mla.mla_write_kv(a)
    status = mla.mla_get_status(ws)
    return kv_d.cpu(), (None if sc_d is None else sc_d.cpu()), status


def _oracle(h, w, kv, scale, bt, sl, kv_dtype, s_q):
    from mla_inputs import bf16_bits, fp8_bits
    hb = om.bf16_to_f64(bf16_bits(h))
    wb = om.bf16_to_f64(bf16_bits(w))
    kvb = bf16_bits(kv) if kv_dtype == "bf16" else fp8_bits(kv)
    sc = None if scale is None else scale.numpy()
    return cw.write_kv(hb, wb[:512], wb[512:], kvb, sc, kv_dtype, bt.numpy(), sl.numpy(), s_q)


def _exact_rows(h, w, bt, sl, s_q):
    from mla_inputs import bf16_bits
    hb = om.bf16_to_f64(bf16_bits(h))
    wb = om.bf16_to_f64(bf16_bits(w))
    out = {}
    for b in range(hb.shape[0]):
        for i in range(s_q):
            pos = int(sl[b]) - s_q + i
            row = np.concatenate([wb[:512] @ hb[b, i], cw.rope(wb[512:] @ hb[b, i], pos)])
            out[(int(bt[b, pos // 64]), pos % 64)] = row
    return out


CASES = [
    # kv, B, s_q, d_h, lens
    ("bf16", 3, 1, 256, [1, 64, 130]),
    ("fp8", 5, 2, 512, [2, 65, 128, 129, 1000]),
    ("bf16", 70, 1, 1024, list(range(1, 141, 2))),
]


def _full_size_inputs(B, s_q, d_h, L, kv_dtype, seed=23):
    """The new tokens of one decode step of a full-size workload (every sequence
    L cached tokens, hidden width d_h).  Only the pages the new rows land in
    matter to the write, so the cache holds 2 pages per sequence: each
    sequence's last logical page maps to a page of its own, its other logical
    pages to arbitrary ones (never written)."""
    g = torch.Generator().manual_seed(seed)
    max_pages = (L + 63) // 64
    num_pages = 2 * B + 3
    perm = torch.randperm(num_pages, generator=g).to(torch.int32)
    bt = torch.randint(0, num_pages, (B, max_pages), generator=g, dtype=torch.int32)
    bt[:, (L - s_q) // 64:] = perm[:B, None]          # the pages the new rows land in
    h = torch.randn(B, s_q, d_h, generator=g).to(torch.bfloat16)
    w = (torch.randn(576, d_h, generator=g) / d_h ** 0.5).to(torch.bfloat16)
    if kv_dtype == "bf16":
        kv = torch.randn(num_pages, 64, 576, generator=g).to(torch.bfloat16)
        scale = None
    else:
        kv = torch.randn(num_pages, 64, 576, generator=g).to(torch.float8_e4m3fn)
        scale = torch.rand(num_pages, 64, generator=g) + 0.5
    return h, w, kv, scale, bt, torch.full((B,), L, dtype=torch.int32)


FULL_SIZE = [
    # the decode workloads' new tokens at a DeepSeek-V3-sized hidden width: 112
    # K chunks of 64, split 16 ways, so every CTA's 4-stage chunk ring wraps
    ("bf16", 64, 1, 7168, 4096),
    ("fp8", 128, 2, 7168, 8192),
]


@pytest.mark.parametrize("kv_dtype,B,s_q,d_h,L", FULL_SIZE)
def test_write_kv_full_size(cuda_lib, kv_dtype, B, s_q, d_h, L):
    a = cuda_lib.WriteKvArgs()
    a.B, a.s_q, a.d_h, a.d_c, a.d_r, a.page_size = B, s_q, d_h, 512, 64, 64
    a.num_pages, a.max_pages_per_seq, a.rope_base = 1, 1, 10000.0
    k_split = (cuda_lib.mla_write_kv_workspace_size(a) - 256) // (B * s_q * 576 * 4)
    assert d_h // 64 > 4 * k_split          # more K chunks per CTA than ring stages
    h, w, kv, scale, bt, sl = _full_size_inputs(B, s_q, d_h, L, kv_dtype)
    _check_write(cuda_lib, h, w, kv, scale, bt, sl, kv_dtype, s_q)


@pytest.mark.parametrize("kv_dtype,B,s_q,d_h,lens", CASES)
def test_write_kv_matches_oracle(cuda_lib, kv_dtype, B, s_q, d_h, lens):
    h, w, kv, scale, bt, sl = _inputs(B, s_q, d_h, lens, kv_dtype)
    _check_write(cuda_lib, h, w, kv, scale, bt, sl, kv_dtype, s_q)


def _check_write(cuda_lib, h, w, kv, scale, bt, sl, kv_dtype, s_q):
    kv_g, sc_g, status = _run(cuda_lib, h, w, kv, scale, bt, sl)
    assert status == 0
    exact = _exact_rows(h, w, bt, sl, s_q)
    from mla_inputs import bf16_bits, fp8_bits
    before = bf16_bits(kv) if kv_dtype == "bf16" else fp8_bits(kv)
    after = bf16_bits(kv_g) if kv_dtype == "bf16" else fp8_bits(kv_g)
    touched = np.zeros(before.shape[:2], dtype=bool)
    for (page, row) in exact:
        touched[page, row] = True
    assert np.array_equal(after[~touched], before[~touched])
    if kv_dtype == "fp8":
        assert torch.equal(sc_g.reshape(-1)[torch.from_numpy(~touched.reshape(-1))],
                           scale.reshape(-1)[torch.from_numpy(~touched.reshape(-1))])
    kv_o, sc_o = _oracle(h, w, kv, scale, bt, sl, kv_dtype, s_q)
    n_code_diff = 0
    for (page, row), want in exact.items():
        if kv_dtype == "bf16":
            got = om.bf16_to_f64(after[page, row])
            assert np.all(np.abs(got - want) <= 2.0 ** -8 * np.abs(want) + 1e-6)
        else:
            s = float(sc_g[page, row])
            assert s == pytest.approx(float(sc_o[page, row]), rel=1e-5)
            got = om.e4m3fn_to_f64(after[page, row]) * s
            assert np.all(np.abs(got - want) <= (2.0 ** -4 + 1e-4) * np.abs(want) + 2.0 ** -9 * s)
            n_code_diff += int((after[page, row] != kv_o[page, row]).sum())
    if kv_dtype == "fp8":
        assert n_code_diff <= 1e-3 * len(exact) * 576


def test_written_tokens_decode_like_the_oracle(cuda_lib):
    """Write the last token of each sequence, then decode: the result matches the
    decode oracle run on the oracle-written cache."""
    import head_latent_attention_06_b200 as mla
    from mla_inputs import WorkloadSpec, make_workload, bf16_bits
    from head_latent_attention_06_b200.step import step_from_workload
    import oracle
    from parity_util import compare_step
    spec = WorkloadSpec("cw", B=3, H=128, s_q=1, lens=[1, 70, 300], kv_dtype="bf16", causal=False,
                        seed=5, permute_pages=True)
    wl = make_workload(spec)
    d_h = 512
    g = torch.Generator().manual_seed(3)
    h = torch.randn(3, 1, d_h, generator=g).to(torch.bfloat16)
    w = (torch.randn(576, d_h, generator=g) / d_h ** 0.5).to(torch.bfloat16)
    st = step_from_workload(wl)
    kv_d, _, bt_d, sl_d = st._keep
    h_d, w_d = h.cuda(), w.cuda()           # kept alive until the write has run
    a = mla.make_write_kv_args(h=h_d, w_dkv=w_d, kv_cache=kv_d, kv_scale=None,
                               block_table=bt_d, seq_lens=sl_d)
    ws = mla.alloc_workspace(a)
    mla.mla_write_kv(a)
    assert mla.mla_get_status(ws) == 0
    st.run()
    torch.cuda.synchronize()
    kv_o, _ = _oracle(h, w, wl.kv_cache, None, wl.block_table, wl.seq_lens, "bf16", 1)
    inp = oracle.from_workload(wl)
    inp.kv = kv_o
    ref = om.decode_absorbed(inp)
    compare_step(st, wl, ref)


def test_bad_block_table_is_reported_and_the_row_skipped(cuda_lib):
    h, w, kv, scale, bt, sl = _inputs(2, 1, 128, [10, 20], "bf16")
    bt[1, 0] = kv.shape[0] + 5
    kv_g, _, status = _run(cuda_lib, h, w, kv, scale, bt, sl)
    assert status == 7                                  # MLA_ERR_BAD_BLOCK_TABLE
    from mla_inputs import bf16_bits
    before, after = bf16_bits(kv), bf16_bits(kv_g)
    changed = np.argwhere((before != after).any(axis=2))
    assert [tuple(x) for x in changed] == [(int(bt[0, 0]), 9)]
