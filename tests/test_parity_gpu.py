"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.

Small cases compare every output element; they span several 32/64-token tiles,
ragged tails, forced split counts, both cache types, causal s_q = 2 and the
head counts 16..128.  The full-size workloads (the five presets, in the launch
configuration bench.py times) compare sampled (sequence, query) rows, all
heads, against the absorbed fp64 oracle, plus a few heads against the
explicit-K/V definition.
"""

import numpy as np
import pytest
import torch

from mla_inputs import WorkloadSpec, make_workload, preset, PRESETS
from oracle import mla_oracle as om
import oracle

from parity_util import TOL, check_close, check_lse, compare_step, errors, oracle_of, report, to_np

pytestmark = pytest.mark.gpu


def _run(cuda_lib, w, splits=0):
    from head_latent_attention_06_b200.step import step_from_workload
    st = step_from_workload(w, num_splits=splits)
    st.run()
    torch.cuda.synchronize()
    assert cuda_lib.mla_get_status(st.workspace) == 0
    return st


def _spec(kv, H, s_q, lens, causal=False, seed=7, permute=True):
    return WorkloadSpec("case", B=len(lens), H=H, s_q=s_q, lens=list(lens), kv_dtype=kv,
                        causal=causal, seed=seed, permute_pages=permute)


def test_tiny_preset_against_definition(cuda_lib):
    w = make_workload(preset("tiny"))
    st = _run(cuda_lib, w)
    ref = oracle_of(w)                         # explicit K/V, every element
    compare_step(st, w, ref)


SMALL = [
    # kv, H, s_q, causal, lens, splits
    ("bf16", 128, 1, False, [1, 63, 64, 65, 200, 1000], 0),
    ("bf16", 128, 1, False, [1, 63, 64, 65, 200, 1000], 1),
    ("bf16", 128, 1, False, [1, 63, 64, 65, 200, 1000], 3),
    ("bf16", 128, 1, False, [1, 63, 64, 65, 200, 1000], 16),
    ("bf16", 128, 2, False, [33, 640], 2),
    ("fp8", 128, 2, True, [2, 64, 130, 777], 1),
    ("fp8", 128, 2, True, [2, 64, 130, 777], 5),
    ("bf16", 16, 1, False, [300, 5000], 0),
    ("bf16", 64, 2, True, [100, 129], 2),
    ("fp8", 32, 1, False, [1000, 31], 0),
    ("fp8", 16, 1, False, [300, 5000], 0),
    ("fp8", 128, 1, False, [1, 63, 64, 65, 200, 1000], 3),
    ("bf16", 48, 1, False, [95], 0),
]


@pytest.mark.parametrize("kv,H,s_q,causal,lens,splits", SMALL)
def test_small_cases_every_element(cuda_lib, kv, H, s_q, causal, lens, splits):
    w = make_workload(_spec(kv, H, s_q, lens, causal))
    st = _run(cuda_lib, w, splits)
    ref = oracle_of(w, absorbed=True)          # pinned equal to the definition (P1)
    report(f"small {kv} H={H} s_q={s_q} causal={causal} lens={lens} splits={splits}", compare_step(st, w, ref))
    # and the explicit K/V definition on a few heads of the longest sequence
    b = int(np.argmax(lens))
    heads = [0, H - 1]
    rows = [(b, i) for i in range(s_q)]
    ref2 = oracle_of(w, rows=rows, heads=heads)
    sel = (np.array([b] * s_q)[:, None], np.arange(s_q)[:, None], np.array(heads)[None, :])
    check_close("o (definition)", to_np(st.out)[sel], ref2["o"][sel], kv)


@pytest.mark.parametrize("lens,splits", [([1, 63, 64, 65, 200, 1000], 1), ([700, 3], 4)])
def test_warp_mma_kernel_on_128_heads(cuda_lib, lens, splits):
    """The portable warp-MMA kernel, forced for a shape the tensor-memory kernel takes."""
    w = make_workload(_spec("bf16", 128, 1, lens))
    cuda_lib.mla_set_decode_kernel(cuda_lib.DECODE_WARP_MMA)
    try:
        st = _run(cuda_lib, w, splits)
    finally:
        cuda_lib.mla_set_decode_kernel(cuda_lib.DECODE_AUTO)
    compare_step(st, w, oracle_of(w, absorbed=True))


def test_empty_and_short_contexts(cuda_lib):
    w = make_workload(_spec("bf16", 16, 2, [0, 1, 2, 70], causal=True))
    for splits in (1, 4):
        st = _run(cuda_lib, w, splits)
        ref = oracle_of(w)
        o, lse = to_np(st.out), to_np(st.lse)
        assert np.all(o[0] == 0) and np.all(np.isneginf(lse[0]))          # L = 0
        assert np.all(o[1, 0] == 0) and np.all(np.isneginf(lse[1, 0]))    # query 0 of L = 1
        compare_step(st, w, ref)


@pytest.mark.parametrize("H", [128, 64])
def test_split_count_invariance(cuda_lib, H):
    w = make_workload(_spec("bf16", H, 1, [3000, 4096, 17]))
    outs = [to_np(_run(cuda_lib, w, s).out) for s in (1, 2, 7, 32)]
    for o in outs[1:]:
        ma, rl = errors(o, outs[0])
        assert ma <= 1e-2 and rl <= 5e-3, (ma, rl)


@pytest.mark.parametrize("kv", ["bf16", "fp8"])
@pytest.mark.parametrize("H", [64, 128])
def test_page_permutation_is_bit_exact(cuda_lib, kv, H):
    a = make_workload(_spec(kv, H, 1, [500, 129], permute=False))
    b = make_workload(_spec(kv, H, 1, [500, 129], permute=True))
    assert not torch.equal(a.block_table, b.block_table)
    oa, ob = _run(cuda_lib, a).out, _run(cuda_lib, b).out
    assert torch.equal(oa, ob)


def _poison_page_tails(w):
    """Fill the cache rows past each sequence's end (and, fp8, their scales) with NaN."""
    for b, L in enumerate(w.lens):
        if L % 64 == 0:
            continue
        pg = int(w.block_table[b, L // 64])
        if w.spec.kv_dtype == "fp8":
            w.kv_cache[pg, L % 64:] = torch.full((64 - L % 64, 576), float("nan")).to(w.kv_cache.dtype)
            w.kv_scale[pg, L % 64:] = float("nan")
        else:
            w.kv_cache[pg, L % 64:] = float("nan")


@pytest.mark.parametrize("kv", ["bf16", "fp8"])
@pytest.mark.parametrize("H", [128, 32])
def test_bytes_past_the_sequence_end_never_reach_the_output(cuda_lib, kv, H):
    """Rows of a last page past the length are not part of the sequence: NaN there changes nothing."""
    w = make_workload(_spec(kv, H, 2, [70, 1000, 129], causal=True))
    clean = _run(cuda_lib, w, 2)
    o_clean, lse_clean = clean.out.clone(), clean.lse.clone()
    _poison_page_tails(w)
    for splits in (1, 2):
        st = _run(cuda_lib, w, splits)
        assert torch.isfinite(st.out).all() and torch.isfinite(st.lse).all()
        ma, rl = errors(to_np(st.out), to_np(o_clean))
        assert ma <= 1e-2 and rl <= 5e-3, (ma, rl)


@pytest.mark.parametrize("factor", [2.0 ** -14, 1.0, 2.0 ** 8])
def test_fp8_scale_magnitudes(cuda_lib, factor):
    """Token scales far from 1 (values near f16's smallest normals, or scores 256x
    larger): the decode kernel alone, given a q_lat that the oracle also uses (the
    oracle's fp64 absorption rounded to bf16, the boundary's type), tracks the
    oracle relative to the value magnitude.  The absorption's own bf16 rounding is
    left out because its score error grows with the score magnitude."""
    from head_latent_attention_06_b200.step import step_from_workload
    w = make_workload(_spec("fp8", 128, 1, [700, 64, 3]))
    w.kv_scale.mul_(factor)
    inp = oracle.from_workload(w)
    q_lat = torch.from_numpy(om.absorb_q(inp.q_nope, inp.w_uk)).to(torch.bfloat16)
    st = step_from_workload(w)
    st.q_lat.copy_(q_lat.to(st.q_lat.device))
    st.attend()
    torch.cuda.synchronize()
    assert cuda_lib.mla_get_status(st.workspace) == 0
    qb = q_lat.double().numpy()
    o_lat, lse = to_np(st.o_lat), to_np(st.lse)
    amax, rl2 = TOL["fp8"]
    for b in range(w.B):
        C = inp.rows(b, inp.visible(b, 0))
        ref_o, ref_lse = om.latent_attention(qb[b, 0], inp.q_pe[b, 0], C, inp.softmax_scale)
        ma, rl = errors(o_lat[b, 0] / factor, ref_o / factor)
        assert ma <= amax and rl <= rl2, (b, ma, rl)
        assert np.abs(lse[b, 0] - ref_lse).max() <= amax


@pytest.mark.parametrize("n_tok,H", [(70, 128), (1, 16), (300, 16), (256, 128), (129, 48)])
def test_projections_against_oracle(cuda_lib, n_tok, H):
    """Token blocks of 64 / 128, a ragged last block, several CTAs per head (few heads)."""
    g = torch.Generator().manual_seed(5)
    q = torch.randn(n_tok, H, 128, generator=g).to(torch.bfloat16)
    w_uk = (torch.randn(H, 128, 512, generator=g) / 512 ** 0.5).to(torch.bfloat16)
    x = torch.randn(n_tok, H, 512, generator=g).to(torch.bfloat16)
    w_uv = (torch.randn(H, 128, 512, generator=g) / 512 ** 0.5).to(torch.bfloat16)
    q_lat = torch.empty(n_tok, H, 512, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(n_tok, H, 128, dtype=torch.bfloat16, device="cuda")
    cuda_lib.mla_absorb_q(q.cuda(), w_uk.cuda(), q_lat)
    cuda_lib.mla_up_proj_v(x.cuda(), w_uv.cuda(), out)
    torch.cuda.synchronize()
    f = lambda t: t.double().numpy()
    ref_q = om.absorb_q(f(q), f(w_uk))
    ref_o = om.up_proj_v(f(x), f(w_uv))
    # bf16 output: one rounding of an fp32 sum
    ma, rl = errors(to_np(q_lat), ref_q)
    assert rl <= 4e-3 and ma <= 2e-2, (ma, rl)
    ma, rl = errors(to_np(out), ref_o)
    assert rl <= 4e-3 and ma <= 4e-2, (ma, rl)


@pytest.mark.parametrize("H", [16, 128])
def test_device_checks_report_bad_block_table_and_length(cuda_lib, H):
    from head_latent_attention_06_b200.step import step_from_workload
    w = make_workload(_spec("bf16", H, 1, [130, 64]))
    st = step_from_workload(w)
    bt = st._keep[2]
    bt[0, 1] = 10_000                     # page id beyond the cache: skipped, reported
    st.run()
    assert cuda_lib.mla_get_status(st.workspace) == 7
    assert cuda_lib.mla_get_status(st.workspace) == 0     # cleared by the read
    bt[0, 1] = int(w.block_table[0, 1])
    lens = st._keep[3]
    lens[1] = 64 * w.max_pages + 1        # longer than the block table allows
    st.run()
    assert cuda_lib.mla_get_status(st.workspace) == 8


# ---------------------------------------------------------------- full-size presets

def _sample_rows(w, k=6, seed=0):
    lens = np.array(w.lens)
    rng = np.random.default_rng(seed)
    bs = {int(np.argmin(lens)), int(np.argmax(lens)), 0, w.B - 1}
    while len(bs) < min(k, w.B):
        bs.add(int(rng.integers(w.B)))
    return [(b, i) for b in sorted(bs) for i in range(w.s_q)]


@pytest.mark.parametrize("name", ["v3", "ragged", "long16", "long128", "fp8"])
def test_full_size_presets_sampled(cuda_lib, name):
    w = make_workload(preset(name))
    st = _run(cuda_lib, w)
    rows = _sample_rows(w)
    ref = oracle_of(w, rows=rows, absorbed=True)
    report(f"full-size {name} (sampled rows)", compare_step(st, w, ref, rows=rows))
    # the explicit-K/V definition on two heads of the first and last sampled row
    for (b, i) in (rows[0], rows[-1]):
        heads = [0, w.H - 1]
        d = oracle_of(w, rows=[(b, i)], heads=heads)
        check_close(f"o definition b={b}", to_np(st.out)[b, i, heads], d["o"][b, i, heads],
                    w.spec.kv_dtype)
    # every output finite
    assert torch.isfinite(st.out).all() and torch.isfinite(st.lse).all()
