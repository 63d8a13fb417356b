"""GPU parity over the blockwise q4_0 cache (ik_llama.cpp docs "FlashMLA",
section "KV cache with MLA": lower-bit blockwise caches; 4-bit codes with one
fp16 scale per 32 values, stored as code + 8, two codes a byte), through the C
ABI: the decode against the fp64 oracle reading the same bytes and scales, and
the cache write against the cache-write oracle.

Tolerance: each value is formed in bf16 from its code and block scale (the
product is exact in fp32 and rounded once), as for q8_0, so the bf16 bounds
apply against the oracle's exact dequantised values."""
import numpy as np
import pytest
import torch

from mla_inputs import WorkloadSpec, make_workload, preset
from parity_util import check_close, compare_step, oracle_of, report, to_np

pytestmark = pytest.mark.gpu


def _run(cuda_lib, w, splits=0, kernel=None):
    from head_latent_attention_06_b200.step import step_from_workload
    if kernel is not None:
        cuda_lib.mla_set_decode_kernel(kernel)
    try:
        st = step_from_workload(w, num_splits=splits)
        st.run()
        torch.cuda.synchronize()
    finally:
        cuda_lib.mla_set_decode_kernel(cuda_lib.DECODE_AUTO)
    assert cuda_lib.mla_get_status(st.workspace) == 0
    return st


CASES = [
    # H, s_q, causal, lens, splits
    (128, 1, False, [1, 63, 64, 65, 200, 1000], 0),
    (128, 1, False, [1, 63, 64, 65, 200, 1000], 3),
    (16, 1, False, [300, 5000], 0),
    (64, 2, True, [2, 64, 130, 777], 2),
    (128, 8, True, [8, 300], 0),
]


@pytest.mark.parametrize("kernel", ["tensor_memory", "warp_mma"])
@pytest.mark.parametrize("H,s_q,causal,lens,splits", CASES)
def test_q4_0_decode_every_element(cuda_lib, H, s_q, causal, lens, splits, kernel):
    """Both decode kernels: the tensor-memory one (converter warps split each byte
    into two codes and expand them into bf16 operands) and the warp-MMA one."""
    w = make_workload(WorkloadSpec("q4c", B=len(lens), H=H, s_q=s_q, lens=lens, kv_dtype="q4_0",
                                   causal=causal, seed=27))
    st = _run(cuda_lib, w, splits, None if kernel == "tensor_memory" else cuda_lib.DECODE_WARP_MMA)
    report(f"q4_0 {kernel} H={H} s_q={s_q} lens={lens} splits={splits}",
           compare_step(st, w, oracle_of(w, absorbed=True)))
    # and the explicit-K/V definition on two heads of the longest sequence
    b = int(np.argmax(lens))
    rows = [(b, i) for i in range(s_q)]
    ref = oracle_of(w, rows=rows, heads=[0, H - 1])
    sel = (np.array([b] * s_q)[:, None], np.arange(s_q)[:, None], np.array([0, H - 1])[None, :])
    check_close("o (definition)", to_np(st.out)[sel], ref["o"][sel], "q4_0")


def test_q4_0_full_size_sampled(cuda_lib):
    w = make_workload(preset("q4"))
    st = _run(cuda_lib, w)
    rows = [(b, 0) for b in (0, 17, 63)]
    report("full-size q4 (sampled rows)", compare_step(st, w, oracle_of(w, rows=rows, absorbed=True), rows=rows))
    assert torch.isfinite(st.out).all()


@pytest.mark.parametrize("kernel", ["tensor_memory", "warp_mma"])
def test_q4_0_bytes_past_the_sequence_end_never_reach_the_output(cuda_lib, kernel):
    k = None if kernel == "tensor_memory" else cuda_lib.DECODE_WARP_MMA
    w = make_workload(WorkloadSpec("q4t", B=2, H=128, s_q=1, lens=[70, 129], kv_dtype="q4_0", seed=19))
    clean = to_np(_run(cuda_lib, w, kernel=k).out)
    for b, L in enumerate(w.lens):
        pg = int(w.block_table[b, L // 64])
        w.kv_cache[pg, L % 64:] = 0xFF
        w.kv_scale[pg, L % 64:] = float("nan")
    st = _run(cuda_lib, w, kernel=k)
    assert torch.isfinite(st.out).all()
    assert np.abs(to_np(st.out) - clean).max() <= 1e-2


def test_q4_0_matches_q8_0_holding_the_same_codes(cuda_lib):
    """The same codes (within [-7, 7]) and scales as a q8_0 cache and as a q4_0
    cache: the two decodes agree to the last bit (the values formed are equal)."""
    w8 = make_workload(WorkloadSpec("q84", B=3, H=128, s_q=1, lens=[100, 700, 64], kv_dtype="q8_0", seed=31))
    w8.kv_cache.clamp_(-7, 7)
    n = (w8.kv_cache.to(torch.int16) + 8).to(torch.uint8)
    w4 = make_workload(WorkloadSpec("q84", B=3, H=128, s_q=1, lens=[100, 700, 64], kv_dtype="q4_0", seed=31))
    w4.kv_cache.copy_(n[..., 0::2] | (n[..., 1::2] << 4))
    w4.kv_scale.copy_(w8.kv_scale)
    a, b = to_np(_run(cuda_lib, w8).out), to_np(_run(cuda_lib, w4).out)
    assert np.array_equal(a, b)


def _unpack(packed: np.ndarray) -> np.ndarray:
    b = packed.astype(np.int64)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.int64)
    out[..., 0::2] = (b & 15) - 8
    out[..., 1::2] = (b >> 4) - 8
    return out


def test_q4_0_cache_write_matches_the_oracle(cuda_lib):
    import head_latent_attention_06_b200 as mla
    from mla_inputs import bf16_bits
    from oracle import cache_write as cw
    from oracle import mla_oracle as om
    g = torch.Generator().manual_seed(37)
    B, s_q, d_h = 5, 2, 512
    lens = [2, 65, 128, 129, 1000]
    max_pages = max((L + 63) // 64 for L in lens)
    P = B * max_pages + 3
    bt = torch.randperm(P, generator=g)[:B * max_pages].reshape(B, max_pages).to(torch.int32)
    h = torch.randn(B, s_q, d_h, generator=g).to(torch.bfloat16)
    w = (torch.randn(576, d_h, generator=g) / d_h ** 0.5).to(torch.bfloat16)
    kv = torch.randint(0, 256, (P, 64, 288), generator=g).to(torch.uint8)
    sc = (torch.rand(P, 64, 18, generator=g) + 0.5).to(torch.float16)
    sl = torch.tensor(lens, dtype=torch.int32)
    # the argument struct holds raw pointers: every device tensor stays referenced
    kv_d, sc_d, h_d, w_d, bt_d, sl_d = kv.cuda(), sc.cuda(), h.cuda(), w.cuda(), bt.cuda(), sl.cuda()
    a = mla.make_write_kv_args(h=h_d, w_dkv=w_d, kv_cache=kv_d, kv_scale=sc_d, block_table=bt_d, seq_lens=sl_d)
    ws = mla.alloc_workspace(a)
    mla.mla_write_kv(a)
    assert mla.mla_get_status(ws) == 0
    hb, wb = om.bf16_to_f64(bf16_bits(h)), om.bf16_to_f64(bf16_bits(w))
    kv_o, sc_o = cw.write_kv(hb, wb[:512], wb[512:], kv.numpy(), sc.numpy(), "q4_0", bt.numpy(), sl.numpy(), s_q)
    got_kv, got_sc = kv_d.cpu().numpy(), sc_d.cpu().numpy()
    touched = np.zeros((P, 64), dtype=bool)
    for b, L in enumerate(lens):
        for i in range(s_q):
            pos = L - s_q + i
            touched[int(bt[b, pos // 64]), pos % 64] = True
    assert np.array_equal(got_kv[~touched], kv.numpy()[~touched])
    assert np.array_equal(got_sc[~touched], sc.numpy()[~touched])
    assert np.array_equal(got_sc[touched], sc_o[touched])
    d = np.abs(_unpack(got_kv[touched]) - _unpack(np.asarray(kv_o)[touched]))
    assert d.max() <= 1 and (d > 0).sum() <= 1e-3 * d.size
