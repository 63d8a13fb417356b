"""GPU parity over the blockwise q8_0 cache (ik_llama.cpp docs "FlashMLA",
section "KV cache with MLA": int8 codes, one fp16 scale per 32 values of a row),
through the C ABI: the decode against the fp64 oracle reading the same codes and
scales, and the cache write against the cache-write oracle."""
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
def test_q8_0_decode_every_element(cuda_lib, H, s_q, causal, lens, splits, kernel):
    """Both decode kernels: the tensor-memory one (converter warps expand the
    codes into bf16 operands) and the warp-MMA one."""
    w = make_workload(WorkloadSpec("q8c", B=len(lens), H=H, s_q=s_q, lens=lens, kv_dtype="q8_0",
                                   causal=causal, seed=17))
    st = _run(cuda_lib, w, splits, None if kernel == "tensor_memory" else cuda_lib.DECODE_WARP_MMA)
    report(f"q8_0 {kernel} H={H} s_q={s_q} lens={lens} splits={splits}",
           compare_step(st, w, oracle_of(w, absorbed=True)))
    # and the explicit-K/V definition on two heads of the longest sequence
    b = int(np.argmax(lens))
    rows = [(b, i) for i in range(s_q)]
    ref = oracle_of(w, rows=rows, heads=[0, H - 1])
    sel = (np.array([b] * s_q)[:, None], np.arange(s_q)[:, None], np.array([0, H - 1])[None, :])
    check_close("o (definition)", to_np(st.out)[sel], ref["o"][sel], "q8_0")


def test_q8_0_full_size_sampled(cuda_lib):
    w = make_workload(preset("q8"))
    st = _run(cuda_lib, w)
    rows = [(b, 0) for b in (0, 17, 63)]
    report("full-size q8 (sampled rows)", compare_step(st, w, oracle_of(w, rows=rows, absorbed=True), rows=rows))
    assert torch.isfinite(st.out).all()


@pytest.mark.parametrize("kernel", ["tensor_memory", "warp_mma"])
def test_q8_0_bytes_past_the_sequence_end_never_reach_the_output(cuda_lib, kernel):
    k = None if kernel == "tensor_memory" else cuda_lib.DECODE_WARP_MMA
    w = make_workload(WorkloadSpec("q8t", B=2, H=128, s_q=1, lens=[70, 129], kv_dtype="q8_0", seed=19))
    clean = to_np(_run(cuda_lib, w, kernel=k).out)
    for b, L in enumerate(w.lens):
        pg = int(w.block_table[b, L // 64])
        w.kv_cache[pg, L % 64:] = 127
        w.kv_scale[pg, L % 64:] = float("nan")
    st = _run(cuda_lib, w, kernel=k)
    assert torch.isfinite(st.out).all()
    assert np.abs(to_np(st.out) - clean).max() <= 1e-2


def test_q8_0_cache_write_matches_the_oracle(cuda_lib):
    import head_latent_attention_06_b200 as mla
    from mla_inputs import f16_bits, int8_bits
    from oracle import cache_write as cw
    from oracle import mla_oracle as om
    g = torch.Generator().manual_seed(29)
    B, s_q, d_h = 5, 2, 512
    lens = [2, 65, 128, 129, 1000]
    max_pages = max((L + 63) // 64 for L in lens)
    P = B * max_pages + 3
    bt = torch.randperm(P, generator=g)[:B * max_pages].reshape(B, max_pages).to(torch.int32)
    h = torch.randn(B, s_q, d_h, generator=g).to(torch.bfloat16)
    w = (torch.randn(576, d_h, generator=g) / d_h ** 0.5).to(torch.bfloat16)
    kv = torch.randint(-127, 128, (P, 64, 576), generator=g).to(torch.int8)
    sc = (torch.rand(P, 64, 18, generator=g) + 0.5).to(torch.float16)
    sl = torch.tensor(lens, dtype=torch.int32)
    kv_d, sc_d = kv.cuda(), sc.cuda()
    h_d, w_d, bt_d, sl_d = h.cuda(), w.cuda(), bt.cuda(), sl.cuda()
    a = mla.make_write_kv_args(h=h_d, w_dkv=w_d, kv_cache=kv_d, kv_scale=sc_d, block_table=bt_d, seq_lens=sl_d)
    ws = mla.alloc_workspace(a)
    mla.mla_write_kv(a)
    assert mla.mla_get_status(ws) == 0
    from mla_inputs import bf16_bits
    hb, wb = om.bf16_to_f64(bf16_bits(h)), om.bf16_to_f64(bf16_bits(w))
    kv_o, sc_o = cw.write_kv(hb, wb[:512], wb[512:], int8_bits(kv), sc.numpy(), "q8_0", bt.numpy(),
                             sl.numpy(), s_q)
    got_kv, got_sc = int8_bits(kv_d.cpu()).view(np.int8), sc_d.cpu().numpy()
    ref_kv = np.asarray(kv_o).view(np.int8)
    touched = np.zeros((P, 64), dtype=bool)
    for b, L in enumerate(lens):
        for i in range(s_q):
            pos = L - s_q + i
            touched[int(bt[b, pos // 64]), pos % 64] = True
    before = int8_bits(kv).view(np.int8)
    assert np.array_equal(got_kv[~touched], before[~touched])
    assert np.array_equal(got_sc[~touched], sc.numpy()[~touched])
    # scales: fp16 values equal; codes equal but for quotients on a rounding boundary
    assert np.array_equal(got_sc[touched], sc_o[touched])
    d = np.abs(got_kv[touched].astype(np.int64) - ref_kv[touched].astype(np.int64))
    assert d.max() <= 1 and (d > 0).sum() <= 1e-3 * d.size
