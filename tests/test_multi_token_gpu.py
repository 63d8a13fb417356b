"""GPU parity of queries with more than two tokens per sequence: speculative
decoding and chunked prefill in the absorbed form (every new token attends to
the latent cache like a decode query, causal among the new tokens).  Both
decode kernels, both cache types, against the fp64 oracle on every element."""
import pytest

from mla_inputs import WorkloadSpec, make_workload
from parity_util import compare_step, oracle_of, report

pytestmark = pytest.mark.gpu


def _spec(kv, H, s_q, lens, causal=True, seed=9):
    return WorkloadSpec("mt", B=len(lens), H=H, s_q=s_q, lens=list(lens), kv_dtype=kv,
                        causal=causal, seed=seed, permute_pages=True)


def _run(cuda_lib, w, splits=0, kernel=None):
    import torch
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
    # kv, H, s_q, lens, splits, causal
    ("bf16", 128, 8, [8, 700], 0, True),
    ("fp8", 128, 8, [8, 129], 2, True),
    ("bf16", 128, 64, [64, 1000], 0, True),
    ("fp8", 128, 64, [100, 640], 0, True),
    ("bf16", 128, 128, [128, 1500], 3, True),
    ("fp8", 128, 128, [130, 2000], 0, True),
    ("bf16", 16, 64, [64, 1000], 0, True),
    ("bf16", 128, 3, [3, 64, 65], 5, True),
    ("bf16", 64, 4, [40, 300], 0, False),
]


@pytest.mark.parametrize("kv,H,s_q,lens,splits,causal", CASES)
def test_multi_token_queries_tensor_memory_kernel(cuda_lib, kv, H, s_q, lens, splits, causal):
    w = make_workload(_spec(kv, H, s_q, lens, causal))
    st = _run(cuda_lib, w, splits)
    report(f"multi-token {kv} H={H} s_q={s_q} lens={lens} splits={splits}",
           compare_step(st, w, oracle_of(w, absorbed=True)))


@pytest.mark.parametrize("kv,H,s_q,lens,splits,causal", [c for c in CASES if c[2] <= 64])
def test_multi_token_queries_warp_mma_kernel(cuda_lib, kv, H, s_q, lens, splits, causal):
    w = make_workload(_spec(kv, H, s_q, lens, causal))
    st = _run(cuda_lib, w, splits, kernel=cuda_lib.DECODE_WARP_MMA)
    compare_step(st, w, oracle_of(w, absorbed=True))


def test_chunk_equals_prefix_decodes(cuda_lib):
    """Query i of a causal chunk equals a one-token decode of the sequence cut at
    its position (the same cache pages, length L - s_q + i + 1)."""
    import dataclasses
    import torch
    from parity_util import errors, to_np
    s_q, L = 16, 300
    w = make_workload(_spec("bf16", 128, s_q, [L]))
    st = _run(cuda_lib, w)
    for i in (0, 7, 15):
        w1 = dataclasses.replace(w, spec=w.spec.with_(s_q=1), q_nope=w.q_nope[:, i:i + 1].clone(),
                                 q_pe=w.q_pe[:, i:i + 1].clone(),
                                 seq_lens=torch.tensor([L - s_q + i + 1], dtype=torch.int32))
        one = _run(cuda_lib, w1)
        ma, rl = errors(to_np(one.out)[0, 0], to_np(st.out)[0, i])
        assert ma <= 1e-2 and rl <= 5e-3, (i, ma, rl)
