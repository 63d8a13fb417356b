"""GPU parity at the edges of the supported sizes: the maximum split count, many
short sequences, an all-empty batch and causal queries across a page boundary."""
import pytest
import torch

from mla_inputs import WorkloadSpec, make_workload
from parity_util import compare_step, oracle_of, report

pytestmark = pytest.mark.gpu


def _run(cuda_lib, w, splits=0):
    from head_latent_attention_06_b200.step import step_from_workload
    st = step_from_workload(w, num_splits=splits)
    st.run()
    torch.cuda.synchronize()
    assert cuda_lib.mla_get_status(st.workspace) == 0
    return st


def _spec(kv, H, s_q, lens, causal=False, seed=13):
    return WorkloadSpec("edge", B=len(lens), H=H, s_q=s_q, lens=list(lens), kv_dtype=kv,
                        causal=causal, seed=seed, permute_pages=True)


def test_maximum_split_count(cuda_lib):
    # 128 splits (the largest count the ABI takes) over one sequence of 2048 pages and a short one
    w = make_workload(_spec("bf16", 128, 1, [131072, 700]))
    st = _run(cuda_lib, w, splits=128)
    rows = [(0, 0), (1, 0)]
    report("edge: 128 splits", compare_step(st, w, oracle_of(w, rows=rows, absorbed=True), rows=rows))


def test_many_short_sequences(cuda_lib):
    # a large batch of one- and two-page sequences (many work units, ragged tails)
    lens = [1 + (37 * i) % 128 for i in range(512)]
    w = make_workload(_spec("bf16", 64, 1, lens))
    st = _run(cuda_lib, w)
    rows = [(b, 0) for b in (0, 1, 2, 255, 511)]
    report("edge: 512 short sequences", compare_step(st, w, oracle_of(w, rows=rows, absorbed=True), rows=rows))


def test_all_empty_batch(cuda_lib):
    w = make_workload(_spec("bf16", 128, 2, [0, 0, 0], causal=True))
    st = _run(cuda_lib, w)
    assert torch.all(st.o_lat == 0) and torch.all(torch.isneginf(st.lse))
    assert torch.all(st.out == 0)


@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_causal_second_query_sees_one_more_token(cuda_lib, kv):
    # lengths 2, 65, 129: query 0 sees 1 / 64 / 128 tokens (page boundaries), query 1 one more
    w = make_workload(_spec(kv, 128, 2, [2, 65, 129], causal=True))
    st = _run(cuda_lib, w)
    compare_step(st, w, oracle_of(w, absorbed=True))
