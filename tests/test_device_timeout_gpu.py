"""The decode kernels' bounded waits, made to run out on purpose.

With the wait limit set to 1 ns, the first wait inside the kernel that is not
satisfied at once gives up: the kernel records MLA_ERR_DEVICE_TIMEOUT in the
workspace's status word, leaves its loops, waits for the copies it already
issued, frees its tensor memory and returns.  Nothing faults or hangs; the next
decode on the same context, with the default limit back, matches the oracle.
"""
import pytest
import torch

from mla_inputs import WorkloadSpec, make_workload
from parity_util import compare_step, oracle_of

pytestmark = pytest.mark.gpu

TIMEOUT = 6


# split count 0: the automatic choice
@pytest.mark.parametrize("kv,splits", [("bf16", 0), ("bf16", 1), ("bf16", 3), ("fp8", 1), ("fp8", 2), ("q8_0", 1),
                                      ("q8_0", 2)])
def test_wait_that_runs_out_is_reported_and_the_context_stays_usable(cuda_lib, kv, splits):
    from head_latent_attention_06_b200.step import step_from_workload
    w = make_workload(WorkloadSpec("to", B=3, H=128, s_q=1, lens=[1000, 300, 70], kv_dtype=kv, seed=31,
                                   permute_pages=True))
    st = step_from_workload(w, num_splits=splits)
    st.absorb()
    torch.cuda.synchronize()
    cuda_lib.mla_set_device_wait_limit(1)
    try:
        cuda_lib.mla_decode_paged(st.args)
        torch.cuda.synchronize()
    finally:
        cuda_lib.mla_set_device_wait_limit(0)
    assert cuda_lib.mla_get_status(st.workspace) == TIMEOUT
    assert cuda_lib.mla_get_status(st.workspace) == 0          # cleared by the read
    st.run()
    torch.cuda.synchronize()
    assert cuda_lib.mla_get_status(st.workspace) == 0
    compare_step(st, w, oracle_of(w, absorbed=True))
