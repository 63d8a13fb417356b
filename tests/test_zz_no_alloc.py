"""The allocation-free decode entry point against the regular one.

mla_decode_paged_noalloc serves callers that cannot call cudaMalloc (an engine
plugin whose host owns all device memory, a path where an allocation could
synchronise the device): it keeps its scratch in an array built into the
library.  It must give the same o_lat and lse as mla_decode_paged followed by
mla_combine_splits with a caller-allocated workspace, call after call.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""

import numpy as np
import pytest
import torch

from mla_inputs import WorkloadSpec, make_workload

from parity_util import TOL, errors, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("H,lens,splits,kv", [
    (128, [700, 129, 3000], 3, "bf16"),   # partials pass through the built-in scratch
    (16, [300, 5000], 0, "bf16"),
    (128, [64, 1000], 1, "fp8"),
])
def test_noalloc_matches_regular_entry_point(cuda_lib, H, lens, splits, kv):
    from head_latent_attention_06_b200.step import step_from_workload
    w = make_workload(WorkloadSpec("na", B=len(lens), H=H, s_q=1, lens=lens, kv_dtype=kv, seed=21))
    st = step_from_workload(w, num_splits=splits)
    st.absorb()
    st.attend()
    torch.cuda.synchronize()
    assert cuda_lib.mla_get_status(st.workspace) == 0
    ref_o, ref_lse = to_np(st.o_lat), to_np(st.lse)
    amax, rl2 = TOL[kv]
    for call in range(2):                       # two calls in a row share the scratch
        st.o_lat.fill_(float("nan"))
        st.lse.fill_(float("nan"))
        cuda_lib.mla_decode_paged_noalloc(st.args)
        torch.cuda.synchronize()
        o, lse = to_np(st.o_lat), to_np(st.lse)
        ma, rl = errors(o, ref_o)
        assert ma <= amax and rl <= rl2, (call, ma, rl)
        assert np.abs(lse - ref_lse).max() <= amax, call


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_lib):
    import ctypes
    a = cuda_lib.DecodeArgs()
    for f in ("q_lat", "q_pe", "kv_cache", "block_table", "seq_lens", "o_lat", "lse"):
        setattr(a, f, 0x10000)
    a.B, a.s_q, a.H = 512, 2, 128
    a.d_c, a.d_r, a.page_size = 512, 64, 64
    a.num_pages, a.max_pages_per_seq = 1024, 64
    a.num_splits, a.softmax_scale = 16, 0.07       # 512*2*128*16 partial rows: 1 GiB of scratch
    assert cuda_lib.load().mla_decode_paged_noalloc(ctypes.byref(a), None) == 4


def test_noalloc_reports_device_status_through_its_accessor(cuda_lib):
    """A page id outside the cache is recorded in the built-in scratch's status
    word; mla_get_status_noalloc returns it once and clears it."""
    from head_latent_attention_06_b200.step import step_from_workload
    cuda_lib.mla_noalloc_init()
    assert cuda_lib.mla_get_status_noalloc() == 0
    w = make_workload(WorkloadSpec("na", B=2, H=128, s_q=1, lens=[130, 64], seed=22))
    st = step_from_workload(w)
    st.absorb()
    st._keep[2][0, 1] = 10_000                  # beyond the cache: skipped and reported
    cuda_lib.mla_decode_paged_noalloc(st.args)
    assert cuda_lib.mla_get_status_noalloc() == 7          # MLA_ERR_BAD_BLOCK_TABLE
    assert cuda_lib.mla_get_status_noalloc() == 0          # cleared by the read
    st._keep[2][0, 1] = int(w.block_table[0, 1])
    cuda_lib.mla_decode_paged_noalloc(st.args)
    assert cuda_lib.mla_get_status_noalloc() == 0
