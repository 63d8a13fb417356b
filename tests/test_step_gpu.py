"""GPU parity of mla_decode_step, the whole decode step in one call (the fused
step: query absorption, paged decode and value up-projection in one launch where
the shape allows), against the fp64 oracle and against the four-kernel sequence
(mla_absorb_q, mla_decode_paged, mla_combine_splits, mla_up_proj_v), which runs
the same tile arithmetic and so gives bit-identical outputs."""
import numpy as np
import pytest
import torch

from mla_inputs import WorkloadSpec, make_workload, preset
from parity_util import TOL, check_close, check_lse, oracle_of, report, to_np

pytestmark = pytest.mark.gpu


def _fused(cuda_lib, w, splits=0, fuse=1):
    from head_latent_attention_06_b200.step import fused_from_workload
    st = fused_from_workload(w, num_splits=splits, fuse=fuse)
    st.run()
    torch.cuda.synchronize()
    assert cuda_lib.mla_get_status(st.workspace) == 0
    return st


def _four(cuda_lib, w, splits=0):
    from head_latent_attention_06_b200.step import step_from_workload
    st = step_from_workload(w, num_splits=splits)
    st.run()
    torch.cuda.synchronize()
    assert cuda_lib.mla_get_status(st.workspace) == 0
    return st


CASES = [
    # H, s_q, causal, lens, kv
    (128, 1, False, [1, 63, 64, 65, 200, 1000, 4096, 77], "bf16"),
    (16, 1, False, [300, 5000, 1], "bf16"),
    (64, 2, True, [2, 64, 130, 777], "bf16"),
    (128, 1, False, [70, 129, 640], "q8_0"),
    (128, 1, False, [70, 129, 640], "q4_0"),
    (128, 4, True, [4, 100, 1000], "bf16"),
]


@pytest.mark.parametrize("H,s_q,causal,lens,kv", CASES)
def test_fused_step_matches_oracle_and_four_kernels(cuda_lib, H, s_q, causal, lens, kv):
    w = make_workload(WorkloadSpec("fs", B=len(lens), H=H, s_q=s_q, lens=lens, kv_dtype=kv, causal=causal,
                                   seed=51))
    st = _fused(cuda_lib, w, splits=1)        # one split: the fused launch
    assert st.launches == 1, st.launches
    ref = oracle_of(w, absorbed=True)
    res = {"o": check_close("o", to_np(st.out), ref["o"], kv)}
    check_lse(to_np(st.lse), ref["lse"], TOL[kv][0])
    report(f"fused step H={H} s_q={s_q} lens={lens} kv={kv}", res)
    four = _four(cuda_lib, w, splits=1)
    assert torch.equal(st.out, four.out) and torch.equal(st.lse, four.lse)


def test_fused_step_repeats(cuda_lib):
    """The flags are cleared by the last CTA of every launch: repeated calls on the
    same workspace (and replays of a captured graph) give the same output."""
    from head_latent_attention_06_b200.step import fused_from_workload
    w = make_workload(WorkloadSpec("fr", B=6, H=128, s_q=1, lens=[100, 2000, 64, 65, 1, 900], seed=52))
    st = fused_from_workload(w, num_splits=1, fuse=1)
    assert st.launches == 1
    st.run()
    torch.cuda.synchronize()
    first = st.out.clone()
    for _ in range(3):
        st.run()
    g = st.capture()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert cuda_lib.mla_get_status(st.workspace) == 0
    assert torch.equal(st.out, first)
    flags = st.workspace[256:512]
    assert int(flags.count_nonzero()) == 0


def test_step_falls_back_to_four_kernels(cuda_lib):
    """Shapes the fused launch does not take (several splits, an e4m3 cache) run the
    four kernels through the same call, against the oracle."""
    for spec, splits in ((WorkloadSpec("fb", B=2, H=16, s_q=1, lens=[20000, 3000], seed=53), 0),
                         (WorkloadSpec("fb8", B=2, H=128, s_q=2, lens=[500, 1500], kv_dtype="fp8", causal=True,
                                       seed=54), 0),
                         (WorkloadSpec("fbs", B=3, H=128, s_q=1, lens=[500, 1500, 64], seed=55), 3)):
        w = make_workload(spec)
        st = _fused(cuda_lib, w, splits)
        assert st.launches in (3, 4)
        ref = oracle_of(w, absorbed=True)
        check_close("o", to_np(st.out), ref["o"], spec.kv_dtype)


def test_fused_step_full_size_sampled(cuda_lib):
    """The V3 decode workload (64 x 4096 tokens, 128 heads) as one launch: sampled
    rows against the oracle, every row against the four kernels."""
    w = make_workload(preset("v3"))
    st = _fused(cuda_lib, w)
    assert st.launches == 1
    rows = [(b, 0) for b in (0, 31, 63)]
    ref = oracle_of(w, rows=rows, absorbed=True)
    bi = tuple(np.array(x) for x in zip(*rows))
    report("fused step v3 (sampled rows)", {"o": check_close("o", to_np(st.out)[bi], ref["o"][bi], "bf16")})
    assert torch.equal(st.out, _four(cuda_lib, w).out)


def test_fused_step_wait_limit_reports_and_recovers(cuda_lib):
    """With a 1 ns device wait limit the step's flag waits give up at once: the
    status word says so, no kernel hangs, and after zeroing the workspace and
    restoring the limit the next call is exact again."""
    from head_latent_attention_06_b200.step import fused_from_workload
    w = make_workload(WorkloadSpec("ft", B=8, H=128, s_q=1, lens=[3000] * 8, seed=56))
    st = fused_from_workload(w, num_splits=1, fuse=1)
    assert st.launches == 1
    cuda_lib.mla_set_device_wait_limit(1)
    try:
        st.run()
        torch.cuda.synchronize()
        status = cuda_lib.mla_get_status(st.workspace)
    finally:
        cuda_lib.mla_set_device_wait_limit(0)
    assert status in (0, 6)
    st.workspace.zero_()
    st.run()
    torch.cuda.synchronize()
    assert cuda_lib.mla_get_status(st.workspace) == 0
    assert torch.equal(st.out, _four(cuda_lib, w, splits=1).out)


def test_automatic_choice_of_one_launch(cuda_lib):
    """fuse = 0: one launch for a q8_0 or q4_0 cache whose grid covers at least half
    the SMs (where it measured faster than four chained launches); the four
    kernels for a bf16 cache, a small grid, or fuse = -1."""
    from head_latent_attention_06_b200.step import fused_from_workload
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    big, small = (sms + 3) // 4, max(1, sms // 8)
    for kv, B, fuse, want in (("q8_0", big, 0, 1), ("q4_0", big, 0, 1), ("q8_0", small, 0, 3),
                              ("bf16", big, 0, 3), ("q8_0", big, -1, 3), ("bf16", big, 1, 1)):
        w = make_workload(WorkloadSpec("fa", B=B, H=128, s_q=1, lens=[64] * B, kv_dtype=kv, seed=57))
        st = fused_from_workload(w, num_splits=1, fuse=fuse)
        assert st.launches == want, (kv, B, fuse, st.launches)


def test_fused_step_two_token_blocks_and_empty_sequences(cuda_lib):
    """More than 64 query tokens: the projection tiles and flags of a second token
    block (two of its 64 rows real, the rest past the end), and sequences with no
    cached token (o = 0, lse = -inf) inside the one launch."""
    B = 66
    lens = [0 if b % 17 == 5 else 64 + 37 * b for b in range(B)]
    w = make_workload(WorkloadSpec("f2b", B=B, H=32, s_q=1, lens=lens, seed=58))
    st = _fused(cuda_lib, w, splits=1)
    if st.launches != 1:
        pytest.skip(f"the device holds fewer than {B} CTA pairs of the fused kernel at once")
    rows = [(b, 0) for b in (0, 5, 22, 63, 64, 65)]
    ref = oracle_of(w, rows=rows, absorbed=True)
    bi = tuple(np.array(x) for x in zip(*rows))
    check_close("o", to_np(st.out)[bi], ref["o"][bi], "bf16")
    check_lse(to_np(st.lse)[bi], ref["lse"][bi], TOL["bf16"][0])
    assert torch.equal(st.out, _four(cuda_lib, w, splits=1).out)
