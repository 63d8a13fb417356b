"""One MLA attention step through the C ABI.

``DecodeStep``: absorb -> paged decode -> combine -> up-project (the absorbed
form); it owns the intermediate device buffers (q_lat, o_lat, lse, out and the
workspace) and replays the four calls on the current stream.  ``FusedStep``: the
same step through ``mla_decode_step`` (one call; one launch where the shape
allows).  ``PrefillStep``: the explicit form for long chunks of new tokens (one
call, two kernels).  None does arithmetic of its own.
"""

from __future__ import annotations

import torch

from . import (D_C, D_N, D_V, alloc_workspace, make_decode_args, make_prefill_args, make_step_args,
               mla_absorb_q, mla_combine_splits, mla_decode_num_splits, mla_decode_paged,
               mla_decode_step, mla_decode_step_launches, mla_prefill, mla_up_proj_v)


class DecodeStep:
    def __init__(self, *, q_nope, q_pe, w_uk, w_uv, kv_cache, kv_scale, block_table, seq_lens,
                 causal, softmax_scale, num_splits=0, max_seq_len=0, out=None):
        B, s_q, H, _ = q_nope.shape
        dev = q_nope.device
        self.B, self.s_q, self.H = B, s_q, H
        self.q_nope, self.q_pe, self.w_uk, self.w_uv = q_nope, q_pe, w_uk, w_uv
        self.q_lat = torch.empty(B, s_q, H, D_C, dtype=torch.bfloat16, device=dev)
        self.o_lat = torch.empty(B, s_q, H, D_C, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(B, s_q, H, dtype=torch.float32, device=dev)
        self.out = out if out is not None else torch.empty(B, s_q, H, D_V, dtype=torch.bfloat16,
                                                           device=dev)
        self.args = make_decode_args(q_lat=self.q_lat, q_pe=q_pe, kv_cache=kv_cache,
                                     kv_scale=kv_scale, block_table=block_table,
                                     seq_lens=seq_lens, o_lat=self.o_lat, lse=self.lse,
                                     causal=causal, softmax_scale=softmax_scale,
                                     num_splits=num_splits, max_seq_len=max_seq_len)
        self.workspace = alloc_workspace(self.args, device=dev)
        self.num_splits = mla_decode_num_splits(self.args)
        self._keep = (kv_cache, kv_scale, block_table, seq_lens)

    def absorb(self, stream=None):
        n_tok = self.B * self.s_q
        mla_absorb_q(self.q_nope.view(n_tok, self.H, D_N), self.w_uk,
                     self.q_lat.view(n_tok, self.H, D_C), stream)

    def attend(self, stream=None):
        mla_decode_paged(self.args, stream)
        mla_combine_splits(self.args, stream)

    def up_project(self, stream=None):
        n_tok = self.B * self.s_q
        mla_up_proj_v(self.o_lat.view(n_tok, self.H, D_C), self.w_uv,
                      self.out.view(n_tok, self.H, D_V), stream)

    def run(self, stream=None):
        self.absorb(stream)
        self.attend(stream)
        self.up_project(stream)
        return self.out

    def capture(self, fn=None):
        """Records ``fn`` (default: the whole step) into a CUDA graph and returns
        it; ``graph.replay()`` then issues all of its launches with one host call.
        The step allocates nothing, so the graph stays valid while the buffers
        (and the arguments captured in it) are unchanged."""
        fn = fn or self.run
        fn()                       # first call outside capture: one-time host setup
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        return g


def step_from_workload(w, device="cuda", num_splits=0):
    """Copy a ``mla_inputs.Workload`` to the device and build its ``DecodeStep``."""
    d = lambda t: None if t is None else t.to(device, non_blocking=False).contiguous()
    return DecodeStep(q_nope=d(w.q_nope), q_pe=d(w.q_pe), w_uk=d(w.w_uk), w_uv=d(w.w_uv),
                      kv_cache=d(w.kv_cache), kv_scale=d(w.kv_scale),
                      block_table=d(w.block_table), seq_lens=d(w.seq_lens), causal=w.causal,
                      softmax_scale=w.softmax_scale, num_splits=num_splits,
                      max_seq_len=max(w.lens) if w.lens else 0)


class FusedStep:
    """The decode step through one ``mla_decode_step`` call: owns out, lse and the
    workspace (which holds q_lat, o_lat and the step's flags)."""

    def __init__(self, *, q_nope, q_pe, w_uk, w_uv, kv_cache, kv_scale, block_table, seq_lens,
                 causal, softmax_scale, num_splits=0, max_seq_len=0, out=None, fuse=0):
        B, s_q, H, _ = q_nope.shape
        dev = q_nope.device
        self.B, self.s_q, self.H = B, s_q, H
        self.lse = torch.empty(B, s_q, H, dtype=torch.float32, device=dev)
        self.out = out if out is not None else torch.empty(B, s_q, H, D_V, dtype=torch.bfloat16,
                                                           device=dev)
        self.args = make_step_args(q_nope=q_nope, q_pe=q_pe, w_uk=w_uk, w_uv=w_uv, kv_cache=kv_cache,
                                   kv_scale=kv_scale, block_table=block_table, seq_lens=seq_lens,
                                   out=self.out, lse=self.lse, causal=causal,
                                   softmax_scale=softmax_scale, num_splits=num_splits,
                                   max_seq_len=max_seq_len, fuse=fuse)
        self.workspace = alloc_workspace(self.args, device=dev)
        self.launches = mla_decode_step_launches(self.args)
        self._keep = (q_nope, q_pe, w_uk, w_uv, kv_cache, kv_scale, block_table, seq_lens)

    def run(self, stream=None):
        mla_decode_step(self.args, stream)
        return self.out

    def capture(self):
        """One CUDA graph of the step (see ``DecodeStep.capture``)."""
        self.run()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.run()
        return g


def fused_from_workload(w, device="cuda", num_splits=0, fuse=0):
    """Copy a ``mla_inputs.Workload`` to the device and build its ``FusedStep``."""
    d = lambda t: None if t is None else t.to(device, non_blocking=False).contiguous()
    return FusedStep(q_nope=d(w.q_nope), q_pe=d(w.q_pe), w_uk=d(w.w_uk), w_uv=d(w.w_uv),
                     kv_cache=d(w.kv_cache), kv_scale=d(w.kv_scale),
                     block_table=d(w.block_table), seq_lens=d(w.seq_lens), causal=w.causal,
                     softmax_scale=w.softmax_scale, num_splits=num_splits,
                     max_seq_len=max(w.lens) if w.lens else 0, fuse=fuse)


class PrefillStep:
    """Explicit-form attention of s_q new tokens per sequence over the paged bf16
    cache: owns out, lse and the workspace (the per-head keys and values)."""

    def __init__(self, *, q_nope, q_pe, w_uk, w_uv, kv_cache, block_table, seq_lens, causal,
                 softmax_scale, max_seq_len, out=None):
        B, s_q, H, _ = q_nope.shape
        dev = q_nope.device
        self.B, self.s_q, self.H = B, s_q, H
        self.lse = torch.empty(B, s_q, H, dtype=torch.float32, device=dev)
        self.out = out if out is not None else torch.empty(B, s_q, H, D_V, dtype=torch.bfloat16,
                                                           device=dev)
        self.args = make_prefill_args(q_nope=q_nope, q_pe=q_pe, w_uk=w_uk, w_uv=w_uv,
                                      kv_cache=kv_cache, block_table=block_table,
                                      seq_lens=seq_lens, out=self.out, lse=self.lse,
                                      max_seq_len=max_seq_len, causal=causal,
                                      softmax_scale=softmax_scale)
        self.workspace = alloc_workspace(self.args, device=dev)
        self._keep = (q_nope, q_pe, w_uk, w_uv, kv_cache, block_table, seq_lens)

    def run(self, stream=None):
        mla_prefill(self.args, stream)
        return self.out


def prefill_from_workload(w, device="cuda", max_seq_len=None):
    """Copy a bf16-cache ``mla_inputs.Workload`` to the device and build its
    ``PrefillStep``."""
    d = lambda t: t.to(device, non_blocking=False).contiguous()
    return PrefillStep(q_nope=d(w.q_nope), q_pe=d(w.q_pe), w_uk=d(w.w_uk), w_uv=d(w.w_uv),
                       kv_cache=d(w.kv_cache), block_table=d(w.block_table),
                       seq_lens=d(w.seq_lens), causal=w.causal, softmax_scale=w.softmax_scale,
                       max_seq_len=max_seq_len or max(max(w.lens), w.spec.s_q))
