#!/usr/bin/env python
"""Benchmark of one MLA decode step (absorb -> paged decode -> combine -> up-project).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config v3] [--impl reference]

Prints one JSON line (rank 0).  The workload is the DeepSeek-V3-shaped decode
(batch 64, 128 heads, 4096 cached tokens per sequence, bf16 cache in 64-token
pages with a shuffled block table); other presets can be chosen with --config.
Under torchrun every rank runs its own batch (different seed, same shape): the
sequences are independent, so ranks exchange nothing on the data path and the
line reports weak scaling, timed on the device as the max over ranks.

Timing: the step is captured once in a CUDA graph (absorb, decode, combine,
up-projection); W untimed warm-up replays, then K replays, each bracketed by
CUDA events on the launching stream, with L2 flushed (a 256 MB write, then
a 256 MB read that leaves no dirty line behind) before each, outside the events.  The parts are then timed the same way one by one.
``value`` is cache GB/s of the whole step (all ranks);
``roofline`` is the decode kernel's own cache bytes over its event-timed
duration against the measured HBM copy bandwidth.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA decode cache GB/s, TFLOP/s & % of B200 roofline; tokens/s per step"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM bytes (read + write) of one decode launch from an ncu capture of the
# workload, recorded with the kernel's source file and the sha256 prefix of that
# file and the device headers it includes, as they were when the capture was
# taken: reported as the roofline's ``traffic`` only while they are unchanged.
MEASURED_TRAFFIC = {
    # ncu (dram__bytes_read.sum + dram__bytes_write.sum), one launch of the V3 workload
    "v3": (314_853_888, "decode_tc.cu", "37924f04a4a9e143"),
    # one launch of the fp8 workload
    "fp8": (774_229_504, "decode_f8.cu", "39ec40f7a33f3d1f"),
    # one launch of each long-context workload
    "long16": (607_507_200, "decode_tc.cu", "37924f04a4a9e143"),
    "long128": (608_263_168, "decode_tc.cu", "37924f04a4a9e143"),
    # one launch of the q8_0 and the q4_0 workloads (the same kernel file, its
    # blockwise instances)
    "q8": (173_468_672, "decode_tc.cu", "37924f04a4a9e143"),
    "q4": (97_926_656, "decode_tc.cu", "37924f04a4a9e143"),
    # both prefill kernels on one sequence of the chunked-prefill workload:
    # 1,148,841,984 bytes, times the 4 sequences of the full workload (traffic
    # grows with the sequences processed)
    "prefill": (4 * 1_148_841_984, "prefill.cu", "740bfda2cf634d5e"),
}
KERNEL_HEADERS = ("sm100.cuh", "common.cuh", "tma_host.cuh")


def kernel_source_digest(src_name: str) -> str:
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "head_latent_attention_06_b200", "csrc")
    for name in (src_name,) + KERNEL_HEADERS:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def decode_traffic(config: str):
    entry = MEASURED_TRAFFIC.get(config)
    if entry is None:
        return None
    nbytes, src_name, sha = entry
    return nbytes if kernel_source_digest(src_name) == sha else None


# Nominal B200 figures, the secondary denominators: HBM3e 7.7 TB/s (HGX), dense
# bf16/f16 tensor 2.25 PFLOP/s, dense fp8 4.5 PFLOP/s.
DATASHEET = {"hbm_gbs": 7700.0, "bf16_tflops": 2250.0, "fp8_tflops": 4500.0}


def datasheet_fracs(cache_bytes: float, flops: float, seconds: float, kv_dtype: str = "bf16") -> dict:
    """The decode's fractions of the nominal figures (the measured peaks are the
    primary denominators); the tensor figure is that of the MMA kind used."""
    tc = DATASHEET["fp8_tflops"] if kv_dtype == "fp8" else DATASHEET["bf16_tflops"]
    t_mem = cache_bytes / (DATASHEET["hbm_gbs"] * 1e9)
    t_tc = flops / (tc * 1e12)
    return {"hbm_gbs": DATASHEET["hbm_gbs"], "tensor_tflops": tc,
            "hbm_frac": round(t_mem / seconds, 4), "tensor_frac": round(t_tc / seconds, 4),
            "binding_frac": round(max(t_mem, t_tc) / seconds, 4)}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown CPU"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def tensor_peak(peaks: dict, kv_dtype: str):
    """Dense tensor peak (TFLOP/s) of the MMA kind the decode runs, and how it was
    obtained: bf16 x bf16 for a bf16 cache (the measured cuBLAS bf16 figure);
    e4m3 x e4m3 for an e4m3 cache: a measured fp8 figure if the peaks file has
    one, else the measured bf16 figure x 2, the ratio of the nominal dense
    figures (4.5 / 2.25 PFLOP/s)."""
    bf16 = float(peaks["bf16_tflops"])
    if kv_dtype != "fp8":
        return bf16, "bf16 x bf16 (measured cuBLAS bf16 GEMM)"
    if "fp8_tflops" in peaks:
        return float(peaks["fp8_tflops"]), "e4m3 x e4m3 (measured fp8 GEMM)"
    return 2.0 * bf16, "e4m3 x e4m3 (measured bf16 GEMM x 2, the nominal fp8 / bf16 ratio)"


def step_flops(lens, H, s_q):
    """Algorithmic decode FLOPs: 2 * (576 + 512) per (cached token, head, query)."""
    return sum(lens) * H * s_q * 2 * (576 + 512)


def proj_flops(n_tok, H):
    return 2 * (2 * n_tok * H * 128 * 512)


def shard_seed(base_seed: int, rank: int) -> int:
    """Each rank decodes its own batch: same shape, its own seed."""
    return base_seed + 1000 * rank


def whole_job_rate(world: int, bytes_per_rank: int, total_ms_max: float, steps: int) -> float:
    """Bytes of all ranks per second over the slowest rank's device time (GB/s)."""
    return world * bytes_per_rank * steps / (total_ms_max * 1e-3) / 1e9


def reduce_max(x: float) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class ClockSampler:
    """nvidia-smi samples during the timed region (SM clock, throttle reasons)."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        import tempfile
        self.path = os.path.join(tempfile.gettempdir(), f"mla_bench_clocks_rank{index}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def oracle_cpu_baseline(spec_name: str, budget_s: float = 12.0):
    """Times the fp64 oracle (absorbed form, the oracle's faster mode) on a bounded
    sample of the workload: whole sequences, all heads, until the budget is used.
    Returns (GB/s of cache processed, description, cores)."""
    import numpy as np
    import torch
    from mla_inputs import make_workload, preset
    import oracle
    from oracle import mla_oracle as om
    spec = preset(spec_name)
    w = make_workload(spec)
    inp = oracle.from_workload(w)
    from mla_inputs import row_bytes as row_bytes_of
    row_bytes = row_bytes_of(spec.kv_dtype)
    done_b, done_tokens, t0 = 0, 0, time.perf_counter()
    while done_b < w.B and time.perf_counter() - t0 < budget_s:
        om.decode_absorbed(inp, rows=[(done_b, i) for i in range(w.s_q)])
        done_tokens += w.lens[done_b]
        done_b += 1
    dt = time.perf_counter() - t0
    cores = torch.get_num_threads()
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        cores = max([d.get("num_threads", 0) for d in info] + [1])
    except Exception:
        pass
    gbs = done_tokens * row_bytes / dt / 1e9
    desc = (f"oracle decode_absorbed (fp64 numpy) on {done_b} of {w.B} sequences "
            f"({done_tokens} cached tokens, all {w.H} heads, {w.s_q} queries) in {dt:.2f} s "
            f"on {cpu_model()}")
    return gbs, desc, cores, dt


def oracle_nonabsorbed_sample(spec_name: str, budget_s: float = 3.0):
    """Times the oracle's non-absorbed form (K and V formed per head, the
    definition itself) on the heads of one query row that fit the budget, and
    extrapolates to the whole workload by cached tokens x heads.  The
    extrapolation is an estimate, labelled as such; the absorbed form above is
    the measured baseline."""
    from mla_inputs import make_workload, preset
    import oracle
    from oracle import mla_oracle as om
    spec = preset(spec_name)
    w = make_workload(spec)
    inp = oracle.from_workload(w)
    b, i = 0, w.s_q - 1
    n = inp.visible(b, i)
    heads, t0 = 0, time.perf_counter()
    while heads < w.H and time.perf_counter() - t0 < budget_s:
        om.decode_nonabsorbed(inp, rows=[(b, i)], heads=[heads])
        heads += 1
    dt = time.perf_counter() - t0
    us_per_token_head = dt * 1e6 / max(1, heads * n)
    work = sum(inp.visible(bb, ii) for bb in range(w.B) for ii in range(w.s_q)) * w.H
    return {"us_per_token_head": round(us_per_token_head, 5),
            "extrapolated_full_s": float(f"{us_per_token_head * work * 1e-6:.4g}"),
            "sample": f"oracle decode_nonabsorbed (fp64 numpy), sequence 0 query {i} "
                      f"({n} cached tokens), {heads} of {w.H} heads in {dt:.2f} s; "
                      f"full-workload time extrapolated by cached tokens x heads"}


def run_reference(args):
    """The oracle timed on the host cores as the reference arm (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    vals, descs, cores = [], [], 1
    for _ in range(args.warmup):
        oracle_cpu_baseline(args.config, budget_s=2.0)
    for _ in range(args.steps):
        v, d, cores, _ = oracle_cpu_baseline(args.config, budget_s=max(2.0, 40.0 / max(1, args.steps)))
        vals.append(v)
        descs.append(d)
    value = statistics.mean(vals)
    line = {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": _config_dict(args.config, None),
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores,
                             "kind": "oracle", "sample": descs[-1]},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


WRITE_METRIC = "MLA cache write GB/s (latent + RoPE key into the paged cache) & % of HBM roofline"


def run_write_kv(args):
    """Times mla_write_kv for the new tokens of one decode step of the workload:
    hidden states of width d_h -> latent c = W_DKV h and rotated RoPE key -> their
    rows of the paged cache (bf16, e4m3 with per-row scales, or q8_0 / q4_0 with
    per-block scales).  One GPU; the
    two launches are replayed from a CUDA graph with L2 flushed before each."""
    import torch
    import head_latent_attention_06_b200 as mla
    from mla_inputs import make_workload, preset
    torch.cuda.set_device(0)
    mla.load()
    spec = preset(args.config)
    w = make_workload(spec)
    d_h = args.d_h
    g = torch.Generator().manual_seed(spec.seed + 1000)
    h = torch.randn(w.B, w.s_q, d_h, generator=g).to(torch.bfloat16).cuda()
    w_dkv = (torch.randn(576, d_h, generator=g) / d_h ** 0.5).to(torch.bfloat16).cuda()
    kv = w.kv_cache.cuda()
    sc = None if w.kv_scale is None else w.kv_scale.cuda()
    bt, sl = w.block_table.cuda(), w.seq_lens.cuda()
    a = mla.make_write_kv_args(h=h, w_dkv=w_dkv, kv_cache=kv, kv_scale=sc, block_table=bt, seq_lens=sl)
    ws = mla.alloc_workspace(a)
    stream = torch.cuda.current_stream()
    mla.mla_write_kv(a)                      # outside capture: one-time host set-up
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        mla.mla_write_kv(a)
    flush_w = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    flush_r = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    for _ in range(max(3, args.warmup)):
        flush_w.zero_()
        torch.sum(flush_r)
        graph.replay()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    with ClockSampler(0) as clk:
        for k in range(args.steps):
            flush_w.zero_()
            torch.sum(flush_r)
            evs[k][0].record(stream)
            graph.replay()
            evs[k][1].record(stream)
        torch.cuda.synchronize()
    assert mla.mla_get_status(ws) == 0
    ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    n_tok = w.B * w.s_q
    from mla_inputs import row_bytes as row_bytes_of
    algo_bytes = 576 * d_h * 2 + n_tok * d_h * 2 + n_tok * row_bytes_of(spec.kv_dtype)
    gbs = algo_bytes / (ms * 1e-3) / 1e9
    peaks, peak_kind = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    cfg = _config_dict(args.config, w)
    cfg.update({"path": "write_kv", "d_h": d_h, "new_tokens": n_tok})
    line = {"metric": WRITE_METRIC, "value": round(gbs, 2), "unit": "GB/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 in, fp32 accumulate, " + {"bf16": "bf16", "fp8": "e4m3", "q8_0": "q8_0",
                                                      "q4_0": "q4_0"}[spec.kv_dtype]
                     + " cache",
            "data": "synthetic (seeded N(0,1) hidden states, N(0,1/d_h) weights)", "config": cfg,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(gbs / hbm, 4), "traffic": None,
                         "peak_kind": f"{peak_kind} HBM copy bandwidth",
                         "kernel": "mla_write_kv (down-projection + finish)",
                         "bytes_per_launch": algo_bytes},
            "gpu_launches": 2 * args.steps, "clocks": clk.summary()}
    print(json.dumps(line), flush=True)
    return 0


PREFILL_METRIC = "MLA chunked-prefill TFLOP/s (explicit K/V form) & % of tensor roofline; tokens/s"


def prefill_flops(lens, H, s_q, causal):
    """Algorithmic FLOPs of the explicit form: per (cached token, head) the two
    up-projections k = W_UK c and v = W_UV c, 2 * 2 * 128 * 512; per (query,
    visible token, head) the 192-wide score and the 128-wide value sum,
    2 * (192 + 128)."""
    up = sum(lens) * H * 2 * 2 * 128 * 512
    vis = 0
    for L in lens:
        if causal:
            vis += s_q * (L - s_q) + s_q * (s_q + 1) // 2
        else:
            vis += s_q * L
    return up + vis * H * 2 * (192 + 128), up


def run_prefill(args):
    """Times mla_prefill on a chunked-prefill workload (s_q new tokens per
    sequence on top of a cached prefix, causal): the per-head key / value
    up-projection and the FlashAttention forward, replayed from a CUDA graph with
    L2 flushed before each call.  The same chunk through the absorbed kernels is
    timed beside it (the form the decode uses), and end to end with the queries
    copied in from pinned host memory and the output copied back."""
    import torch
    import head_latent_attention_06_b200 as mla
    from head_latent_attention_06_b200.step import prefill_from_workload, step_from_workload
    from mla_inputs import make_workload, preset
    torch.cuda.set_device(0)
    mla.load()
    spec = preset(args.config)
    w = make_workload(spec)
    st = prefill_from_workload(w)
    stream = torch.cuda.current_stream()
    st.run()                                 # outside capture: one-time host set-up
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        st.run()
    flush_w = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    flush_r = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device="cuda")

    def timed_loop(g, n):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
        for k in range(n):
            flush_w.zero_()
            torch.sum(flush_r)
            evs[k][0].record(stream)
            g.replay()
            evs[k][1].record(stream)
        return evs

    timed_loop(graph, max(3, args.warmup))
    torch.cuda.synchronize()
    assert mla.mla_get_status(st.workspace) == 0
    with ClockSampler(0) as clk:
        evs = timed_loop(graph, args.steps)
        torch.cuda.synchronize()
    assert mla.mla_get_status(st.workspace) == 0
    ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps

    absorbed_ms = None
    if w.s_q <= 1024:
        dec = step_from_workload(w)
        g_dec = dec.capture()
        timed_loop(g_dec, 3)
        torch.cuda.synchronize()
        n_dec = max(3, min(args.steps, 50))
        ev = timed_loop(g_dec, n_dec)
        torch.cuda.synchronize()
        assert mla.mla_get_status(dec.workspace) == 0
        absorbed_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / n_dec
        del dec, g_dec

    # end to end: queries, block table and lengths from pinned host memory, the
    # output back to pinned host memory, every call
    h_in = (w.q_nope.pin_memory(), w.q_pe.pin_memory(), w.block_table.pin_memory(), w.seq_lens.pin_memory())
    d_in = (st._keep[0], st._keep[1], st._keep[5], st._keep[6])
    h_out = torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory()
    n_e2e = max(3, min(args.steps, 50))
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for rep in range(2):
        n = 3 if rep == 0 else n_e2e
        torch.cuda.synchronize()
        t0.record(stream)
        for _ in range(n):
            for d, h in zip(d_in, h_in):
                d.copy_(h, non_blocking=True)
            st.run()
            h_out.copy_(st.out, non_blocking=True)
        t1.record(stream)
        torch.cuda.synchronize()
    e2e_ms = t0.elapsed_time(t1) / n_e2e
    assert torch.equal(h_out, st.out.cpu())
    h2d = sum(t.numel() * t.element_size() for t in h_in)
    d2h = h_out.numel() * h_out.element_size()

    flops, up_flops = prefill_flops(w.lens, w.H, w.s_q, w.causal)
    tflops = flops / (ms * 1e-3) / 1e12
    peaks, peak_kind = load_peaks()
    tc_peak, tc_kind = tensor_peak(peaks, "bf16")
    n_tok = w.B * w.s_q
    cfg = _config_dict(args.config, w)
    cfg.update({"path": "prefill", "form": "explicit: per-head K = [W_UK c ; k_pe], V = W_UV c, "
                                           "then FlashAttention forward"})
    line = {"metric": PREFILL_METRIC, "value": round(tflops, 2), "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 (fp32 accumulate; K, V and P in bf16)",
            "data": "synthetic (seeded, N(0,1) activations and cache, N(0,1/512) weights)", "config": cfg,
            "tokens_per_s": round(n_tok / (ms * 1e-3), 1),
            "flops_per_step": flops, "kv_up_flops_per_step": up_flops,
            "absorbed_form_ms": None if absorbed_ms is None else round(absorbed_ms, 4),
            "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "peak": tc_peak, "unit": "TFLOP/s",
                         "frac": round(tflops / tc_peak, 4), "traffic": decode_traffic(args.config),
                         "peak_kind": f"{peak_kind}: {tc_kind}",
                         "kernel": "mla_prefill (kv_up_kernel + prefill_attn_kernel, one call)"},
            "e2e": {"value": round(flops / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 5)},
            "gpu_launches": 2 * args.steps, "clocks": clk.summary()}
    print(json.dumps(line), flush=True)
    return 0


def _config_dict(name, w, splits=None):
    from mla_inputs import preset
    s = preset(name)
    d = {"workload": f"{name}: {s.note}", "B": s.B, "H": s.H, "s_q": s.s_q,
         "kv_cache": s.kv_dtype, "page_size": 64, "d_c": 512, "d_r": 64,
         "causal": s.causal, "l2": "flushed between timed steps (256 MB write, then 256 MB read)"}
    if w is not None:
        d["cached_tokens"] = sum(w.lens)
    if splits is not None:
        d["splits"] = splits
    return d


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    # enough steps that the timed region lasts about a second (the clock sampler
    # reads every 200 ms)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="v3")
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--splits", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--path", default="decode", choices=["decode", "write_kv", "prefill"],
                    help="decode: the decode step (default); write_kv: the cache write of its new "
                         "tokens; prefill: the explicit-form chunked prefill (--config prefill)")
    ap.add_argument("--d-h", dest="d_h", type=int, default=7168, help="hidden width for --path write_kv")
    args = ap.parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.path == "write_kv":
        return run_write_kv(args)
    if args.path == "prefill":
        return run_prefill(args)

    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    import head_latent_attention_06_b200 as mla
    from head_latent_attention_06_b200.step import step_from_workload
    from mla_inputs import make_workload, preset
    mla.load()

    spec = preset(args.config)
    spec = spec.with_(seed=shard_seed(spec.seed, rank))
    w = make_workload(spec)
    st = step_from_workload(w, num_splits=args.splits)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    # L2 flush: write a 256 MB buffer (twice the 126 MB L2), then read another
    # one.  The write evicts everything the step left in L2; the read then
    # replaces the written (dirty) lines with clean ones, so that the timed step
    # does not pay for writing back the flush buffer itself.
    flush_w = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    flush_r = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device="cuda")

    def flush_l2():
        flush_w.zero_()
        torch.sum(flush_r)
    cache_bytes = w.cache_bytes()
    flops = step_flops(w.lens, w.H, w.s_q)

    # The step and its parts are replayed from CUDA graphs: one host call issues
    # all launches of a part, so the device never waits on the host and the
    # events measure device time only.
    g_step = st.capture()
    g_absorb = st.capture(st.absorb)
    g_decode = st.capture(lambda: mla.mla_decode_paged(st.args))
    g_tail = st.capture(lambda: (mla.mla_combine_splits(st.args), st.up_project()))
    # the same step through mla_decode_step (one launch where the shape allows)
    from head_latent_attention_06_b200.step import FusedStep
    fst = FusedStep(q_nope=st.q_nope, q_pe=st.q_pe, w_uk=st.w_uk, w_uv=st.w_uv, kv_cache=st._keep[0],
                    kv_scale=st._keep[1], block_table=st._keep[2], seq_lens=st._keep[3], causal=w.causal,
                    softmax_scale=w.softmax_scale, num_splits=args.splits,
                    max_seq_len=max(w.lens) if w.lens else 0, fuse=1)
    g_fused = fst.capture()

    def timed(graph, ev):
        flush_l2()
        ev[0].record(stream)
        graph.replay()
        ev[1].record(stream)

    for _ in range(max(3, args.warmup)):
        flush_l2()
        g_step.replay()
    torch.cuda.synchronize()
    assert mla.mla_get_status(st.workspace) == 0

    def new_events():
        return [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]

    evs, ev_abs, ev_dec, ev_tail, ev_fused = new_events(), new_events(), new_events(), new_events(), new_events()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    # The clock record covers both timed loops: the steps, then the parts one by
    # one (each after an L2 flush), whose decode figure is the roofline's.
    with ClockSampler(local) as clk:
        for k in range(args.steps):
            timed(g_step, evs[k])
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        for k in range(args.steps):
            timed(g_absorb, ev_abs[k])
            timed(g_decode, ev_dec[k])
            timed(g_tail, ev_tail[k])
        torch.cuda.synchronize()
        for k in range(args.steps):
            timed(g_fused, ev_fused[k])
        torch.cuda.synchronize()
    assert mla.mla_get_status(st.workspace) == 0
    assert mla.mla_get_status(fst.workspace) == 0
    g_step.replay()
    torch.cuda.synchronize()
    fused_same = bool(torch.equal(fst.out, st.out))
    ms = lambda ev: [e[0].elapsed_time(e[1]) for e in ev]
    step_ms, dec_ms, absorb_ms, tail_ms, fused_ms = ms(evs), ms(ev_dec), ms(ev_abs), ms(ev_tail), ms(ev_fused)
    total_ms = reduce_max(sum(step_ms))
    dec_avg_ms = reduce_max(sum(dec_ms) / len(dec_ms))
    ms_per_step = total_ms / args.steps

    # End to end through the public API, the way a serving loop drives it: every
    # step's queries, block table and lengths come from pinned host memory and its
    # output goes back to pinned host memory.  Two sets of step buffers (the cache
    # and weights are shared model state), each with a CUDA graph of its whole
    # step (host->device copies, the four library calls, the device->host copy),
    # replayed alternately on two streams, so that one step's copies overlap the
    # other step's decode and the host issues one call per step.  The cache
    # (302 MB at V3) is larger than L2, so no flush is needed between these steps.
    from head_latent_attention_06_b200.step import DecodeStep
    st2 = DecodeStep(q_nope=torch.empty_like(st.q_nope), q_pe=torch.empty_like(st.q_pe), w_uk=st.w_uk,
                     w_uv=st.w_uv, kv_cache=st._keep[0], kv_scale=st._keep[1],
                     block_table=torch.empty_like(st._keep[2]), seq_lens=torch.empty_like(st._keep[3]),
                     causal=w.causal, softmax_scale=w.softmax_scale, num_splits=st.num_splits,
                     max_seq_len=max(w.lens) if w.lens else 0)
    sts = [st, st2]
    h_in = [(w.q_nope.pin_memory(), w.q_pe.pin_memory(), w.block_table.pin_memory(), w.seq_lens.pin_memory())
            for _ in range(2)]
    h_out = [torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in h_in[0])
    d2h = h_out[0].numel() * h_out[0].element_size()

    def e2e_step(x, hi, ho):
        x.q_nope.copy_(hi[0], non_blocking=True)
        x.q_pe.copy_(hi[1], non_blocking=True)
        x._keep[2].copy_(hi[2], non_blocking=True)
        x._keep[3].copy_(hi[3], non_blocking=True)
        x.run()
        ho.copy_(x.out, non_blocking=True)

    e2e_graphs = []
    for i, x in enumerate(sts):
        e2e_step(x, h_in[i], h_out[i])         # outside capture: one-time host set-up
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            e2e_step(x, h_in[i], h_out[i])
        e2e_graphs.append(g)
    e2e_streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def e2e_run(n):
        for s2 in e2e_streams:
            s2.wait_stream(stream)
        for k in range(n):
            with torch.cuda.stream(e2e_streams[k % 2]):
                e2e_graphs[k % 2].replay()
        for s2 in e2e_streams:
            stream.wait_stream(s2)

    e2e_run(max(3, args.warmup))
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t_start.record(stream)
    e2e_run(args.steps)
    t_end.record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(t_start.elapsed_time(t_end)) / args.steps
    for i, x in enumerate(sts):
        assert mla.mla_get_status(x.workspace) == 0
        assert torch.equal(h_out[i], st.out.cpu())   # both buffer sets decode the same step

    peaks, peak_kind = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    value = whole_job_rate(world, cache_bytes, total_ms, args.steps)
    dec_gbs = cache_bytes / (dec_avg_ms * 1e-3) / 1e9
    dec_tflops = flops / (dec_avg_ms * 1e-3) / 1e12
    t_mem = cache_bytes / (hbm * 1e9)
    tc_peak, tc_peak_kind = tensor_peak(peaks, spec.kv_dtype)
    t_tc = flops / (tc_peak * 1e12)
    tensor_bound = t_tc > t_mem
    # absorb, decode, up-projection, and the merge unless one split was used
    launches_per_step = 3 + (1 if st.num_splits != 1 else 0)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": {"fp8": "e4m3 cache, e4m3 x e4m3 MMA (two-term operand split)",
                  "q8_0": "q8_0 cache (int8 codes x fp16 block scales formed in bf16), bf16 MMA",
                  "q4_0": "q4_0 cache (4-bit codes x fp16 block scales formed in bf16), bf16 MMA",
                  "bf16": "bf16"}[spec.kv_dtype],
        "data": "synthetic (seeded, N(0,1) activations and cache, N(0,1/512) weights)",
        "config": _config_dict(args.config, w, st.num_splits),
        "tflops": round(world * (flops + proj_flops(w.n_tok, w.H)) / (ms_per_step * 1e-3) / 1e12, 2),
        "tokens_per_s": round(world * w.n_tok / (ms_per_step * 1e-3), 1),
        "decode_us": round(dec_avg_ms * 1e3, 2),
        "absorb_us": round(1e3 * sum(absorb_ms) / len(absorb_ms), 2),
        "combine_up_proj_us": round(1e3 * sum(tail_ms) / len(tail_ms), 2),
        # mla_decode_step with fuse = 1: the same step in one call (one launch
        # where the shape allows), timed the same way; its output equals the
        # four-kernel step's bit for bit
        "fused_step": {"us": round(1e3 * reduce_max(sum(fused_ms)) / len(fused_ms), 2),
                       "launches": fst.launches, "same_output": fused_same},
        "roofline": {
            # the binding side: cache bytes at the HBM copy bandwidth, or the
            # algorithmic FLOPs at the tensor peak of the MMA kind used
            **({"bound": "tensor", "achieved": round(dec_tflops, 1), "peak": tc_peak, "unit": "TFLOP/s",
                "frac": round(dec_tflops / tc_peak, 4), "peak_kind": f"{peak_kind}: {tc_peak_kind}"}
               if tensor_bound else
               {"bound": "hbm", "achieved": round(dec_gbs, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(dec_gbs / hbm, 4), "peak_kind": f"{peak_kind} HBM copy bandwidth"}),
            "traffic": decode_traffic(args.config),
            "kernel": "mla_decode_paged",
            "hbm": {"achieved_gbs": round(dec_gbs, 1), "peak_gbs": hbm, "frac": round(dec_gbs / hbm, 4)},
            "tensor": {"achieved_tflops": round(dec_tflops, 1), "peak_tflops": tc_peak,
                       "peak_kind": tc_peak_kind, "frac": round(dec_tflops / tc_peak, 4)},
            "binding_roofline_frac": round(max(t_mem, t_tc) / (dec_avg_ms * 1e-3), 4),
            "datasheet": datasheet_fracs(cache_bytes, flops, dec_avg_ms * 1e-3, spec.kv_dtype),
        },
        "cached_tokens_per_s": round(world * sum(w.lens) / (dec_avg_ms * 1e-3), 1),
        "e2e": {"value": round(world * cache_bytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 5),
                "pipeline": "two step buffer sets, one CUDA graph each (copies + step), replayed "
                            "alternately on two streams; host copies overlap the other step's decode"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc, cores, _ = oracle_cpu_baseline(args.config)
        line["cpu_baseline"] = {"value": round(v, 4), "unit": "GB/s", "cores": cores,
                                "kind": "oracle", "sample": desc,
                                "nonabsorbed": oracle_nonabsorbed_sample(args.config)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
