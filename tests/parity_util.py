"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (final output o, bf16 out, fp32 accumulation): bf16 cache max-abs
<= 2e-2 and relative L2 <= 1e-2; fp8 cache 6e-2 / 3e-2.  The same bounds are
applied to o_lat; lse is compared with an absolute bound of 2e-2 (bf16 cache)
or 6e-2 (fp8 cache) since it is a log of a sum whose terms carry the same
relative error as the scores.
"""

import numpy as np
import torch

import oracle
from oracle import mla_oracle as om

# q8_0: each value is formed in bf16 from its code and block scale, so the bf16
# cache's bounds apply (against the oracle's exact dequantised values)
TOL = {"bf16": (2e-2, 1e-2), "fp8": (6e-2, 3e-2), "q8_0": (2e-2, 1e-2), "q4_0": (2e-2, 1e-2)}


def errors(got: np.ndarray, ref: np.ndarray):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = got - ref
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    nrm = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(d) / nrm) if nrm > 0 else float(np.linalg.norm(d))
    return max_abs, rel


def check_lse(got, ref, tol):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    inf = np.isneginf(ref)
    assert np.array_equal(inf, np.isneginf(got)), "empty rows must give lse = -inf"
    if (~inf).any():
        assert np.abs(got[~inf] - ref[~inf]).max() <= tol


def check_close(name, got, ref, kv, rows=None):
    """rows: optional boolean/index selection (sampled rows) applied to both."""
    amax, rl2 = TOL[kv]
    if rows is not None:
        got, ref = got[rows], ref[rows]
    ma, rl = errors(got, ref)
    assert ma <= amax and rl <= rl2, f"{name}: max_abs {ma:.3e} (<= {amax}), rel_l2 {rl:.3e} (<= {rl2})"
    return ma, rl


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def compare_step(step, w, ref, rows=None):
    """Compare a finished DecodeStep against an oracle result dict."""
    kv = w.spec.kv_dtype
    o = to_np(step.out)
    o_lat = to_np(step.o_lat)
    lse = to_np(step.lse)
    if rows is None:
        sel = (slice(None),) * 2
        res = {
            "o": check_close("o", o, ref["o"], kv),
            "o_lat": check_close("o_lat", o_lat, ref["o_lat"], kv),
        }
        check_lse(lse, ref["lse"], TOL[kv][0])
    else:
        bi = tuple(np.array(x) for x in zip(*rows))
        res = {
            "o": check_close("o", o[bi], ref["o"][bi], kv),
            "o_lat": check_close("o_lat", o_lat[bi], ref["o_lat"][bi], kv),
        }
        check_lse(lse[bi], ref["lse"][bi], TOL[kv][0])
    return res


def report(label, res):
    """Appends the achieved errors of one comparison as a JSON line to the file
    named by MLA_PARITY_REPORT (nothing when it is unset)."""
    import json
    import os
    path = os.environ.get("MLA_PARITY_REPORT")
    if not path:
        return
    line = {"case": label}
    for key, (ma, rl) in res.items():
        line[key] = {"max_abs": ma, "rel_l2": rl}
    with open(path, "a") as f:
        f.write(json.dumps(line) + "\n")


def oracle_of(w, rows=None, absorbed=False, heads=None):
    inp = oracle.from_workload(w)
    fn = om.decode_absorbed if absorbed else om.decode_nonabsorbed
    return fn(inp, rows=rows, heads=heads)
