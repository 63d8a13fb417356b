"""fp64 CPU oracle for MLA decode over a paged latent KV cache.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code with
the CUDA library (``head_latent_attention_06_b200``) and never imports it.

What it follows (page titles and sections of the pages this method comes from):

* "MLA: Multi-Head Latent Attention — DeepSeek-AI Explained", section
  "Architecture": the cache holds the latent ``c_t`` (width d_c); keys and values
  are its up-projections ``k_t = W_UK c_t`` and ``v_t = W_UV c_t``.
* snowgate thread 35, replies on the 576-value latent record: the latent (512)
  is stored beside a decoupled RoPE key (64) shared by every head; the RoPE slice
  is handled apart from the up-projection.
* nnets.ru "Как технология MLA ...", section "Суть MLA": the weight-absorbing
  trick folds W_UK into the query and W_UV into the output side, so the full K
  and V are never formed.  ``decode_absorbed`` states that form.
* Standard softmax attention with a log-sum-exp output; split partials merge by
  the log-sum-exp identity (``combine_splits``).

Readings taken where the pages are silent:
RoPE is already applied to the cached ``k_pe`` and to ``q_pe`` (the kernel
rotates nothing); the softmax scale is 1/sqrt(qk_nope + rope) = 1/sqrt(192);
``W_UK[h]`` and ``W_UV[h]`` are the per-head [128 x 512] slices; with causal
decoding the s_q new tokens are the last s_q cached positions and query i sees
positions 0 .. L - s_q + i; lse is a natural logarithm.

Pinned by ``tests/test_oracle_pins.py`` (closed forms, a library attention
routine, invariants); no function here is "parity unpinned".
"""

from __future__ import annotations

import math
from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np

PAGE = 64
D_C = 512
D_R = 64
Q8_BLOCK = 32


# ----------------------------------------------------------------------------
# Storage formats, decoded from their bit definitions
# ----------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 is the upper half of an IEEE binary32: shift the 16 bits up."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def e4m3fn_to_f64(bits: np.ndarray) -> np.ndarray:
    """OCP FP8 E4M3 ("fn": finite, no infinities): 1 sign, 4 exponent (bias 7),
    3 mantissa bits; exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN."""
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    sub = (m / 8.0) * 2.0 ** -6
    v = np.where(e == 0, sub, normal) * sign
    return np.where((e == 15) & (m == 7), np.nan, v)


def f16_to_f64(bits: np.ndarray) -> np.ndarray:
    """IEEE binary16: 1 sign, 5 exponent (bias 15), 10 mantissa bits; exponent 0
    is subnormal (m/1024 * 2^-14); exponent 31 is inf (m = 0) or NaN."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.int64)
    sign = np.where(b & 0x8000, -1.0, 1.0)
    e = (b >> 10) & 0x1F
    m = (b & 0x3FF).astype(np.float64)
    normal = (1.0 + m / 1024.0) * np.exp2(e.astype(np.float64) - 15.0)
    sub = (m / 1024.0) * 2.0 ** -14
    v = np.where(e == 0, sub, normal)
    v = np.where(e == 31, np.where(m == 0, np.inf, np.nan), v)
    return v * sign


# ----------------------------------------------------------------------------
# Inputs
# ----------------------------------------------------------------------------

class OracleInputs:
    """Raw bits of one decode step, as the cache and the queries hold them.

    q_nope [B][s_q][H][128] and q_pe [B][s_q][H][64] as bf16 bits; w_uk, w_uv
    [H][128][512] bf16 bits; kv [num_pages][64][576] as bf16 (uint16), e4m3
    (uint8) or q8_0 (int8 codes, as uint8) bits, or [num_pages][64][288] packed
    q4_0 codes (uint8); kv_scale fp32 [num_pages][64] for e4m3, fp16 bits
    [num_pages][64][18] (one scale per 32-value block) for q8_0 and q4_0, else
    None; block_table int [B][max_pages]; seq_lens int [B] (lengths include the
    s_q new tokens).

    q8_0 and q4_0 (ik_llama.cpp docs "FlashMLA", section "KV cache with MLA":
    q8_0 is the recommended quantised MLA cache, lower-bit types are used with a
    Hadamard rotation): value = code * the block's scale, blocks of 32
    consecutive values of the 576-value row.  The docs fix no byte layout for
    q4_0; the reading taken here: codes in [-7, 7] stored as the 4-bit number
    code + 8, value 2j of the row in the low half of byte j and value 2j + 1 in
    its high half (288 bytes a row).
    """

    def __init__(self, q_nope, q_pe, w_uk, w_uv, kv, kv_dtype, kv_scale, block_table,
                 seq_lens, softmax_scale, causal):
        self.q_nope = bf16_to_f64(q_nope)
        self.q_pe = bf16_to_f64(q_pe)
        self.w_uk = bf16_to_f64(w_uk)
        self.w_uv = bf16_to_f64(w_uv)
        self.kv = np.asarray(kv)
        self.kv_dtype = kv_dtype
        if kv_dtype in ("q8_0", "q4_0"):
            self.kv_scale = f16_to_f64(kv_scale)
        else:
            self.kv_scale = None if kv_scale is None else np.asarray(kv_scale, dtype=np.float64)
        self.block_table = np.asarray(block_table, dtype=np.int64)
        self.seq_lens = np.asarray(seq_lens, dtype=np.int64)
        self.softmax_scale = float(softmax_scale)
        self.causal = bool(causal)
        self.B, self.s_q, self.H, _ = self.q_nope.shape
        assert kv_dtype in ("bf16", "fp8", "q8_0", "q4_0")

    def visible(self, b: int, i: int) -> int:
        """Number of cached tokens query i of sequence b attends to."""
        L = int(self.seq_lens[b])
        if not self.causal:
            return L
        return max(0, L - self.s_q + i + 1)

    def rows(self, b: int, n: int) -> np.ndarray:
        """The first n cached rows [n][576] of sequence b in fp64, through the block
        table: token j lives in physical page block_table[b][j // 64], row j % 64."""
        if n == 0:
            return np.zeros((0, D_C + D_R))
        npg = (n + PAGE - 1) // PAGE
        pages = self.block_table[b, :npg]
        raw = self.kv[pages].reshape(npg * PAGE, -1)[:n]
        if self.kv_dtype == "bf16":
            return bf16_to_f64(raw)
        if self.kv_dtype == "q8_0":
            codes = raw.astype(np.uint8).view(np.int8).astype(np.float64)          # [n][576]
            block = self.kv_scale[pages].reshape(npg * PAGE, -1)[:n]               # [n][18]
            return codes * np.repeat(block, Q8_BLOCK, axis=1)
        if self.kv_dtype == "q4_0":
            byte = raw.astype(np.int64)                                            # [n][288]
            codes = np.empty((n, D_C + D_R))
            codes[:, 0::2] = (byte & 0xF) - 8
            codes[:, 1::2] = (byte >> 4) - 8
            block = self.kv_scale[pages].reshape(npg * PAGE, -1)[:n]               # [n][18]
            return codes * np.repeat(block, Q8_BLOCK, axis=1)
        scale = self.kv_scale[pages].reshape(npg * PAGE)[:n]
        return e4m3fn_to_f64(raw) * scale[:, None]


def _all_rows(inp: OracleInputs, rows):
    if rows is None:
        return [(b, i) for b in range(inp.B) for i in range(inp.s_q)]
    return list(rows)


def _empty_out(inp: OracleInputs):
    B, s_q, H = inp.B, inp.s_q, inp.H
    return {
        "o": np.full((B, s_q, H, inp.w_uv.shape[1]), np.nan),
        "o_lat": np.full((B, s_q, H, D_C), np.nan),
        "lse": np.full((B, s_q, H), np.nan),
    }


def _softmax_lse(s: np.ndarray):
    """Softmax along axis 0 and its natural-log partition function."""
    m = s.max(axis=0)
    e = np.exp(s - m)
    z = e.sum(axis=0)
    return e / z, m + np.log(z)


# ----------------------------------------------------------------------------
# The definition: explicit K and V per head (non-absorbed)
# ----------------------------------------------------------------------------

def decode_nonabsorbed(inp: OracleInputs, rows: Optional[Iterable[Tuple[int, int]]] = None,
                       heads: Optional[Sequence[int]] = None):
    """MLA decode as the architecture defines it.  For each (b, i) in ``rows`` and
    head h in ``heads``: k_j = [W_UK[h] c_j ; k_pe_j], v_j = W_UV[h] c_j,
    q = [q_nope ; q_pe], s_j = scale * q . k_j, p = softmax(s), o = sum_j p_j v_j,
    o_lat = sum_j p_j c_j (the latent-space output the absorbed form produces),
    lse = log sum_j exp(s_j).  An empty context gives o = 0, o_lat = 0,
    lse = -inf.  Entries not requested stay NaN."""
    out = _empty_out(inp)
    heads = list(range(inp.H)) if heads is None else list(heads)
    cache = {}
    for b, i in _all_rows(inp, rows):
        n = inp.visible(b, i)
        if n == 0:
            for h in heads:
                out["o"][b, i, h] = 0.0
                out["o_lat"][b, i, h] = 0.0
                out["lse"][b, i, h] = -np.inf
            continue
        key = (b, n)
        if key not in cache:
            cache.clear()
            cache[key] = inp.rows(b, n)
        C = cache[key]
        c, k_pe = C[:, :D_C], C[:, D_C:]
        for h in heads:
            K = np.concatenate([c @ inp.w_uk[h].T, k_pe], axis=1)     # [n][192]
            V = c @ inp.w_uv[h].T                                      # [n][128]
            q = np.concatenate([inp.q_nope[b, i, h], inp.q_pe[b, i, h]])
            s = inp.softmax_scale * (K @ q)
            p, lse = _softmax_lse(s)
            out["o"][b, i, h] = p @ V
            out["o_lat"][b, i, h] = p @ c
            out["lse"][b, i, h] = lse
    return out


# ----------------------------------------------------------------------------
# The absorbed form (same mathematics, K and V never formed)
# ----------------------------------------------------------------------------

def absorb_q(q_nope: np.ndarray, w_uk: np.ndarray) -> np.ndarray:
    """q_lat[..., h, :] = W_UK[h]^T q_nope[..., h, :]   (512 <- 128)."""
    return np.einsum("...hn,hnc->...hc", q_nope, w_uk)


def up_proj_v(o_lat: np.ndarray, w_uv: np.ndarray) -> np.ndarray:
    """o[..., h, :] = W_UV[h] o_lat[..., h, :]   (128 <- 512)."""
    return np.einsum("...hc,hvc->...hv", o_lat, w_uv)


def latent_attention(q_lat: np.ndarray, q_pe: np.ndarray, C: np.ndarray, scale: float):
    """Attention of H absorbed queries over n cached rows, all in latent space:
    s[j, h] = scale * (q_lat[h] . c_j + q_pe[h] . k_pe_j); returns o_lat [H][512]
    and lse [H].  n = 0 gives zeros and -inf."""
    H = q_lat.shape[0]
    if C.shape[0] == 0:
        return np.zeros((H, D_C)), np.full(H, -np.inf)
    s = scale * (C[:, :D_C] @ q_lat.T + C[:, D_C:] @ q_pe.T)          # [n][H]
    p, lse = _softmax_lse(s)
    return p.T @ C[:, :D_C], lse


def decode_absorbed(inp: OracleInputs, rows: Optional[Iterable[Tuple[int, int]]] = None,
                    heads: Optional[Sequence[int]] = None):
    """The weight-absorbed decode: q_lat = W_UK^T q_nope, latent attention over
    [c ; k_pe], o = W_UV o_lat.  Same outputs as ``decode_nonabsorbed``."""
    out = _empty_out(inp)
    heads = np.arange(inp.H) if heads is None else np.asarray(list(heads))
    q_lat = absorb_q(inp.q_nope[:, :, heads], inp.w_uk[heads])          # [B][s_q][h][512]
    cache = {}
    for b, i in _all_rows(inp, rows):
        n = inp.visible(b, i)
        key = (b, n)
        if key not in cache:
            cache.clear()
            cache[key] = inp.rows(b, n)
        o_lat, lse = latent_attention(q_lat[b, i], inp.q_pe[b, i, heads], cache[key],
                                      inp.softmax_scale)
        out["o_lat"][b, i, heads] = o_lat
        out["lse"][b, i, heads] = lse
        out["o"][b, i, heads] = up_proj_v(o_lat, inp.w_uv[heads])
    return out


# ----------------------------------------------------------------------------
# Split-KV partials and their log-sum-exp merge
# ----------------------------------------------------------------------------

def combine_splits(o_parts: np.ndarray, lse_parts: np.ndarray):
    """Merge S partial results over disjoint token ranges.  Axis 0 indexes the
    split.  lse = log sum_s exp(lse_s); o = sum_s exp(lse_s - lse) o_s.  Splits with
    lse_s = -inf (no tokens) weigh nothing; if every split is empty the result is
    o = 0, lse = -inf."""
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = lse_parts.max(axis=0)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    w = np.exp(lse_parts - m_safe)                                       # exp(-inf) = 0
    z = w.sum(axis=0)
    lse = np.where(finite, m_safe + np.log(np.where(finite, z, 1.0)), -np.inf)
    wn = np.where(finite, w / np.where(finite, z, 1.0), 0.0)
    o = (wn[..., None] * o_parts).sum(axis=0)
    return o, lse

