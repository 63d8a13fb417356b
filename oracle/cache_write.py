"""fp64 CPU oracle for writing new tokens into the paged latent KV cache.

TEST INFRASTRUCTURE ONLY, like ``mla_oracle``: only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may call it; it shares no
code with the CUDA library and never imports it.

What it follows (page titles and sections of the pages this method comes from):

* "MLA: Multi-Head Latent Attention — DeepSeek-AI Explained", section
  "Architecture": the cache stores the down-projection ``c_t = W_DKV h_t``
  (width d_c = 512) of the token's hidden state.
* snowgate thread 35, replies on the 576-value latent record: beside the latent
  sits a 64-wide RoPE key shared by every head, kept apart from the
  up-projections (so it is rotated before it is stored).
* ik_llama.cpp docs "FlashMLA", section "KV cache with MLA": the latent cache may
  be stored quantised.

Readings taken where the pages are silent (each one is listed with the design):

* The RoPE key is ``k_pe_t = RoPE(W_KR h_t, pos_t)`` with its own projection
  ``W_KR`` [64 x d_h] (the pages give the 64 values, not their source).
* RoPE is the rotary embedding in its original form: value pairs (2i, 2i+1)
  rotate by the angle ``pos * base**(-2i / 64)``, base 10000.
* The s_q new tokens of sequence b sit at positions L_b - s_q + i (lengths count
  the new tokens), row ``pos % 64`` of page ``block_table[b][pos // 64]``.
* bf16 cache: each value is rounded to nearest even.  e4m3 cache: one fp32 scale
  per 576-value row, ``scale = amax / 448`` computed in fp32 (1 for an all-zero
  row), codes = the fp32 quotient ``value / scale`` rounded to nearest even and
  saturated at +-448.  The decision takes fp32 inputs, so the fp64 row is first
  rounded to fp32.
* q8_0 and q4_0 caches: blocks of 32 values, one fp16 scale ``d = amax / levels``
  (127 or 7, computed in fp32), codes = the fp32 quotients ``value / d`` rounded
  to nearest even and clamped to +-levels (0 for an all-zero block).  q4_0 codes
  are stored as the 4-bit number code + 8, value 2j of the row in the low half of
  byte j and value 2j + 1 in the high half (the docs name the type, not its
  byte layout).

Pinned by ``tests/test_cache_write_oracle.py``: the encoders against torch's
casts, RoPE against closed forms and its relative-position identity, the paged
write by brute force, and the whole write read back through the decode oracle.
"""

from __future__ import annotations

from typing import Optional, Tuple

import numpy as np

PAGE = 64
D_C = 512
D_R = 64
ROW = D_C + D_R
E4M3_MAX = 448.0


# ----------------------------------------------------------------------------
# Storage encoders (round to nearest even), written from the bit formats
# ----------------------------------------------------------------------------

def _round_to_grid(a: np.ndarray, mant_bits: int, min_exp: int) -> np.ndarray:
    """Non-negative fp64 values rounded to nearest even on the grid of a binary
    format with ``mant_bits`` stored mantissa bits whose smallest normal is
    2**min_exp (below it the spacing stays 2**(min_exp - mant_bits))."""
    _, e = np.frexp(a)                          # a = m * 2**e, m in [0.5, 1)
    lead = np.maximum(e - 1, min_exp)           # exponent of the leading bit
    quantum = np.ldexp(1.0, lead - mant_bits)
    return np.rint(a / quantum) * quantum       # np.rint: ties to even; a / quantum is exact


def f64_to_e4m3fn(x) -> np.ndarray:
    """OCP e4m3fn bits (uint8) of x: 1 sign, 4 exponent (bias 7), 3 mantissa bits,
    no infinities; finite values beyond 448 saturate to 448; NaN -> 0x7F."""
    x = np.asarray(x, dtype=np.float64)
    sign = np.signbit(x).astype(np.uint8)
    a = np.minimum(np.abs(np.nan_to_num(x, nan=0.0)), E4M3_MAX)
    v = _round_to_grid(a, 3, -6)
    _, ve = np.frexp(v)
    normal = v >= 2.0 ** -6
    exp_field = np.where(normal, ve - 1 + 7, 0)
    mant = np.where(normal, v / np.ldexp(1.0, ve - 1) * 8 - 8, v / 2.0 ** -9)
    bits = (sign << 7) | (exp_field.astype(np.uint8) << 3) | mant.astype(np.uint8)
    return np.where(np.isnan(x), np.uint8(0x7F) | (sign << 7), bits).astype(np.uint8)


def f64_to_bf16(x) -> np.ndarray:
    """bf16 bits (uint16) of finite x, rounded to nearest even (8 significant
    bits; normals from 2**-126)."""
    x = np.asarray(x, dtype=np.float64)
    v = np.copysign(_round_to_grid(np.abs(x), 7, -126), x)
    return (v.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


# ----------------------------------------------------------------------------
# The steps of a cache write
# ----------------------------------------------------------------------------

def compress(h: np.ndarray, w_dkv: np.ndarray, w_kr: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """c = W_DKV h (512) and the unrotated RoPE key W_KR h (64), per token.
    h [n][d_h], w_dkv [512][d_h], w_kr [64][d_h]."""
    return h @ w_dkv.T, h @ w_kr.T


def rope(x: np.ndarray, pos, base: float = 10000.0) -> np.ndarray:
    """Rotary embedding of x [..., d] at integer positions pos [...]: pair i =
    (x[2i], x[2i+1]) turns by the angle pos * base**(-2i/d)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    theta = base ** (-np.arange(0, d, 2, dtype=np.float64) / d)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * theta
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


def quantise_row_e4m3(row: np.ndarray) -> Tuple[np.ndarray, np.float32]:
    """One 576-value row -> (e4m3 codes, fp32 scale), value ~ code * scale.  The
    row is taken at fp32 precision and the scale and quotients are fp32 IEEE
    operations, as the stored format fixes."""
    r32 = np.asarray(row, dtype=np.float64).astype(np.float32)
    amax = np.float32(np.max(np.abs(r32))) if r32.size else np.float32(0.0)
    scale = np.float32(amax / np.float32(E4M3_MAX)) if amax > 0 else np.float32(1.0)
    q = (r32 / scale).astype(np.float32)
    return f64_to_e4m3fn(np.clip(q.astype(np.float64), -E4M3_MAX, E4M3_MAX)), scale


def _quantise_row_blocks(row: np.ndarray, levels: int) -> Tuple[np.ndarray, np.ndarray]:
    r32 = np.asarray(row, dtype=np.float64).astype(np.float32).reshape(-1, 32)
    amax = np.max(np.abs(r32), axis=1)
    d16 = (amax / np.float32(levels)).astype(np.float32).astype(np.float16)
    d32 = d16.astype(np.float32)
    safe = np.where(d32 > 0, d32, np.float32(1.0))
    q = np.rint((r32 / safe[:, None]).astype(np.float32))
    q = np.clip(q, -levels, levels)
    q = np.where(d32[:, None] > 0, q, 0)
    return q.astype(np.int8).reshape(-1), d16


def quantise_row_q8_0(row: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """One 576-value row -> (int8 codes [576], fp16 scales [18]) of the q8_0 format
    (ik_llama.cpp docs "FlashMLA", section "KV cache with MLA"; blocks of 32
    values, d = amax / 127 rounded to fp16, codes round(x / d) in [-127, 127]).
    The row is taken at fp32 precision and amax / 127 and the quotients are fp32
    IEEE operations, as for the e4m3 row."""
    return _quantise_row_blocks(row, 127)


def quantise_row_q4_0(row: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """One 576-value row -> (packed codes uint8 [288], fp16 scales [18]) of the
    q4_0 format: as q8_0 with d = amax / 7 and codes in [-7, 7]; byte j holds
    code 2j + 8 in its low four bits and code 2j+1 + 8 in its high four bits."""
    q, d16 = _quantise_row_blocks(row, 7)
    n = (q.astype(np.int64) + 8).astype(np.uint8)
    return (n[0::2] | (n[1::2] << 4)).astype(np.uint8), d16


def slot_of(block_table: np.ndarray, seq_lens: np.ndarray, s_q: int, b: int, i: int,
            num_pages: int) -> Tuple[int, int]:
    """(physical page, row) of new token i of sequence b."""
    pos = int(seq_lens[b]) - s_q + i
    if pos < 0:
        raise ValueError(f"sequence {b}: length {int(seq_lens[b])} < {s_q} new tokens")
    if pos // PAGE >= block_table.shape[1]:
        raise ValueError(f"sequence {b}: position {pos} beyond the block table")
    page = int(block_table[b, pos // PAGE])
    if not 0 <= page < num_pages:
        raise ValueError(f"sequence {b}: page id {page} outside the cache")
    return page, pos % PAGE


def write_kv(h: np.ndarray, w_dkv: np.ndarray, w_kr: np.ndarray, kv: np.ndarray,
             kv_scale: Optional[np.ndarray], kv_dtype: str, block_table: np.ndarray,
             seq_lens: np.ndarray, s_q: int, rope_base: float = 10000.0):
    """Writes the s_q new tokens of every sequence into a copy of the cache and
    returns (kv, kv_scale).

    h [B][s_q][d_h] (fp64 values), w_dkv [512][d_h], w_kr [64][d_h]; kv holds raw
    bits [num_pages][64][576] (uint16 bf16, uint8 e4m3, int8 q8_0 codes) or
    [num_pages][64][288] (uint8 packed q4_0 codes); kv_scale is fp32
    [num_pages][64] for e4m3, fp16 [num_pages][64][18] for q8_0 and q4_0.  Every
    row other than the new tokens' is left as it was."""
    assert kv_dtype in ("bf16", "fp8", "q8_0", "q4_0")
    B = h.shape[0]
    kv = np.array(kv, copy=True)
    if kv_dtype in ("q8_0", "q4_0"):
        kv_scale = np.array(kv_scale, dtype=np.float16, copy=True)
    else:
        kv_scale = None if kv_scale is None else np.array(kv_scale, dtype=np.float32, copy=True)
    for b in range(B):
        c, kr = compress(h[b], w_dkv, w_kr)                       # [s_q][512], [s_q][64]
        pos = int(seq_lens[b]) - s_q + np.arange(s_q)
        k_pe = rope(kr, pos, rope_base)
        for i in range(s_q):
            page, row = slot_of(block_table, seq_lens, s_q, b, i, kv.shape[0])
            full = np.concatenate([c[i], k_pe[i]])
            if kv_dtype == "bf16":
                kv[page, row] = f64_to_bf16(full)
            elif kv_dtype == "q8_0":
                kv[page, row], kv_scale[page, row] = quantise_row_q8_0(full)
            elif kv_dtype == "q4_0":
                kv[page, row], kv_scale[page, row] = quantise_row_q4_0(full)
            else:
                kv[page, row], kv_scale[page, row] = quantise_row_e4m3(full)
    return kv, kv_scale
