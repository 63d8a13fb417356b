"""fp64 CPU oracle for a blockwise low-bit latent cache with an optional Hadamard
rotation (test infrastructure only, like ``mla_oracle``: only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may call it; it shares no
code with the CUDA library and never imports it).

What it follows: ik_llama.cpp docs "FlashMLA", section "KV cache with MLA": the
MLA cache may be stored as ``q8_0`` (the recommended type) and, below 6 bits, a
Hadamard transform applied to the K cache before quantisation recovers quality.

Readings taken where the pages are silent (each one is listed with the design):

* ``q8_0``: the 576 values of a cached row in blocks of 32, one scale per block
  ``d = amax / 127`` (kept at fp16 precision), codes ``round(x / d)`` in
  [-127, 127]; ``q4_0``: the same with ``d = amax / 7`` and codes in [-7, 7].
  Rounding is to nearest, ties to even; an all-zero block has ``d = 0`` and
  zero codes.  Value = code * d.
* The Hadamard transform is the orthonormal Sylvester matrix ``H`` of size 512
  applied to the latent part ``c`` of every row (the RoPE key is left as it is).
  Because ``H`` is symmetric and orthonormal, ``q_lat . c = (H q_lat) . (H c)``
  and ``sum_j p_j (H c_j) = H o_lat``: the rotation folds into the weights,
  ``W_DKV -> H W_DKV``, ``W_UK[h] -> W_UK[h] H``, ``W_UV[h] -> W_UV[h] H``, and
  attention over the rotated cache with the folded weights equals attention over
  the plain cache with the plain weights.

Pinned by ``tests/test_lowbit_cache_oracle.py``.
"""

from __future__ import annotations

from typing import Tuple

import numpy as np

BLOCK = 32
D_C = 512
LEVELS = {"q8_0": 127, "q4_0": 7}


def hadamard(n: int) -> np.ndarray:
    """Orthonormal Sylvester-Hadamard matrix of size n (a power of two)."""
    assert n >= 1 and n & (n - 1) == 0
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h / np.sqrt(n)


def fold_hadamard(w_dkv: np.ndarray, w_uk: np.ndarray, w_uv: np.ndarray):
    """The weights that make attention over the rotated cache equal attention over
    the plain one: H W_DKV [512 x d_h], W_UK[h] H and W_UV[h] H [H][128][512]."""
    h = hadamard(D_C)
    return h @ w_dkv, w_uk @ h, w_uv @ h


def rotate_latent(rows: np.ndarray) -> np.ndarray:
    """Rows [..., 576] with their latent part c replaced by H c."""
    out = np.array(rows, dtype=np.float64, copy=True)
    out[..., :D_C] = out[..., :D_C] @ hadamard(D_C).T
    return out


def quantise_blocks(row: np.ndarray, kind: str) -> Tuple[np.ndarray, np.ndarray]:
    """A row of length multiple of 32 -> (int codes [n], fp16-precision scales
    [n / 32]) of the blockwise format ``kind`` ("q8_0" or "q4_0")."""
    levels = LEVELS[kind]
    x = np.asarray(row, dtype=np.float64).reshape(-1, BLOCK)
    amax = np.abs(x).max(axis=1)
    d = (amax / levels).astype(np.float16).astype(np.float64)
    safe = np.where(d > 0, d, 1.0)
    q = np.clip(np.rint(x / safe[:, None]), -levels, levels)
    q = np.where(d[:, None] > 0, q, 0.0)
    return q.astype(np.int8).reshape(-1), d


def dequantise_blocks(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Value = code * block scale."""
    q = np.asarray(codes, dtype=np.float64).reshape(-1, BLOCK)
    return (q * np.asarray(scales, dtype=np.float64)[:, None]).reshape(-1)
