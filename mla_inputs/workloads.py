"""Workload presets and the seeded generator.

Draw recipe (fixed; changing it changes every stored expectation):

* one ``torch.Generator`` seeded with the preset's seed, CPU, draws in this order:
  sequence lengths (ragged presets only), physical page permutation, q_nope,
  q_pe, W_UK, W_UV, then the cache rows page by page;
* activations, RoPE parts and cache values are N(0, 1) in fp32, weights are
  N(0, std = 1/sqrt(512)); all are rounded to bf16 (round to nearest even) by
  the cast, except the fp8 cache below;
* fp8 cache: each 576-value row is scaled by ``amax(row) / 448`` and cast to
  float8 e4m3fn (round to nearest even); the fp32 scale is stored per token;
* q8_0 cache: each block of 32 consecutive values of a row gets the scale
  ``d = amax(block) / 127`` rounded to fp16, and int8 codes ``round(x / d)``
  (nearest even, in fp32, clamped to [-127, 127]; 0 for an all-zero block);
* q4_0 cache: the same with ``d = amax(block) / 7`` and codes in [-7, 7], each
  stored as the 4-bit number code + 8, value 2j of a row in the low half of
  byte j and value 2j + 1 in the high half (288 bytes a row);
* rows of a sequence's last page at positions >= its length hold finite values
  50x larger than the real rows, so that a kernel that forgets to mask them
  produces a visibly wrong answer.

The quantisation above only produces a cache in the stored format; the decode
step never quantises anything.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import numpy as np
import torch

D_C = 512      # latent width c_KV
D_R = 64       # decoupled RoPE key width
D_N = 128      # per-head no-position query/key width (qk_nope)
D_V = 128      # per-head value width
PAGE = 64      # tokens per cache page
ROW = D_C + D_R  # 576 values per cached token
SOFTMAX_SCALE = 1.0 / math.sqrt(D_N + D_R)  # 1/sqrt(192)
TAIL_GAIN = 50.0
FP8_MAX = 448.0
Q8_BLOCK = 32     # q8_0: values per scale block
Q8_LEVELS = 127   # q8_0: largest code
Q4_LEVELS = 7     # q4_0: largest code


@dataclass
class WorkloadSpec:
    name: str
    B: int
    H: int
    s_q: int
    lens: Optional[Sequence[int]]  # explicit lengths; None => ragged draw
    kv_dtype: str = "bf16"  # "bf16" | "fp8" | "q8_0" | "q4_0"
    causal: bool = False
    seed: int = 0
    permute_pages: bool = True
    ragged_max: int = 0  # for lens=None: lengths uniform in [1, ragged_max]
    note: str = ""

    def with_(self, **kw) -> "WorkloadSpec":
        d = dict(self.__dict__)
        d.update(kw)
        return WorkloadSpec(**d)


# The five workload shapes (DeepSeek-V2/V3 MLA dims: d_c=512, d_r=64, qk_nope=128,
# v_head=128, softmax scale 1/sqrt(192)).
PRESETS = {
    "tiny": WorkloadSpec("tiny", B=1, H=16, s_q=1, lens=[256], seed=0, permute_pages=False,
                         note="batch 1, 16 heads, 256 tokens, contiguous cache"),
    "v3": WorkloadSpec("v3", B=64, H=128, s_q=1, lens=[4096] * 64, seed=1,
                       note="DeepSeek-V3-shaped: batch 64, 128 heads, 4096 tokens, bf16 paged"),
    "ragged": WorkloadSpec("ragged", B=128, H=128, s_q=1, lens=None, ragged_max=32768, seed=2,
                           note="batch 128, 128 heads, lengths uniform in [1, 32768]"),
    "long16": WorkloadSpec("long16", B=4, H=16, s_q=1, lens=[131072] * 4, seed=3,
                           note="batch 4, 131072 tokens, 16 heads, split-KV"),
    "long128": WorkloadSpec("long128", B=4, H=128, s_q=1, lens=[131072] * 4, seed=3,
                            note="batch 4, 131072 tokens, 128 heads, split-KV"),
    "fp8": WorkloadSpec("fp8", B=128, H=128, s_q=2, lens=[8192] * 128, kv_dtype="fp8",
                        causal=True, seed=4,
                        note="batch 128, 128 heads, 8192 tokens, e4m3 cache + fp32 per-token "
                             "scale, 2 causal query tokens"),
    # the V3 shape over the blockwise q8_0 cache (ik_llama.cpp's recommended MLA cache type)
    "prefill": WorkloadSpec("prefill", B=4, H=128, s_q=1024, lens=[8192] * 4, causal=True, seed=6,
                            note="chunked prefill: batch 4, 128 heads, 1024 new tokens appended "
                                 "to 7168 cached (8192 in all), causal, bf16 paged"),
    "prefill1": WorkloadSpec("prefill1", B=1, H=128, s_q=1024, lens=[8192], causal=True, seed=6,
                             note="one sequence of the chunked-prefill workload (for profiler "
                                  "captures): 128 heads, 1024 new tokens on 7168 cached, causal"),
    "q8": WorkloadSpec("q8", B=64, H=128, s_q=1, lens=[4096] * 64, kv_dtype="q8_0", seed=5,
                       note="DeepSeek-V3-shaped: batch 64, 128 heads, 4096 tokens, q8_0 cache "
                            "(int8 codes, fp16 scale per 32 values)"),
    # the same over the 4-bit blockwise cache
    "q4": WorkloadSpec("q4", B=64, H=128, s_q=1, lens=[4096] * 64, kv_dtype="q4_0", seed=6,
                       note="DeepSeek-V3-shaped: batch 64, 128 heads, 4096 tokens, q4_0 cache "
                            "(4-bit codes, fp16 scale per 32 values)"),
}


def preset(name: str) -> WorkloadSpec:
    return PRESETS[name]


@dataclass
class Workload:
    """Host (CPU) tensors of one decode step, in the layouts the C ABI takes."""
    spec: WorkloadSpec
    seq_lens: torch.Tensor        # int32 [B]
    block_table: torch.Tensor     # int32 [B][max_pages]
    q_nope: torch.Tensor          # bf16 [B][s_q][H][128]
    q_pe: torch.Tensor            # bf16 [B][s_q][H][64]
    w_uk: torch.Tensor            # bf16 [H][128][512]   k = W_UK[h] . c
    w_uv: torch.Tensor            # bf16 [H][128][512]   v = W_UV[h] . c
    kv_cache: torch.Tensor        # bf16 or float8_e4m3fn [num_pages][64][576]
    kv_scale: Optional[torch.Tensor]  # fp32 [num_pages][64] (fp8), fp16 [num_pages][64][18] (q8_0, q4_0)
    raw_rows: Optional[torch.Tensor] = None  # fp32 [num_pages][64][576] draws (keep_raw only)
    softmax_scale: float = SOFTMAX_SCALE
    extra: dict = field(default_factory=dict)

    @property
    def B(self): return self.spec.B

    @property
    def H(self): return self.spec.H

    @property
    def s_q(self): return self.spec.s_q

    @property
    def causal(self): return self.spec.causal

    @property
    def num_pages(self): return int(self.kv_cache.shape[0])

    @property
    def max_pages(self): return int(self.block_table.shape[1])

    @property
    def lens(self) -> List[int]:
        return [int(x) for x in self.seq_lens.tolist()]

    @property
    def n_tok(self): return self.spec.B * self.spec.s_q

    def cache_bytes(self) -> int:
        """Bytes of cache rows the step must read: sum of lengths x row bytes."""
        return sum(self.lens) * row_bytes(self.spec.kv_dtype)


def row_bytes(kv_dtype: str) -> int:
    """Bytes one cached token occupies: 576 values, plus their scales."""
    return {"bf16": 2 * ROW, "fp8": ROW + 4, "q8_0": ROW + 2 * (ROW // Q8_BLOCK),
            "q4_0": ROW // 2 + 2 * (ROW // Q8_BLOCK)}[kv_dtype]


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """uint16 view of a bf16 tensor (the bits the oracle decodes itself)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def fp8_bits(t: torch.Tensor) -> np.ndarray:
    """uint8 view of a float8_e4m3fn tensor."""
    assert t.dtype == torch.float8_e4m3fn
    return t.contiguous().view(torch.uint8).numpy()


def int8_bits(t: torch.Tensor) -> np.ndarray:
    """uint8 view of an int8 tensor."""
    assert t.dtype == torch.int8
    return t.contiguous().view(torch.uint8).numpy()


def f16_bits(t: torch.Tensor) -> np.ndarray:
    """uint16 view of a float16 tensor."""
    assert t.dtype == torch.float16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _quantise_rows_e4m3(rows: torch.Tensor):
    amax = rows.abs().amax(dim=-1, keepdim=True)
    scale = torch.where(amax > 0, amax / FP8_MAX, torch.ones_like(amax))
    q = (rows / scale).clamp_(-FP8_MAX, FP8_MAX).to(torch.float8_e4m3fn)
    return q, scale.squeeze(-1).to(torch.float32)


def _quantise_rows_blocks(rows: torch.Tensor, levels: int):
    blocks = rows.reshape(*rows.shape[:-1], ROW // Q8_BLOCK, Q8_BLOCK)
    d = (blocks.abs().amax(dim=-1) / levels).to(torch.float16)
    df = d.to(torch.float32)
    safe = torch.where(df > 0, df, torch.ones_like(df))
    q = torch.round(blocks / safe[..., None]).clamp_(-levels, levels)
    q = torch.where(df[..., None] > 0, q, torch.zeros_like(q))
    return q.to(torch.int8).reshape(rows.shape), d


def _quantise_rows_q8_0(rows: torch.Tensor):
    return _quantise_rows_blocks(rows, Q8_LEVELS)


def _quantise_rows_q4_0(rows: torch.Tensor):
    """(packed uint8 [..., 288], fp16 scales [..., 18])."""
    q, d = _quantise_rows_blocks(rows, Q4_LEVELS)
    n = (q.to(torch.int16) + 8).to(torch.uint8)
    return n[..., 0::2] | (n[..., 1::2] << 4), d


def make_workload(spec: WorkloadSpec, keep_raw: bool = False) -> Workload:
    g = torch.Generator().manual_seed(int(spec.seed))
    B, H, s_q = spec.B, spec.H, spec.s_q
    if spec.lens is None:
        lens = torch.randint(1, spec.ragged_max + 1, (B,), generator=g, dtype=torch.int64)
        lens = [int(x) for x in lens.tolist()]
    else:
        lens = [int(x) for x in spec.lens]
        assert len(lens) == B
    assert all(L >= 0 for L in lens)
    pages_per = [(L + PAGE - 1) // PAGE for L in lens]
    num_pages = max(1, sum(pages_per))
    max_pages = max(1, max(pages_per))
    # The permutation is always drawn so that the logical contents do not depend
    # on whether pages are shuffled.
    perm = torch.randperm(num_pages, generator=g, dtype=torch.int64)
    if not spec.permute_pages:
        perm = torch.arange(num_pages, dtype=torch.int64)
    block_table = torch.zeros(B, max_pages, dtype=torch.int32)
    off = 0
    for b, n in enumerate(pages_per):
        block_table[b, :n] = perm[off:off + n].to(torch.int32)
        off += n

    q_nope = torch.randn(B, s_q, H, D_N, generator=g).to(torch.bfloat16)
    q_pe = torch.randn(B, s_q, H, D_R, generator=g).to(torch.bfloat16)
    w_std = 1.0 / math.sqrt(D_C)
    w_uk = (torch.randn(H, D_N, D_C, generator=g) * w_std).to(torch.bfloat16)
    w_uv = (torch.randn(H, D_V, D_C, generator=g) * w_std).to(torch.bfloat16)

    # Cache rows, drawn in logical order (sequence by sequence, page by page) and
    # stored at their physical page.  Tail rows of a last page get TAIL_GAIN.
    fp8 = spec.kv_dtype == "fp8"
    q8 = spec.kv_dtype == "q8_0"
    q4 = spec.kv_dtype == "q4_0"
    if fp8:
        kv_cache = torch.zeros(num_pages, PAGE, ROW, dtype=torch.float8_e4m3fn)
        kv_scale = torch.ones(num_pages, PAGE, dtype=torch.float32)
    elif q8:
        kv_cache = torch.zeros(num_pages, PAGE, ROW, dtype=torch.int8)
        kv_scale = torch.zeros(num_pages, PAGE, ROW // Q8_BLOCK, dtype=torch.float16)
    elif q4:
        kv_cache = torch.zeros(num_pages, PAGE, ROW // 2, dtype=torch.uint8)
        kv_scale = torch.zeros(num_pages, PAGE, ROW // Q8_BLOCK, dtype=torch.float16)
    else:
        kv_cache = torch.zeros(num_pages, PAGE, ROW, dtype=torch.bfloat16)
        kv_scale = None
    raw = torch.zeros(num_pages, PAGE, ROW, dtype=torch.float32) if keep_raw else None
    CH = 2048  # pages per chunk, bounds host memory for the large presets
    for b, n in enumerate(pages_per):
        if n == 0:
            continue
        phys = block_table[b, :n].to(torch.int64)
        for c0 in range(0, n, CH):
            c1 = min(n, c0 + CH)
            rows = torch.randn(c1 - c0, PAGE, ROW, generator=g)
            if c1 == n and lens[b] % PAGE:
                rows[-1, lens[b] % PAGE:, :] *= TAIL_GAIN
            idx = phys[c0:c1]
            if raw is not None:
                raw[idx] = rows
            if fp8:
                q, sc = _quantise_rows_e4m3(rows)
                kv_cache[idx] = q
                kv_scale[idx] = sc
            elif q8:
                q, sc = _quantise_rows_q8_0(rows)
                kv_cache[idx] = q
                kv_scale[idx] = sc
            elif q4:
                q, sc = _quantise_rows_q4_0(rows)
                kv_cache[idx] = q
                kv_scale[idx] = sc
            else:
                kv_cache[idx] = rows.to(torch.bfloat16)
    return Workload(spec=spec, seq_lens=torch.tensor(lens, dtype=torch.int32),
                    block_table=block_table, q_nope=q_nope, q_pe=q_pe, w_uk=w_uk, w_uv=w_uv,
                    kv_cache=kv_cache, kv_scale=kv_scale, raw_rows=raw)
