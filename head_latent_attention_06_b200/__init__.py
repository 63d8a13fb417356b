"""B200 (sm_100a) MLA decode over a paged latent KV cache.

A thin ctypes binding over ``libmla_b200.so`` (C ABI in ``include/mla.h``).  The
functions keep the C names and only marshal arguments: torch tensors become
device pointers and sizes, the current torch stream becomes the CUDA stream.
Every step of the computation runs in the library's CUDA kernels; there is no
fallback, and calling into a missing library raises.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmla_b200.so")

D_C, D_R, D_N, D_V, PAGE = 512, 64, 128, 128, 64
MAX_SPLITS = 128
KV_BF16, KV_FP8_E4M3, KV_Q8_0, KV_Q4_0 = 0, 1, 2, 3
Q8_BLOCKS = (D_C + D_R) // 32   # q8_0: scale blocks of a 576-value row

STATUS = {
    0: "MLA_OK", 1: "MLA_ERR_INVALID_VALUE", 2: "MLA_ERR_UNSUPPORTED", 3: "MLA_ERR_MISALIGNED",
    4: "MLA_ERR_WORKSPACE_TOO_SMALL", 5: "MLA_ERR_CUDA", 6: "MLA_ERR_DEVICE_TIMEOUT",
    7: "MLA_ERR_BAD_BLOCK_TABLE", 8: "MLA_ERR_BAD_SEQ_LEN",
}

# Every symbol include/mla.h declares.
EXPORTS = ("mla_absorb_q", "mla_decode_workspace_size", "mla_decode_num_splits",
           "mla_decode_paged", "mla_combine_splits", "mla_up_proj_v", "mla_get_status",
           "mla_status_string", "mla_decode_paged_noalloc", "mla_noalloc_init",
           "mla_get_status_noalloc", "mla_write_kv_workspace_size", "mla_write_kv",
           "mla_set_decode_kernel", "mla_set_device_wait_limit", "mla_fold_hadamard", "mla_prefill_workspace_size",
           "mla_prefill", "mla_decode_step_workspace_size", "mla_decode_step_launches", "mla_decode_step")

DECODE_AUTO, DECODE_WARP_MMA = 0, 1


class MlaError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")
        self.code = code


class DecodeArgs(ctypes.Structure):
    """Mirror of ``mla_decode_args_t`` (field order and types must match)."""
    _fields_ = [
        ("q_lat", ctypes.c_void_p), ("q_pe", ctypes.c_void_p),
        ("kv_cache", ctypes.c_void_p), ("kv_scale", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
        ("o_lat", ctypes.c_void_p), ("lse", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("B", ctypes.c_int32), ("s_q", ctypes.c_int32), ("H", ctypes.c_int32),
        ("d_c", ctypes.c_int32), ("d_r", ctypes.c_int32), ("page_size", ctypes.c_int32),
        ("num_pages", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32),
        ("kv_dtype", ctypes.c_int32), ("causal", ctypes.c_int32),
        ("num_splits", ctypes.c_int32), ("max_seq_len", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float),
    ]


class WriteKvArgs(ctypes.Structure):
    """Mirror of ``mla_write_kv_args_t`` (field order and types must match)."""
    _fields_ = [
        ("h", ctypes.c_void_p), ("w_dkv", ctypes.c_void_p),
        ("kv_cache", ctypes.c_void_p), ("kv_scale", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("B", ctypes.c_int32), ("s_q", ctypes.c_int32), ("d_h", ctypes.c_int32),
        ("d_c", ctypes.c_int32), ("d_r", ctypes.c_int32), ("page_size", ctypes.c_int32),
        ("num_pages", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32),
        ("kv_dtype", ctypes.c_int32), ("rope_base", ctypes.c_float),
    ]


class PrefillArgs(ctypes.Structure):
    """Mirror of ``mla_prefill_args_t`` (field order and types must match)."""
    _fields_ = [
        ("q_nope", ctypes.c_void_p), ("q_pe", ctypes.c_void_p),
        ("w_uk", ctypes.c_void_p), ("w_uv", ctypes.c_void_p),
        ("kv_cache", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
        ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("B", ctypes.c_int32), ("s_q", ctypes.c_int32), ("H", ctypes.c_int32),
        ("d_c", ctypes.c_int32), ("d_r", ctypes.c_int32), ("page_size", ctypes.c_int32),
        ("num_pages", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32),
        ("kv_dtype", ctypes.c_int32), ("causal", ctypes.c_int32),
        ("max_seq_len", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
    ]


class StepArgs(ctypes.Structure):
    """Mirror of ``mla_step_args_t`` (field order and types must match)."""
    _fields_ = [
        ("q_nope", ctypes.c_void_p), ("q_pe", ctypes.c_void_p),
        ("w_uk", ctypes.c_void_p), ("w_uv", ctypes.c_void_p),
        ("kv_cache", ctypes.c_void_p), ("kv_scale", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
        ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("B", ctypes.c_int32), ("s_q", ctypes.c_int32), ("H", ctypes.c_int32),
        ("d_c", ctypes.c_int32), ("d_r", ctypes.c_int32), ("page_size", ctypes.c_int32),
        ("num_pages", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32),
        ("kv_dtype", ctypes.c_int32), ("causal", ctypes.c_int32), ("num_splits", ctypes.c_int32),
        ("max_seq_len", ctypes.c_int32), ("softmax_scale", ctypes.c_float), ("fuse", ctypes.c_int32),
    ]


_lib: Optional[ctypes.CDLL] = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (built by ``head_latent_attention_06_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: run `python -m head_latent_attention_06_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32 = ctypes.c_void_p, ctypes.c_int32
    lib.mla_absorb_q.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp]
    lib.mla_up_proj_v.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp]
    pa = ctypes.POINTER(DecodeArgs)
    lib.mla_decode_workspace_size.argtypes = [pa, ctypes.POINTER(ctypes.c_size_t)]
    lib.mla_decode_num_splits.argtypes = [pa, ctypes.POINTER(ctypes.c_int32)]
    lib.mla_decode_paged.argtypes = [pa, vp]
    lib.mla_combine_splits.argtypes = [pa, vp]
    lib.mla_decode_paged_noalloc.argtypes = [pa, vp]
    lib.mla_noalloc_init.argtypes = []
    lib.mla_get_status_noalloc.argtypes = [vp]
    lib.mla_set_decode_kernel.argtypes = [i32]
    lib.mla_set_device_wait_limit.argtypes = [ctypes.c_uint64]
    pw = ctypes.POINTER(WriteKvArgs)
    lib.mla_write_kv_workspace_size.argtypes = [pw, ctypes.POINTER(ctypes.c_size_t)]
    lib.mla_write_kv.argtypes = [pw, vp]
    pp = ctypes.POINTER(PrefillArgs)
    lib.mla_prefill_workspace_size.argtypes = [pp, ctypes.POINTER(ctypes.c_size_t)]
    lib.mla_prefill.argtypes = [pp, vp]
    lib.mla_get_status.argtypes = [vp, vp]
    ps = ctypes.POINTER(StepArgs)
    lib.mla_decode_step_workspace_size.argtypes = [ps, ctypes.POINTER(ctypes.c_size_t)]
    lib.mla_decode_step_launches.argtypes = [ps, ctypes.POINTER(ctypes.c_int32)]
    lib.mla_decode_step.argtypes = [ps, vp]
    lib.mla_fold_hadamard.argtypes = [vp, i32, vp, vp, i32, vp]
    lib.mla_status_string.argtypes = [ctypes.c_int]
    lib.mla_status_string.restype = ctypes.c_char_p
    for name in EXPORTS:
        if name != "mla_status_string":
            getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    return int(stream) if isinstance(stream, int) else int(stream.cuda_stream)


def _check(fn, code):
    if code != 0:
        raise MlaError(fn, code)


def _want(specs):
    """Argument check of the tensor builders.  ``specs``: (tensor, name, dtype or
    tuple of dtypes, shape or None, optional).  Every tensor's dtype, shape and
    contiguity are checked first, then every tensor's device; the first problem
    raises ValueError naming the field."""
    for t, name, dtypes, shape, optional in specs:
        if t is None:
            if optional:
                continue
            raise ValueError(f"{name} is required")
        dtypes = dtypes if isinstance(dtypes, tuple) else (dtypes,)
        if t.dtype not in dtypes:
            raise ValueError(f"{name}: dtype {t.dtype}, expected {' or '.join(str(d) for d in dtypes)}")
        if shape is not None and tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    for t, name, _, _, _ in specs:
        if t is not None and not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")


def _tokens(t, name, H, d):
    """Token count of a [..., H, d] tensor (any leading token dimensions)."""
    if t.dim() < 2 or tuple(t.shape[-2:]) != (H, d):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected [..., {H}, {d}]")
    return t.numel() // (H * d)


# ------------------------------------------------------------------ entry points

def mla_absorb_q(q_nope, w_uk, q_lat, stream=None):
    """q_lat[t][h] = W_UK[h]^T q_nope[t][h]; q_nope [n_tok][H][128], w_uk [H][128][512],
    q_lat [n_tok][H][512], all bf16 on the device."""
    import torch
    H = w_uk.shape[0]
    n_tok = _tokens(q_nope, "q_nope", H, D_N)
    if _tokens(q_lat, "q_lat", H, D_C) != n_tok:
        raise ValueError("q_lat must hold as many tokens as q_nope")
    _want([(q_nope, "q_nope", torch.bfloat16, None, False), (w_uk, "w_uk", torch.bfloat16, (H, D_N, D_C), False),
           (q_lat, "q_lat", torch.bfloat16, None, False)])
    _check("mla_absorb_q", load().mla_absorb_q(_ptr(q_nope), _ptr(w_uk), _ptr(q_lat), n_tok, H,
                                               w_uk.shape[1], w_uk.shape[2], _stream(stream)))


def mla_up_proj_v(o_lat, w_uv, out, stream=None):
    """out[t][h] = W_UV[h] o_lat[t][h]; o_lat [n_tok][H][512], w_uv [H][128][512],
    out [n_tok][H][128], all bf16 on the device."""
    import torch
    H = w_uv.shape[0]
    n_tok = _tokens(o_lat, "o_lat", H, D_C)
    if _tokens(out, "out", H, D_V) != n_tok:
        raise ValueError("out must hold as many tokens as o_lat")
    _want([(o_lat, "o_lat", torch.bfloat16, None, False), (w_uv, "w_uv", torch.bfloat16, (H, D_V, D_C), False),
           (out, "out", torch.bfloat16, None, False)])
    _check("mla_up_proj_v", load().mla_up_proj_v(_ptr(o_lat), _ptr(w_uv), _ptr(out), n_tok, H,
                                                 w_uv.shape[1], w_uv.shape[2], _stream(stream)))


def mla_fold_hadamard(w_dkv=None, w_uk=None, w_uv=None, stream=None):
    """Folds the orthonormal 512-point Hadamard rotation into the weights, in place:
    w_dkv [576][d_h] (rows 0..511 -> H W_DKV), w_uk and w_uv [H][128][512] (each row
    -> row H); bf16 on the device, any of them may be None."""
    import torch
    H = (w_uk if w_uk is not None else w_uv).shape[0] if (w_uk is not None or w_uv is not None) else 0
    d_h = w_dkv.shape[1] if w_dkv is not None else 0
    _want([(w_dkv, "w_dkv", torch.bfloat16, (D_C + D_R, d_h), True),
           (w_uk, "w_uk", torch.bfloat16, (H, D_N, D_C), True),
           (w_uv, "w_uv", torch.bfloat16, (H, D_V, D_C), True)])
    _check("mla_fold_hadamard", load().mla_fold_hadamard(_ptr(w_dkv), d_h, _ptr(w_uk), _ptr(w_uv), H,
                                                         _stream(stream)))


def _cache_kind(kv_cache):
    """(kv_dtype code, scale dtype, scale shape tail, row width) of a cache tensor's
    dtype: bf16 values; float8_e4m3fn codes with fp32 row scales [pages][64]; int8
    q8_0 codes with fp16 block scales [pages][64][18]; uint8 q4_0 bytes (two codes
    a byte, 288 a row) with fp16 block scales [pages][64][18]."""
    import torch
    if kv_cache.dtype == torch.float8_e4m3fn:
        return KV_FP8_E4M3, torch.float32, (), D_C + D_R
    if kv_cache.dtype == torch.int8:
        return KV_Q8_0, torch.float16, (Q8_BLOCKS,), D_C + D_R
    if kv_cache.dtype == torch.uint8:
        return KV_Q4_0, torch.float16, (Q8_BLOCKS,), (D_C + D_R) // 2
    return KV_BF16, None, (), D_C + D_R


def make_decode_args(*, q_lat, q_pe, kv_cache, kv_scale, block_table, seq_lens, o_lat, lse,
                     workspace=None, causal=False, softmax_scale, num_splits=0,
                     max_seq_len=0) -> DecodeArgs:
    """Fill a ``DecodeArgs`` from device tensors.  Shapes: q_lat [B][s_q][H][512],
    q_pe [B][s_q][H][64], kv_cache [num_pages][64][576] (bf16, float8_e4m3fn or
    int8 for q8_0) or [num_pages][64][288] uint8 (q4_0), kv_scale [num_pages][64]
    fp32 (e4m3), [num_pages][64][18] fp16 (q8_0, q4_0) or None (bf16), block_table
    [B][max_pages] int32, seq_lens [B] int32, o_lat like q_lat, lse [B][s_q][H]
    fp32 or None."""
    import torch
    bf16, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    if q_lat.dim() != 4 or kv_cache.dim() != 3 or block_table.dim() != 2:
        raise ValueError("q_lat must be [B][s_q][H][512], kv_cache [pages][64][576], block_table [B][pages]")
    B, s_q, H, _ = q_lat.shape
    P = kv_cache.shape[0]
    kind, sc_dtype, sc_tail, width = _cache_kind(kv_cache)
    _want([(q_lat, "q_lat", bf16, (B, s_q, H, D_C), False),
           (q_pe, "q_pe", bf16, (B, s_q, H, D_R), False),
           (kv_cache, "kv_cache", (bf16, torch.float8_e4m3fn, torch.int8, torch.uint8), (P, PAGE, width), False),
           (kv_scale, "kv_scale", sc_dtype or f32, (P, PAGE) + sc_tail, kind == KV_BF16),
           (block_table, "block_table", i32, (B, block_table.shape[1]), False),
           (seq_lens, "seq_lens", i32, (B,), False),
           (o_lat, "o_lat", bf16, (B, s_q, H, D_C), False),
           (lse, "lse", f32, (B, s_q, H), True),
           (workspace, "workspace", torch.uint8, None, True)])
    a = DecodeArgs()
    a.q_lat, a.q_pe = _ptr(q_lat), _ptr(q_pe)
    a.kv_cache, a.kv_scale = _ptr(kv_cache), _ptr(kv_scale)
    a.block_table, a.seq_lens = _ptr(block_table), _ptr(seq_lens)
    a.o_lat, a.lse = _ptr(o_lat), _ptr(lse)
    a.B, a.s_q, a.H = B, s_q, H
    a.d_c, a.d_r, a.page_size = D_C, D_R, PAGE
    a.num_pages = kv_cache.shape[0]
    a.max_pages_per_seq = block_table.shape[1]
    a.kv_dtype = kind
    a.causal = int(bool(causal))
    a.num_splits = int(num_splits)
    a.max_seq_len = int(max_seq_len)
    a.softmax_scale = float(softmax_scale)
    if workspace is not None:
        a.workspace, a.workspace_bytes = _ptr(workspace), workspace.numel() * workspace.element_size()
    return a


def mla_decode_workspace_size(args: DecodeArgs) -> int:
    n = ctypes.c_size_t(0)
    _check("mla_decode_workspace_size", load().mla_decode_workspace_size(ctypes.byref(args), ctypes.byref(n)))
    return int(n.value)


def mla_decode_num_splits(args: DecodeArgs) -> int:
    n = ctypes.c_int32(0)
    _check("mla_decode_num_splits", load().mla_decode_num_splits(ctypes.byref(args), ctypes.byref(n)))
    return int(n.value)


def mla_decode_paged(args: DecodeArgs, stream=None):
    _check("mla_decode_paged", load().mla_decode_paged(ctypes.byref(args), _stream(stream)))


def mla_combine_splits(args: DecodeArgs, stream=None):
    _check("mla_combine_splits", load().mla_combine_splits(ctypes.byref(args), _stream(stream)))


def mla_decode_paged_noalloc(args: DecodeArgs, stream=None):
    """Decode plus split merge with the library's built-in scratch (args.workspace is
    ignored); for callers that cannot allocate device memory."""
    _check("mla_decode_paged_noalloc", load().mla_decode_paged_noalloc(ctypes.byref(args), _stream(stream)))


def mla_noalloc_init():
    """Set-up of the built-in scratch on the current device (address lookup, status
    word zeroed); call at start-up, before any stream capture."""
    _check("mla_noalloc_init", load().mla_noalloc_init())


def mla_get_status_noalloc(stream=None) -> int:
    """Waits for the stream and returns (and clears) the built-in scratch's device
    status word."""
    return int(load().mla_get_status_noalloc(_stream(stream)))


def mla_set_decode_kernel(kernel: int):
    """Process-wide decode kernel choice: DECODE_AUTO or DECODE_WARP_MMA."""
    _check("mla_set_decode_kernel", load().mla_set_decode_kernel(int(kernel)))


def mla_set_device_wait_limit(ns: int):
    """Process-wide limit of the decode kernels' bounded waits (0: the 2 s default)."""
    _check("mla_set_device_wait_limit", load().mla_set_device_wait_limit(int(ns)))


def make_write_kv_args(*, h, w_dkv, kv_cache, kv_scale, block_table, seq_lens, workspace=None,
                       rope_base=10000.0) -> WriteKvArgs:
    """Fill a ``WriteKvArgs`` from device tensors.  Shapes: h [B][s_q][d_h] bf16,
    w_dkv [576][d_h] bf16 (W_DKV rows, then W_KR rows), kv_cache [num_pages][64][576]
    (bf16, float8_e4m3fn or int8 for q8_0) or [num_pages][64][288] uint8 (q4_0),
    kv_scale [num_pages][64] fp32 (e4m3), [num_pages][64][18] fp16 (q8_0, q4_0) or
    None (bf16), block_table [B][max_pages] int32, seq_lens [B] int32."""
    import torch
    bf16, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    if h.dim() != 3 or kv_cache.dim() != 3 or block_table.dim() != 2:
        raise ValueError("h must be [B][s_q][d_h], kv_cache [pages][64][576], block_table [B][pages]")
    B, s_q, d_h = h.shape
    P = kv_cache.shape[0]
    kind, sc_dtype, sc_tail, width = _cache_kind(kv_cache)
    _want([(h, "h", bf16, (B, s_q, d_h), False),
           (w_dkv, "w_dkv", bf16, (D_C + D_R, d_h), False),
           (kv_cache, "kv_cache", (bf16, torch.float8_e4m3fn, torch.int8, torch.uint8), (P, PAGE, width), False),
           (kv_scale, "kv_scale", sc_dtype or f32, (P, PAGE) + sc_tail, kind == KV_BF16),
           (block_table, "block_table", i32, (B, block_table.shape[1]), False),
           (seq_lens, "seq_lens", i32, (B,), False),
           (workspace, "workspace", torch.uint8, None, True)])
    a = WriteKvArgs()
    a.h, a.w_dkv = _ptr(h), _ptr(w_dkv)
    a.kv_cache, a.kv_scale = _ptr(kv_cache), _ptr(kv_scale)
    a.block_table, a.seq_lens = _ptr(block_table), _ptr(seq_lens)
    a.B, a.s_q, a.d_h = B, s_q, d_h
    a.d_c, a.d_r, a.page_size = D_C, D_R, PAGE
    a.num_pages = kv_cache.shape[0]
    a.max_pages_per_seq = block_table.shape[1]
    a.kv_dtype = kind
    a.rope_base = float(rope_base)
    if workspace is not None:
        a.workspace, a.workspace_bytes = _ptr(workspace), workspace.numel() * workspace.element_size()
    return a


def mla_write_kv_workspace_size(args: WriteKvArgs) -> int:
    n = ctypes.c_size_t(0)
    _check("mla_write_kv_workspace_size", load().mla_write_kv_workspace_size(ctypes.byref(args), ctypes.byref(n)))
    return int(n.value)


def mla_write_kv(args: WriteKvArgs, stream=None):
    """Appends the new tokens' latent and RoPE key rows to the paged cache."""
    _check("mla_write_kv", load().mla_write_kv(ctypes.byref(args), _stream(stream)))


def make_step_args(*, q_nope, q_pe, w_uk, w_uv, kv_cache, kv_scale, block_table, seq_lens, out, lse,
                   workspace=None, causal=False, softmax_scale, num_splits=0, max_seq_len=0,
                   fuse=0) -> StepArgs:
    """Fill a ``StepArgs`` (the whole decode step, ``mla_decode_step``) from device
    tensors.  Shapes: q_nope [B][s_q][H][128], q_pe [B][s_q][H][64], w_uk and w_uv
    [H][128][512] bf16; the cache, scales, block table and lengths as for
    ``make_decode_args``; out [B][s_q][H][128] bf16, lse [B][s_q][H] fp32 or None;
    fuse: 0 automatic, 1 one launch wherever possible, -1 never."""
    import torch
    bf16, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    if q_nope.dim() != 4 or kv_cache.dim() != 3 or block_table.dim() != 2:
        raise ValueError("q_nope must be [B][s_q][H][128], kv_cache [pages][64][row], block_table [B][pages]")
    B, s_q, H, _ = q_nope.shape
    P = kv_cache.shape[0]
    kind, sc_dtype, sc_tail, width = _cache_kind(kv_cache)
    _want([(q_nope, "q_nope", bf16, (B, s_q, H, D_N), False),
           (q_pe, "q_pe", bf16, (B, s_q, H, D_R), False),
           (w_uk, "w_uk", bf16, (H, D_N, D_C), False),
           (w_uv, "w_uv", bf16, (H, D_V, D_C), False),
           (kv_cache, "kv_cache", (bf16, torch.float8_e4m3fn, torch.int8, torch.uint8), (P, PAGE, width), False),
           (kv_scale, "kv_scale", sc_dtype or f32, (P, PAGE) + sc_tail, kind == KV_BF16),
           (block_table, "block_table", i32, (B, block_table.shape[1]), False),
           (seq_lens, "seq_lens", i32, (B,), False),
           (out, "out", bf16, (B, s_q, H, D_V), False),
           (lse, "lse", f32, (B, s_q, H), True),
           (workspace, "workspace", torch.uint8, None, True)])
    a = StepArgs()
    a.q_nope, a.q_pe, a.w_uk, a.w_uv = _ptr(q_nope), _ptr(q_pe), _ptr(w_uk), _ptr(w_uv)
    a.kv_cache, a.kv_scale = _ptr(kv_cache), _ptr(kv_scale)
    a.block_table, a.seq_lens = _ptr(block_table), _ptr(seq_lens)
    a.out, a.lse = _ptr(out), _ptr(lse)
    a.B, a.s_q, a.H = B, s_q, H
    a.d_c, a.d_r, a.page_size = D_C, D_R, PAGE
    a.num_pages = P
    a.max_pages_per_seq = block_table.shape[1]
    a.kv_dtype = kind
    a.causal = int(bool(causal))
    a.num_splits = int(num_splits)
    a.max_seq_len = int(max_seq_len)
    a.softmax_scale = float(softmax_scale)
    a.fuse = int(fuse)
    if workspace is not None:
        a.workspace, a.workspace_bytes = _ptr(workspace), workspace.numel() * workspace.element_size()
    return a


def mla_decode_step_workspace_size(args: StepArgs) -> int:
    n = ctypes.c_size_t(0)
    _check("mla_decode_step_workspace_size",
           load().mla_decode_step_workspace_size(ctypes.byref(args), ctypes.byref(n)))
    return int(n.value)


def mla_decode_step_launches(args: StepArgs) -> int:
    """Kernel launches one mla_decode_step call makes (1: fused)."""
    n = ctypes.c_int32(0)
    _check("mla_decode_step_launches", load().mla_decode_step_launches(ctypes.byref(args), ctypes.byref(n)))
    return int(n.value)


def mla_decode_step(args: StepArgs, stream=None):
    """The whole decode step (absorption, decode, split merge, up-projection)."""
    _check("mla_decode_step", load().mla_decode_step(ctypes.byref(args), _stream(stream)))


def make_prefill_args(*, q_nope, q_pe, w_uk, w_uv, kv_cache, block_table, seq_lens, out, lse,
                      max_seq_len, workspace=None, causal=True, softmax_scale) -> PrefillArgs:
    """Fill a ``PrefillArgs`` from device tensors.  Shapes: q_nope [B][s_q][H][128],
    q_pe [B][s_q][H][64], w_uk [H][128][512], w_uv [H][128][512], kv_cache
    [num_pages][64][576] bf16, block_table [B][max_pages] int32, seq_lens [B] int32,
    out [B][s_q][H][128] bf16, lse [B][s_q][H] fp32 or None; max_seq_len bounds
    seq_lens and sizes the workspace."""
    import torch
    bf16, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    if q_nope.dim() != 4 or kv_cache.dim() != 3 or block_table.dim() != 2:
        raise ValueError("q_nope must be [B][s_q][H][128], kv_cache [pages][64][576], block_table [B][pages]")
    B, s_q, H, _ = q_nope.shape
    P = kv_cache.shape[0]
    _want([(q_nope, "q_nope", bf16, (B, s_q, H, D_N), False),
           (q_pe, "q_pe", bf16, (B, s_q, H, D_R), False),
           (w_uk, "w_uk", bf16, (H, D_N, D_C), False),
           (w_uv, "w_uv", bf16, (H, D_V, D_C), False),
           (kv_cache, "kv_cache", bf16, (P, PAGE, D_C + D_R), False),
           (block_table, "block_table", i32, (B, block_table.shape[1]), False),
           (seq_lens, "seq_lens", i32, (B,), False),
           (out, "out", bf16, (B, s_q, H, D_V), False),
           (lse, "lse", f32, (B, s_q, H), True),
           (workspace, "workspace", torch.uint8, None, True)])
    a = PrefillArgs()
    a.q_nope, a.q_pe, a.w_uk, a.w_uv = _ptr(q_nope), _ptr(q_pe), _ptr(w_uk), _ptr(w_uv)
    a.kv_cache = _ptr(kv_cache)
    a.block_table, a.seq_lens = _ptr(block_table), _ptr(seq_lens)
    a.out, a.lse = _ptr(out), _ptr(lse)
    a.B, a.s_q, a.H = B, s_q, H
    a.d_c, a.d_r, a.page_size = D_C, D_R, PAGE
    a.num_pages = P
    a.max_pages_per_seq = block_table.shape[1]
    a.kv_dtype = KV_BF16
    a.causal = int(bool(causal))
    a.max_seq_len = int(max_seq_len)
    a.softmax_scale = float(softmax_scale)
    if workspace is not None:
        a.workspace, a.workspace_bytes = _ptr(workspace), workspace.numel() * workspace.element_size()
    return a


def mla_prefill_workspace_size(args: PrefillArgs) -> int:
    n = ctypes.c_size_t(0)
    _check("mla_prefill_workspace_size", load().mla_prefill_workspace_size(ctypes.byref(args), ctypes.byref(n)))
    return int(n.value)


def mla_prefill(args: PrefillArgs, stream=None):
    """Explicit-form attention of the s_q new tokens of every sequence (per-head
    keys and values formed in the workspace, then a FlashAttention forward)."""
    _check("mla_prefill", load().mla_prefill(ctypes.byref(args), _stream(stream)))


def mla_get_status(workspace, stream=None) -> int:
    """Waits for the stream and returns (and clears) the device status word."""
    return int(load().mla_get_status(_ptr(workspace), _stream(stream)))


def mla_status_string(code: int) -> str:
    return load().mla_status_string(int(code)).decode()


def alloc_workspace(args, device="cuda"):
    """A zeroed workspace tensor sized for ``args`` (``DecodeArgs``,
    ``WriteKvArgs`` or ``PrefillArgs``); also stored into ``args``."""
    import torch
    if isinstance(args, WriteKvArgs):
        n = mla_write_kv_workspace_size(args)
    elif isinstance(args, StepArgs):
        n = mla_decode_step_workspace_size(args)
    elif isinstance(args, PrefillArgs):
        n = mla_prefill_workspace_size(args)
    else:
        n = mla_decode_workspace_size(args)
    ws = torch.zeros(n, dtype=torch.uint8, device=device)
    args.workspace, args.workspace_bytes = _ptr(ws), n
    return ws
