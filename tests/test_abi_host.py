"""Host-side checks of the C ABI: the library loads without a GPU, exports every
symbol include/mla.h declares, and rejects bad arguments before touching the
device (no call here reaches a CUDA launch)."""

import ctypes
import os
import re
import subprocess

import pytest

import head_latent_attention_06_b200 as mla
from head_latent_attention_06_b200 import build as mla_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla.h")

OK, INVALID, UNSUPPORTED, MISALIGNED, WS_SMALL = 0, 1, 2, 3, 4


@pytest.fixture(scope="module")
def lib():
    mla_build.build()
    return mla.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_what_binding_expects():
    assert declared_functions() == sorted(mla.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", mla.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (mla_\w+)", out))
    for name in declared_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None


def test_status_strings(lib):
    for code, name in mla.STATUS.items():
        assert mla.mla_status_string(code) == name
    assert mla.mla_status_string(99) == "MLA_ERR_UNKNOWN"


def _args(B=2, s_q=1, H=128, splits=0, max_len=4096, **kw):
    a = mla.DecodeArgs()
    fake = 0x10000
    for f in ("q_lat", "q_pe", "kv_cache", "block_table", "seq_lens", "o_lat", "lse"):
        setattr(a, f, fake)
    a.B, a.s_q, a.H = B, s_q, H
    a.d_c, a.d_r, a.page_size = 512, 64, 64
    a.num_pages, a.max_pages_per_seq = 128, 64
    a.kv_dtype, a.causal, a.num_splits, a.max_seq_len = 0, 0, splits, max_len
    a.softmax_scale = 0.0722
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_workspace_size_is_host_only_and_grows_with_splits(lib):
    one = mla.mla_decode_workspace_size(_args(splits=1))
    assert one == 256
    four = mla.mla_decode_workspace_size(_args(splits=4))
    rows = 2 * 1 * 128 * 4
    assert four >= 256 + rows * 512 * 4 + rows * 4
    assert four % 256 == 0


def test_auto_split_count(lib):
    # few sequences, long context: many splits; a batch that fills the GPU: one
    assert mla.mla_decode_num_splits(_args(B=4, H=16, max_len=131072)) >= 16
    assert mla.mla_decode_num_splits(_args(B=4, H=128, max_len=131072)) >= 16
    assert mla.mla_decode_num_splits(_args(B=64, H=128, max_len=4096)) == 1
    assert mla.mla_decode_num_splits(_args(B=1, H=16, max_len=64)) == 1
    assert mla.mla_decode_num_splits(_args(B=4, H=16, splits=7)) == 7
    # e4m3 cache: the same model
    assert mla.mla_decode_num_splits(_args(B=4, H=128, max_len=131072, kv_dtype=1)) >= 16
    assert mla.mla_decode_num_splits(_args(B=128, H=128, max_len=8192, s_q=2, kv_dtype=1)) <= 2


@pytest.mark.parametrize("field,value,code", [
    ("d_c", 256, UNSUPPORTED), ("d_r", 32, UNSUPPORTED), ("page_size", 32, UNSUPPORTED),
    ("H", 24, UNSUPPORTED), ("H", 256, UNSUPPORTED), ("s_q", 1025, UNSUPPORTED),
    ("kv_dtype", 4, UNSUPPORTED), ("kv_dtype", -1, UNSUPPORTED), ("H", 0, INVALID), ("s_q", 0, INVALID),
    ("B", -1, INVALID),
    ("num_splits", 129, INVALID), ("max_pages_per_seq", 0, INVALID),
])
def test_decode_rejects_bad_shapes(lib, field, value, code):
    a = _args(**{field: value})
    assert lib.mla_decode_paged(ctypes.byref(a), None) == code
    assert lib.mla_combine_splits(ctypes.byref(a), None) == code
    n = ctypes.c_size_t(0)
    assert lib.mla_decode_workspace_size(ctypes.byref(a), ctypes.byref(n)) == code


def test_decode_rejects_bad_pointers_and_workspace(lib):
    a = _args()
    assert lib.mla_decode_paged(ctypes.byref(a), None) == INVALID          # no workspace
    a.workspace, a.workspace_bytes = 0x20001, 1 << 30
    assert lib.mla_decode_paged(ctypes.byref(a), None) == MISALIGNED
    a.workspace, a.workspace_bytes = 0x20000, 16
    a.num_splits = 4
    assert lib.mla_decode_paged(ctypes.byref(a), None) == WS_SMALL
    a.workspace_bytes = 1 << 30
    a.q_lat = None
    assert lib.mla_decode_paged(ctypes.byref(a), None) == INVALID
    a.q_lat = 0x10008
    assert lib.mla_decode_paged(ctypes.byref(a), None) == MISALIGNED
    a.q_lat = 0x10000
    a.kv_dtype, a.kv_scale = 1, None                                       # fp8 needs scales
    assert lib.mla_decode_paged(ctypes.byref(a), None) == INVALID


def test_decode_with_empty_batch_enqueues_nothing(lib):
    a = _args(B=0)
    a.workspace, a.workspace_bytes = 0x20000, 256
    assert lib.mla_decode_paged(ctypes.byref(a), None) == OK
    assert lib.mla_combine_splits(ctypes.byref(a), None) == OK


@pytest.mark.parametrize("fn", ["mla_absorb_q", "mla_up_proj_v"])
def test_projection_argument_checks(lib, fn):
    f = getattr(lib, fn)
    p = 0x10000
    assert f(p, p, p, 0, 128, 128, 512, None) == OK            # n_tok = 0: nothing to do
    assert f(p, p, p, 4, 128, 64, 512, None) == UNSUPPORTED
    assert f(p, p, p, 4, 128, 128, 256, None) == UNSUPPORTED
    assert f(p, p, p, -1, 128, 128, 512, None) == INVALID
    assert f(p, p, p, 4, 0, 128, 512, None) == INVALID
    assert f(None, p, p, 4, 128, 128, 512, None) == INVALID
    assert f(p, p + 2, p, 4, 128, 128, 512, None) == MISALIGNED


def test_get_status_rejects_null(lib):
    assert lib.mla_get_status(None, None) == INVALID


# ---------------------------------------------------------------- cache write

def _wargs(B=64, s_q=1, d_h=7168, **kw):
    a = mla.WriteKvArgs()
    fake = 0x10000
    for f in ("h", "w_dkv", "kv_cache", "block_table", "seq_lens"):
        setattr(a, f, fake)
    a.B, a.s_q, a.d_h = B, s_q, d_h
    a.d_c, a.d_r, a.page_size = 512, 64, 64
    a.num_pages, a.max_pages_per_seq = 4096, 64
    a.kv_dtype, a.rope_base = 0, 10000.0
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_write_kv_workspace_holds_the_split_partials(lib):
    # 64 tokens: 9 column tiles of one token block, split 16 ways along d_h
    assert mla.mla_write_kv_workspace_size(_wargs()) == 256 + 16 * 64 * 576 * 4
    # 4096 tokens fill the GPU without a split
    assert mla.mla_write_kv_workspace_size(_wargs(B=2048, s_q=2)) == 256 + 4096 * 576 * 4
    # never more splits than 64-wide chunks of d_h
    assert mla.mla_write_kv_workspace_size(_wargs(B=1, d_h=128)) == 256 + 2 * 576 * 4


@pytest.mark.parametrize("field,value,code", [
    ("d_c", 256, UNSUPPORTED), ("d_r", 32, UNSUPPORTED), ("page_size", 32, UNSUPPORTED),
    ("d_h", 100, UNSUPPORTED), ("kv_dtype", 5, UNSUPPORTED), ("d_h", 0, INVALID),
    ("s_q", 0, INVALID), ("B", -1, INVALID), ("max_pages_per_seq", 0, INVALID),
    ("rope_base", 0.0, INVALID), ("rope_base", float("nan"), INVALID), ("rope_base", float("inf"), INVALID),
])
def test_write_kv_rejects_bad_shapes(lib, field, value, code):
    a = _wargs(**{field: value})
    a.workspace, a.workspace_bytes = 0x20000, 1 << 30
    assert lib.mla_write_kv(ctypes.byref(a), None) == code
    n = ctypes.c_size_t(0)
    assert lib.mla_write_kv_workspace_size(ctypes.byref(a), ctypes.byref(n)) == code


def test_write_kv_rejects_bad_pointers_and_workspace(lib):
    a = _wargs()
    assert lib.mla_write_kv(ctypes.byref(a), None) == INVALID               # no workspace
    a.workspace, a.workspace_bytes = 0x20008, 1 << 30
    assert lib.mla_write_kv(ctypes.byref(a), None) == MISALIGNED
    a.workspace, a.workspace_bytes = 0x20000, 256
    assert lib.mla_write_kv(ctypes.byref(a), None) == WS_SMALL
    a.workspace_bytes = 1 << 30
    a.h = None
    assert lib.mla_write_kv(ctypes.byref(a), None) == INVALID
    a.h = 0x10008
    assert lib.mla_write_kv(ctypes.byref(a), None) == MISALIGNED
    a.h = 0x10000
    a.kv_dtype, a.kv_scale = 1, None                                        # e4m3 needs scales
    assert lib.mla_write_kv(ctypes.byref(a), None) == INVALID
    a.kv_scale = 0x30002
    assert lib.mla_write_kv(ctypes.byref(a), None) == MISALIGNED


def test_write_kv_with_empty_batch_enqueues_nothing(lib):
    a = _wargs(B=0)
    a.workspace, a.workspace_bytes = 0x20000, 256
    assert lib.mla_write_kv(ctypes.byref(a), None) == OK


# ---------------------------------------------------------------- prefill

def _pargs(B=4, s_q=1024, H=128, max_len=8192, **kw):
    a = mla.PrefillArgs()
    fake = 0x10000
    for f in ("q_nope", "q_pe", "w_uk", "w_uv", "kv_cache", "block_table", "seq_lens", "out", "lse"):
        setattr(a, f, fake)
    a.B, a.s_q, a.H = B, s_q, H
    a.d_c, a.d_r, a.page_size = 512, 64, 64
    a.num_pages, a.max_pages_per_seq = 512, 128
    a.kv_dtype, a.causal, a.max_seq_len = 0, 1, max_len
    a.softmax_scale = 0.0722
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_prefill_workspace_holds_keys_and_values(lib):
    # per-head keys and values (128 bf16 each) of every sequence, rows padded to 256
    assert mla.mla_prefill_workspace_size(_pargs()) == 256 + 2 * 4 * 128 * 8192 * 256
    assert mla.mla_prefill_workspace_size(_pargs(B=1, H=1, s_q=1, max_len=1)) == 256 + 2 * 256 * 256
    assert mla.mla_prefill_workspace_size(_pargs(B=2, H=16, s_q=100, max_len=129)) == 256 + 2 * 32 * 256 * 256


@pytest.mark.parametrize("field,value,code", [
    ("d_c", 256, UNSUPPORTED), ("d_r", 32, UNSUPPORTED), ("page_size", 32, UNSUPPORTED),
    ("kv_dtype", 1, UNSUPPORTED), ("kv_dtype", 2, UNSUPPORTED), ("kv_dtype", 3, UNSUPPORTED),
    ("H", 129, UNSUPPORTED),
    ("H", 0, INVALID), ("s_q", 0, INVALID), ("B", -1, INVALID), ("max_pages_per_seq", 0, INVALID),
    ("max_seq_len", 1023, INVALID), ("softmax_scale", float("nan"), INVALID),
    ("max_seq_len", 1 << 30, UNSUPPORTED), ("B", 65536, UNSUPPORTED),
])
def test_prefill_rejects_bad_shapes(lib, field, value, code):
    a = _pargs(**{field: value})
    a.workspace, a.workspace_bytes = 0x20000, 1 << 40
    assert lib.mla_prefill(ctypes.byref(a), None) == code
    n = ctypes.c_size_t(0)
    assert lib.mla_prefill_workspace_size(ctypes.byref(a), ctypes.byref(n)) == code


def test_prefill_rejects_bad_pointers_and_workspace(lib):
    a = _pargs()
    assert lib.mla_prefill(ctypes.byref(a), None) == INVALID                # no workspace
    a.workspace, a.workspace_bytes = 0x20008, 1 << 40
    assert lib.mla_prefill(ctypes.byref(a), None) == MISALIGNED
    a.workspace, a.workspace_bytes = 0x20000, 256
    assert lib.mla_prefill(ctypes.byref(a), None) == WS_SMALL
    a.workspace_bytes = 1 << 40
    for f in ("q_nope", "w_uv", "out"):
        setattr(a, f, None)
        assert lib.mla_prefill(ctypes.byref(a), None) == INVALID, f
        setattr(a, f, 0x10008)
        assert lib.mla_prefill(ctypes.byref(a), None) == MISALIGNED, f
        setattr(a, f, 0x10000)
    a.lse = 0x10002
    assert lib.mla_prefill(ctypes.byref(a), None) == MISALIGNED
    a.lse = None                                                            # lse is optional
    a.num_pages = 0
    assert lib.mla_prefill(ctypes.byref(a), None) == INVALID


def test_prefill_with_empty_batch_enqueues_nothing(lib):
    a = _pargs(B=0)
    a.workspace, a.workspace_bytes = 0x20000, 256
    assert lib.mla_prefill(ctypes.byref(a), None) == OK


def test_q4_0_cache_is_accepted_and_needs_scales(lib):
    a = _args(kv_dtype=3)
    n = ctypes.c_size_t(0)
    assert lib.mla_decode_workspace_size(ctypes.byref(a), ctypes.byref(n)) == OK
    a.workspace, a.workspace_bytes = 0x20000, 1 << 30
    a.kv_scale = None
    assert lib.mla_decode_paged(ctypes.byref(a), None) == INVALID
    a.kv_scale = 0x30002                                                   # fp16 scales: 4-byte aligned
    assert lib.mla_decode_paged(ctypes.byref(a), None) == MISALIGNED


def test_fold_hadamard_argument_checks(lib):
    f = lib.mla_fold_hadamard
    p = 0x10000
    assert f(None, 0, None, None, 0, None) == OK                   # nothing to fold
    assert f(p, 7168, p, p, -1, None) == INVALID
    assert f(p, 0, None, None, 0, None) == INVALID                 # w_dkv needs d_h > 0
    assert f(p, 100, None, None, 0, None) == UNSUPPORTED           # d_h a multiple of 64
    assert f(None, 0, p, p, 129, None) == UNSUPPORTED
    assert f(p + 8, 7168, None, None, 0, None) == MISALIGNED
    assert f(None, 0, p, p + 4, 16, None) == MISALIGNED


def _sargs(B=2, s_q=1, H=128, splits=0, max_len=4096, **kw):
    a = mla.StepArgs()
    fake = 0x10000
    for f in ("q_nope", "q_pe", "w_uk", "w_uv", "kv_cache", "block_table", "seq_lens", "out", "lse"):
        setattr(a, f, fake)
    a.B, a.s_q, a.H = B, s_q, H
    a.d_c, a.d_r, a.page_size = 512, 64, 64
    a.num_pages, a.max_pages_per_seq = 128, 64
    a.kv_dtype, a.causal, a.num_splits, a.max_seq_len = 0, 0, splits, max_len
    a.softmax_scale = 0.0722
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_step_workspace_holds_the_decode_flags_and_both_latents(lib):
    # the decode's part (256 bytes at one split), 256 bytes of flags, then q_lat and
    # o_lat (B * s_q * H * 512 bf16 each, 256-byte aligned)
    lat = 2 * 1 * 128 * 512 * 2
    assert mla.mla_decode_step_workspace_size(_sargs(splits=1)) == 256 + 256 + 2 * lat
    four = mla.mla_decode_step_workspace_size(_sargs(splits=4))
    assert four == mla.mla_decode_workspace_size(_args(splits=4)) + 256 + 2 * lat


@pytest.mark.parametrize("field,value,code", [
    ("d_c", 256, UNSUPPORTED), ("H", 24, UNSUPPORTED), ("s_q", 1025, UNSUPPORTED), ("kv_dtype", 4, UNSUPPORTED),
    ("H", 0, INVALID), ("B", -1, INVALID), ("num_splits", 129, INVALID),
])
def test_step_rejects_bad_shapes(lib, field, value, code):
    a = _sargs(**{field: value})
    a.workspace, a.workspace_bytes = 0x20000, 1 << 40
    assert lib.mla_decode_step(ctypes.byref(a), None) == code
    n = ctypes.c_size_t(0)
    assert lib.mla_decode_step_workspace_size(ctypes.byref(a), ctypes.byref(n)) == code
    k = ctypes.c_int32(0)
    assert lib.mla_decode_step_launches(ctypes.byref(a), ctypes.byref(k)) == code


def test_step_rejects_bad_pointers_and_workspace(lib):
    a = _sargs()
    assert lib.mla_decode_step(ctypes.byref(a), None) == INVALID              # no workspace
    a.workspace, a.workspace_bytes = 0x20008, 1 << 40
    assert lib.mla_decode_step(ctypes.byref(a), None) == MISALIGNED
    a.workspace, a.workspace_bytes = 0x20000, 1024
    assert lib.mla_decode_step(ctypes.byref(a), None) == WS_SMALL
    a.workspace_bytes = 1 << 40
    for f in ("q_nope", "w_uk", "w_uv", "out", "q_pe", "kv_cache"):
        setattr(a, f, None)
        assert lib.mla_decode_step(ctypes.byref(a), None) == INVALID, f
        setattr(a, f, 0x10008)
        assert lib.mla_decode_step(ctypes.byref(a), None) == MISALIGNED, f
        setattr(a, f, 0x10000)
    a.kv_dtype, a.kv_scale = 3, None                                         # q4_0 needs scales
    assert lib.mla_decode_step(ctypes.byref(a), None) == INVALID


def test_step_with_empty_batch_enqueues_nothing(lib):
    a = _sargs(B=0)
    a.workspace, a.workspace_bytes = 0x20000, 1024
    assert lib.mla_decode_step(ctypes.byref(a), None) == OK
    assert mla.mla_decode_step_launches(a) == 0
    # without a device the step is never fused: the four-kernel sequence (three at one split)
    assert mla.mla_decode_step_launches(_sargs(splits=1)) in (1, 3)
    assert mla.mla_decode_step_launches(_sargs(splits=4)) == 4
    assert mla.mla_decode_step_launches(_sargs(splits=1, kv_dtype=1)) == 3   # e4m3: never fused
    assert mla.mla_decode_step_launches(_sargs(splits=1, fuse=-1)) == 3
