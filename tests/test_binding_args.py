"""Argument checks of the Python binding's tensor builders (CPU): dtype, shape,
contiguity and device are checked before any pointer reaches the C ABI."""

import pytest
import torch

import head_latent_attention_06_b200 as mla

bf16, f32, i32 = torch.bfloat16, torch.float32, torch.int32


def _decode_tensors(B=2, s_q=1, H=16, P=8, fp8=False):
    return dict(
        q_lat=torch.zeros(B, s_q, H, 512, dtype=bf16), q_pe=torch.zeros(B, s_q, H, 64, dtype=bf16),
        kv_cache=torch.zeros(P, 64, 576, dtype=torch.float8_e4m3fn if fp8 else bf16),
        kv_scale=torch.ones(P, 64, dtype=f32) if fp8 else None,
        block_table=torch.zeros(B, 4, dtype=i32), seq_lens=torch.ones(B, dtype=i32),
        o_lat=torch.zeros(B, s_q, H, 512, dtype=bf16), lse=torch.zeros(B, s_q, H, dtype=f32))


def _write_tensors(B=2, s_q=1, d_h=128, P=8, fp8=False):
    return dict(
        h=torch.zeros(B, s_q, d_h, dtype=bf16), w_dkv=torch.zeros(576, d_h, dtype=bf16),
        kv_cache=torch.zeros(P, 64, 576, dtype=torch.float8_e4m3fn if fp8 else bf16),
        kv_scale=torch.ones(P, 64, dtype=f32) if fp8 else None,
        block_table=torch.zeros(B, 4, dtype=i32), seq_lens=torch.ones(B, dtype=i32))


def test_decode_args_need_device_tensors():
    with pytest.raises(ValueError, match="q_lat must be a CUDA tensor"):
        mla.make_decode_args(**_decode_tensors(), softmax_scale=0.07)


@pytest.mark.parametrize("field,bad,msg", [
    ("q_lat", torch.zeros(2, 1, 16, 512, dtype=f32), "q_lat: dtype"),
    ("q_pe", torch.zeros(2, 1, 16, 32, dtype=bf16), "q_pe: shape"),
    ("kv_cache", torch.zeros(8, 32, 576, dtype=bf16), "kv_cache: shape"),
    ("block_table", torch.zeros(2, 4, dtype=torch.int64), "block_table: dtype"),
    ("seq_lens", torch.ones(3, dtype=i32), "seq_lens: shape"),
    ("o_lat", torch.zeros(2, 1, 16, 512, dtype=torch.float16), "o_lat: dtype"),
    ("lse", torch.zeros(2, 1, 8, dtype=f32), "lse: shape"),
    ("q_pe", torch.zeros(2, 1, 64, 16, dtype=bf16).transpose(2, 3), "q_pe must be contiguous"),
])
def test_decode_args_reject_bad_tensors(field, bad, msg):
    t = _decode_tensors()
    t[field] = bad
    with pytest.raises(ValueError, match=msg):
        mla.make_decode_args(**t, softmax_scale=0.07)


def test_decode_args_fp8_cache_needs_scales():
    t = _decode_tensors(fp8=True)
    t["kv_scale"] = None
    with pytest.raises(ValueError, match="kv_scale is required"):
        mla.make_decode_args(**t, softmax_scale=0.07)
    t["kv_scale"] = torch.ones(8, 64, dtype=torch.float64)
    with pytest.raises(ValueError, match="kv_scale: dtype"):
        mla.make_decode_args(**t, softmax_scale=0.07)


def test_write_kv_args_need_device_tensors():
    with pytest.raises(ValueError, match="h must be a CUDA tensor"):
        mla.make_write_kv_args(**_write_tensors())


@pytest.mark.parametrize("field,bad,msg", [
    ("h", torch.zeros(2, 1, 128, dtype=f32), "h: dtype"),
    ("w_dkv", torch.zeros(512, 128, dtype=bf16), "w_dkv: shape"),
    ("w_dkv", torch.zeros(576, 64, dtype=bf16), "w_dkv: shape"),
    ("kv_cache", torch.zeros(8, 64, 512, dtype=bf16), "kv_cache: shape"),
    ("seq_lens", torch.ones(2, dtype=torch.int64), "seq_lens: dtype"),
])
def test_write_kv_args_reject_bad_tensors(field, bad, msg):
    t = _write_tensors()
    t[field] = bad
    with pytest.raises(ValueError, match=msg):
        mla.make_write_kv_args(**t)


def test_write_kv_args_fp8_cache_needs_scales():
    t = _write_tensors(fp8=True)
    t["kv_scale"] = None
    with pytest.raises(ValueError, match="kv_scale is required"):
        mla.make_write_kv_args(**t)


def test_projection_calls_check_shapes_before_the_device():
    H = 4
    q = torch.zeros(3, H, 128, dtype=bf16)
    w = torch.zeros(H, 128, 512, dtype=bf16)
    with pytest.raises(ValueError, match="q_lat must hold as many tokens"):
        mla.mla_absorb_q(q, w, torch.zeros(2, H, 512, dtype=bf16))
    with pytest.raises(ValueError, match="w_uk: shape"):
        mla.mla_absorb_q(q, torch.zeros(H, 128, 256, dtype=bf16), torch.zeros(3, H, 512, dtype=bf16))
    with pytest.raises(ValueError, match="q_nope: shape"):
        mla.mla_absorb_q(torch.zeros(3, H, 64, dtype=bf16), w, torch.zeros(3, H, 512, dtype=bf16))
    with pytest.raises(ValueError, match="q_nope must be a CUDA tensor"):
        mla.mla_absorb_q(q, w, torch.zeros(3, H, 512, dtype=bf16))
    x = torch.zeros(3, H, 512, dtype=bf16)
    with pytest.raises(ValueError, match="out must hold as many tokens"):
        mla.mla_up_proj_v(x, w, torch.zeros(4, H, 128, dtype=bf16))
    with pytest.raises(ValueError, match="out: dtype"):
        mla.mla_up_proj_v(x, w, torch.zeros(3, H, 128, dtype=f32))


def _step_tensors(B=2, s_q=1, H=16, P=8, kind="bf16"):
    cache = {"bf16": torch.zeros(P, 64, 576, dtype=bf16), "q8_0": torch.zeros(P, 64, 576, dtype=torch.int8),
             "q4_0": torch.zeros(P, 64, 288, dtype=torch.uint8)}[kind]
    scale = None if kind == "bf16" else torch.ones(P, 64, 18, dtype=torch.float16)
    return dict(
        q_nope=torch.zeros(B, s_q, H, 128, dtype=bf16), q_pe=torch.zeros(B, s_q, H, 64, dtype=bf16),
        w_uk=torch.zeros(H, 128, 512, dtype=bf16), w_uv=torch.zeros(H, 128, 512, dtype=bf16),
        kv_cache=cache, kv_scale=scale, block_table=torch.zeros(B, 4, dtype=i32), seq_lens=torch.ones(B, dtype=i32),
        out=torch.zeros(B, s_q, H, 128, dtype=bf16), lse=torch.zeros(B, s_q, H, dtype=f32))


def test_step_args_need_device_tensors():
    with pytest.raises(ValueError, match="q_nope must be a CUDA tensor"):
        mla.make_step_args(**_step_tensors(), softmax_scale=0.07)


@pytest.mark.parametrize("field,bad,msg", [
    ("q_nope", torch.zeros(2, 1, 16, 128, dtype=f32), "q_nope: dtype"),
    ("w_uk", torch.zeros(16, 128, 256, dtype=bf16), "w_uk: shape"),
    ("w_uv", torch.zeros(8, 128, 512, dtype=bf16), "w_uv: shape"),
    ("out", torch.zeros(2, 1, 16, 512, dtype=bf16), "out: shape"),
    ("kv_cache", torch.zeros(8, 64, 576, dtype=torch.uint8), "kv_cache: shape"),   # uint8 is q4_0: 288 a row
])
def test_step_args_reject_bad_tensors(field, bad, msg):
    t = _step_tensors()
    t[field] = bad
    with pytest.raises(ValueError, match=msg):
        mla.make_step_args(**t, softmax_scale=0.07)


@pytest.mark.parametrize("kind", ["q8_0", "q4_0"])
def test_step_args_blockwise_cache_needs_fp16_block_scales(kind):
    t = _step_tensors(kind=kind)
    t["kv_scale"] = None
    with pytest.raises(ValueError, match="kv_scale is required"):
        mla.make_step_args(**t, softmax_scale=0.07)
    t["kv_scale"] = torch.ones(8, 64, dtype=torch.float16)
    with pytest.raises(ValueError, match="kv_scale: shape"):
        mla.make_step_args(**t, softmax_scale=0.07)


def test_fold_hadamard_checks_its_weights():
    with pytest.raises(ValueError, match="w_uk: shape"):
        mla.mla_fold_hadamard(w_uk=torch.zeros(4, 128, 256, dtype=bf16))
    with pytest.raises(ValueError, match="w_dkv must be a CUDA tensor"):
        mla.mla_fold_hadamard(w_dkv=torch.zeros(576, 128, dtype=bf16))
