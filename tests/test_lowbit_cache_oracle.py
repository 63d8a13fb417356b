"""Pins for the low-bit cache oracle (``oracle/lowbit_cache.py``).

* the Hadamard matrix against scipy's construction (library routine), its
  orthonormality and symmetry;
* folding the rotation into W_DKV, W_UK and W_UV leaves attention unchanged: the
  rotated cache with the folded weights gives the plain output and lse, and the
  latent output comes out rotated (an identity of orthonormal matrices);
* blockwise q8_0 / q4_0: every value within half a step of its block (plus the
  fp16 rounding of the scale), block extremes on the outermost code, zero blocks,
  blocks independent of one another;
* the pages' claim that the rotation helps at low bit widths, on rows with an
  outlier: the q4_0 error after rotate -> quantise -> rotate back is smaller;
* the decode oracle's q8_0 and q4_0 caches: rows read back as the blockwise
  dequantisation of the raw draw, a hand-made q4_0 row pins the byte layout, a
  q4_0 cache equals a q8_0 cache holding the same codes, and the absorbed form
  equals the definition over both.
"""

import numpy as np
import pytest
import scipy.linalg

from oracle import lowbit_cache as lb
from oracle import mla_oracle as om


@pytest.mark.parametrize("n", [1, 2, 64, 512])
def test_hadamard_matches_scipy(n):
    ref = scipy.linalg.hadamard(n).astype(np.float64) / np.sqrt(n)
    assert np.array_equal(lb.hadamard(n), ref)


def test_hadamard_is_orthonormal_and_symmetric():
    h = lb.hadamard(512)
    assert np.allclose(h @ h.T, np.eye(512), atol=1e-12)
    assert np.array_equal(h, h.T)


def test_folded_weights_leave_attention_unchanged():
    rng = np.random.default_rng(0)
    H, n, d_h = 4, 150, 96
    q_nope = rng.standard_normal((H, 128))
    q_pe = rng.standard_normal((H, 64))
    w_uk = rng.standard_normal((H, 128, 512)) / np.sqrt(512)
    w_uv = rng.standard_normal((H, 128, 512)) / np.sqrt(512)
    w_dkv = rng.standard_normal((512, d_h)) / np.sqrt(d_h)
    hs = rng.standard_normal((n, d_h))
    C = np.concatenate([hs @ w_dkv.T, rng.standard_normal((n, 64))], axis=1)
    scale = 1 / np.sqrt(192)
    o_lat, lse = om.latent_attention(om.absorb_q(q_nope, w_uk), q_pe, C, scale)
    o = om.up_proj_v(o_lat, w_uv)
    f_dkv, f_uk, f_uv = lb.fold_hadamard(w_dkv, w_uk, w_uv)
    C_rot = lb.rotate_latent(C)
    # the cache written with the folded W_DKV is the rotated cache
    assert np.allclose(hs @ f_dkv.T, C_rot[:, :512], atol=1e-12)
    o_lat2, lse2 = om.latent_attention(om.absorb_q(q_nope, f_uk), q_pe, C_rot, scale)
    o2 = om.up_proj_v(o_lat2, f_uv)
    assert np.allclose(lse2, lse, atol=1e-12)
    assert np.allclose(o2, o, atol=1e-12)
    assert np.allclose(o_lat2, o_lat @ lb.hadamard(512).T, atol=1e-12)


@pytest.mark.parametrize("kind,levels", [("q8_0", 127), ("q4_0", 7)])
def test_blocks_within_half_a_step(kind, levels):
    rng = np.random.default_rng(1)
    x = rng.standard_normal(576) * np.repeat(rng.uniform(1e-3, 1e2, 18), 32)
    x[32:64] = 0.0                                           # a zero block
    q, d = lb.quantise_blocks(x, kind)
    assert q.shape == (576,) and d.shape == (18,)
    assert np.all(np.abs(q) <= levels)
    assert d[1] == 0 and np.all(q[32:64] == 0)
    y = lb.dequantise_blocks(q, d)
    bound = np.repeat(d / 2 + levels * d * 2.0 ** -10, 32)
    assert np.all(np.abs(y - x) <= bound)
    # the largest magnitude of each non-zero block sits on the outermost code
    for b in range(18):
        if d[b] > 0:
            j = 32 * b + np.argmax(np.abs(x[32 * b:32 * b + 32]))
            assert abs(q[j]) == levels
    # fp16 scales
    assert np.array_equal(d, d.astype(np.float16).astype(np.float64))


def test_blocks_are_independent():
    rng = np.random.default_rng(2)
    x = rng.standard_normal(576)
    q, d = lb.quantise_blocks(x, "q8_0")
    x2 = x.copy()
    x2[:32] *= 1000.0                                        # change block 0 only
    q2, d2 = lb.quantise_blocks(x2, "q8_0")
    assert np.array_equal(q2[32:], q[32:]) and np.array_equal(d2[1:], d[1:])


def test_rotation_reduces_low_bit_error_with_outliers():
    rng = np.random.default_rng(3)
    h = lb.hadamard(512)
    err_plain, err_rot = 0.0, 0.0
    for _ in range(50):
        c = rng.standard_normal(512)
        c[rng.integers(0, 512, 3)] *= 30.0                   # a few outlier channels
        q, d = lb.quantise_blocks(c, "q4_0")
        err_plain += np.sum((lb.dequantise_blocks(q, d) - c) ** 2)
        q, d = lb.quantise_blocks(h @ c, "q4_0")
        err_rot += np.sum((h.T @ lb.dequantise_blocks(q, d) - c) ** 2)
    assert err_rot < 0.5 * err_plain


# ---------------------------------------------------------------- q8_0 cache in the decode oracle

def test_f16_decoder_matches_numpy_on_every_code():
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = om.f16_to_f64(bits)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])


def _q8_workload(lens=(70, 130), H=16, seed=3):
    from mla_inputs import WorkloadSpec, make_workload
    return make_workload(WorkloadSpec("q8", B=len(lens), H=H, s_q=1, lens=list(lens), kv_dtype="q8_0",
                                      seed=seed), keep_raw=True)


def test_q8_0_cache_rows_are_the_blockwise_dequantisation():
    """The decode oracle reads a q8_0 cache row as code * block scale: the same
    values the low-bit oracle's quantiser gives for the raw fp32 draw."""
    import oracle
    w = _q8_workload()
    inp = oracle.from_workload(w)
    raw = w.raw_rows.double().numpy()
    for b, L in enumerate(w.lens):
        C = inp.rows(b, L)
        for j in (0, 31, L - 1):
            pg, rr = int(w.block_table[b, j // 64]), j % 64
            codes, d = lb.quantise_blocks(raw[pg, rr], "q8_0")
            assert np.array_equal(C[j], lb.dequantise_blocks(codes, d))
            # every value within half a step of its block (plus the fp16 rounding of d)
            step = np.repeat(d, 32)
            assert np.all(np.abs(C[j] - raw[pg, rr]) <= 0.5 * step + 1e-3 * np.abs(raw[pg, rr]) + 1e-12)


def test_q8_0_decode_absorbed_equals_the_definition():
    import oracle
    w = _q8_workload(lens=(1, 200), H=16)
    inp = oracle.from_workload(w)
    a = om.decode_absorbed(inp)
    d = om.decode_nonabsorbed(inp)
    for key in ("o", "o_lat", "lse"):
        assert np.allclose(a[key], d[key], rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- q4_0 cache in the decode oracle

def _q4_workload(lens=(70, 130), H=16, seed=3):
    from mla_inputs import WorkloadSpec, make_workload
    return make_workload(WorkloadSpec("q4", B=len(lens), H=H, s_q=1, lens=list(lens), kv_dtype="q4_0",
                                      seed=seed), keep_raw=True)


def test_q4_0_byte_layout():
    """One hand-made row: byte 0 = 0x1F holds code 15 - 8 = 7 (value 0, low four
    bits) and 1 - 8 = -7 (value 1, high four bits); byte 0x88 is two zeros."""
    kv = np.full((1, 64, 288), 0x88, dtype=np.uint8)
    kv[0, 0, 0] = 0x1F
    kv[0, 0, 17] = 0xA3                              # values 34, 35: 3 - 8, 10 - 8
    sc = np.zeros((1, 64, 18), dtype=np.float16)
    sc[0, 0, :] = 0.5
    sc[0, 0, 1] = 2.0
    z = np.zeros((1, 1, 16, 128), dtype=np.uint16)
    inp = om.OracleInputs(z, np.zeros((1, 1, 16, 64), np.uint16), np.zeros((16, 128, 512), np.uint16),
                          np.zeros((16, 128, 512), np.uint16), kv, "q4_0", sc.view(np.uint16),
                          np.zeros((1, 1), np.int64), np.array([1]), 1.0, False)
    row = inp.rows(0, 1)[0]
    want = np.zeros(576)
    want[0], want[1] = 3.5, -3.5
    want[34], want[35] = -10.0, 4.0
    assert np.array_equal(row, want)


def test_q4_0_cache_rows_are_the_blockwise_dequantisation():
    """The decode oracle reads a q4_0 row as code * block scale: the values the
    low-bit oracle's quantiser gives for the raw fp32 draw."""
    import oracle
    w = _q4_workload()
    inp = oracle.from_workload(w)
    raw = w.raw_rows.double().numpy()
    for b, L in enumerate(w.lens):
        C = inp.rows(b, L)
        for j in (0, 31, L - 1):
            pg, rr = int(w.block_table[b, j // 64]), j % 64
            codes, d = lb.quantise_blocks(raw[pg, rr], "q4_0")
            assert np.array_equal(C[j], lb.dequantise_blocks(codes, d))


def test_q4_0_equals_q8_0_on_the_same_codes():
    """A q4_0 cache and a q8_0 cache holding the same codes (all within [-7, 7])
    and scales give the same attention: the 4-bit storage is only addressing."""
    import oracle
    from mla_inputs import WorkloadSpec, make_workload
    w = make_workload(WorkloadSpec("q8", B=2, H=16, s_q=1, lens=[70, 130], kv_dtype="q8_0", seed=8))
    inp8 = oracle.from_workload(w)
    codes = np.clip(inp8.kv.view(np.int8).astype(np.int64), -7, 7)
    inp8.kv = codes.astype(np.int8).view(np.uint8)
    n = (codes + 8).astype(np.uint8)
    kv4 = n[..., 0::2] | (n[..., 1::2] << 4)
    from mla_inputs import bf16_bits, f16_bits
    inp4 = om.OracleInputs(bf16_bits(w.q_nope), bf16_bits(w.q_pe), bf16_bits(w.w_uk), bf16_bits(w.w_uv),
                           kv4, "q4_0", f16_bits(w.kv_scale), w.block_table.numpy(), w.seq_lens.numpy(),
                           w.softmax_scale, False)
    a, b = om.decode_absorbed(inp8), om.decode_absorbed(inp4)
    for key in ("o", "o_lat", "lse"):
        assert np.array_equal(a[key], b[key])


def test_q4_0_decode_absorbed_equals_the_definition():
    import oracle
    w = _q4_workload(lens=(1, 200), H=16)
    inp = oracle.from_workload(w)
    a = om.decode_absorbed(inp)
    d = om.decode_nonabsorbed(inp)
    for key in ("o", "o_lat", "lse"):
        assert np.allclose(a[key], d[key], rtol=1e-10, atol=1e-12)
