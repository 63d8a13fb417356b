"""Pins for the cache-write oracle (``oracle/cache_write.py``): facts fixed by the
storage formats, by the mathematics of the rotary embedding and by brute force,
none of which re-types the oracle's own formulas.

* the bf16 and e4m3 encoders against torch's casts (library routines), ties
  included, and the e4m3 encoder as the inverse of the decoder on every code;
* per-row e4m3 quantisation against the torch route the input generator uses;
* RoPE: identity at position 0, norm of every pair kept, pair 0 turning by
  exactly ``pos`` radians, a geometric ladder of frequencies, the
  relative-position identity and composition of rotations;
* the paged write by brute force (only the new rows change, page order is
  addressing only) and its error cases;
* the whole write read back through the decode oracle: one cached token gives
  ``o = W_UV c`` with ``c = W_DKV h`` (closed form);
* the q8_0 and q4_0 row quantisers against the low-bit oracle's blockwise
  quantiser, q4_0's zero block, extremes and packing by hand, and the paged
  q8_0 / q4_0 writes by brute force.
"""

import numpy as np
import pytest
import torch

from oracle import cache_write as cw
from oracle import mla_oracle as om


# ---------------------------------------------------------------- encoders

def _e4m3_grid():
    codes = np.arange(256, dtype=np.uint8)
    vals = om.e4m3fn_to_f64(codes)
    keep = ~np.isnan(vals)
    return codes[keep], vals[keep]


def test_e4m3_encoder_inverts_the_decoder_on_every_code():
    codes, vals = _e4m3_grid()
    assert np.array_equal(cw.f64_to_e4m3fn(vals), codes)       # -0.0 keeps its sign bit
    assert cw.f64_to_e4m3fn(np.nan) & 0x7F == 0x7F


def test_e4m3_encoder_matches_torch_cast_with_ties_and_saturation():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(100000) * 50.0,
                        rng.standard_normal(20000) * 2.0 ** -7,      # subnormal range
                        [0.0, -0.0, 448.0, -448.0, 1e6, -1e6, 464.0, 449.0]]).astype(np.float32)
    # exact midpoints between neighbouring positive codes: ties go to the even code
    _, vals = _e4m3_grid()
    pos = np.unique(vals[vals > 0])
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids])
    clipped = np.clip(x, -448.0, 448.0)
    ref = torch.from_numpy(clipped).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(cw.f64_to_e4m3fn(x.astype(np.float64)), ref)


def test_bf16_encoder_matches_torch_cast_with_ties():
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-30, 30, 100000),
                        [0.0, -0.0, 1.0, -3.0]]).astype(np.float32)
    # fp32 values exactly half-way between two bf16 values (low 16 bits 0x8000)
    ties = ((rng.integers(0x3F00, 0x4100, 5000, dtype=np.uint32) << 16) | 0x8000).view(np.float32)
    x = np.concatenate([x, ties, -ties])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(cw.f64_to_bf16(x.astype(np.float64)), ref)


def test_row_quantisation_matches_the_torch_route():
    from mla_inputs.workloads import _quantise_rows_e4m3
    rng = np.random.default_rng(3)
    rows = (rng.standard_normal((64, cw.ROW)) * rng.uniform(1e-3, 1e3, (64, 1))).astype(np.float32)
    rows[5] = 0.0                                               # the all-zero row: scale 1
    q_ref, s_ref = _quantise_rows_e4m3(torch.from_numpy(rows))
    q_ref = q_ref.view(torch.uint8).numpy()
    s_ref = s_ref.reshape(-1).numpy()
    for r in range(rows.shape[0]):
        q, s = cw.quantise_row_e4m3(rows[r].astype(np.float64))
        assert s == s_ref[r]
        assert np.array_equal(q, q_ref[r])
    q, s = cw.quantise_row_e4m3(rows[0])
    amax_at = np.argmax(np.abs(rows[0]))
    assert q[amax_at] & 0x7F == 0x7E                           # the largest value maps to +-448


# ---------------------------------------------------------------- RoPE

def test_rope_closed_forms():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((5, cw.D_R))
    assert np.array_equal(cw.rope(x, np.zeros(5)), x)           # position 0: identity
    p = np.array([1, 7, 100, 4095, 131071])
    y = cw.rope(x, p)
    # every pair keeps its length
    assert np.allclose(np.hypot(y[:, 0::2], y[:, 1::2]), np.hypot(x[:, 0::2], x[:, 1::2]), rtol=1e-13)
    # pair 0 turns by exactly p radians (its frequency is base**0 = 1)
    e = np.zeros((5, cw.D_R))
    e[:, 0] = 1.0
    z = cw.rope(e, p)
    assert np.allclose(z[:, 0], np.cos(p), atol=1e-12) and np.allclose(z[:, 1], np.sin(p), atol=1e-12)


def test_rope_frequencies_form_a_geometric_ladder():
    # the angle of each pair after one position, read back with atan2: pair 0
    # turns 1 radian, the last pair turns base**(-(d-2)/d), and neighbouring pairs
    # differ by the constant ratio base**(-2/d)
    e = np.zeros((cw.D_R // 2, cw.D_R))
    for i in range(cw.D_R // 2):
        e[i, 2 * i] = 1.0
    z = cw.rope(e, np.ones(cw.D_R // 2))
    ang = np.array([np.arctan2(z[i, 2 * i + 1], z[i, 2 * i]) for i in range(cw.D_R // 2)])
    ratio = ang[1:] / ang[:-1]
    assert ang[0] == pytest.approx(1.0, abs=1e-14)
    assert np.allclose(ratio, ratio[0], rtol=1e-12)
    assert ratio[0] ** (cw.D_R // 2) == pytest.approx(1.0 / 10000.0, rel=1e-10)


def test_rope_scores_depend_on_relative_position_only():
    rng = np.random.default_rng(5)
    q, k = rng.standard_normal(cw.D_R), rng.standard_normal(cw.D_R)
    for m, n in [(10, 3), (4100, 4096), (131071, 5), (7, 7)]:
        lhs = cw.rope(q, m) @ cw.rope(k, n)
        rhs = cw.rope(q, m - n) @ k
        assert lhs == pytest.approx(rhs, rel=1e-9, abs=1e-9)
    x = rng.standard_normal(cw.D_R)
    assert np.allclose(cw.rope(cw.rope(x, 37), 1000), cw.rope(x, 1037), atol=1e-10)


# ---------------------------------------------------------------- paged write

def _setup(kv_dtype, lens, s_q, d_h=96, num_pages=20, seed=6):
    rng = np.random.default_rng(seed)
    B = len(lens)
    max_pages = 4
    pages = rng.permutation(num_pages)[:B * max_pages].reshape(B, max_pages)
    if kv_dtype == "bf16":
        kv = rng.integers(0, 1 << 16, (num_pages, cw.PAGE, cw.ROW), dtype=np.uint32).astype(np.uint16)
        scale = None
    else:
        kv = rng.integers(0, 0x78, (num_pages, cw.PAGE, cw.ROW), dtype=np.uint8)
        scale = rng.uniform(0.1, 2.0, (num_pages, cw.PAGE)).astype(np.float32)
    h = rng.standard_normal((B, s_q, d_h))
    w_dkv = rng.standard_normal((cw.D_C, d_h)) / np.sqrt(d_h)
    w_kr = rng.standard_normal((cw.D_R, d_h)) / np.sqrt(d_h)
    return h, w_dkv, w_kr, kv, scale, pages.astype(np.int64), np.array(lens, dtype=np.int64)


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
def test_only_the_new_rows_change(kv_dtype):
    lens, s_q = [1, 64, 65, 200], 1
    h, w_dkv, w_kr, kv, scale, bt, sl = _setup(kv_dtype, lens, s_q)
    kv2, scale2 = cw.write_kv(h, w_dkv, w_kr, kv, scale, kv_dtype, bt, sl, s_q)
    touched = np.zeros(kv.shape[:2], dtype=bool)
    for b, L in enumerate(lens):
        pos = L - 1
        page, row = bt[b, pos // 64], pos % 64
        touched[page, row] = True
        # brute force: the row holds c = W_DKV h and the rotated W_KR h
        want = np.concatenate([w_dkv @ h[b, 0], cw.rope(w_kr @ h[b, 0], pos)])
        if kv_dtype == "bf16":
            got = om.bf16_to_f64(kv2[page, row])
            assert np.allclose(got, want, rtol=2.0 ** -8, atol=0)
        else:
            got = om.e4m3fn_to_f64(kv2[page, row]) * np.float64(scale2[page, row])
            assert np.all(np.abs(got - want) <= 2.0 ** -4 * np.abs(want) + 2.0 ** -9 * scale2[page, row])
    assert np.array_equal(kv2[~touched], kv[~touched])
    if scale is not None:
        assert np.array_equal(scale2[~touched], scale[~touched])


def test_two_new_tokens_land_at_the_end_of_the_sequence():
    lens, s_q = [2, 66, 130], 2
    h, w_dkv, w_kr, kv, scale, bt, sl = _setup("bf16", lens, s_q)
    kv2, _ = cw.write_kv(h, w_dkv, w_kr, kv, scale, "bf16", bt, sl, s_q)
    for b, L in enumerate(lens):
        for i in range(s_q):
            pos = L - s_q + i
            want = np.concatenate([w_dkv @ h[b, i], cw.rope(w_kr @ h[b, i], pos)])
            got = om.bf16_to_f64(kv2[bt[b, pos // 64], pos % 64])
            assert np.allclose(got, want, rtol=2.0 ** -8, atol=0)


def test_page_order_is_addressing_only():
    lens, s_q = [70, 5], 1
    h, w_dkv, w_kr, kv, scale, bt, sl = _setup("fp8", lens, s_q)
    kv_a, sc_a = cw.write_kv(h, w_dkv, w_kr, kv, scale, "fp8", bt, sl, s_q)
    perm = np.random.default_rng(9).permutation(kv.shape[0])     # physical page p -> perm[p]
    kv_p = np.empty_like(kv)
    sc_p = np.empty_like(scale)
    kv_p[perm], sc_p[perm] = kv, scale
    kv_b, sc_b = cw.write_kv(h, w_dkv, w_kr, kv_p, sc_p, "fp8", perm[bt], sl, s_q)
    assert np.array_equal(kv_b[perm], kv_a) and np.array_equal(sc_b[perm], sc_a)


def test_write_errors():
    h, w_dkv, w_kr, kv, scale, bt, sl = _setup("bf16", [1, 10], 2)
    with pytest.raises(ValueError):                              # length 1 < 2 new tokens
        cw.write_kv(h, w_dkv, w_kr, kv, scale, "bf16", bt, sl, 2)
    h, w_dkv, w_kr, kv, scale, bt, sl = _setup("bf16", [300], 1)
    with pytest.raises(ValueError):                              # beyond the 4-page table
        cw.write_kv(h, w_dkv, w_kr, kv, scale, "bf16", bt, sl, 1)
    h, w_dkv, w_kr, kv, scale, bt, sl = _setup("bf16", [3], 1)
    bt[0, 0] = kv.shape[0]
    with pytest.raises(ValueError):                              # page id outside the cache
        cw.write_kv(h, w_dkv, w_kr, kv, scale, "bf16", bt, sl, 1)


# ---------------------------------------------------------------- read back

def test_single_written_token_decodes_to_w_uv_c():
    rng = np.random.default_rng(10)
    d_h, H = 64, 2
    h, w_dkv, w_kr, kv, scale, bt, sl = _setup("bf16", [1], 1, d_h=d_h)
    kv2, _ = cw.write_kv(h, w_dkv, w_kr, kv, scale, "bf16", bt, sl, 1)
    to_bits = lambda a: cw.f64_to_bf16(a)
    q_nope = to_bits(rng.standard_normal((1, 1, H, 128)))
    q_pe = to_bits(rng.standard_normal((1, 1, H, 64)))
    w_uk = to_bits(rng.standard_normal((H, 128, 512)) / np.sqrt(512))
    w_uv = to_bits(rng.standard_normal((H, 128, 512)) / np.sqrt(512))
    inp = om.OracleInputs(q_nope, q_pe, w_uk, w_uv, kv2, "bf16", None, bt, sl,
                          1.0 / np.sqrt(192.0), False)
    out = om.decode_nonabsorbed(inp)
    c = w_dkv @ h[0, 0]
    k_pe = cw.rope(w_kr @ h[0, 0], 0)                             # position 0: unrotated
    for hh in range(H):
        o_want = om.bf16_to_f64(w_uv[hh]) @ c
        assert np.allclose(out["o"][0, 0, hh], o_want, rtol=0, atol=2e-2 * np.abs(o_want).max())
        s = (om.bf16_to_f64(q_nope[0, 0, hh]) @ (om.bf16_to_f64(w_uk[hh]) @ c)
             + om.bf16_to_f64(q_pe[0, 0, hh]) @ k_pe) / np.sqrt(192.0)
        assert out["lse"][0, 0, hh] == pytest.approx(s, rel=2e-2, abs=2e-2)


def test_q8_0_row_quantisation_matches_the_blockwise_format():
    """The cache write's q8_0 row (fp32 arithmetic) against the low-bit oracle's
    blockwise quantiser (fp64): scales equal, codes equal except where an fp32
    quotient falls on the other side of a rounding boundary than the exact one."""
    from oracle import lowbit_cache as lb
    rng = np.random.default_rng(11)
    diff = 0
    for _ in range(200):
        row = rng.standard_normal(576) * rng.uniform(0.01, 50.0)
        row32 = row.astype(np.float32).astype(np.float64)
        codes, d = cw.quantise_row_q8_0(row)
        ref_codes, ref_d = lb.quantise_blocks(row32, "q8_0")
        assert np.array_equal(d.astype(np.float64), ref_d)
        diff += int((codes.astype(np.int64) != ref_codes).sum())
        assert np.abs(codes.astype(np.int64) - ref_codes).max() <= 1
    assert diff <= 2e-4 * 200 * 576


def test_q8_0_write_touches_only_the_new_rows():
    rng = np.random.default_rng(12)
    B, s_q, d_h, P = 2, 2, 64, 6
    h = rng.standard_normal((B, s_q, d_h))
    w_dkv, w_kr = rng.standard_normal((512, d_h)) / 8, rng.standard_normal((64, d_h)) / 8
    kv = rng.integers(-127, 128, size=(P, 64, 576)).astype(np.int8)
    sc = rng.random((P, 64, 18)).astype(np.float16)
    bt = np.array([[3, 1], [0, 5]])
    lens = np.array([66, 10])
    kv2, sc2 = cw.write_kv(h, w_dkv, w_kr, kv, sc, "q8_0", bt, lens, s_q)
    changed = np.argwhere((kv2 != kv).any(axis=2) | (sc2 != sc).any(axis=2))
    assert sorted(map(tuple, changed)) == [(0, 8), (0, 9), (1, 0), (1, 1)]
    # the written row decodes to the compressed row within half a step per block
    c, kr = cw.compress(h[0], w_dkv, w_kr)
    full = np.concatenate([c[1], cw.rope(kr, np.array([65]), 10000.0)[1]])
    got = kv2[1, 1].astype(np.float64) * np.repeat(sc2[1, 1].astype(np.float64), 32)
    step = np.repeat(sc2[1, 1].astype(np.float64), 32)
    assert np.all(np.abs(got - full) <= 0.5 * step + 1e-3 * np.abs(full) + 1e-9)


def _unpack_q4(packed: np.ndarray) -> np.ndarray:
    """Codes of a packed q4_0 row: value 2j in the low four bits of byte j, value
    2j + 1 in the high four, each stored as code + 8."""
    b = packed.astype(np.int64)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.int64)
    out[..., 0::2] = (b & 15) - 8
    out[..., 1::2] = (b >> 4) - 8
    return out


def test_q4_0_row_quantisation_matches_the_blockwise_format():
    """The cache write's q4_0 row (fp32 arithmetic, packed) against the low-bit
    oracle's blockwise quantiser (fp64): scales equal, codes equal except where an
    fp32 quotient falls on the other side of a rounding boundary."""
    from oracle import lowbit_cache as lb
    rng = np.random.default_rng(13)
    diff = 0
    for _ in range(200):
        row = rng.standard_normal(576) * rng.uniform(0.01, 50.0)
        row32 = row.astype(np.float32).astype(np.float64)
        packed, d = cw.quantise_row_q4_0(row)
        assert packed.shape == (288,) and packed.dtype == np.uint8
        codes = _unpack_q4(packed)
        ref_codes, ref_d = lb.quantise_blocks(row32, "q4_0")
        assert np.array_equal(d.astype(np.float64), ref_d)
        diff += int((codes != ref_codes).sum())
        assert np.abs(codes - ref_codes).max() <= 1
    assert diff <= 2e-4 * 200 * 576


def test_q4_0_zero_block_and_extremes():
    row = np.zeros(576)
    row[32:64] = np.linspace(-3.5, 7.0, 32)          # block 1: amax 7 -> d = 1
    packed, d = cw.quantise_row_q4_0(row)
    codes = _unpack_q4(packed)
    assert d[0] == 0 and np.all(codes[:32] == 0)      # an all-zero block: zero codes
    assert d[1] == 1.0 and codes[63] == 7 and codes[32] == -4  # -3.5 rounds to even
    assert packed[0] == 0x88                          # two zero codes: 8 | 8 << 4


def test_q4_0_write_touches_only_the_new_rows():
    rng = np.random.default_rng(14)
    B, s_q, d_h, P = 2, 2, 64, 6
    h = rng.standard_normal((B, s_q, d_h))
    w_dkv, w_kr = rng.standard_normal((512, d_h)) / 8, rng.standard_normal((64, d_h)) / 8
    kv = rng.integers(0, 256, size=(P, 64, 288)).astype(np.uint8)
    sc = rng.random((P, 64, 18)).astype(np.float16)
    bt = np.array([[3, 1], [0, 5]])
    lens = np.array([66, 10])
    kv2, sc2 = cw.write_kv(h, w_dkv, w_kr, kv, sc, "q4_0", bt, lens, s_q)
    changed = np.argwhere((kv2 != kv).any(axis=2) | (sc2 != sc).any(axis=2))
    assert sorted(map(tuple, changed)) == [(0, 8), (0, 9), (1, 0), (1, 1)]
    c, kr = cw.compress(h[0], w_dkv, w_kr)
    full = np.concatenate([c[1], cw.rope(kr, np.array([65]), 10000.0)[1]])
    step = np.repeat(sc2[1, 1].astype(np.float64), 32)
    got = _unpack_q4(kv2[1, 1]) * step
    assert np.all(np.abs(got - full) <= 0.5 * step + 1e-3 * np.abs(full) + 1e-9)
