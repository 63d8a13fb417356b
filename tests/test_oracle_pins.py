"""Pins for the fp64 oracle: facts fixed by the pages and by mathematics, none of
which re-types the oracle's own formula.

* storage formats against torch's own casts (library routines);
* fp8 round trip within e4m3's half-ulp;
* absorbed form == explicit-K/V definition (the weight-absorbing identity);
* single cached token -> o = W_UV c_0, lse = the one score (closed form);
* zero query -> uniform weights: o = mean of V, lse = log n exactly;
* torch's scaled_dot_product_attention on explicitly built K, V (library routine);
* causal reduction, page-permutation invariance, split/LSE identity.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from oracle import mla_oracle as om
from mla_inputs import WorkloadSpec, make_workload, bf16_bits, SOFTMAX_SCALE


def _bf16(x):
    return bf16_bits(torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16))


def _small(kv="bf16", s_q=1, causal=False, lens=(1, 70, 130), H=4, seed=11, keep_raw=False,
           permute=True):
    spec = WorkloadSpec("pin", B=len(lens), H=H, s_q=s_q, lens=list(lens), kv_dtype=kv,
                        causal=causal, seed=seed, permute_pages=permute)
    return make_workload(spec, keep_raw=keep_raw)


# ---------------------------------------------------------------- formats

def test_bf16_decode_matches_torch_cast():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 1 << 16, size=200000, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):
        ours = om.bf16_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(ours))
    assert np.array_equal(ours[~nan], ref[~nan])


def test_e4m3_decode_matches_torch_cast_all_codes():
    bits = np.arange(256, dtype=np.uint8)
    ours = om.e4m3fn_to_f64(bits)
    ref = torch.from_numpy(bits).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert nan.sum() == 2                      # 0x7F and 0xFF
    assert np.array_equal(nan, np.isnan(ours))
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.nanmax(ours) == 448.0 and om.e4m3fn_to_f64(np.uint8(1)) == 2.0 ** -9


def test_fp8_round_trip_within_half_ulp():
    w = _small(kv="fp8", keep_raw=True, lens=(1, 64, 200))
    inp = oracle.from_workload(w)
    for b, L in enumerate(w.lens):
        got = inp.rows(b, L)
        pages = w.block_table[b, :(L + 63) // 64].long()
        raw = w.raw_rows[pages].reshape(-1, 576)[:L].double().numpy()
        scale = w.kv_scale[pages].reshape(-1)[:L].double().numpy()[:, None]
        x = raw / scale                                   # value before the cast
        bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10) * scale
        assert np.all(np.abs(got - raw) <= bound * (1 + 1e-6))
        assert np.all(np.abs(x) <= 448.0 * (1 + 1e-6))


# ---------------------------------------------------------------- P1 absorbed == definition

@pytest.mark.parametrize("kv,s_q,causal", [("bf16", 1, False), ("bf16", 2, True), ("fp8", 2, True)])
def test_absorbed_equals_nonabsorbed(kv, s_q, causal):
    w = _small(kv=kv, s_q=s_q, causal=causal, lens=(2, 70, 130))
    inp = oracle.from_workload(w)
    a = om.decode_absorbed(inp)
    n = om.decode_nonabsorbed(inp)
    for k in ("o", "o_lat", "lse"):
        assert np.all(np.isfinite(a[k])) and np.all(np.isfinite(n[k]))
        err = np.abs(a[k] - n[k]).max() / max(1e-300, np.abs(n[k]).max())
        assert err < 1e-12, (k, err)


# ---------------------------------------------------------------- P2 single token

def test_single_token_closed_form():
    w = _small(lens=(1,), H=3)
    inp = oracle.from_workload(w)
    # q_nope = 0 and q_pe = a e_5  =>  the only score is scale * a * k_pe_0[5]
    inp.q_nope[:] = 0.0
    inp.q_pe[:] = 0.0
    inp.q_pe[0, 0, :, 5] = 2.5
    c0 = inp.rows(0, 1)[0]
    out = om.decode_nonabsorbed(inp)
    for h in range(3):
        np.testing.assert_allclose(out["o"][0, 0, h], inp.w_uv[h] @ c0[:512], rtol=1e-13, atol=1e-15)
        np.testing.assert_array_equal(out["o_lat"][0, 0, h], c0[:512])
        assert out["lse"][0, 0, h] == pytest.approx(SOFTMAX_SCALE * 2.5 * c0[512 + 5], rel=1e-14)
    # with a random query, one token still gives o = W_UV c_0 exactly (weight 1)
    inp2 = oracle.from_workload(w)
    out2 = om.decode_nonabsorbed(inp2)
    np.testing.assert_allclose(out2["o"][0, 0], inp2.w_uv @ c0[:512], rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- P3 uniform weights

@pytest.mark.parametrize("kv,s_q,causal", [("bf16", 1, False), ("fp8", 2, True)])
def test_zero_query_gives_mean_of_v_and_log_n(kv, s_q, causal):
    w = _small(kv=kv, s_q=s_q, causal=causal, lens=(3, 64, 129))
    inp = oracle.from_workload(w)
    inp.q_nope[:] = 0.0
    inp.q_pe[:] = 0.0
    out = om.decode_nonabsorbed(inp)
    for b in range(inp.B):
        for i in range(s_q):
            n = inp.visible(b, i)
            C = inp.rows(b, n)
            mean_c = C[:, :512].mean(axis=0)
            assert np.all(out["lse"][b, i] == math.log(n))
            np.testing.assert_allclose(out["o_lat"][b, i], np.broadcast_to(mean_c, (inp.H, 512)),
                                       rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(out["o"][b, i], inp.w_uv @ mean_c, rtol=1e-11, atol=1e-14)


# ---------------------------------------------------------------- P4 library attention

@pytest.mark.parametrize("kv,s_q,causal", [("bf16", 1, False), ("bf16", 2, True), ("fp8", 2, True)])
def test_matches_torch_sdpa_on_explicit_kv(kv, s_q, causal):
    w = _small(kv=kv, s_q=s_q, causal=causal, lens=(5, 97, 190), H=3)
    inp = oracle.from_workload(w)
    out = om.decode_nonabsorbed(inp)
    for b in range(inp.B):
        L = int(inp.seq_lens[b])
        C = torch.from_numpy(inp.rows(b, L))
        for h in range(inp.H):
            K = torch.cat([C[:, :512] @ torch.from_numpy(inp.w_uk[h]).T, C[:, 512:]], dim=1)
            V = C[:, :512] @ torch.from_numpy(inp.w_uv[h]).T
            Q = torch.cat([torch.from_numpy(inp.q_nope[b, :, h]), torch.from_numpy(inp.q_pe[b, :, h])], 1)
            mask = torch.ones(s_q, L, dtype=torch.bool)
            if causal:
                pos = torch.arange(L)[None, :]
                mask = pos <= (L - s_q + torch.arange(s_q))[:, None]
            ref = torch.nn.functional.scaled_dot_product_attention(
                Q[None, None], K[None, None], V[None, None], attn_mask=mask[None, None],
                scale=SOFTMAX_SCALE)[0, 0]
            logits = (Q @ K.T) * SOFTMAX_SCALE
            lse = torch.logsumexp(logits.masked_fill(~mask, -math.inf), dim=1)
            np.testing.assert_allclose(out["o"][b, :, h], ref.numpy(), rtol=1e-11, atol=1e-13)
            np.testing.assert_allclose(out["lse"][b, :, h], lse.numpy(), rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- P5 causal reduction

def test_causal_query0_equals_shorter_context():
    lens = (2, 65, 128)
    w2 = _small(s_q=2, causal=True, lens=lens)
    inp2 = oracle.from_workload(w2)
    out2 = om.decode_absorbed(inp2)
    inp1 = oracle.from_workload(w2)
    inp1.s_q = 1
    inp1.causal = False
    inp1.q_nope = inp2.q_nope[:, :1].copy()
    inp1.q_pe = inp2.q_pe[:, :1].copy()
    inp1.seq_lens = inp2.seq_lens - 1
    out1 = om.decode_absorbed(inp1)
    for k in ("o", "o_lat", "lse"):
        np.testing.assert_array_equal(out2[k][:, 0], out1[k][:, 0])
    # the last query sees the whole context
    inp3 = oracle.from_workload(w2)
    inp3.s_q, inp3.causal = 1, False
    inp3.q_nope, inp3.q_pe = inp2.q_nope[:, 1:].copy(), inp2.q_pe[:, 1:].copy()
    out3 = om.decode_absorbed(inp3)
    np.testing.assert_array_equal(out2["lse"][:, 1], out3["lse"][:, 0])


def test_causal_multi_token_equals_single_token_prefixes():
    """Eight new tokens with the causal mask (a chunked-prefill shape): query i
    gives exactly the one-query result over the first L - 8 + i + 1 tokens,
    through the definition itself."""
    s_q = 8
    w = _small(s_q=s_q, causal=True, lens=(8, 70, 140), H=2)
    inp = oracle.from_workload(w)
    out = om.decode_nonabsorbed(inp)
    for i in range(s_q):
        one = oracle.from_workload(w)
        one.s_q, one.causal = 1, False
        one.q_nope = inp.q_nope[:, i:i + 1].copy()
        one.q_pe = inp.q_pe[:, i:i + 1].copy()
        one.seq_lens = inp.seq_lens - s_q + i + 1
        ref = om.decode_nonabsorbed(one)
        for k in ("o", "o_lat", "lse"):
            np.testing.assert_array_equal(out[k][:, i], ref[k][:, 0])


# ---------------------------------------------------------------- P6 paging invariance

@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_page_permutation_invariance(kv):
    a = oracle.from_workload(_small(kv=kv, permute=False, lens=(70, 200, 1)))
    b = oracle.from_workload(_small(kv=kv, permute=True, lens=(70, 200, 1)))
    assert not np.array_equal(a.block_table, b.block_table)
    oa, ob = om.decode_nonabsorbed(a), om.decode_nonabsorbed(b)
    for k in ("o", "o_lat", "lse"):
        np.testing.assert_array_equal(oa[k], ob[k])


# ---------------------------------------------------------------- P7 split identity

def test_split_lse_combine_identity():
    w = _small(lens=(300,), H=5)
    inp = oracle.from_workload(w)
    q_lat = om.absorb_q(inp.q_nope, inp.w_uk)[0, 0]
    C = inp.rows(0, 300)
    whole_o, whole_lse = om.latent_attention(q_lat, inp.q_pe[0, 0], C, inp.softmax_scale)
    cuts = [0, 1, 64, 64, 200, 300]       # includes an empty range
    parts = [om.latent_attention(q_lat, inp.q_pe[0, 0], C[a:b], inp.softmax_scale)
             for a, b in zip(cuts[:-1], cuts[1:])]
    o, lse = om.combine_splits([p[0] for p in parts], [p[1] for p in parts])
    np.testing.assert_allclose(o, whole_o, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, whole_lse, rtol=1e-13)
    # every split empty -> zeros and -inf
    o0, l0 = om.combine_splits(np.zeros((3, 5, 512)), np.full((3, 5), -np.inf))
    assert np.all(o0 == 0) and np.all(l0 == -np.inf)


# ---------------------------------------------------------------- edge cases

def test_empty_context_is_zero_and_minus_inf():
    w = _small(lens=(0, 5))
    inp = oracle.from_workload(w)
    for fn in (om.decode_nonabsorbed, om.decode_absorbed):
        out = fn(inp)
        assert np.all(out["o"][0] == 0) and np.all(out["o_lat"][0] == 0)
        assert np.all(out["lse"][0] == -np.inf)
        assert np.all(np.isfinite(out["o"][1]))
    # causal with fewer cached tokens than queries: query 0 of a length-1
    # sequence with s_q = 2 sees nothing, query 1 sees one token
    w2 = _small(lens=(1,), s_q=2, causal=True)
    inp2 = oracle.from_workload(w2)
    out2 = om.decode_nonabsorbed(inp2)
    assert np.all(out2["lse"][0, 0] == -np.inf) and np.all(out2["o"][0, 0] == 0)
    c0 = inp2.rows(0, 1)[0]
    np.testing.assert_allclose(out2["o"][0, 1], inp2.w_uv @ c0[:512], rtol=1e-13, atol=1e-15)


def test_tail_rows_of_last_page_are_not_attended():
    # positions >= L in the last page hold 50x values; changing them must not matter
    w = _small(lens=(70,), H=2)
    inp = oracle.from_workload(w)
    before = om.decode_nonabsorbed(inp)
    page = int(inp.block_table[0, 1])
    inp.kv = inp.kv.copy()
    inp.kv[page, 6:] = _bf16(np.full((58, 576), 7.0))
    after = om.decode_nonabsorbed(inp)
    np.testing.assert_array_equal(before["o"], after["o"])


@pytest.mark.parametrize("name", ["v3", "ragged", "fp8"])
def test_absorbed_equals_definition_on_full_size_samples(name):
    """The absorbed mode (the one the full-size GPU comparisons use) agrees with the
    non-absorbed definition on sampled rows of the full-size workloads: the
    shortest and longest sequence and one more, two heads each, to 1e-10."""
    from mla_inputs import preset
    w = make_workload(preset(name))
    inp = oracle.from_workload(w)
    lens = np.asarray(w.lens)
    bs = sorted({int(np.argmin(lens)), int(np.argmax(lens)), len(lens) // 3})
    rows = [(b, i) for b in bs for i in range(w.s_q)]
    heads = [0, w.H - 1]
    a = om.decode_absorbed(inp, rows=rows, heads=heads)
    d = om.decode_nonabsorbed(inp, rows=rows, heads=heads)
    for b, i in rows:
        for key in ("o", "o_lat"):
            x, y = a[key][b, i, heads], d[key][b, i, heads]
            assert np.linalg.norm(x - y) <= 1e-10 * max(np.linalg.norm(y), 1e-300), (name, b, i, key)
        x, y = a["lse"][b, i, heads], d["lse"][b, i, heads]
        assert np.all(np.abs(x - y) <= 1e-10 * np.maximum(np.abs(y), 1.0))
