"""GPU parity of mla_fold_hadamard (the 512-point orthonormal Hadamard rotation
folded into W_DKV, W_UK and W_UV; ik_llama.cpp docs "FlashMLA", section "KV
cache with MLA") against the fp64 low-bit oracle, and the rotation at work: a
q4_0 cache written and read with folded weights against the plain bf16 path.

Tolerance of the fold: each output is an fp32 transform rounded once to bf16,
so |gpu - oracle| <= 2^-8 |oracle| plus a fp32 summation term far below it
(bounded here by 1e-5 of the largest output)."""
import numpy as np
import pytest
import torch

from mla_inputs import bf16_bits
from oracle import lowbit_cache as lb
from oracle import mla_oracle as om

pytestmark = pytest.mark.gpu


def _weights(H, d_h, seed):
    g = torch.Generator().manual_seed(seed)
    w_dkv = (torch.randn(576, d_h, generator=g) / d_h ** 0.5).to(torch.bfloat16)
    w_uk = (torch.randn(H, 128, 512, generator=g) / 512 ** 0.5).to(torch.bfloat16)
    w_uv = (torch.randn(H, 128, 512, generator=g) / 512 ** 0.5).to(torch.bfloat16)
    return w_dkv, w_uk, w_uv


def _close(got, ref):
    d = np.abs(got - ref)
    assert np.all(d <= 2.0 ** -8 * np.abs(ref) + 1e-5 * np.abs(ref).max()), float(d.max())


@pytest.mark.parametrize("H,d_h", [(16, 1024), (128, 7168)])
def test_fold_matches_the_oracle(cuda_lib, H, d_h):
    import head_latent_attention_06_b200 as mla
    w_dkv, w_uk, w_uv = _weights(H, d_h, seed=H + d_h)
    g_dkv, g_uk, g_uv = w_dkv.cuda(), w_uk.cuda(), w_uv.cuda()
    mla.mla_fold_hadamard(g_dkv, g_uk, g_uv)
    torch.cuda.synchronize()
    f = lambda t: om.bf16_to_f64(bf16_bits(t))
    r_dkv, r_uk, r_uv = lb.fold_hadamard(f(w_dkv)[:512], f(w_uk), f(w_uv))
    got_dkv = f(g_dkv.cpu())
    _close(got_dkv[:512], r_dkv)
    assert np.array_equal(got_dkv[512:], f(w_dkv)[512:])          # the RoPE rows stay
    _close(f(g_uk.cpu()), r_uk)
    _close(f(g_uv.cpu()), r_uv)


def test_fold_skips_missing_weights_and_twice_restores(cuda_lib):
    import head_latent_attention_06_b200 as mla
    w_dkv, w_uk, w_uv = _weights(32, 512, seed=5)
    g_uk, g_uv = w_uk.cuda(), w_uv.cuda()
    mla.mla_fold_hadamard(None, g_uk, None)
    torch.cuda.synchronize()
    assert torch.equal(g_uv.cpu(), w_uv)
    mla.mla_fold_hadamard(None, g_uk, None)                        # H H = I
    torch.cuda.synchronize()
    a, b = om.bf16_to_f64(bf16_bits(g_uk.cpu())), om.bf16_to_f64(bf16_bits(w_uk))
    # two bf16 roundings of at most 2^-9 of each vector's L2 norm (H keeps norms)
    d = np.linalg.norm(a - b, axis=-1)
    assert np.all(d <= 1.01 * 2.0 ** -8 * np.linalg.norm(b, axis=-1) + 1e-6), float((d / np.linalg.norm(b, axis=-1)).max())


def _run_q4_path(cuda_lib, h, w_dkv, w_uk, w_uv, q_nope, q_pe, lens, fold):
    """Cache write (q4_0) of every token, then absorb, decode and up-projection
    through the C ABI; with ``fold`` the weights are folded first.  Returns the
    output and the written cache (bytes, scales)."""
    import head_latent_attention_06_b200 as mla
    B, L, d_h = h.shape
    P = B * ((L + 63) // 64)
    w_dkv, w_uk, w_uv = w_dkv.cuda(), w_uk.cuda(), w_uv.cuda()
    if fold:
        mla.mla_fold_hadamard(w_dkv, w_uk, w_uv)
    kv = torch.zeros(P, 64, 288, dtype=torch.uint8, device="cuda")
    sc = torch.zeros(P, 64, 18, dtype=torch.float16, device="cuda")
    bt = torch.arange(P, dtype=torch.int32, device="cuda").reshape(B, -1)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    # the argument structs hold raw pointers: every device tensor stays referenced
    h_d, sl_w = h.cuda(), torch.full((B,), L, dtype=torch.int32, device="cuda")
    a = mla.make_write_kv_args(h=h_d, w_dkv=w_dkv, kv_cache=kv, kv_scale=sc, block_table=bt, seq_lens=sl_w)
    ws = mla.alloc_workspace(a)
    mla.mla_write_kv(a)
    assert mla.mla_get_status(ws) == 0
    H = w_uk.shape[0]
    q_lat = torch.empty(B, 1, H, 512, dtype=torch.bfloat16, device="cuda")
    q_nope_d, q_pe_d = q_nope.cuda(), q_pe.cuda()
    mla.mla_absorb_q(q_nope_d, w_uk, q_lat)
    o_lat = torch.empty_like(q_lat)
    d = mla.make_decode_args(q_lat=q_lat, q_pe=q_pe_d, kv_cache=kv, kv_scale=sc, block_table=bt, seq_lens=sl,
                             o_lat=o_lat, lse=None, softmax_scale=1 / 192 ** 0.5)
    ws2 = mla.alloc_workspace(d)
    mla.mla_decode_paged(d)
    mla.mla_combine_splits(d)
    out = torch.empty(B, 1, H, 128, dtype=torch.bfloat16, device="cuda")
    mla.mla_up_proj_v(o_lat, w_uv, out)
    assert mla.mla_get_status(ws2) == 0
    return (out.float().cpu().numpy().astype(np.float64), kv.cpu().numpy().reshape(B, -1, 288),
            sc.cpu().numpy().astype(np.float64).reshape(B, -1, 18))


def _latent_of(kv, sc):
    """Values of a q4_0 cache's latent part: (low or high four bits - 8) * scale."""
    b = kv.astype(np.int64)
    codes = np.empty(b.shape[:-1] + (576,))
    codes[..., 0::2] = (b & 15) - 8
    codes[..., 1::2] = (b >> 4) - 8
    return (codes * np.repeat(sc, 32, axis=-1))[..., :512]


def test_rotation_shrinks_the_q4_0_error_with_outlier_channels(cuda_lib):
    """Hidden states whose latent has three channels 30x larger than the rest
    (W_DKV rows scaled): in a plain q4_0 cache the other values of those blocks
    lose their resolution; with the folded weights the cache holds H c, where the
    outliers are spread over every block.  Checked: the latent read back from the
    written cache (rotated back with H for the folded path) is at least twice as
    close to the exact latent in squared error, and the decode through either path
    stays within the 4-bit error of the fp64 plain-weight reference, the rotated
    one closer.  Every written row is a new token at position 0 .. L-1; the query
    of sequence b attends to the first lens[b] of them."""
    from oracle import cache_write as cw
    g = torch.Generator().manual_seed(41)
    B, L, H, d_h = 2, 256, 32, 512
    lens = [256, 150]
    h = torch.randn(B, L, d_h, generator=g).to(torch.bfloat16)
    w_dkv = torch.randn(576, d_h, generator=g) / d_h ** 0.5
    w_dkv[[37, 200, 411]] *= 30.0
    w_dkv = w_dkv.to(torch.bfloat16)
    w_uk = (torch.randn(H, 128, 512, generator=g) / 512 ** 0.5).to(torch.bfloat16)
    w_uv = (torch.randn(H, 128, 512, generator=g) / 512 ** 0.5).to(torch.bfloat16)
    q_nope = torch.randn(B, 1, H, 128, generator=g).to(torch.bfloat16)
    q_pe = torch.randn(B, 1, H, 64, generator=g).to(torch.bfloat16)
    # fp64 reference: exact latent rows and plain weights, positions 0 .. L-1
    f = lambda t: om.bf16_to_f64(bf16_bits(t))
    hb, wb = f(h), f(w_dkv)
    ref = np.zeros((B, 1, H, 128))
    exact_c = []
    for b in range(B):
        c, kr = cw.compress(hb[b], wb[:512], wb[512:])
        exact_c.append(c)
        k_pe = cw.rope(kr, np.arange(L), 10000.0)
        C = np.concatenate([c, k_pe], axis=1)[:lens[b]]
        for hh in range(H):
            q_lat = f(q_nope)[b, 0, hh] @ f(w_uk)[hh]
            s = (C[:, :512] @ q_lat + C[:, 512:] @ f(q_pe)[b, 0, hh]) / np.sqrt(192.0)
            p = np.exp(s - s.max())
            p /= p.sum()
            ref[b, 0, hh] = f(w_uv)[hh] @ (p @ C[:, :512])
    exact_c = np.stack(exact_c)
    err, lat = {}, {}
    for fold in (False, True):
        got, kv, sc = _run_q4_path(cuda_lib, h, w_dkv, w_uk, w_uv, q_nope, q_pe, lens, fold)
        err[fold] = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
        c_back = _latent_of(kv, sc)
        if fold:
            c_back = c_back @ lb.hadamard(512)                      # H is symmetric: H^T H c' = c
        lat[fold] = float(np.sum((c_back - exact_c) ** 2))
    assert lat[True] < 0.5 * lat[False], lat
    assert err[True] < err[False] and err[True] < 0.15, err
