// Per-head projections on both sides of the latent attention:
//   mla_absorb_q  : q_lat[t][h][:] = W_UK[h]^T q_nope[t][h][:]   (512 <- 128)
//   mla_up_proj_v : out[t][h][:]   = W_UV[h]   o_lat[t][h][:]    (128 <- 512)
// (weight absorption, nnets.ru article section "Суть MLA"; the up-projections
// k = W_UK c, v = W_UV c of "MLA ... Explained", section "Architecture").
//
// Both are a batch of H small GEMMs out[t][n] = sum_k X[t][k] W(k, n) whose
// weight (16.8 MB at H = 128) is read once per 64-token block; they are
// HBM-bound on the weight.  One CTA computes a 64-token x 128-column tile of one
// head, streaming K in 64-wide chunks through a cp.async double buffer, with
// warp-level bf16 MMAs (fp32 accumulation).
#include "common.cuh"

namespace mla {
namespace {

constexpr int TM = 64, TN = 128, TK = 64;
constexpr int XS = TK + 8;   // padded smem row (elements) of the X chunk
constexpr int WKN = TN + 8;  // padded row of a [k][n] weight chunk
constexpr int WNK = TK + 8;  // padded row of a [n][k] weight chunk

// W_KN: weight stored [K][N] per head (W_UK for absorption); otherwise [N][K]
// (W_UV for the up-projection).
template <int K, int N, bool W_KN>
__global__ void __launch_bounds__(128) proj_kernel(const __nv_bfloat16* __restrict__ X,
                                                   const __nv_bfloat16* __restrict__ W,
                                                   __nv_bfloat16* __restrict__ Y, int n_tok,
                                                   int H) {
  constexpr int XCH = TM * XS;
  constexpr int WCH = W_KN ? TK * WKN : TN * WNK;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(smem_raw);  // [2][TM][XS]
  __nv_bfloat16* ws = xs + 2 * XCH;                                  // [2][WCH]

  const int n0 = blockIdx.x * TN, t0 = blockIdx.y * TM, h = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp >> 1, wn = warp & 1;  // warp tile: 32 tokens x 64 columns
  const __nv_bfloat16* Wh = W + (size_t)h * K * N;
  pdl_trigger();
  // The weight is never written by the kernel this one may overlap with: its rows
  // for this CTA go to L2 before waiting for the activations.
  if (tid < (W_KN ? K : TN)) {
    const __nv_bfloat16* row = W_KN ? Wh + (size_t)tid * N + n0 : Wh + (size_t)(n0 + tid) * K;
    asm volatile("prefetch.global.L2 [%0];" ::"l"(row) : "memory");
  }
  pdl_wait();

  auto load_chunk = [&](int kc, int buf) {
    const int k0 = kc * TK;
    __nv_bfloat16* xb = xs + buf * XCH;
    for (int v = tid; v < TM * (TK / 8); v += 128) {
      int r = v / (TK / 8), c = (v % (TK / 8)) * 8;
      int t = t0 + r;
      if (t < n_tok) {
        cp_async16(xb + r * XS + c, X + ((size_t)t * H + h) * K + k0 + c);
      } else {
        *reinterpret_cast<uint4*>(xb + r * XS + c) = make_uint4(0, 0, 0, 0);
      }
    }
    __nv_bfloat16* wb = ws + buf * WCH;
    if (W_KN) {
      for (int v = tid; v < TK * (TN / 8); v += 128) {
        int r = v / (TN / 8), c = (v % (TN / 8)) * 8;
        cp_async16(wb + r * WKN + c, Wh + (size_t)(k0 + r) * N + n0 + c);
      }
    } else {
      for (int v = tid; v < TN * (TK / 8); v += 128) {
        int r = v / (TK / 8), c = (v % (TK / 8)) * 8;
        cp_async16(wb + r * WNK + c, Wh + (size_t)(n0 + r) * K + k0 + c);
      }
    }
    cp_async_commit();
  };

  float acc[2][8][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;

  constexpr int NK = K / TK;
  load_chunk(0, 0);
  for (int kc = 0; kc < NK; ++kc) {
    if (kc + 1 < NK) {
      load_chunk(kc + 1, (kc + 1) & 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const __nv_bfloat16* xb = xs + (kc & 1) * XCH;
    const __nv_bfloat16* wb = ws + (kc & 1) * WCH;
#pragma unroll
    for (int ks = 0; ks < TK / 16; ++ks) {
      uint32_t a[2][4];
#pragma unroll
      for (int mi = 0; mi < 2; ++mi)
        ldmatrix_x4(a[mi][0], a[mi][1], a[mi][2], a[mi][3],
                    xb + (wm * 32 + mi * 16 + (lane & 15)) * XS + ks * 16 + (lane >> 4) * 8);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        if (W_KN) {
          ldmatrix_x4_trans(b0, b1, b2, b3,
                            wb + (ks * 16 + (lane & 15)) * WKN + wn * 64 + np * 16 + (lane >> 4) * 8);
        } else {
          ldmatrix_x4(b0, b1, b2, b3,
                      wb + (wn * 64 + np * 16 + (lane & 7) + 8 * (lane >> 4)) * WNK + ks * 16 +
                          8 * ((lane >> 3) & 1));
        }
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
          mma_bf16_16816(acc[mi][2 * np], a[mi], b0, b1);
          mma_bf16_16816(acc[mi][2 * np + 1], a[mi], b2, b3);
        }
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int mi = 0; mi < 2; ++mi) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      int t = t0 + wm * 32 + mi * 16 + (lane >> 2) + half * 8;
      if (t >= n_tok) continue;
      __nv_bfloat16* yrow = Y + ((size_t)t * H + h) * N + n0 + wn * 64 + 2 * (lane & 3);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        *reinterpret_cast<uint32_t*>(yrow + j * 8) =
            pack_bf16(acc[mi][j][2 * half], acc[mi][j][2 * half + 1]);
      }
    }
  }
}

template <int K, int N, bool W_KN>
cudaError_t launch_proj(const void* X, const void* W, void* Y, int n_tok, int H,
                        cudaStream_t stream) {
  constexpr int WCH = W_KN ? TK * WKN : TN * WNK;
  const size_t smem = 2 * (TM * XS + WCH) * sizeof(__nv_bfloat16);
  auto kern = proj_kernel<K, N, W_KN>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  dim3 grid(N / TN, (n_tok + TM - 1) / TM, H);
  return launch_pdl(kern, grid, dim3(128), smem, stream, static_cast<const __nv_bfloat16*>(X),
                    static_cast<const __nv_bfloat16*>(W), static_cast<__nv_bfloat16*>(Y), n_tok, H);
}

}  // namespace

cudaError_t launch_absorb_q(const void* q_nope, const void* w_uk, void* q_lat, int n_tok, int H,
                            cudaStream_t stream) {
  return launch_proj<kDn, kDc, true>(q_nope, w_uk, q_lat, n_tok, H, stream);
}

cudaError_t launch_up_proj_v(const void* o_lat, const void* w_uv, void* out, int n_tok, int H,
                             cudaStream_t stream) {
  return launch_proj<kDc, kDv, false>(o_lat, w_uv, out, n_tok, H, stream);
}

}  // namespace mla
