// Hadamard rotation of the latent space, folded into the weights.
//
// ik_llama.cpp docs "FlashMLA", section "KV cache with MLA": below 6 bits a
// Hadamard transform applied to the cache before quantisation recovers quality.
// With the orthonormal Sylvester matrix H of size 512 (symmetric, H H = I) the
// rotation needs no work in the decode: the cache holds c' = H c when the
// down-projection is H W_DKV, and then
//   q_lat . c   = (H q_lat) . c'     (fold into W_UK: W_UK[h] -> W_UK[h] H)
//   W_UV o_lat  = W_UV H (H o_lat)   (fold into W_UV: W_UV[h] -> W_UV[h] H)
// since the attention over c' returns H o_lat.  This file applies H to the
// 512-value vectors of the three weights once, in place: the columns of the
// first 512 rows of the stacked down-projection, and every row of W_UK and W_UV
// (a row times H is H times the row, H being symmetric).  The RoPE rows and
// the RoPE key stay as they are.
//
// One warp per vector: lane l holds elements l + 32 e (e = 0..15).  The fast
// Walsh-Hadamard transform takes the nine butterfly stages of the index bits,
// bits 5..8 inside the lane and bits 0..4 across lanes by shuffles, in fp32;
// the sum is scaled by 2^-4.5 and rounded once to bf16.
#include "common.cuh"

namespace mla {
namespace {

constexpr int kVecWarps = 8;
// 2^-4.5 = 1 / sqrt(512), correctly rounded to fp32
constexpr float kInvSqrt512 = 0.044194173824159220f;

MLA_DEVI void fwht512(float (&x)[16], int lane) {
#pragma unroll
  for (int h = 1; h < 16; h <<= 1)
#pragma unroll
    for (int e = 0; e < 16; ++e)
      if ((e & h) == 0) {
        const float a = x[e], b = x[e + h];
        x[e] = a + b;
        x[e + h] = a - b;
      }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float y = __shfl_xor_sync(0xffffffffu, x[e], m);
      x[e] = upper ? y - x[e] : x[e] + y;
    }
  }
}

// vector v, element i at base[v * vec_stride + i * elem_stride]
__global__ void __launch_bounds__(32 * kVecWarps) fwht_kernel(__nv_bfloat16* base, int n_vec, int64_t vec_stride,
                                                               int64_t elem_stride) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int v = blockIdx.x * kVecWarps + (threadIdx.x >> 5);
  if (v >= n_vec) return;
  __nv_bfloat16* p = base + (int64_t)v * vec_stride;
  float x[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) x[e] = __bfloat162float(p[(int64_t)(lane + 32 * e) * elem_stride]);
  fwht512(x, lane);
#pragma unroll
  for (int e = 0; e < 16; ++e) p[(int64_t)(lane + 32 * e) * elem_stride] = __float2bfloat16_rn(x[e] * kInvSqrt512);
}

cudaError_t launch_fwht(void* base, int n_vec, int64_t vec_stride, int64_t elem_stride, cudaStream_t stream) {
  if (n_vec == 0) return cudaSuccess;
  const dim3 grid((n_vec + kVecWarps - 1) / kVecWarps);
  return launch_pdl(fwht_kernel, grid, dim3(32 * kVecWarps), 0, stream, static_cast<__nv_bfloat16*>(base), n_vec,
                    vec_stride, elem_stride);
}

}  // namespace

cudaError_t launch_fold_hadamard(void* w_dkv, int d_h, void* w_uk, void* w_uv, int H, cudaStream_t stream) {
  cudaError_t e = cudaSuccess;
  if (w_dkv) e = launch_fwht(w_dkv, d_h, 1, d_h, stream);  // columns of rows 0..511
  if (e == cudaSuccess && w_uk) e = launch_fwht(w_uk, H * kDn, kDc, 1, stream);
  if (e == cudaSuccess && w_uv) e = launch_fwht(w_uv, H * kDv, kDc, 1, stream);
  return e;
}

}  // namespace mla
