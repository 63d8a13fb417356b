// Split-KV merge (flash-decoding): each split s of a sequence produced a
// normalised partial o_s over its token range and that range's log-sum-exp
// lse_s.  The whole-range result is
//   lse = log sum_s exp(lse_s),   o = sum_s exp(lse_s - lse) o_s .
// One warp per (token, head) row: the split weights come from a warp-shuffle
// max / sum over the lse values, then each lane accumulates 16 of the 512
// latent columns with float4 loads.  Empty splits carry lse_s = -inf and weigh 0.
#include <math_constants.h>

#include "common.cuh"

namespace mla {
namespace {

template <int kBatch>
__global__ void __launch_bounds__(128) combine_kernel(const float* __restrict__ o_part,
                                                      const float* __restrict__ lse_part,
                                                      __nv_bfloat16* __restrict__ o_lat,
                                                      float* __restrict__ lse_out, int rows,
                                                      int splits) {
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  pdl_trigger();
  pdl_wait();
  if (row >= rows) return;
  const float* lp = lse_part + (size_t)row * splits;
  float m = -CUDART_INF_F;
  for (int s = lane; s < splits; s += 32) m = fmaxf(m, lp[s]);
#pragma unroll
  for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  const float ref = m == -CUDART_INF_F ? 0.f : m;
  float z = 0.f;
  for (int s = lane; s < splits; s += 32) z += __expf(lp[s] - ref);
#pragma unroll
  for (int off = 16; off; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
  const bool empty = !(z > 0.f);
  const float inv_z = empty ? 0.f : 1.f / z;

  float4 acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  const float* op = o_part + (size_t)row * splits * kDc;
  // splits in batches of kBatch whose loads are all in flight before the first
  // use: one memory latency per batch rather than per split
  for (int s0 = 0; s0 < splits; s0 += kBatch) {
    float w[kBatch];
    float4 v[kBatch][4];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int s = s0 + j;
      const float ls = s < splits ? lp[s] : -CUDART_INF_F;
      w[j] = ls == -CUDART_INF_F ? 0.f : __expf(ls - ref) * inv_z;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        v[j][k] = w[j] != 0.f ? *reinterpret_cast<const float4*>(op + (size_t)s * kDc + k * 128 + lane * 4)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc[k].x += w[j] * v[j][k].x;
        acc[k].y += w[j] * v[j][k].y;
        acc[k].z += w[j] * v[j][k].z;
        acc[k].w += w[j] * v[j][k].w;
      }
  }
  __nv_bfloat16* dst = o_lat + (size_t)row * kDc;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint2 pk;
    pk.x = pack_bf16(acc[k].x, acc[k].y);
    pk.y = pack_bf16(acc[k].z, acc[k].w);
    *reinterpret_cast<uint2*>(dst + k * 128 + lane * 4) = pk;
  }
  if (lse_out && lane == 0) lse_out[row] = empty ? -CUDART_INF_F : ref + __logf(z);
}

}  // namespace

cudaError_t launch_combine(const mla_decode_args_t* a, int splits, cudaStream_t stream) {
  const int n_tok = a->B * a->s_q;
  const int rows = n_tok * a->H;
  WorkspaceLayout wl = workspace_layout(n_tok, a->H, splits);
  const unsigned char* ws = static_cast<const unsigned char*>(a->workspace);
  // few splits: a small batch keeps the registers low and the warps many
  auto kern = splits <= 2 ? combine_kernel<2> : combine_kernel<6>;
  return launch_pdl(kern, dim3((rows + 3) / 4), dim3(128), 0, stream,
                    reinterpret_cast<const float*>(ws + wl.o_part_off),
                    reinterpret_cast<const float*>(ws + wl.lse_part_off),
                    static_cast<__nv_bfloat16*>(a->o_lat), a->lse, rows, splits);
}

}  // namespace mla
