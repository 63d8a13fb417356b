// Per-head projections on both sides of the latent attention:
//   mla_absorb_q  : q_lat[t][h][:] = W_UK[h]^T q_nope[t][h][:]   (512 <- 128)
//   mla_up_proj_v : out[t][h][:]   = W_UV[h]   o_lat[t][h][:]    (128 <- 512)
// (weight absorption, nnets.ru article section "Суть MLA"; the up-projections
// k = W_UK c, v = W_UV c of "MLA ... Explained", section "Architecture").
//
// Both are a batch of H small GEMMs out[t][n] = sum_k X[t][k] W(k, n).  At decode
// sizes (tens to hundreds of tokens) they are bound by reading the weight
// (128 KB per head, 16.8 MB at H = 128).  A CTA owns one head, one block of 64
// tokens and one slice of NC output columns, so that the weight streams into
// every SM through several CTAs at once (four per SM) rather than one: TMA brings
// the slice's weight and the block's activations, K chunk by K chunk, into
// 128-byte-swizzled shared memory, and four warps (16 tokens each) run warp-level
// bf16 MMAs with fp32 accumulation over all NC columns.
#include "proj_tile.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int TM = proj::TM;

template <int K, int N, int NC, bool W_KN, int STAGES>
struct ProjCfg {
  using T = proj::Cfg<K, N, NC, W_KN, STAGES>;
  static constexpr int NT = proj::kGroupThreads;
  static constexpr size_t smem = (size_t)T::RING + 1024 + 64;  // + alignment, barriers
};

// One tile per CTA: head blockIdx.y, tokens 64 blockIdx.x .., columns NC blockIdx.z ..
template <int K, int N, int NC, bool W_KN, int STAGES>
__global__ void __launch_bounds__(proj::kGroupThreads) proj_kernel(const __grid_constant__ CUtensorMap tm_x,
                                                                   const __grid_constant__ CUtensorMap tm_w,
                                                                   __nv_bfloat16* __restrict__ Y, int n_tok,
                                                                   int H) {
  using T = proj::Cfg<K, N, NC, W_KN, STAGES>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sa = (raw + 1023u) & ~1023u;
  const uint32_t bar0 = sa + T::RING;
  const int tid = threadIdx.x;
  pdl_trigger();
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(bar0 + 8 * s, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // the weight is never written by the kernel this one may overlap with, the
  // activations are: the first thread requests weight chunks before waiting for
  // it, the others wait at once
  if (tid != 0) pdl_wait();
  int abort = 0;
  proj::tile<K, N, NC, W_KN, STAGES>(&tm_x, &tm_w, Y, n_tok, H, blockIdx.x * TM, blockIdx.y, blockIdx.z * NC, sa,
                                     smem_raw + (sa - raw), bar0, 0, tid, 1, []() { pdl_wait(); }, abort,
                                     nullptr);
}

template <int K, int N, int NC, bool W_KN, int STAGES>
cudaError_t launch_proj(const void* X, const void* W, void* Y, int n_tok, int H, cudaStream_t stream) {
  using C = ProjCfg<K, N, NC, W_KN, STAGES>;
  CUtensorMap tm_x, tm_w;
  // X [n_tok][H][K]: dims (K, H, n_tok), boxes of 64 tokens x 1 head x 64 values
  if (!tma_map_3d(&tm_x, X, K, H, n_tok, (uint64_t)K * 2, (uint64_t)H * K * 2, 64, 1, TM))
    return cudaErrorInvalidValue;
  const bool ok = W_KN ? tma_map_2d(&tm_w, W, N, (uint64_t)H * K, (uint64_t)N * 2, 64, proj::TK)
                       : tma_map_2d(&tm_w, W, K, (uint64_t)H * N, (uint64_t)K * 2, 64, NC);
  if (!ok) return cudaErrorInvalidValue;
  auto kern = proj_kernel<K, N, NC, W_KN, STAGES>;
  static PerDeviceOnce attrs;
  cudaError_t e = once_per_device(
      attrs, [&]() { return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::smem); });
  if (e != cudaSuccess) return e;
  dim3 grid((n_tok + TM - 1) / TM, H, N / NC);
  return launch_pdl(kern, grid, dim3(C::NT), C::smem, stream, tm_x, tm_w, static_cast<__nv_bfloat16*>(Y),
                    n_tok, H);
}

}  // namespace

// absorption: K = 128 (2 chunks, both in flight), N = 512 in 4 slices of 128
// columns; 48 KB of shared memory per CTA
cudaError_t launch_absorb_q(const void* q_nope, const void* w_uk, void* q_lat, int n_tok, int H,
                            cudaStream_t stream) {
  return launch_proj<kDn, kDc, 128, true, 2>(q_nope, w_uk, q_lat, n_tok, H, stream);
}

// up-projection: K = 512 (8 chunks, 4 in flight), N = 128 in 4 slices of 32
// columns; 48 KB of shared memory per CTA
cudaError_t launch_up_proj_v(const void* o_lat, const void* w_uv, void* out, int n_tok, int H,
                             cudaStream_t stream) {
  return launch_proj<kDc, kDv, 32, false, 4>(o_lat, w_uv, out, n_tok, H, stream);
}

}  // namespace mla
