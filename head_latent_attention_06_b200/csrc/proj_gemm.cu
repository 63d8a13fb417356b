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
#include "sm100.cuh"
#include "tma_host.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int TM = 64;   // tokens per CTA, 16 per warp
constexpr int TK = 64;   // K per chunk: one 128-byte swizzled row per matrix row
constexpr int NWARPS = 4;
constexpr uint64_t kProjWaitNs = 2000000000ull;

MLA_DEVI void tma_load_2d(uint32_t dst, const void* tmap, uint32_t mbar, int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(tmap), "r"(mbar), "r"(x), "r"(y)
      : "memory");
}
MLA_DEVI void tma_load_3d(uint32_t dst, const void* tmap, uint32_t mbar, int32_t x, int32_t y, int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(tmap), "r"(mbar), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Address of the 16-byte unit holding columns c0 .. c0+7 of row r in a block of
// 128-byte rows written by TMA with the 128-byte swizzle (block 1024-aligned).
MLA_DEVI uint32_t sw128(uint32_t base, int r, int c0) {
  return base + r * 128 + ((((c0 >> 3) ^ (r & 7)) & 7) << 4);
}

// W_KN: weight stored [K][N] per head (W_UK for absorption); otherwise [N][K]
// (W_UV for the up-projection).  NC: output columns per CTA.
template <int K, int N, int NC, bool W_KN, int STAGES>
struct ProjCfg {
  static constexpr int NT = NWARPS * 32;
  static constexpr uint32_t XBYTES = TM * 128;            // X chunk: 64 rows x 64 bf16
  static constexpr uint32_t WBYTES = (uint32_t)NC * 128;  // weight chunk: NC x 64 (either layout)
  static constexpr uint32_t STAGE = XBYTES + WBYTES;
  static constexpr int NK = K / TK;
  static constexpr size_t smem = (size_t)STAGES * STAGE + 1024 + 64;  // + alignment, barriers
  static_assert(NC % 64 == 0 || !W_KN, "K-by-N weight slices come in 64-column boxes");
  static_assert(NC % 16 == 0, "column pairs of n-tiles");
};

template <int K, int N, int NC, bool W_KN, int STAGES>
__global__ void __launch_bounds__(NWARPS * 32) proj_kernel(const __grid_constant__ CUtensorMap tm_x,
                                                           const __grid_constant__ CUtensorMap tm_w,
                                                           __nv_bfloat16* __restrict__ Y, int n_tok,
                                                           int H) {
  using C = ProjCfg<K, N, NC, W_KN, STAGES>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sa = (raw + 1023u) & ~1023u;
  const uint32_t bar0 = sa + STAGES * C::STAGE;

  const int t0 = blockIdx.x * TM, h = blockIdx.y, n0 = blockIdx.z * NC;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_trigger();
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(bar0 + 8 * s, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  // the weight is never written by the kernel this one may overlap with, the
  // activations are: weight chunks are requested before waiting for it
  auto load_w = [&](int kc, int s) {
    const uint32_t dst = sa + s * C::STAGE + C::XBYTES, mb = bar0 + 8 * s;
    if (W_KN) {
      for (int g = 0; g < NC / 64; ++g)
        tma_load_2d(dst + g * (TK * 128), &tm_w, mb, n0 + 64 * g, h * K + kc * TK);
    } else {
      tma_load_2d(dst, &tm_w, mb, kc * TK, h * N + n0);
    }
  };
  auto load_x = [&](int kc, int s) { tma_load_3d(sa + s * C::STAGE, &tm_x, bar0 + 8 * s, kc * TK, h, t0); };
  if (tid == 0) {
    for (int s = 0; s < STAGES && s < C::NK; ++s) {
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar0 + 8 * s),
                   "r"(C::STAGE)
                   : "memory");
      load_w(s, s);
    }
  }
  pdl_wait();
  if (tid == 0)
    for (int s = 0; s < STAGES && s < C::NK; ++s) load_x(s, s);

  constexpr int NJ = NC / 8;  // n-tiles of 8 columns
  float acc[NJ][4];
#pragma unroll
  for (int j = 0; j < NJ; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;

  int no_abort = 0;
#pragma unroll 1
  for (int kc = 0; kc < C::NK; ++kc) {
    const int s = kc % STAGES;
    mbar_wait(bar0 + 8 * s, (kc / STAGES) & 1, &no_abort, nullptr, kProjWaitNs);
    const uint32_t xb = sa + s * C::STAGE, wb = xb + C::XBYTES;
#pragma unroll
    for (int ks = 0; ks < TK / 16; ++ks) {
      uint32_t a[4];
      {
        const uint32_t ad = sw128(xb, warp * 16 + (lane & 15), ks * 16 + (lane >> 4) * 8);
        asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                     : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                     : "r"(ad));
      }
#pragma unroll
      for (int np = 0; np < NJ / 2; ++np) {
        uint32_t b0, b1, b2, b3;
        if (W_KN) {
          const int col = np * 16 + (lane >> 4) * 8;
          const uint32_t ad = sw128(wb + (col >> 6) * (TK * 128), ks * 16 + (lane & 15), col & 63);
          asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                       : "=r"(b0), "=r"(b1), "=r"(b2), "=r"(b3)
                       : "r"(ad));
        } else {
          const uint32_t ad = sw128(wb, np * 16 + (lane & 7) + 8 * (lane >> 4), ks * 16 + 8 * ((lane >> 3) & 1));
          asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                       : "=r"(b0), "=r"(b1), "=r"(b2), "=r"(b3)
                       : "r"(ad));
        }
        mma_bf16_16816(acc[2 * np], a, b0, b1);
        mma_bf16_16816(acc[2 * np + 1], a, b2, b3);
      }
    }
    __syncthreads();  // everyone is done with stage s
    const int nk = kc + STAGES;
    if (tid == 0 && nk < C::NK) {
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar0 + 8 * s),
                   "r"(C::STAGE)
                   : "memory");
      load_w(nk, s);
      load_x(nk, s);
    }
  }

  // epilogue: the bf16 tile goes through shared memory (the stages are free after
  // the loop's last barrier), then out in 16-byte pieces, consecutive threads on
  // consecutive pieces of a row
  constexpr int kPitch = NC * 2 + 16;  // bytes per staged row; the pad spreads banks
  static_assert(TM * kPitch <= (int)C::STAGE * STAGES, "output tile fits the stages");
  unsigned char* stile = smem_raw + (sa - raw);
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const int rl = warp * 16 + (lane >> 2) + hf * 8;
#pragma unroll
    for (int j = 0; j < NJ; ++j)
      *reinterpret_cast<uint32_t*>(stile + rl * kPitch + (j * 8 + 2 * (lane & 3)) * 2) =
          pack_bf16(acc[j][2 * hf], acc[j][2 * hf + 1]);
  }
  __syncthreads();
  constexpr int kPieces = NC / 8;  // 16-byte pieces per row
  for (int i = tid; i < TM * kPieces; i += C::NT) {
    const int rl = i / kPieces, pc = i % kPieces;
    const int t = t0 + rl;
    if (t < n_tok)
      *reinterpret_cast<uint4*>(Y + ((size_t)t * H + h) * N + n0 + pc * 8) =
          *reinterpret_cast<const uint4*>(stile + rl * kPitch + pc * 16);
  }
}

template <int K, int N, int NC, bool W_KN, int STAGES>
cudaError_t launch_proj(const void* X, const void* W, void* Y, int n_tok, int H, cudaStream_t stream) {
  using C = ProjCfg<K, N, NC, W_KN, STAGES>;
  CUtensorMap tm_x, tm_w;
  // X [n_tok][H][K]: dims (K, H, n_tok), boxes of 64 tokens x 1 head x 64 values
  if (!tma_map_3d(&tm_x, X, K, H, n_tok, (uint64_t)K * 2, (uint64_t)H * K * 2, 64, 1, TM))
    return cudaErrorInvalidValue;
  const bool ok = W_KN ? tma_map_2d(&tm_w, W, N, (uint64_t)H * K, (uint64_t)N * 2, 64, TK)
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
