// One tile of the per-head projections (query absorption, value up-projection),
// for a group of four warps: out[t][h][n0 .. n0+NC) = sum_k X[t][h][k] W(k, n)
// for the 64 tokens t0 .. t0+63 of head h.  TMA brings the weight slice and the
// activations, K chunk by K chunk, into 128-byte-swizzled shared memory (STAGES
// stages of X (64 x 64 bf16) then W (NC x 64 bf16)); each warp runs warp-level
// bf16 MMAs with fp32 accumulation for 16 tokens over all NC columns; the bf16
// tile goes out through shared memory in 16-byte pieces.
//
// Used by the standalone projection kernels (one tile per CTA) and by the fused
// decode step (three groups per CTA, several tiles each): the group's 128
// threads synchronise on their own named barrier, and the stage barriers' phases
// continue from tile to tile (`tile_iter` counts the tiles the group has done).
#pragma once

#include <cuda.h>

#include "sm100.cuh"

namespace mla {
namespace proj {

using namespace sm100;

constexpr int TM = 64;   // tokens per tile, 16 per warp
constexpr int TK = 64;   // K per chunk: one 128-byte swizzled row per matrix row
constexpr int kGroupThreads = 128;
constexpr uint64_t kWaitNs = 2000000000ull;

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

MLA_DEVI void group_sync(int bar_id) {
  asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "n"(kGroupThreads) : "memory");
}

// W_KN: weight stored [K][N] per head (W_UK for absorption); otherwise [N][K]
// (W_UV for the up-projection).  NC: output columns per tile.
template <int K, int N, int NC, bool W_KN, int STAGES>
struct Cfg {
  static constexpr uint32_t XBYTES = TM * 128;            // X chunk: 64 rows x 64 bf16
  static constexpr uint32_t WBYTES = (uint32_t)NC * 128;  // weight chunk: NC x 64 (either layout)
  static constexpr uint32_t STAGE = XBYTES + WBYTES;
  static constexpr uint32_t RING = STAGES * STAGE;        // shared memory of one group (1024-aligned base)
  static constexpr int NK = K / TK;
  static_assert(NC % 64 == 0 || !W_KN, "K-by-N weight slices come in 64-column boxes");
  static_assert(NC % 16 == 0, "column pairs of n-tiles");
  static_assert(NK % STAGES == 0, "each stage completes the same number of phases per tile");
  static constexpr int kPitch = NC * 2 + 16;  // bytes per staged output row; the pad spreads banks
  static_assert(TM * kPitch <= (int)RING, "output tile fits the stages");
};

// sa: the group's 1024-aligned ring (shared address), sgen the same as a generic
// pointer; bar0: STAGES mbarriers (count 1) of the group.  before_x() runs in
// the group's first thread after the first weight chunks are requested and
// before the activations are (a wait for their producer).  `abort` (per thread,
// kept across tiles) is set when a wait gives up: every later wait then returns
// at once, and the caller stops giving the group tiles.
template <int K, int N, int NC, bool W_KN, int STAGES, typename BeforeX>
MLA_DEVI void tile(const CUtensorMap* tm_x, const CUtensorMap* tm_w, __nv_bfloat16* __restrict__ Y, int n_tok,
                   int H, int t0, int h, int n0, uint32_t sa, unsigned char* sgen, uint32_t bar0,
                   uint32_t tile_iter, int gtid, int bar_id, BeforeX before_x, int& abort, uint32_t* status) {
  using C = Cfg<K, N, NC, W_KN, STAGES>;
  const int warp = gtid >> 5, lane = gtid & 31;
  auto load_w = [&](int kc, int s) {
    const uint32_t dst = sa + s * C::STAGE + C::XBYTES, mb = bar0 + 8 * s;
    if (W_KN) {
      for (int g = 0; g < NC / 64; ++g) tma_load_2d(dst + g * (TK * 128), tm_w, mb, n0 + 64 * g, h * K + kc * TK);
    } else {
      tma_load_2d(dst, tm_w, mb, kc * TK, h * N + n0);
    }
  };
  auto load_x = [&](int kc, int s) { tma_load_3d(sa + s * C::STAGE, tm_x, bar0 + 8 * s, kc * TK, h, t0); };
  if (gtid == 0) {
    for (int s = 0; s < STAGES && s < C::NK; ++s) {
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar0 + 8 * s), "r"(C::STAGE)
                   : "memory");
      load_w(s, s);
    }
    before_x();
    for (int s = 0; s < STAGES && s < C::NK; ++s) load_x(s, s);
  }

  constexpr int NJ = NC / 8;  // n-tiles of 8 columns
  float acc[NJ][4];
#pragma unroll
  for (int j = 0; j < NJ; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;

  constexpr uint32_t kPhasesPerTile = C::NK / STAGES;
#pragma unroll 1
  for (int kc = 0; kc < C::NK; ++kc) {
    const int s = kc % STAGES;
    mbar_wait(bar0 + 8 * s, (tile_iter * kPhasesPerTile + kc / STAGES) & 1, &abort, status, kWaitNs);
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
    group_sync(bar_id);  // the group is done with stage s
    const int nk = kc + STAGES;
    if (gtid == 0 && nk < C::NK && !abort) {
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar0 + 8 * s), "r"(C::STAGE)
                   : "memory");
      load_w(nk, s);
      load_x(nk, s);
    }
  }

  // epilogue: the bf16 tile goes through shared memory (the stages are free after
  // the loop's last barrier), then out in 16-byte pieces, consecutive threads on
  // consecutive pieces of a row
  constexpr int kPitch = C::kPitch;
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const int rl = warp * 16 + (lane >> 2) + hf * 8;
#pragma unroll
    for (int j = 0; j < NJ; ++j)
      *reinterpret_cast<uint32_t*>(sgen + rl * kPitch + (j * 8 + 2 * (lane & 3)) * 2) =
          pack_bf16(acc[j][2 * hf], acc[j][2 * hf + 1]);
  }
  group_sync(bar_id);
  constexpr int kPieces = NC / 8;  // 16-byte pieces per row
  for (int i = gtid; i < TM * kPieces; i += kGroupThreads) {
    const int rl = i / kPieces, pc = i % kPieces;
    const int t = t0 + rl;
    if (t < n_tok)
      *reinterpret_cast<uint4*>(Y + ((size_t)t * H + h) * N + n0 + pc * 8) =
          *reinterpret_cast<const uint4*>(sgen + rl * kPitch + pc * 16);
  }
  group_sync(bar_id);  // the staging area is free again
}

}  // namespace proj
}  // namespace mla
