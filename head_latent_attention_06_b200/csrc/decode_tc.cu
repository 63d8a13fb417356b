// Paged latent-attention decode on the 5th-generation tensor cores (sm_100a):
// tcgen05 MMAs over a CTA pair, accumulators in tensor memory (TMEM), cache
// pages streamed by TMA.  This is the path for a bf16 cache and up to 128 heads
// (fewer heads pad the 128-row tile with zero rows: the step stays bound by the
// cache stream, so the idle rows cost tensor work only).
//
// What it computes (absorbed MLA decode; nnets.ru article, sections "Суть MLA"
// and "MLA и FlashAttention"; snowgate thread 35 on the 512 + 64 latent record):
// for the 128 heads of one query token of sequence b,
//   S = Q . C^T   with Q = [q_lat | q_pe] (128 x 576), C = cache rows (tokens x 576)
//   online softmax over the tokens, O = P . C[:, :512]
// Scores and output share the one latent tile: V is the latent itself.
//
// Decomposition.  A cluster of two CTAs owns (sequence, query, split).  The MMA
// is the paired form (cta_group::2, M = 128): CTA r holds the Q rows of heads
// 64r .. 64r+63 and receives their S and O rows in its TMEM.  Per 64-token page:
//   S  (M=128, N=64,  K=576): B = the page's tokens; CTA r supplies its 32
//        tokens x 576 (9 TMA boxes of 32 x 64).
//   PV (M=128, N=256, K=64) twice (latent 0..255, 256..511): B = all 64 tokens x
//        the CTA's 128-column half of each N tile (4 TMA boxes of 64 x 64, a
//        second read of the page that hits L2).
// The cache streams through two rings, one for the score operand (S stages of
// 36 KB) and one for the value operand (V stages of 32 KB), in the order the
// MMAs consume them.  Only the even CTA posts the expected byte count of a stage
// (both CTAs' bytes) on its own barrier; the odd CTA's TMA completes its bytes
// there without arriving; each slot is released by the commit of the MMAs that read it, so
// the producer refills it at once.  Each CTA also prefetches its half of the
// page four tiles ahead into L2 with a bulk prefetch.
// TMEM per CTA (2x2 datapath layout of the paired M = 128 MMA): O takes 256
// columns, each S buffer 32 columns (two buffers).  Lane l < 64 holds head row l
// for the first half of every N tile, lane 64 + l the same row for the second.
//
// Warp roles (384 threads): warp 0 TMA producer, warp 1 TMEM allocator and (in
// the even CTA) issuer of the score MMAs, warp 2 (even CTA) issuer of the P.V
// MMAs, warp 3 idle, warps 4..11 softmax / correction / epilogue, two warps per
// TMEM lane quadrant, each thread 16 scores of a row half per page.
// Two S buffers let S(t+2) run on the tensor pipe while the softmax of t+1 runs;
// each softmax warp signals its own P rows to the P.V issuer.
// P is double-buffered in shared memory, so the softmax of t+1 never waits for
// P.V of t.  The output rescale is lazy: the reference maximum moves only when
// the tile maximum exceeds it by more than 2^8, so O in TMEM is rarely touched.
//
// Every mbarrier wait is bounded (MLA_ERR_DEVICE_TIMEOUT in the status word,
// then an orderly exit that drains issued MMAs and frees TMEM).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include "sm100.cuh"
#include "tma_host.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kThreads = 384;
constexpr uint32_t kChunkQ = 64 * 128;              // 64 rows x 64 bf16
#ifndef MLA_TC_Q_TMEM_CHUNKS
#define MLA_TC_Q_TMEM_CHUNKS 6
#endif
#ifndef MLA_TC_S_STAGES
#define MLA_TC_S_STAGES 3
#endif
#ifndef MLA_TC_PREFETCH
#define MLA_TC_PREFETCH 4
#endif
constexpr int kQTmemChunks = MLA_TC_Q_TMEM_CHUNKS;  // Q chunks 0..5 (latent 0..383) live in TMEM
constexpr int kQSmemChunks = 9 - kQTmemChunks;      // chunks 6..8 (latent 384..511, q_pe) in smem
constexpr uint32_t kQBytes = kQSmemChunks * kChunkQ;
constexpr uint32_t kChunkS = 32 * 128;              // 32 tokens x 64 bf16
constexpr uint32_t kSStage = 9 * kChunkS;           // 36864: the CTA's 32 tokens x 576
constexpr uint32_t kChunkV = 64 * 128;              // 64 tokens x 64 bf16
constexpr uint32_t kVStage = 4 * kChunkV;           // 32768: 64 tokens x the CTA's 4 latent chunks
constexpr int kSStages = MLA_TC_S_STAGES;           // score-operand stages
constexpr int kVStages = 2;                         // value-operand stages
constexpr uint32_t kPBytes = 64 * 128;              // 64 rows x 64 tokens bf16
constexpr uint32_t kQOff = 0;
constexpr uint32_t kSOff = kQOff + kQBytes;
constexpr uint32_t kVOff = kSOff + kSStages * kSStage;
constexpr uint32_t kPOff = kVOff + kVStages * kVStage;  // two P buffers
constexpr uint32_t kBarOff = kPOff + 2 * kPBytes;
// barrier indices
constexpr int S_FULL = 0;                  // [kSStages] in the even CTA: stage filled in both CTAs
constexpr int S_EMPTY = S_FULL + kSStages; // [kSStages] in each CTA: stage consumed by the MMAs
constexpr int V_FULL = S_EMPTY + kSStages; // [kVStages]
constexpr int V_EMPTY = V_FULL + kVStages;
constexpr int Q_FULL = V_EMPTY + kVStages; // smem part of Q landed (TMA bytes)
constexpr int Q_TMEM = Q_FULL + 1;         // TMEM part of Q written by the softmax warps
constexpr int S_READY = Q_TMEM + 1;        // [2]
constexpr int P_READY = S_READY + 2;      // [2] in the even CTA
constexpr int O_DONE = P_READY + 2;       // [2]
constexpr int DRAIN = O_DONE + 2;        // [2] one per MMA-issuing warp
constexpr int NBARS = DRAIN + 2;
constexpr int kSoftmaxWarps = 8;          // warps 4..11: two per TMEM lane quadrant
constexpr int kPrefetchTiles = MLA_TC_PREFETCH;      // L2 prefetch distance of the cache stream
constexpr uint32_t kMiscOff = kBarOff + 8 * NBARS;
constexpr uint32_t kXmaxOff = kMiscOff + 16;         // float [2 tiles][2 column halves][128 lanes]
constexpr uint32_t kXlOff = kXmaxOff + 4 * 128 * 4;  // float [2][128]
constexpr uint32_t kSmemUsed = kXlOff + 2 * 128 * 4;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;    // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 256;                     // S buffers at columns 256, 288
constexpr uint32_t kTmemQ = 320;                     // Q chunks 0..5: columns 320..511 (2 bf16 each)
static_assert(kTmemQ + kQTmemChunks * 32 <= kTmemCols, "TMEM budget");
constexpr uint64_t kWaitLimitNs = 2000000000ull;     // 2 s
constexpr float kRescaleThreshold = 8.0f;            // log2 units

constexpr uint32_t kIdescS = idesc_bf16_f32(128, 64, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 256, false, true);

struct TcParams {
  const __nv_bfloat16* q_lat;
  const uint8_t* kv;
  const int32_t* block_table;
  const int32_t* seq_lens;
  __nv_bfloat16* o_lat;
  float* lse;
  float* o_part;
  float* lse_part;
  uint32_t* status;
  int B, s_q, H, num_pages, max_pages, causal, splits;
  float scale_log2;
};

// 2^x with the hardware approximation (MUFU), flushing subnormal results to 0.
MLA_DEVI float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qpe,
                     const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_kv,
                     const TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
  uint8_t* sm = smem_raw + pad;
  const uint32_t sa = raw_addr + pad;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t r = cluster_ctarank();
  const int split = blockIdx.x >> 1, g = blockIdx.y, b = blockIdx.z;

  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kMiscOff + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kMiscOff);
  float* xmax = reinterpret_cast<float*>(sm + kXmaxOff);
  float* xl = reinterpret_cast<float*>(sm + kXlOff);
  auto own_bar = [&](int i) -> uint32_t { return sa + kBarOff + 8u * i; };
  auto lead_bar = [&](int i) -> uint32_t { return mapa(sa + kBarOff + 8u * i, 0); };

  // ---- the work unit: tiles [t0, t1) of sequence b, query g
  int L = p.seq_lens[b];
  const bool bad_len = L < 0 || L > p.max_pages * kPage;
  if (bad_len) L = 0;
  const int n_tiles = (L + kPage - 1) / kPage;
  const int per = (n_tiles + p.splits - 1) / p.splits;
  const int t0 = min(n_tiles, split * per);
  const int t1 = min(n_tiles, t0 + per);
  const int n = t1 - t0;
  const int j_end = min(L, t1 * kPage);
  const int vis = p.causal ? L - p.s_q + g + 1 : L;
  const int32_t* bt = p.block_table + (size_t)b * p.max_pages;

  if (threadIdx.x == 0) {
    if (bad_len && r == 0 && g == 0 && split == 0) set_status(p.status, MLA_ERR_BAD_SEQ_LEN);
    *abort_flag = 0;
    for (int i = 0; i < kSStages; ++i) {
      mbar_init(own_bar(S_FULL + i), 1);
      mbar_init(own_bar(S_EMPTY + i), 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(own_bar(V_FULL + i), 1);
      mbar_init(own_bar(V_EMPTY + i), 1);
    }
    mbar_init(own_bar(Q_TMEM), 2 * kSoftmaxWarps);
    mbar_init(own_bar(Q_FULL), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(own_bar(S_READY + i), 1);
      mbar_init(own_bar(P_READY + i), 2 * kSoftmaxWarps);
      mbar_init(own_bar(O_DONE + i), 1);
    }
    mbar_init(own_bar(DRAIN), 1);
    mbar_init(own_bar(DRAIN + 1), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  __syncthreads();
  cluster_arrive();
  cluster_wait();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();

  if (warp == 0) {
    // =========================== TMA producer ===========================
    // Ring order = MMA order: S(0), S(1), V(0), S(2), V(1), ... where S(u) is the
    // CTA's 32 tokens x 576 of page u (9 slots) and V(u) the page's 64 tokens x
    // the CTA's latent columns of both P.V halves (8 slots of 16 tokens x 128).
    if (n > 0) {
      if (lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_qpe);
        prefetch_tmap(&tm_ks);
        prefetch_tmap(&tm_kv);
      }
      // physical pages, fetched 32 at a time by the whole warp
      int blk_s = -1, pg_s = 0, blk_v = -1, pg_v = 0, blk_p = -1, pg_p = 0;
      auto page_of = [&](int u, int& blk, int& pg) -> int {
        if ((u >> 5) != blk) {
          blk = u >> 5;
          const int idx = t0 + (blk << 5) + lane;
          int v = idx < t1 ? bt[idx] : 0;
          if (v < 0 || v >= p.num_pages) {
            if (idx < t1) set_status(p.status, MLA_ERR_BAD_BLOCK_TABLE);
            v = 0;
          }
          pg = v;
        }
        return __shfl_sync(0xffffffffu, pg, u & 31);
      };
      // the CTA's half page (32 contiguous rows) of tile u, into L2 ahead of its TMA
      auto prefetch = [&](int u) {
        const int pg = page_of(u, blk_p, pg_p);
        if (lane == 0) prefetch_l2_bulk(p.kv + ((size_t)pg * kPage + 32 * r) * kRow * 2, kSStage);
      };
      for (int u = 0; u < n && u < kPrefetchTiles; ++u) prefetch(u);
      auto load_s = [&](int u) -> bool {
        const int st = u % kSStages;
        const uint32_t ph = ((u / kSStages) & 1) ^ 1;
        if (!mbar_wait_converged(own_bar(S_EMPTY + st), ph, abort_flag, p.status, kWaitLimitNs)) return false;
        const int pg = page_of(u, blk_s, pg_s);
        const uint32_t fb = lead_bar(S_FULL + st);
        if (r == 0) mbar_arrive_expect_tx_local_elect(own_bar(S_FULL + st), 2 * kSStage);
        const uint32_t dst = sa + kSOff + st * kSStage;
        for (int c = 0; c < 9; ++c)
          tma_load_2d_pair_elect(dst + c * kChunkS, &tm_ks, fb, 64 * c, pg * kPage + 32 * (int)r);
        if (u + kPrefetchTiles < n) prefetch(u + kPrefetchTiles);
        return true;
      };
      auto load_v = [&](int u) -> bool {
        const int st = u % kVStages;
        const uint32_t ph = ((u / kVStages) & 1) ^ 1;
        if (!mbar_wait_converged(own_bar(V_EMPTY + st), ph, abort_flag, p.status, kWaitLimitNs)) return false;
        const int pg = page_of(u, blk_v, pg_v);
        const uint32_t fb = lead_bar(V_FULL + st);
        if (r == 0) mbar_arrive_expect_tx_local_elect(own_bar(V_FULL + st), 2 * kVStage);
        const uint32_t dst = sa + kVOff + st * kVStage;
        for (int j = 0; j < 4; ++j) {
          const int lc = 4 * (j >> 1) + 2 * (int)r + (j & 1);  // latent chunk: halves {2r, 2r+1}, {4+2r, 5+2r}
          tma_load_2d_pair_elect(dst + j * kChunkV, &tm_kv, fb, 64 * lc, pg * kPage);
        }
        return true;
      };
      // The cache, block table and lengths are not written by the kernel this one
      // may overlap with (the query absorption); q_lat is, so Q waits for it.
      bool ok = load_s(0);
      pdl_wait();
      if (lane == 0) {
        // 3-D maps (values, heads, query tokens): heads >= H come in as zeros
        const int qtok = b * p.s_q + g, h0 = 64 * (int)r;
        const uint32_t qb = lead_bar(Q_FULL);
        if (r == 0) mbar_arrive_expect_tx_local(own_bar(Q_FULL), 2 * kQBytes);
        for (int c = kQTmemChunks; c < 8; ++c)
          tma_load_3d_pair(sa + kQOff + (c - kQTmemChunks) * kChunkQ, &tm_q, qb, 64 * c, h0, qtok);
        tma_load_3d_pair(sa + kQOff + (8 - kQTmemChunks) * kChunkQ, &tm_qpe, qb, 0, h0, qtok);
      }
      __syncwarp();
      for (int u = 0; ok && u < n; ++u) {
        if (u + 1 < n) ok = load_s(u + 1);
        if (ok) ok = load_v(u);
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ============ MMA issuers (even CTA): warp 1 scores, warp 2 P.V ============
    // The two streams touch disjoint TMEM (S buffers / O) and shared memory
    // (Q and the S ring / P and the V ring), so they are issued independently.
    if (r == 0 && n > 0) {
      const uint64_t dq = desc_sw128(sa + kQOff, 16, 1024);
      const uint64_t ds = desc_sw128(sa + kSOff, 16, 1024);
      const uint64_t dv = desc_sw128(sa + kVOff, kChunkV, 1024);
      const uint64_t dp = desc_sw128(sa + kPOff, 16, 1024);
      bool ok = true;
      if (warp == 1) {
        ok = mbar_wait_converged(own_bar(Q_FULL), 0, abort_flag, p.status, kWaitLimitNs) &&
             mbar_wait_converged(own_bar(Q_TMEM), 0, abort_flag, p.status, kWaitLimitNs);
        for (int u = 0; ok && u < n; ++u) {
          const int st = u % kSStages, sb = u & 1;
          // S buffer sb was last read by the softmax of tile u-2
          if (u >= 2 && !mbar_wait_converged(own_bar(P_READY + sb), ((u - 2) >> 1) & 1, abort_flag, p.status,
                                             kWaitLimitNs))
            break;
          if (!mbar_wait_converged(own_bar(S_FULL + st), (u / kSStages) & 1, abort_flag, p.status, kWaitLimitNs))
            break;
          tc_fence_after();
          const uint32_t d = tmem + kTmemS + 32u * sb;
          const uint64_t bs0 = ds + ((st * kSStage) >> 4);
          // K chunks 0..5: A (Q) from TMEM, only B is read from shared memory
#pragma unroll
          for (int c = 0; c < kQTmemChunks; ++c) {
            const uint32_t aq = tmem + kTmemQ + 32u * c;
            const uint64_t bs = bs0 + ((c * kChunkS) >> 4);
            mma_pair_ts_elect(d, aq, bs, kIdescS, c != 0);
            mma_pair_ts_elect(d, aq + 8, bs + 2, kIdescS, 1);
            mma_pair_ts_elect(d, aq + 16, bs + 4, kIdescS, 1);
            mma_pair_ts_elect(d, aq + 24, bs + 6, kIdescS, 1);
          }
#pragma unroll
          for (int c = kQTmemChunks; c < 9; ++c) {
            const uint64_t aq = dq + (((c - kQTmemChunks) * kChunkQ) >> 4), bs = bs0 + ((c * kChunkS) >> 4);
            mma_pair_elect(d, aq, bs, kIdescS, c != 0);
            mma_pair_elect(d, aq + 2, bs + 2, kIdescS, 1);
            mma_pair_elect(d, aq + 4, bs + 4, kIdescS, 1);
            mma_pair_elect(d, aq + 6, bs + 6, kIdescS, 1);
          }
          commit_pair_mc_elect(own_bar(S_EMPTY + st), 0x3);
          commit_pair_mc_elect(own_bar(S_READY + sb), 0x3);
        }
      } else {
        for (int t = 0; t < n; ++t) {
          const int pb = t & 1, st = t % kVStages;
          if (!mbar_wait_converged(own_bar(P_READY + pb), (t >> 1) & 1, abort_flag, p.status, kWaitLimitNs))
            break;
          if (!mbar_wait_converged(own_bar(V_FULL + st), (t / kVStages) & 1, abort_flag, p.status, kWaitLimitNs))
            break;
          tc_fence_after();
          const uint64_t ap = dp + ((pb * kPBytes) >> 4);
          const uint64_t bv = dv + ((st * kVStage) >> 4);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_pair_elect(tmem + 128u * h, ap + kk * 2, bv + ((2 * h * kChunkV + kk * 2048) >> 4), kIdescPV,
                             (t > 0 || kk > 0) ? 1u : 0u);
          }
          commit_pair_mc_elect(own_bar(V_EMPTY + st), 0x3);
          commit_pair_mc_elect(own_bar(O_DONE + pb), 0x3);
        }
      }
      // every MMA this warp issued has completed before TMEM is released
      const int db = DRAIN + (warp == 2 ? 1 : 0);
      commit_pair_mc_elect(own_bar(db), 0x1);
      int dummy = 0;
      mbar_wait_converged(own_bar(db), 0, &dummy, p.status, kWaitLimitNs);
    }
  } else if (warp >= 4) {
    // ====================== softmax / correction / epilogue ======================
    // Thread = (TMEM lane lt, column half ch).  Lane lt holds head row m = lt % 64
    // for tokens 32*half .. 32*half+31 of the page (half = lt / 64); the two warps
    // of a lane quadrant take 16 of those scores each, and half of the row's O
    // columns each.  A row's four threads (lt, lt ^ 64, both ch) agree on the
    // reference maximum through shared memory.
    const int wq = warp & 3;                 // TMEM lane quadrant of this warp
    const int ch = (warp - 4) >> 2;          // column half
    const int lt = wq * 32 + lane;
    const int m = lt & 63, half = lt >> 6;
    const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t grp_bar = 3 + (wq & 1);   // the 4 warps of quadrants {q, q^2}
    // Q row m, latent columns 0 .. 64*kQTmemChunks-1, into this lane's TMEM columns
    // (A operand of the score MMA: each 32-bit column holds two consecutive bf16;
    // lanes l and 64 + l both hold row l, the duplicated layout of the paired MMA)
    pdl_wait();
    const int head = 64 * (int)r + m;        // rows beyond H pad the 128-row MMA tile
    const bool row_ok = head < p.H;
    if (n > 0) {
      const uint4* qsrc =
          reinterpret_cast<const uint4*>(p.q_lat + (((size_t)b * p.s_q + g) * p.H + (row_ok ? head : 0)) * kDc);
      constexpr int kPerWarp = (kQTmemChunks + 1) / 2;
#pragma unroll 1
      for (int c = ch * kPerWarp; c < kQTmemChunks && c < (ch + 1) * kPerWarp; ++c) {
        uint32_t qv[32];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint4 v = row_ok ? __ldg(qsrc + c * 8 + k) : make_uint4(0u, 0u, 0u, 0u);
          qv[4 * k] = v.x;
          qv[4 * k + 1] = v.y;
          qv[4 * k + 2] = v.z;
          qv[4 * k + 3] = v.w;
        }
        tmem_st32(tl + kTmemQ + 32u * c, qv);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(lead_bar(Q_TMEM));
    }
    float m_used = -CUDART_INF_F, l = 0.f;
    const int lim = min(vis, j_end);
    // Control flow stays uniform even if a wait gives up (the kernel is then
    // aborting and every later wait returns at once): no barrier is skipped.
    for (int t = 0; t < n; ++t) {
      const int sb = t & 1;
      mbar_wait(own_bar(S_READY + sb), (t >> 1) & 1, abort_flag, p.status, kWaitLimitNs);
      tc_fence_after();
      uint32_t sv[16];
      tmem_ld16(tl + kTmemS + 32u * sb + 16u * ch, sv);
      tmem_wait_ld();
      const int j0 = (t0 + t) * kPage + 32 * half + 16 * ch;
      const int nv = max(0, min(16, lim - j0));
      float s[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) s[j] = j < nv ? __uint_as_float(sv[j]) : -CUDART_INF_F;
      float mx[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) mx[k] = fmaxf(fmaxf(s[k], s[k + 4]), fmaxf(s[k + 8], s[k + 12]));
      // the softmax scale is positive: scaling commutes with the maximum
      const float lmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.scale_log2;
      float* xm = xmax + sb * 256;
      xm[ch * 128 + lt] = lmax;
      named_bar_sync(grp_bar, 128);
      const float tmax = fmaxf(fmaxf(xm[lt], xm[lt ^ 64]), fmaxf(xm[128 + lt], xm[128 + (lt ^ 64)]));
      float alpha = 1.f;
      bool resc = false;
      if (tmax > -CUDART_INF_F) {
        if (m_used == -CUDART_INF_F) {
          m_used = tmax;                       // nothing accumulated yet: O and l are zero
        } else if (tmax > m_used + kRescaleThreshold) {
          alpha = ex2_approx(m_used - tmax);
          m_used = tmax;
          resc = true;
          l *= alpha;
        }
      }
      // p = 2^(s * scale_log2 - ref); a row with nothing visible yet keeps ref = 0
      // so that no (-inf) - (-inf) appears
      const float nref = m_used == -CUDART_INF_F ? 0.f : -m_used;
      uint32_t pk[8];
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        const float p0 = ex2_approx(fmaf(s[j], p.scale_log2, nref));
        const float p1 = ex2_approx(fmaf(s[j + 1], p.scale_log2, nref));
        ls[(j >> 1) & 3] += p0 + p1;
        pk[j >> 1] = pack_bf16(p0, p1);
      }
      l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      // P buffer sb was last read by PV(t-2)
      if (t >= 2) mbar_wait(own_bar(O_DONE + sb), ((t - 2) >> 1) & 1, abort_flag, p.status, kWaitLimitNs);
      // this warp's O columns may only be rescaled once PV(t-1) has accumulated into them
      if (__any_sync(0xffffffffu, resc)) {
        if (t >= 1) {
          mbar_wait(own_bar(O_DONE + (sb ^ 1)), ((t - 1) >> 1) & 1, abort_flag, p.status, kWaitLimitNs);
          tc_fence_after();
        }
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t ov[32];
          const uint32_t col = 128u * ch + 32u * c;
          tmem_ld32(tl + col, ov);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
          tmem_st32(tl + col, ov);
        }
        tmem_wait_st();
      }
      // P row m, tokens 32*half + 16*ch .. +15: two 16-byte chunks of the 128-byte row
      uint8_t* prow = sm + kPOff + sb * kPBytes + m * 128;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int q = 4 * half + 2 * ch + k;
        *reinterpret_cast<uint4*>(prow + ((q ^ (m & 7)) << 4)) =
            make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(lead_bar(P_READY + sb));
    }
    if (n > 0) {
      mbar_wait(own_bar(O_DONE + ((n - 1) & 1)), ((n - 1) >> 1) & 1, abort_flag, p.status, kWaitLimitNs);
      tc_fence_after();
    }
    xl[ch * 128 + lt] = l;
    named_bar_sync(1, 256);
    const bool alive = *abort_flag == 0;
    const float ltot = (xl[lt] + xl[lt ^ 64]) + (xl[128 + lt] + xl[128 + (lt ^ 64)]);
    const bool empty = !(ltot > 0.f) || !alive;
    const float inv = empty ? 0.f : 1.f / ltot;
    const float lse = empty ? -CUDART_INF_F : (m_used + log2f(ltot)) * 0.6931471805599453f;
    const size_t orow = ((size_t)b * p.s_q + g) * p.H + (row_ok ? head : 0);
    const bool read_o = alive && n > 0;
    // TMEM columns 128*ch .. +127 of this lane: latent half*128 + 256*ch + 0..127
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t ov[32];
      if (read_o) {
        tmem_ld32(tl + 128u * ch + 32u * c, ov);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) ov[j] = 0u;
      }
      const int col = 256 * ch + half * 128 + 32 * c;
      if (!row_ok) continue;
      if (p.splits == 1) {
        uint4* dst = reinterpret_cast<uint4*>(p.o_lat + orow * kDc + col);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint4 v;
          v.x = pack_bf16(__uint_as_float(ov[8 * k + 0]) * inv, __uint_as_float(ov[8 * k + 1]) * inv);
          v.y = pack_bf16(__uint_as_float(ov[8 * k + 2]) * inv, __uint_as_float(ov[8 * k + 3]) * inv);
          v.z = pack_bf16(__uint_as_float(ov[8 * k + 4]) * inv, __uint_as_float(ov[8 * k + 5]) * inv);
          v.w = pack_bf16(__uint_as_float(ov[8 * k + 6]) * inv, __uint_as_float(ov[8 * k + 7]) * inv);
          dst[k] = v;
        }
      } else {
        float4* dst = reinterpret_cast<float4*>(p.o_part + (orow * p.splits + split) * kDc + col);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          dst[k] = make_float4(__uint_as_float(ov[4 * k]) * inv, __uint_as_float(ov[4 * k + 1]) * inv,
                               __uint_as_float(ov[4 * k + 2]) * inv, __uint_as_float(ov[4 * k + 3]) * inv);
      }
    }
    if (half == 0 && ch == 0 && row_ok) {
      if (p.splits == 1) {
        if (p.lse) p.lse[orow] = lse;
      } else {
        p.lse_part[orow * p.splits + split] = lse;
      }
    }
    tc_fence_before();
  }

  // ---- teardown: both CTAs done with TMEM and shared memory
  __syncthreads();
  if (*abort_flag) {
    // let TMA copies already issued land before the shared memory is released
    const uint64_t t_end = globaltimer() + 2000000ull;
    while (globaltimer() < t_end) {
    }
  }
  cluster_arrive();
  cluster_wait();
  if (warp == 1) tmem_dealloc_pair(tmem, kTmemCols);
}

// ---------------------------------------------------------------- host side
}  // namespace

bool decode_tc_supported(const mla_decode_args_t* a) {
  // any head count up to 128 (rows beyond H pad the 128-row tile), bf16 cache
  return a->H % 16 == 0 && a->H <= 128 && a->kv_dtype == MLA_KV_BF16;
}

int decode_tc_clusters_per_split(const mla_decode_args_t* a) { return a->B * a->s_q; }

cudaError_t launch_decode_tc(const mla_decode_args_t* a, int splits, cudaStream_t stream) {
  CUtensorMap tm_q, tm_qpe, tm_ks, tm_kv;
  const uint64_t rows_kv = (uint64_t)a->num_pages * kPage;
  const int n_tok = a->B * a->s_q;
  // query maps are 3-D (values, heads, tokens) so that a 64-head box past H reads zeros
  if (!tma_map_3d(&tm_q, a->q_lat, kDc, a->H, n_tok, kDc * 2, (uint64_t)a->H * kDc * 2, 64, 64, 1) ||
      !tma_map_3d(&tm_qpe, a->q_pe, kDr, a->H, n_tok, kDr * 2, (uint64_t)a->H * kDr * 2, 64, 64, 1) ||
      !tma_map_2d(&tm_ks, a->kv_cache, kRow, rows_kv, kRow * 2, 64, 32) ||
      !tma_map_2d(&tm_kv, a->kv_cache, kRow, rows_kv, kRow * 2, 64, 64))
    return cudaErrorInvalidValue;
  TcParams p;
  p.q_lat = static_cast<const __nv_bfloat16*>(a->q_lat);
  p.kv = static_cast<const uint8_t*>(a->kv_cache);
  p.block_table = a->block_table;
  p.seq_lens = a->seq_lens;
  p.o_lat = static_cast<__nv_bfloat16*>(a->o_lat);
  p.lse = a->lse;
  WorkspaceLayout wl = workspace_layout(n_tok, a->H, splits);
  unsigned char* ws = static_cast<unsigned char*>(a->workspace);
  p.status = reinterpret_cast<uint32_t*>(ws + wl.status_off);
  p.o_part = reinterpret_cast<float*>(ws + wl.o_part_off);
  p.lse_part = reinterpret_cast<float*>(ws + wl.lse_part_off);
  p.B = a->B;
  p.s_q = a->s_q;
  p.H = a->H;
  p.num_pages = a->num_pages;
  p.max_pages = a->max_pages_per_seq;
  p.causal = a->causal;
  p.splits = splits;
  p.scale_log2 = a->softmax_scale * kLog2e;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  dim3 grid(2 * splits, a->s_q, a->B);
  return launch_pdl(decode_tc_kernel, grid, dim3(kThreads), kSmemBytes, stream, tm_q, tm_qpe, tm_ks, tm_kv, p);
}

}  // namespace mla
