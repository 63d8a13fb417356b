// Paged latent-attention decode on the 5th-generation tensor cores (sm_100a):
// tcgen05 MMAs over a CTA pair, accumulators in tensor memory (TMEM), cache
// pages streamed by TMA.  This is the path for 128 heads and a bf16 cache.
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
// Warp roles (192 threads): warp 0 TMA producer, warp 1 TMEM allocator and (in
// the even CTA) the single MMA issuer, warps 2..5 softmax / correction /
// epilogue, one thread per TMEM lane.  The MMA order S(0), S(1), PV(0), S(2),
// PV(1), ... lets S(t+2) run on the tensor pipe while the softmax of t+1 runs.
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

namespace mla {
namespace {

using namespace sm100;

constexpr int kThreads = 192;
constexpr uint32_t kChunkQ = 64 * 128;              // 64 rows x 64 bf16
constexpr uint32_t kQBytes = 9 * kChunkQ;           // 73728
constexpr uint32_t kChunkS = 32 * 128;              // 32 tokens x 64 bf16
constexpr uint32_t kSStage = 9 * kChunkS;           // 36864: the CTA's 32 tokens x 576
constexpr uint32_t kChunkV = 64 * 128;              // 64 tokens x 64 bf16
constexpr uint32_t kVStage = 4 * kChunkV;           // 32768: 64 tokens x the CTA's 4 latent chunks
constexpr int kStages = 2;
constexpr uint32_t kPBytes = 64 * 128;              // 64 rows x 64 tokens bf16
constexpr uint32_t kQOff = 0;
constexpr uint32_t kSOff = kQOff + kQBytes;
constexpr uint32_t kVOff = kSOff + kStages * kSStage;
constexpr uint32_t kPOff = kVOff + kStages * kVStage;  // two P buffers
constexpr uint32_t kBarOff = kPOff + 2 * kPBytes;
// barrier indices
constexpr int S_FULL = 0;                 // [kStages] in the even CTA: stage filled in both CTAs
constexpr int S_EMPTY = S_FULL + kStages; // [kStages] in each CTA: stage consumed by the MMAs
constexpr int V_FULL = S_EMPTY + kStages;
constexpr int V_EMPTY = V_FULL + kStages;
constexpr int Q_FULL = V_EMPTY + kStages;
constexpr int S_READY = Q_FULL + 1;       // [2]
constexpr int P_READY = S_READY + 2;      // [2] in the even CTA
constexpr int O_DONE = P_READY + 2;       // [2]
constexpr int DRAIN = O_DONE + 2;
constexpr int NBARS = DRAIN + 1;
constexpr int kPrefetchTiles = 4;                    // L2 prefetch distance of the cache stream
constexpr uint32_t kMiscOff = kBarOff + 8 * NBARS;
constexpr uint32_t kXmaxOff = kMiscOff + 16;         // float [2][128]
constexpr uint32_t kXlOff = kXmaxOff + 2 * 128 * 4;  // float [128]
constexpr uint32_t kSmemUsed = kXlOff + 128 * 4;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;    // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 256;                     // S buffers at columns 256, 288
constexpr uint64_t kWaitLimitNs = 2000000000ull;     // 2 s
constexpr float kRescaleThreshold = 8.0f;            // log2 units

constexpr uint32_t kIdescS = idesc_bf16_f32(128, 64, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 256, false, true);

struct TcParams {
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

MLA_DEVI bool group_any(bool pred) {  // OR over the 128 softmax threads (named barrier 2)
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0;
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
    for (int i = 0; i < kStages; ++i) {
      mbar_init(own_bar(S_FULL + i), 1);
      mbar_init(own_bar(S_EMPTY + i), 1);
      mbar_init(own_bar(V_FULL + i), 1);
      mbar_init(own_bar(V_EMPTY + i), 1);
    }
    mbar_init(own_bar(Q_FULL), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(own_bar(S_READY + i), 1);
      mbar_init(own_bar(P_READY + i), 2);
      mbar_init(own_bar(O_DONE + i), 1);
    }
    mbar_init(own_bar(DRAIN), 1);
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
        const int qrow = (b * p.s_q + g) * p.H + 64 * (int)r;
        const uint32_t qb = lead_bar(Q_FULL);
        if (r == 0) mbar_arrive_expect_tx_local(own_bar(Q_FULL), 2 * kQBytes);
        for (int c = 0; c < 8; ++c) tma_load_2d_pair(sa + kQOff + c * kChunkQ, &tm_q, qb, 64 * c, qrow);
        tma_load_2d_pair(sa + kQOff + 8 * kChunkQ, &tm_qpe, qb, 0, qrow);
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
        const int st = u % kStages;
        const uint32_t ph = ((u / kStages) & 1) ^ 1;
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
        const int st = u % kStages;
        const uint32_t ph = ((u / kStages) & 1) ^ 1;
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
      bool ok = load_s(0);
      for (int u = 0; ok && u < n; ++u) {
        if (u + 1 < n) ok = load_s(u + 1);
        if (ok) ok = load_v(u);
      }
    }
  } else if (warp == 1) {
    // =========================== MMA issuer (even CTA) ===========================
    if (r == 0 && n > 0) {
      bool ok = mbar_wait_converged(own_bar(Q_FULL), 0, abort_flag, p.status, kWaitLimitNs);
      const uint64_t dq = desc_sw128(sa + kQOff, 16, 1024);
      const uint64_t ds = desc_sw128(sa + kSOff, 16, 1024);
      const uint64_t dv = desc_sw128(sa + kVOff, kChunkV, 1024);
      const uint64_t dp = desc_sw128(sa + kPOff, 16, 1024);
      auto issue_s = [&](int u) -> bool {
        const int st = u % kStages, sb = u & 1;
        if (!mbar_wait_converged(own_bar(S_FULL + st), (u / kStages) & 1, abort_flag, p.status, kWaitLimitNs))
          return false;
        tc_fence_after();
        const uint32_t d = tmem + kTmemS + 32u * sb;
        const uint64_t bs0 = ds + ((st * kSStage) >> 4);
#pragma unroll
        for (int c = 0; c < 9; ++c) {
          const uint64_t aq = dq + ((c * kChunkQ) >> 4), bs = bs0 + ((c * kChunkS) >> 4);
          mma_pair_elect(d, aq, bs, kIdescS, c != 0);
          mma_pair_elect(d, aq + 2, bs + 2, kIdescS, 1);
          mma_pair_elect(d, aq + 4, bs + 4, kIdescS, 1);
          mma_pair_elect(d, aq + 6, bs + 6, kIdescS, 1);
        }
        commit_pair_mc_elect(own_bar(S_EMPTY + st), 0x3);
        commit_pair_mc_elect(own_bar(S_READY + sb), 0x3);
        return true;
      };
      auto issue_pv = [&](int t) -> bool {
        const int pb = t & 1, st = t % kStages;
        if (!mbar_wait_converged(own_bar(P_READY + pb), (t >> 1) & 1, abort_flag, p.status, kWaitLimitNs))
          return false;
        if (!mbar_wait_converged(own_bar(V_FULL + st), (t / kStages) & 1, abort_flag, p.status, kWaitLimitNs))
          return false;
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
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && n > 1) ok = issue_s(1);
      for (int t = 0; ok && t < n; ++t) {
        ok = issue_pv(t);
        if (ok && t + 2 < n) ok = issue_s(t + 2);
      }
      // every issued MMA has completed before TMEM is released
      commit_pair_mc_elect(own_bar(DRAIN), 0x1);
      int dummy = 0;
      mbar_wait_converged(own_bar(DRAIN), 0, &dummy, p.status, kWaitLimitNs);
    }
  } else {
    // ====================== softmax / correction / epilogue ======================
    const int wq = warp & 3;                 // TMEM lane quadrant of this warp
    const int lt = wq * 32 + lane;           // TMEM lane = thread's row slot
    const int m = lt & 63, half = lt >> 6;   // head row in this CTA, token / column half
    const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);
    float m_used = -CUDART_INF_F, l = 0.f;
    bool alive = true;
    const int lim = min(vis, j_end);
    for (int t = 0; t < n; ++t) {
      const int sb = t & 1;
      bool w = mbar_wait(own_bar(S_READY + sb), (t >> 1) & 1, abort_flag, p.status, kWaitLimitNs);
      if (group_any(!w)) { alive = false; break; }
      tc_fence_after();
      uint32_t sv[32];
      tmem_ld32(tl + kTmemS + 32u * sb, sv);
      tmem_wait_ld();
      const int j0 = (t0 + t) * kPage + 32 * half;
      const int nv = max(0, min(32, lim - j0));
      float s[32];
      float lmax = -CUDART_INF_F;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        s[j] = j < nv ? __uint_as_float(sv[j]) * p.scale_log2 : -CUDART_INF_F;
        lmax = fmaxf(lmax, s[j]);
      }
      xmax[sb * 128 + lt] = lmax;
      named_bar_sync(1, 128);
      const float tmax = fmaxf(lmax, xmax[sb * 128 + (lt ^ 64)]);
      float alpha = 1.f;
      bool resc = false;
      if (tmax > -CUDART_INF_F) {
        if (m_used == -CUDART_INF_F) {
          m_used = tmax;                       // nothing accumulated yet: O and l are zero
        } else if (tmax > m_used + kRescaleThreshold) {
          alpha = exp2f(m_used - tmax);
          m_used = tmax;
          resc = true;
          l *= alpha;
        }
      }
      // reference point of the exponentials; a row with nothing visible yet keeps
      // 0 so that no (-inf) - (-inf) appears
      const float ref = m_used == -CUDART_INF_F ? 0.f : m_used;
      uint32_t pk[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float p0 = exp2f(s[j] - ref), p1 = exp2f(s[j + 1] - ref);
        l += p0 + p1;
        pk[j >> 1] = pack_bf16(p0, p1);
      }
      // P buffer sb was last read by PV(t-2)
      if (t >= 2) {
        w = mbar_wait(own_bar(O_DONE + sb), ((t - 2) >> 1) & 1, abort_flag, p.status, kWaitLimitNs);
        if (group_any(!w)) { alive = false; break; }
      }
      // O may only be rescaled once PV(t-1) has finished accumulating into it
      const bool any_resc = group_any(resc);
      if (any_resc && t >= 1) {
        w = mbar_wait(own_bar(O_DONE + (sb ^ 1)), ((t - 1) >> 1) & 1, abort_flag, p.status, kWaitLimitNs);
        if (group_any(!w)) { alive = false; break; }
        tc_fence_after();
      }
      if (any_resc) {
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t ov[32];
          tmem_ld32(tl + 32u * c, ov);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
          tmem_st32(tl + 32u * c, ov);
        }
        tmem_wait_st();
      }
      // P row m, tokens 32*half .. +31: four 16-byte chunks of the 128-byte row
      uint8_t* prow = sm + kPOff + sb * kPBytes + m * 128;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int q = 4 * half + k;
        *reinterpret_cast<uint4*>(prow + ((q ^ (m & 7)) << 4)) =
            make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(1, 128);
      if (lt == 0) mbar_arrive_remote(lead_bar(P_READY + sb));
    }
    if (alive && n > 0) {
      bool w = mbar_wait(own_bar(O_DONE + ((n - 1) & 1)), ((n - 1) >> 1) & 1, abort_flag, p.status,
                         kWaitLimitNs);
      if (group_any(!w)) alive = false;
      tc_fence_after();
    }
    xl[lt] = l;
    named_bar_sync(1, 128);
    const float ltot = l + xl[lt ^ 64];
    const bool empty = !(ltot > 0.f) || !alive;
    const float inv = empty ? 0.f : 1.f / ltot;
    const float lse = empty ? -CUDART_INF_F : (m_used + log2f(ltot)) * 0.6931471805599453f;
    const size_t orow = ((size_t)b * p.s_q + g) * p.H + 64 * r + m;
    const bool read_o = alive && n > 0;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      uint32_t ov[32];
      if (read_o) {
        tmem_ld32(tl + 32u * c, ov);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) ov[j] = 0u;
      }
      const int col = (c < 4) ? half * 128 + 32 * c : 256 + half * 128 + 32 * (c - 4);
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
    if (half == 0) {
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
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

bool encode_2d(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint64_t row_bytes,
               uint32_t box_cols, uint32_t box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult res = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS;
}

}  // namespace

bool decode_tc_supported(const mla_decode_args_t* a) {
  return a->H == 128 && a->kv_dtype == MLA_KV_BF16;
}

int decode_tc_clusters_per_split(const mla_decode_args_t* a) { return a->B * a->s_q; }

cudaError_t launch_decode_tc(const mla_decode_args_t* a, int splits, cudaStream_t stream) {
  CUtensorMap tm_q, tm_qpe, tm_ks, tm_kv;
  const uint64_t rows_q = (uint64_t)a->B * a->s_q * a->H;
  const uint64_t rows_kv = (uint64_t)a->num_pages * kPage;
  if (!encode_2d(&tm_q, a->q_lat, kDc, rows_q, kDc * 2, 64, 64) ||
      !encode_2d(&tm_qpe, a->q_pe, kDr, rows_q, kDr * 2, 64, 64) ||
      !encode_2d(&tm_ks, a->kv_cache, kRow, rows_kv, kRow * 2, 64, 32) ||
      !encode_2d(&tm_kv, a->kv_cache, kRow, rows_kv, kRow * 2, 64, 64))
    return cudaErrorInvalidValue;
  TcParams p;
  p.kv = static_cast<const uint8_t*>(a->kv_cache);
  p.block_table = a->block_table;
  p.seq_lens = a->seq_lens;
  p.o_lat = static_cast<__nv_bfloat16*>(a->o_lat);
  p.lse = a->lse;
  const int n_tok = a->B * a->s_q;
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
  cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(2 * splits, a->s_q, a->B);
  decode_tc_kernel<<<grid, kThreads, kSmemBytes, stream>>>(tm_q, tm_qpe, tm_ks, tm_kv, p);
  return cudaGetLastError();
}

}  // namespace mla
