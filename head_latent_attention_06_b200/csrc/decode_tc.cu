// Paged latent-attention decode on the 5th-generation tensor cores (sm_100a):
// tcgen05 MMAs over a CTA pair, accumulators in tensor memory (TMEM), cache
// pages streamed by TMA.  This is the path for a bf16 or e4m3 cache and 16 to 128
// heads (fewer heads pad the 128-row tile with zero rows: the step stays bound by
// the cache stream, so the idle rows cost tensor work only).
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
//        tokens x 576 (one 3-D TMA box: 64 values x 32 rows x 9 chunks).
//   PV (M=128, N=256, K=64) twice (latent 0..255, 256..511): B = all 64 tokens x
//        the CTA's 128-column half of each N tile (one 4-D TMA box of 4 chunks of
//        64 x 64, a second read of the page that hits L2).
// The cache streams through two rings, one for the score operand (S stages of
// 36 KB) and one for the value operand (V stages of 32 KB), in the order the
// MMAs consume them.  Only the even CTA posts the expected byte count of a stage
// (both CTAs' bytes) on its own barrier; the odd CTA's TMA completes its bytes
// there without arriving; each slot is released by the commit of the MMAs that
// read it, so the producer refills it at once.  Each CTA also prefetches its half
// of the page two tiles ahead into L2 with a bulk prefetch.
// Q: latent chunks 0..5 are the A operand from TMEM; they are staged by TMA in the
// value ring (idle until page 0's value operand) and moved into TMEM by the
// softmax warps; chunks 6..7 and q_pe stay in shared memory.
// TMEM per CTA (2x2 datapath layout of the paired M = 128 MMA): O takes 256
// columns, each S buffer 32 columns (two buffers).  Lane l < 64 holds head row l
// for the first half of every N tile, lane 64 + l the same row for the second.
//
// Warp roles (384 threads; fp8 512): warp 0 TMA producer, warp 1 TMEM allocator
// and (in the even CTA) issuer of the score MMAs (bf16: of even pages, warp 3 of
// odd ones), warp 2 (even CTA) issuer of the P.V MMAs, warps 4..11 softmax /
// correction / epilogue, two warps per TMEM lane quadrant, each thread 16
// scores of a row half per page; fp8: warps 12..15 convert, warp 3 relays the
// value stages' completion.
// Two S buffers: each softmax warp releases its S buffer as soon as its scores
// are in registers, so S(t+2) is issued while the softmax of t is still running
// and the tensor pipe does not wait on it; each softmax warp signals its own P
// rows to the P.V issuer.
// P is double-buffered in shared memory, so the softmax of t+1 never waits for
// P.V of t.  The output rescale is lazy: the reference maximum moves only when
// the tile maximum exceeds it by more than 2^8, so O in TMEM is rarely touched.
//
// fp8 (e4m3) cache with a per-token scale: the MMAs run on f16 operands.  Every
// e4m3 value is exactly an f16 value, so the cache needs only a format change:
// the producer brings the raw bytes of the CTA's 32 score rows into the back half
// of their stage slot (one bulk copy), four converter warps (12..15) read the
// whole stage, then write it back as f16 in the layout the TMA gives the bf16
// cache, and mark the slot full.  The value operand is assembled from both
// CTAs' converted score stages by shared-memory bulk copies (see copy_v).  Q is
// rounded from bf16 to f16 once (exact inside f16's normal range).  The token
// scales stay out of the operands: the softmax multiplies
// the raw scores by them, and P by them before the P.V MMA, so that
// O = sum_t p_t * scale_t * code_t.  Rows past the sequence end are written as
// zeros in the value operand, so that whatever bytes they hold cannot reach O.
//
// Every mbarrier wait is bounded (MLA_ERR_DEVICE_TIMEOUT in the status word,
// then an orderly exit that drains issued MMAs and frees TMEM).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <math_constants.h>
#include <string.h>

#include "sm100.cuh"
#include "tma_host.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kThreadsBf16 = 384;            // warps 0..11
constexpr int kConvWarps = 4;                // fp8: converter warps 12..15
constexpr int kThreadsFp8 = kThreadsBf16 + 32 * kConvWarps;
constexpr int kScRing = 8;                   // fp8: per-tile token scales (64 floats each)
constexpr uint32_t kChunkQ = 64 * 128;              // 64 rows x 64 bf16
#ifndef MLA_TC_Q_TMEM_CHUNKS
#define MLA_TC_Q_TMEM_CHUNKS 6
#endif
#ifndef MLA_TC_S_STAGES
#define MLA_TC_S_STAGES 3
#endif
#ifndef MLA_TC_PREFETCH
#define MLA_TC_PREFETCH 2
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
constexpr uint32_t kScOff = kPOff + 2 * kPBytes;      // fp8 token scales [kScRing][64]
constexpr uint32_t kBarOff = kScOff + kScRing * 256;
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
constexpr int DRAIN = O_DONE + 2;        // [3] one per MMA-issuing warp
constexpr int S_FREE = DRAIN + 3;         // [2] in the even CTA: the softmax has read S buffer sb
constexpr int RAW_S = S_FREE + 2;         // [kSStages] fp8: raw bytes of a score stage landed
constexpr int RAW_V = RAW_S + kSStages;   // [kVStages] bf16: a last page's value stage landed here;
                                          // fp8: both CTAs' copies into this CTA's value stage landed
constexpr int SC_FULL = RAW_V + kVStages; // [kScRing]  fp8: token scales of a tile landed
constexpr int Q_STAGE = SC_FULL + kScRing; // bf16: Q chunks 0..5 landed in the value ring (this CTA)
constexpr int Q_MOVED = Q_STAGE + 1;        // bf16: the softmax warps have moved them into TMEM
constexpr int NBARS = Q_MOVED + 1;
// A scale entry is reloaded for tile u + kScRing only after the score stage of
// tile u + kScRing - kSStages was consumed; that score MMA waited for every
// softmax warp to release the S buffer of tile u + kScRing - kSStages - 2, which
// each does only after finishing tile u + kScRing - kSStages - 3.  Tile u must
// be among the finished ones.
static_assert(kScRing >= kSStages + 3, "scale ring too short");
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

template <bool FP8>
constexpr uint32_t idesc_s() { return FP8 ? idesc_f16_f32(128, 64, false, false) : idesc_bf16_f32(128, 64, false, false); }
template <bool FP8>
constexpr uint32_t idesc_pv() { return FP8 ? idesc_f16_f32(128, 256, false, true) : idesc_bf16_f32(128, 256, false, true); }

struct TcParams {
  const __nv_bfloat16* q_lat;
  const __nv_bfloat16* q_pe;
  const uint8_t* kv;
  const float* kv_scale;  // fp8: [num_pages][64]
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

// bf16 pair -> f16 pair (round to nearest even; exact inside f16's normal range)
MLA_DEVI uint32_t bf16x2_to_f16x2(uint32_t x) {
  const __half2 h = __floats2half2_rn(__uint_as_float(x << 16), __uint_as_float(x & 0xFFFF0000u));
  return *reinterpret_cast<const uint32_t*>(&h);
}

MLA_DEVI uint32_t pack_f16(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// 16 e4m3 codes (16 bytes, lowest address first) -> 16 f16 values, exactly
MLA_DEVI void e4m3x16_to_f16(const uint4 v, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __half2_raw a = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[k] & 0xFFFFu), __NV_E4M3);
    const __half2_raw b = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[k] >> 16), __NV_E4M3);
    o[2 * k] = (uint32_t)a.x | ((uint32_t)a.y << 16);
    o[2 * k + 1] = (uint32_t)b.x | ((uint32_t)b.y << 16);
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

template <bool FP8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(FP8 ? kThreadsFp8 : kThreadsBf16, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qpe,
                     const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_kv,
                     const __grid_constant__ CUtensorMap tm_o, const TcParams p) {
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

  // The length and (for the first split, which starts at page 0) the producer's
  // first 32 block-table entries are requested here and used after the barrier
  // set-up, TMEM allocation and cluster sync, so that their latencies overlap.
  const int L_in = p.seq_lens[b];
  const int32_t* bt = p.block_table + (size_t)b * p.max_pages;
  int bt_first = 0;
  if (warp == 0 && split == 0 && lane < p.max_pages) bt_first = __ldg(bt + lane);

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    // bf16: a full score stage is the even CTA's expect_tx plus both CTAs' TMA
    // bytes, a full value stage that and the odd CTA's arrival (a last, partial
    // page instead takes one arrival per CTA after its tail rows are zeroed);
    // fp8: the arrivals of both CTAs' converter warps
    const uint32_t full_count = FP8 ? 2 * kConvWarps : 1;
    for (int i = 0; i < kSStages; ++i) {
      mbar_init(own_bar(S_FULL + i), full_count);
      // fp8: a stage is free once its score MMAs are done and the value-operand
      // copies have read it
      mbar_init(own_bar(S_EMPTY + i), FP8 ? 2 : 1);
      mbar_init(own_bar(RAW_S + i), 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(own_bar(V_FULL + i), 2);
      mbar_init(own_bar(V_EMPTY + i), 1);
      mbar_init(own_bar(RAW_V + i), 1);
    }
    for (int i = 0; i < kScRing; ++i) mbar_init(own_bar(SC_FULL + i), 1);
    mbar_init(own_bar(Q_TMEM), 2 * kSoftmaxWarps);
    mbar_init(own_bar(Q_FULL), 1);
    mbar_init(own_bar(Q_STAGE), 1);
    mbar_init(own_bar(Q_MOVED), kSoftmaxWarps);
    for (int i = 0; i < 2; ++i) {
      mbar_init(own_bar(S_READY + i), 1);
      mbar_init(own_bar(P_READY + i), 2 * kSoftmaxWarps);
      mbar_init(own_bar(S_FREE + i), 2 * kSoftmaxWarps);
      mbar_init(own_bar(O_DONE + i), 1);
    }
    for (int i = 0; i < 3; ++i) mbar_init(own_bar(DRAIN + i), 1);
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

  // ---- the work unit: tiles [t0, t1) of sequence b, query g
  const bool bad_len = L_in < 0 || L_in > p.max_pages * kPage;
  const int L = bad_len ? 0 : L_in;
  if (bad_len && threadIdx.x == 0 && r == 0 && g == 0 && split == 0) set_status(p.status, MLA_ERR_BAD_SEQ_LEN);
  // tokens this query sees: a causal query stops at its own position, so its
  // work unit covers only the pages up to there
  const int vis = p.causal ? max(0, L - p.s_q + g + 1) : L;
  const int n_tiles = (vis + kPage - 1) / kPage;
  const int per = (n_tiles + p.splits - 1) / p.splits;
  const int t0 = min(n_tiles, split * per);
  const int t1 = min(n_tiles, t0 + per);
  const int n = t1 - t0;
  const int j_end = min(vis, t1 * kPage);

  if (warp == 0) {
    // =========================== TMA producer ===========================
    // Ring order = MMA order: S(0), S(1), V(0), S(2), V(1), ... where S(u) is the
    // CTA's 32 tokens x 576 of page u (one 36 KB score stage) and V(u) the page's
    // 64 tokens x the CTA's latent columns of both P.V halves (one 32 KB value
    // stage).
    if (n > 0) {
      // physical pages, fetched 32 at a time by the whole warp
      int blk_s = -1, pg_s = 0, blk_v = -1, pg_v = 0, blk_p = -1, pg_p = 0;
      auto page_of = [&](int u, int& blk, int& pg) -> int {
        if ((u >> 5) != blk) {
          blk = u >> 5;
          const int idx = t0 + (blk << 5) + lane;
          int v = idx < t1 ? (blk == 0 && split == 0 ? bt_first : bt[idx]) : 0;
          if (v < 0 || v >= p.num_pages) {
            if (idx < t1) set_status(p.status, MLA_ERR_BAD_BLOCK_TABLE);
            v = 0;
          }
          pg = v;
        }
        return __shfl_sync(0xffffffffu, pg, u & 31);
      };
      // the CTA's half page (32 contiguous rows) of tile u, into L2 ahead of its TMA
      constexpr int kElem = FP8 ? 1 : 2;  // bytes per cached value
      auto prefetch = [&](int u) {
        const int pg = page_of(u, blk_p, pg_p);
        if (lane == 0) prefetch_l2_bulk(p.kv + ((size_t)pg * kPage + 32 * r) * kRow * kElem, 32 * kRow * kElem);
      };
      auto load_s = [&](int u) -> bool {
        const int st = u % kSStages;
        const uint32_t ph = ((u / kSStages) & 1) ^ 1;
        if (!mbar_wait_converged(own_bar(S_EMPTY + st), ph, abort_flag, p.status, kWaitLimitNs)) return false;
        const int pg = page_of(u, blk_s, pg_s);
        const uint32_t dst = sa + kSOff + st * kSStage;
        if constexpr (FP8) {
          // raw e4m3 rows 32r .. 32r+31 of the page (contiguous) into the back half
          // of the slot, and the page's 64 token scales
          if (lane == 0) {
            mbar_arrive_expect_tx_local(own_bar(RAW_S + st), kSStage / 2);
            bulk_load_cta(dst + kSStage / 2, p.kv + ((size_t)pg * kPage + 32 * r) * kRow, kSStage / 2,
                          own_bar(RAW_S + st));
            const int e = u % kScRing;
            mbar_arrive_expect_tx_local(own_bar(SC_FULL + e), 256);
            bulk_load_cta(sa + kScOff + 256 * e, p.kv_scale + (size_t)pg * kPage, 256, own_bar(SC_FULL + e));
          }
          __syncwarp();
        } else {
          // one box: (64 values, 32 rows, 9 chunks) lands chunk-major, 9 x 4 KB
          const uint32_t fb = lead_bar(S_FULL + st);
          if (r == 0) mbar_arrive_expect_tx_local_elect(own_bar(S_FULL + st), 2 * kSStage);
          tma_load_3d_pair_elect(dst, &tm_ks, fb, 0, pg * kPage + 32 * (int)r, 0);
        }
        if (u > 0 && u + kPrefetchTiles < n) prefetch(u + kPrefetchTiles);
        return true;
      };
      auto load_v = [&](int u) -> bool {
        const int st = u % kVStages;
        const uint32_t ph = ((u / kVStages) & 1) ^ 1;
        if (!mbar_wait_converged(own_bar(V_EMPTY + st), ph, abort_flag, p.status, kWaitLimitNs)) return false;
        const int pg = page_of(u, blk_v, pg_v);
        const uint32_t dst = sa + kVOff + st * kVStage;
        {  // bf16 only: the fp8 value operand is copied from the converted score stages
          const int nvalid = j_end - (t0 + u) * kPage;  // cached rows of this page inside the sequence
          if (nvalid >= kPage) {
            // one box: (64 values, 64 rows, chunks 2r and 2r+1, groups 0 and 1): latent
            // chunks {2r, 2r+1, 4+2r, 5+2r} of the page, 4 x 8 KB
            const uint32_t fb = lead_bar(V_FULL + st);
            if (r == 0) mbar_arrive_expect_tx_local_elect(own_bar(V_FULL + st), 2 * kVStage);
            else if (lane == 0) mbar_arrive_remote_relaxed(fb);
            tma_load_4d_pair_elect(dst, &tm_kv, fb, 0, pg * kPage, 2 * (int)r, 0);
          } else {
            // The last page of the sequence: P is 0 past the end, but 0 * NaN is
            // not, so whatever those rows hold is replaced by zeros before the MMA.
            // The stage lands on this CTA's own barrier (once per work unit).
            if (lane == 0) {
              mbar_arrive_expect_tx_local(own_bar(RAW_V + st), kVStage);
              tma_load_4d_cta(dst, &tm_kv, own_bar(RAW_V + st), 0, pg * kPage, 2 * (int)r, 0);
            }
            __syncwarp();
            if (!mbar_wait_converged(own_bar(RAW_V + st), 0, abort_flag, p.status, kWaitLimitNs)) return false;
            const int units = (kPage - nvalid) * 8;  // 16-byte units per chunk past the end
            for (int q = lane; q < 4 * units; q += 32) {
              const int j = q / units, rem = q - j * units;
              *reinterpret_cast<uint4*>(sm + kVOff + st * kVStage + j * kChunkV + (nvalid + (rem >> 3)) * 128 +
                                        (rem & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(lead_bar(V_FULL + st));
          }
        }
        return true;
      };
      // The cache, block table and lengths are not written by any kernel this one
      // may overlap with (the query absorption, or what the absorption overlaps;
      // the cache write lets nothing after it start early); q_lat is, so Q waits
      // for its producer.
      // page 0's score stage and Q first: every CTA asks for its first bytes at
      // the same moment, and these two gate the first score MMA; the L2
      // prefetch of the next pages only after them
      bool ok = load_s(0);
      pdl_wait();
      if (!FP8 && lane == 0) {
        // 3-D maps (values, heads, query tokens): heads >= H come in as zeros.
        // Chunks 6.. (the MMA's shared-memory A operand) into the Q region; chunks
        // 0..5 (the TMEM part) staged in the value ring, which V(0) may only
        // overwrite once the softmax warps have moved them into TMEM.
        const int qtok = b * p.s_q + g, h0 = 64 * (int)r;
        const uint32_t qb = lead_bar(Q_FULL);
        if (r == 0) mbar_arrive_expect_tx_local(own_bar(Q_FULL), 2 * kQBytes);
        for (int c = kQTmemChunks; c < 8; ++c)
          tma_load_3d_pair(sa + kQOff + (c - kQTmemChunks) * kChunkQ, &tm_q, qb, 64 * c, h0, qtok);
        tma_load_3d_pair(sa + kQOff + (8 - kQTmemChunks) * kChunkQ, &tm_qpe, qb, 0, h0, qtok);
        mbar_arrive_expect_tx_local(own_bar(Q_STAGE), kQTmemChunks * kChunkQ);
        for (int c = 0; c < kQTmemChunks; ++c)
          tma_load_3d_cta(sa + kVOff + c * kChunkQ, &tm_q, own_bar(Q_STAGE), 64 * c, h0, qtok);
      }
      __syncwarp();
      // bf16: nothing else is requested until Q has landed: at start-up every CTA
      // asks for its first bytes at once, and Q and page 0 gate the first MMA
      if (!FP8 && ok) ok = mbar_wait_converged(own_bar(Q_STAGE), 0, abort_flag, p.status, kWaitLimitNs);
      for (int u = 1; u < n && u <= kPrefetchTiles; ++u) prefetch(u);
      for (int u = 0; ok && u < n; ++u) {
        if (u + 1 < n) ok = load_s(u + 1);
        if (!FP8 && u == 0 && ok)
          ok = mbar_wait_converged(own_bar(Q_MOVED), 0, abort_flag, p.status, kWaitLimitNs);
        if (!FP8 && ok) ok = load_v(u);
      }
    }
  } else if (warp == 1 || warp == 2 || (!FP8 && warp == 3)) {
    // ==== MMA issuers (even CTA): warp 1 (bf16: and 3) scores, warp 2 P.V ====
    // The two streams touch disjoint TMEM (S buffers / O) and shared memory
    // (Q and the S ring / P and the V ring), so they are issued independently.
    if (r == 0 && n > 0) {
      const uint64_t dq = desc_sw128(sa + kQOff, 16, 1024);
      const uint64_t ds = desc_sw128(sa + kSOff, 16, 1024);
      const uint64_t dv = desc_sw128(sa + kVOff, kChunkV, 1024);
      const uint64_t dp = desc_sw128(sa + kPOff, 16, 1024);
      bool ok = true;
      if (warp != 2) {
        // fp8: the softmax warps write all of Q (TMEM and shared memory parts)
        ok = (FP8 || mbar_wait_converged(own_bar(Q_FULL), 0, abort_flag, p.status, kWaitLimitNs)) &&
             mbar_wait_converged(own_bar(Q_TMEM), 0, abort_flag, p.status, kWaitLimitNs);
        // bf16: warp 1 issues the even pages, warp 3 the odd ones.  Issuing 36 MMAs
        // takes the issue slots of the warp's SM sub-partition, whose softmax warps
        // then fall behind; two issuers halve that.  Each page's waits (S buffer
        // free, then stage full) imply that the stage's previous phase has
        // completed, so that parity waits stay exact with two issuers.  (fp8: the
        // converter warp on warp 3's sub-partition needs those slots; warp 1 alone.)
        constexpr int kStep = FP8 ? 1 : 2;
        for (int u = warp == 3 ? 1 : 0; ok && u < n; u += kStep) {
          const int st = u % kSStages, sb = u & 1;
          // S buffer sb was last read by the softmax of tile u-2 (released as soon as
          // its scores are in registers)
          if (u >= 2 && !mbar_wait_converged(own_bar(S_FREE + sb), ((u - 2) >> 1) & 1, abort_flag, p.status,
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
            mma_pair_ts_elect(d, aq, bs, idesc_s<FP8>(), c != 0);
            mma_pair_ts_elect(d, aq + 8, bs + 2, idesc_s<FP8>(), 1);
            mma_pair_ts_elect(d, aq + 16, bs + 4, idesc_s<FP8>(), 1);
            mma_pair_ts_elect(d, aq + 24, bs + 6, idesc_s<FP8>(), 1);
          }
#pragma unroll
          for (int c = kQTmemChunks; c < 9; ++c) {
            const uint64_t aq = dq + (((c - kQTmemChunks) * kChunkQ) >> 4), bs = bs0 + ((c * kChunkS) >> 4);
            mma_pair_elect(d, aq, bs, idesc_s<FP8>(), c != 0);
            mma_pair_elect(d, aq + 2, bs + 2, idesc_s<FP8>(), 1);
            mma_pair_elect(d, aq + 4, bs + 4, idesc_s<FP8>(), 1);
            mma_pair_elect(d, aq + 6, bs + 6, idesc_s<FP8>(), 1);
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
              mma_pair_elect(tmem + 128u * h, ap + kk * 2, bv + ((2 * h * kChunkV + kk * 2048) >> 4), idesc_pv<FP8>(),
                             (t > 0 || kk > 0) ? 1u : 0u);
          }
          commit_pair_mc_elect(own_bar(V_EMPTY + st), 0x3);
          commit_pair_mc_elect(own_bar(O_DONE + pb), 0x3);
        }
      }
      // every MMA this warp issued has completed before TMEM is released
      const int db = DRAIN + warp - 1;
      commit_pair_mc_elect(own_bar(db), 0x1);
      int dummy = 0;
      mbar_wait_converged(own_bar(db), 0, &dummy, p.status, kWaitLimitNs);
    }
  } else if (FP8 && warp >= 12) {
    // ====================== fp8 -> f16 converters (fp8 only) ======================
    // Same stage order as the producer: S(0), S(1), V(0), S(2), V(1), ...  Each
    // stage is read whole into registers, the four warps meet, and the f16 values
    // are written over the slot (the raw bytes sit in its back half).
    const int ct = threadIdx.x - kThreadsBf16;  // 0 .. 127
    auto convert_s = [&](int u) {
      const int st = u % kSStages;
      mbar_wait(own_bar(RAW_S + st), (u / kSStages) & 1, abort_flag, p.status, kWaitLimitNs);
      const uint32_t slot = sa + kSOff + st * kSStage;
      const uint32_t raw = slot + kSStage / 2;  // 32 rows x 576 bytes
      // rows i (even) and i + 1 share a quarter-warp, four 16-byte units each: the
      // reads (576-byte row pitch) and the swizzled writes both hit 8 distinct bank groups
      const int i = 2 * (ct >> 3) + ((ct >> 2) & 1), w = 2 * (ct & 3);
      // rows past the sequence end become zeros: the value operand is copied from here
      const bool live = 32 * (int)r + i < j_end - (t0 + u) * kPage;
      uint4 v[9];
#pragma unroll
      for (int c = 0; c < 9; ++c)
        v[c] = lds128(raw + i * kRow + 16 * (4 * c + (ct & 3)));
      named_bar_sync(5, 32 * kConvWarps);
#pragma unroll
      for (int c = 0; c < 9; ++c) {
        // values 64c + 16(ct&3) .. +15 of row i: f16 units w, w + 1 of chunk c
        uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = lo;
        if (live) e4m3x16_to_f16(v[c], lo, hi);
        const uint32_t row = slot + c * kChunkS + i * 128;
        sts128(row + ((w ^ (i & 7)) << 4), lo);
        sts128(row + (((w + 1) ^ (i & 7)) << 4), hi);
      }
      fence_proxy_async_smem();
      named_bar_sync(5, 32 * kConvWarps);  // the whole stage is written before it is copied
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(lead_bar(S_FULL + st));
    };
    // The value operand of page u: the converted latent chunks of this CTA's 32
    // rows go to the CTA that holds their columns (chunks {2d, 2d+1, 4+2d, 5+2d}
    // belong to CTA d), into rows 32r .. 32r+31 of its value stage: eight 4 KB
    // bulk copies, four to this CTA and four to the peer, counted on the
    // destination's RAW_V barrier.  The 128-byte swizzle depends on the row mod 8
    // only, so a block copied 32 rows down keeps its layout.  Both CTAs' value
    // slots are released by the same multicast commit, so waiting for our own is
    // enough for both destinations.  A score stage may be refilled once its copies
    // have read it: the arrival on S_EMPTY for page u is made when the copies of
    // page u+1 are issued (or never, for pages with no later refill).
    auto copy_v = [&](int u) {
      if (ct != 0) return;
      const int st = u % kVStages, ss = u % kSStages;
      mbar_wait(own_bar(V_EMPTY + st), ((u / kVStages) & 1) ^ 1, abort_flag, p.status, kWaitLimitNs);
#pragma unroll 1
      for (int lc = 0; lc < 8; ++lc) {
        const uint32_t d = (lc >> 1) & 1, j = 2 * (lc >> 2) + (lc & 1);
        const uint32_t dst = sa + kVOff + st * kVStage + j * kChunkV + r * (32 * 128);
        bulk_copy_s2s(mapa(dst, d), sa + kSOff + ss * kSStage + lc * kChunkS, kChunkS, mapa(own_bar(RAW_V + st), d));
      }
      bulk_commit_group();
      if (u >= 1) {
        bulk_wait_read<1>();  // page u-1's copies have read their stage
        mbar_arrive_remote(own_bar(S_EMPTY + (u - 1) % kSStages));
      }
    };
    if (n > 0) {
      convert_s(0);
      for (int u = 0; u < n; ++u) {
        if (u + 1 < n) convert_s(u + 1);
        copy_v(u);
      }
      if (ct == 0) bulk_wait_all();  // every copy has landed before shared memory is released
    }
  } else if (FP8 && warp == 3) {
    // ============ fp8: value-stage relay (one thread) ============
    // Posts the expected bytes of each value stage of this CTA (both CTAs' copies),
    // waits for them, and arrives on the even CTA's V_FULL (count 2: one per CTA).
    if (n > 0 && lane == 0) {
      for (int u = 0; u < n; ++u) {
        const int st = u % kVStages;
        mbar_arrive_expect_tx_local(own_bar(RAW_V + st), kVStage);
        if (!mbar_wait(own_bar(RAW_V + st), (u / kVStages) & 1, abort_flag, p.status, kWaitLimitNs)) break;
        mbar_arrive_remote(lead_bar(V_FULL + st));
      }
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 12) {
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
      static_assert(kQTmemChunks % 2 == 0, "Q chunks split evenly between the column halves");
      constexpr int kPerWarp = kQTmemChunks / 2;
      if constexpr (!FP8) {
        // bf16: the chunks were staged by TMA (128-byte swizzled rows of 64 heads);
        // read this row's, store them into TMEM, then free the staging area
        mbar_wait(own_bar(Q_STAGE), 0, abort_flag, p.status, kWaitLimitNs);
#pragma unroll
        for (int i = 0; i < kPerWarp; ++i) {
          const int c = ch * kPerWarp + i;
          uint32_t qv[32];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint4 v = lds128(sa + kVOff + c * kChunkQ + m * 128 + ((k ^ (m & 7)) << 4));
            qv[4 * k] = v.x;
            qv[4 * k + 1] = v.y;
            qv[4 * k + 2] = v.z;
            qv[4 * k + 3] = v.w;
          }
          tmem_st32(tl + kTmemQ + 32u * c, qv);
        }
      }
      // fp8: from global memory, rounded to f16 on the way
      constexpr int kBatch = 1;
#pragma unroll 1
      for (int c0 = ch * kPerWarp; FP8 && c0 < (ch + 1) * kPerWarp; c0 += kBatch) {
        uint32_t qv[kBatch][32];
#pragma unroll
        for (int i = 0; i < kBatch; ++i)
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint4 v = row_ok ? __ldg(qsrc + (c0 + i) * 8 + k) : make_uint4(0u, 0u, 0u, 0u);
            qv[i][4 * k] = FP8 ? bf16x2_to_f16x2(v.x) : v.x;
            qv[i][4 * k + 1] = FP8 ? bf16x2_to_f16x2(v.y) : v.y;
            qv[i][4 * k + 2] = FP8 ? bf16x2_to_f16x2(v.z) : v.z;
            qv[i][4 * k + 3] = FP8 ? bf16x2_to_f16x2(v.w) : v.w;
          }
#pragma unroll
        for (int i = 0; i < kBatch; ++i) tmem_st32(tl + kTmemQ + 32u * (c0 + i), qv[i]);
      }
      if constexpr (FP8) {
        // the shared-memory chunks of Q as f16 (128-byte swizzled rows, the layout
        // TMA gives the bf16 path); the row's four threads take six 16-byte units each
        static_assert(kQSmemChunks * 8 % 4 == 0, "Q units per thread");
        constexpr int kUnits = kQSmemChunks * 8 / 4;
        const size_t qr = ((size_t)b * p.s_q + g) * p.H + (row_ok ? head : 0);
        const int qi = 2 * half + ch;
#pragma unroll
        for (int k = 0; k < kUnits; ++k) {
          const int gu = qi * kUnits + k, cs = gu >> 3, w = gu & 7, c = kQTmemChunks + cs;
          const uint4* src = c < 8 ? reinterpret_cast<const uint4*>(p.q_lat + qr * kDc + 64 * c + 8 * w)
                                   : reinterpret_cast<const uint4*>(p.q_pe + qr * kDr + 8 * w);
          uint4 v = row_ok ? __ldg(src) : make_uint4(0u, 0u, 0u, 0u);
          v = make_uint4(bf16x2_to_f16x2(v.x), bf16x2_to_f16x2(v.y), bf16x2_to_f16x2(v.z), bf16x2_to_f16x2(v.w));
          *reinterpret_cast<uint4*>(sm + kQOff + cs * kChunkQ + m * 128 + ((w ^ (m & 7)) << 4)) = v;
        }
        fence_proxy_async_smem();
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_remote(lead_bar(Q_TMEM));
        if (!FP8) mbar_arrive_remote(own_bar(Q_MOVED));
      }
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
      // the scores are in registers: S buffer sb may take S(t+2)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(lead_bar(S_FREE + sb));
      const int j0 = (t0 + t) * kPage + 32 * half + 16 * ch;
      const int nv = max(0, min(16, lim - j0));
      // fp8: token scales of these 16 columns (0 where masked, so that nothing a
      // masked row holds reaches P)
      float sc[16];
      if constexpr (FP8) {
        mbar_wait(own_bar(SC_FULL + t % kScRing), (t / kScRing) & 1, abort_flag, p.status, kWaitLimitNs);
        const float4* sp = reinterpret_cast<const float4*>(sm + kScOff + 256 * (t % kScRing)) + 8 * half + 4 * ch;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 f = sp[k];
          sc[4 * k] = 4 * k < nv ? f.x : 0.f;
          sc[4 * k + 1] = 4 * k + 1 < nv ? f.y : 0.f;
          sc[4 * k + 2] = 4 * k + 2 < nv ? f.z : 0.f;
          sc[4 * k + 3] = 4 * k + 3 < nv ? f.w : 0.f;
        }
      }
      float s[16];
#pragma unroll
      for (int j = 0; j < 16; ++j)
        s[j] = j < nv ? (FP8 ? __uint_as_float(sv[j]) * sc[j] : __uint_as_float(sv[j])) : -CUDART_INF_F;
      float mx[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) mx[k] = fmaxf(fmaxf(s[k], s[k + 4]), fmaxf(s[k + 8], s[k + 12]));
      // the softmax scale is positive: scaling commutes with the maximum
      float lmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.scale_log2;
      if constexpr (FP8) {
        // the reference of O (and l) bounds x_t + log2(scale_t) rather than x_t, so
        // that every P entry p_t * scale_t stays at or below 2^8 whatever the scales
        float scm = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) scm = fmaxf(scm, sc[j]);
        if (nv > 0) lmax += __log2f(fmaxf(scm, 0x1p-64f));
      }
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
        // fp8: the P.V operand carries the token scale (the cache operand is the raw code)
        pk[j >> 1] = FP8 ? pack_f16(p0 * sc[j], p1 * sc[j + 1]) : pack_bf16(p0, p1);
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
    // TMEM columns 128*ch .. +127 of this lane: latent half*128 + 256*ch + 0..127,
    // loaded kEpi x 32 columns at a time (one wait per group)
    constexpr int kEpi = FP8 ? 1 : 2;  // fp8 threads have fewer registers to spare
#pragma unroll 1
    for (int c0 = 0; c0 < 4; c0 += kEpi) {
      uint32_t ovs[kEpi][32];
      if (read_o) {
#pragma unroll
        for (int i = 0; i < kEpi; ++i) tmem_ld32(tl + 128u * ch + 32u * (c0 + i), ovs[i]);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < kEpi; ++i)
#pragma unroll
          for (int j = 0; j < 32; ++j) ovs[i][j] = 0u;
      }
#pragma unroll
      for (int i = 0; i < kEpi; ++i) {
        const uint32_t (&ov)[32] = ovs[i];
        const int c = c0 + i;
        const int col = 256 * ch + half * 128 + 32 * c;
        if (p.splits == 1) {
          // bf16 row m, latent col .. col+31 into the staging area (the score ring,
          // idle now): 64-column chunks of 64 rows x 128 bytes, 128-byte swizzled
          const int chunk = col >> 6;
          const uint32_t base = sa + kSOff + chunk * (64 * 128) + m * 128;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint4 v;
            v.x = pack_bf16(__uint_as_float(ov[8 * k + 0]) * inv, __uint_as_float(ov[8 * k + 1]) * inv);
            v.y = pack_bf16(__uint_as_float(ov[8 * k + 2]) * inv, __uint_as_float(ov[8 * k + 3]) * inv);
            v.z = pack_bf16(__uint_as_float(ov[8 * k + 4]) * inv, __uint_as_float(ov[8 * k + 5]) * inv);
            v.w = pack_bf16(__uint_as_float(ov[8 * k + 6]) * inv, __uint_as_float(ov[8 * k + 7]) * inv);
            const int u = ((col & 63) >> 3) + k;
            sts128(base + ((u ^ (m & 7)) << 4), v);
          }
        } else {
          if (!row_ok) continue;
          float4* dst = reinterpret_cast<float4*>(p.o_part + (orow * p.splits + split) * kDc + col);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            dst[k] = make_float4(__uint_as_float(ov[4 * k]) * inv, __uint_as_float(ov[4 * k + 1]) * inv,
                                 __uint_as_float(ov[4 * k + 2]) * inv, __uint_as_float(ov[4 * k + 3]) * inv);
        }
      }
    }
    if (p.splits == 1) {
      // one thread stores the 8 chunks of this CTA's 64 rows (rows past H are
      // outside the map and not written)
      fence_proxy_async_smem();
      named_bar_sync(1, 256);
      if (warp == 4 && lane == 0) {
        const int qtok = b * p.s_q + g;
        for (int c = 0; c < 8; ++c) tma_store_3d(&tm_o, sa + kSOff + c * (64 * 128), 64 * c, 64 * (int)r, qtok);
        bulk_commit_group();
        bulk_wait_all();
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
template <bool FP8>
cudaError_t launch_tc(const mla_decode_args_t* a, int splits, cudaStream_t stream) {
  CUtensorMap tm_q, tm_qpe, tm_ks, tm_kv, tm_o;  // tm_o: o_lat, the single-split result
  const uint64_t rows_kv = (uint64_t)a->num_pages * kPage;
  const int n_tok = a->B * a->s_q;
  // query maps are 3-D (values, heads, tokens) so that a 64-head box past H reads zeros
  if (!tma_map_3d(&tm_q, a->q_lat, kDc, a->H, n_tok, kDc * 2, (uint64_t)a->H * kDc * 2, 64, 64, 1) ||
      !tma_map_3d(&tm_qpe, a->q_pe, kDr, a->H, n_tok, kDr * 2, (uint64_t)a->H * kDr * 2, 64, 64, 1) ||
      !tma_map_3d(&tm_o, a->o_lat, kDc, a->H, n_tok, kDc * 2, (uint64_t)a->H * kDc * 2, 64, 64, 1))
    return cudaErrorInvalidValue;
  if (FP8) {
    // unused: the raw e4m3 rows come by plain bulk copies and the value operand is
    // copied from the converted score stages
    memset(&tm_ks, 0, sizeof(tm_ks));
    tm_kv = tm_ks;
  } else {
    // score operand: (64 values, rows, 9 chunks 128 bytes apart), one box per stage;
    // value operand: (64 values, rows, 4 chunks 128 bytes apart, 2 groups 512 bytes
    // apart), one box of 2 x 2 chunks per stage
    const uint64_t dks[3] = {64, rows_kv, 9}, sks[2] = {kRow * 2, 128};
    const uint32_t bks[3] = {64, 32, 9};
    const uint64_t dkv[4] = {64, rows_kv, 4, 2}, skv[3] = {kRow * 2, 128, 512};
    const uint32_t bkv[4] = {64, 64, 2, 2};
    if (!tma_map_nd(&tm_ks, a->kv_cache, 3, dks, sks, bks) || !tma_map_nd(&tm_kv, a->kv_cache, 4, dkv, skv, bkv))
      return cudaErrorInvalidValue;
  }
  TcParams p;
  p.q_lat = static_cast<const __nv_bfloat16*>(a->q_lat);
  p.q_pe = static_cast<const __nv_bfloat16*>(a->q_pe);
  p.kv = static_cast<const uint8_t*>(a->kv_cache);
  p.kv_scale = a->kv_scale;
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
  auto kern = decode_tc_kernel<FP8>;
  static PerDeviceOnce attrs;
  cudaError_t e = once_per_device(attrs, [&]() {
    cudaError_t e2 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e2 != cudaSuccess) return e2;
    return cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  });
  if (e != cudaSuccess) return e;
  dim3 grid(2 * splits, a->s_q, a->B);
  return launch_pdl(kern, grid, dim3(FP8 ? kThreadsFp8 : kThreadsBf16), kSmemBytes, stream, tm_q, tm_qpe, tm_ks,
                    tm_kv, tm_o, p);
}

}  // namespace

bool decode_tc_supported(const mla_decode_args_t* a) {
  // any head count up to 128 (rows beyond H pad the 128-row tile); a bf16 cache,
  // or an e4m3 cache whose scale array starts on 16 bytes (bulk copies)
  if (a->H % 16 != 0 || a->H > 128) return false;
  if (a->kv_dtype == MLA_KV_BF16) return true;
  return a->kv_dtype == MLA_KV_FP8_E4M3 && (reinterpret_cast<uintptr_t>(a->kv_scale) & 15u) == 0;
}

int decode_tc_clusters_per_split(const mla_decode_args_t* a) { return a->B * a->s_q; }

cudaError_t launch_decode_tc(const mla_decode_args_t* a, int splits, cudaStream_t stream) {
  return a->kv_dtype == MLA_KV_FP8_E4M3 ? launch_tc<true>(a, splits, stream) : launch_tc<false>(a, splits, stream);
}

}  // namespace mla
