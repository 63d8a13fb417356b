// Paged latent-attention decode over an e4m3 cache on the e4m3 x e4m3 tensor
// path (tcgen05 kind::f8f6f4, fp32 accumulation in TMEM): the cache codes feed
// both contractions as they are stored, with no conversion pass.
//
// What it computes (absorbed MLA decode; nnets.ru article, sections "Суть MLA"
// and "MLA и FlashAttention"; the fp8 latent record of snowgate thread 35; the
// quantised latent cache of the ik_llama.cpp "FlashMLA" docs): for the heads of
// one query token, scores s_j = scale * (q_lat . c_j + q_pe . k_pe_j) with
// c_j || k_pe_j = code_j * scale_j (one fp32 scale per cached token), an online
// softmax over the visible tokens and o_lat = sum_j p_j c_j.
//
// Operands.  Only the cache side is in e4m3 by storage; the other side of each
// contraction is split into two e4m3 terms so that the product keeps about 7
// significant bits more than one e4m3 rounding would:
//   scores:  Q ~ s_h (Q_hi + Q_lo) per head row, s_h a power of two with
//            |Q| / s_h <= 448, Q_hi = e4m3(Q / s_h), Q_lo = e4m3(Q / s_h - Q_hi);
//            both terms multiply the same cache codes and accumulate into the
//            same TMEM columns: S_raw = (Q_hi + Q_lo) . code, score = S_raw s_h scale_j.
//   values:  P~_j = p_j scale_j, which the softmax reference keeps at or below
//            2^8 (inside e4m3's range, no scale needed); P~ = P_hi + P_lo and
//            O += (P_hi + P_lo) . code.
// A numerical model of the fp8 workload (8192 tokens per sequence) puts the
// result within 7e-4 relative L2 of the exact one; one e4m3 term each would
// give about 3e-2.
//
// Decomposition (as the bf16 kernel): a cluster of two CTAs owns (sequence,
// query, split) and issues the paired MMA (cta_group::2, M = 128 head rows, 64
// per CTA; rows past H are zero).  Per 64-token page:
//   S  (N = 64, K = 576 in steps of 32): B = the page's tokens, CTA r supplying
//      its 32 tokens x 576 codes (one 3-D TMA box, 9 chunks of 64 bytes per row,
//      64-byte swizzle, K-major); 36 MMAs (9 chunks x 2 K-steps x 2 terms).
//   PV (N = 256, K = 64) twice: B = all 64 tokens x the CTA's 128 latent columns
//      of the N tile (one 4-D TMA box, 128-byte rows, 128-byte swizzle,
//      MN-major); 8 MMAs (2 tiles x 2 K-steps x 2 terms).
// Q: K 0..383 of both terms live in TMEM as the score MMA's A operand (4 codes
// per 32-bit column; lanes l and 64 + l both hold head row l, the duplicated
// layout of the paired M = 128 MMA), K 384..575 in shared memory; the softmax
// warps split and write both.  P: two buffers x two terms of 64 rows x 64
// tokens in shared memory (64-byte swizzle).
//
// Warp roles (384 threads): warp 0 TMA producer (score stages two tiles ahead of
// value stages, the page's token scales with each score stage), warps 1 and 3
// (even CTA) score MMAs of even / odd pages, warp 2 (even CTA) P.V MMAs, warps
// 4..11 softmax (two per TMEM lane quadrant, 16 scores of a row half each),
// lazy rescale of O (the reference moves only when the maximum grows by more
// than 2^8), epilogue.
//
// Every mbarrier wait is bounded; on expiry the status word gets
// MLA_ERR_DEVICE_TIMEOUT, every role leaves its loop, issued MMAs are drained,
// and before the CTAs exit the even CTA reconciles and waits for every copy
// either CTA issued (see the teardown), then TMEM is freed.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <math_constants.h>

#include "sm100.cuh"
#include "tma_host.cuh"

namespace mla {
uint64_t device_wait_limit_ns();

namespace {

using namespace sm100;

constexpr int kThreads = 384;
constexpr int kScRing = 8;                      // per-tile token scales (64 floats each)
constexpr int kSStages = 4;                     // score-operand stages
constexpr int kVStages = 3;                     // value-operand stages
constexpr uint32_t kChunkS = 32 * 64;           // 32 tokens x 64 codes
constexpr uint32_t kSStage = 9 * kChunkS;       // 18432: the CTA's 32 tokens x 576 codes
constexpr uint32_t kVHalf = 64 * 128;           // 64 tokens x the CTA's 128 codes of one N tile
constexpr uint32_t kVStage = 2 * kVHalf;        // 16384: both N tiles
constexpr uint32_t kQChunk = 64 * 64;           // 64 rows x 64 codes
constexpr int kQTmemK = 384;                    // K values of each term held in TMEM
constexpr int kQSmemChunks = 3;                 // K 384..575 in shared memory
constexpr uint32_t kQBytes = 2 * kQSmemChunks * kQChunk;
constexpr uint32_t kPTerm = 64 * 64;            // 64 rows x 64 tokens
constexpr uint32_t kQOff = 0;
constexpr uint32_t kSOff = kQOff + kQBytes;               // 24576
constexpr uint32_t kVOff = kSOff + kSStages * kSStage;    // 98304
constexpr uint32_t kPOff = kVOff + kVStages * kVStage;    // 147456
constexpr uint32_t kScOff = kPOff + 4 * kPTerm;           // 163840
constexpr uint32_t kBarOff = kScOff + kScRing * 256;
static_assert(kSOff % 1024 == 0 && kVOff % 1024 == 0 && kPOff % 1024 == 0, "operand alignment");
// the single-split epilogue stages o_lat (8 chunks of 64 rows x 128 bytes) in the score ring
static_assert(kSStages * kSStage >= 8 * 64 * 128, "epilogue staging");
// barrier indices
constexpr int S_FULL = 0;                  // [kSStages] even CTA: both CTAs' score stage landed
constexpr int S_EMPTY = S_FULL + kSStages; // [kSStages] each CTA: the stage's score MMAs are done
constexpr int V_FULL = S_EMPTY + kSStages; // [kVStages] even CTA
constexpr int V_EMPTY = V_FULL + kVStages; // [kVStages] each CTA
constexpr int Q_TMEM = V_EMPTY + kVStages; // even CTA: every softmax warp of both CTAs wrote Q
constexpr int S_READY = Q_TMEM + 1;        // [2]
constexpr int P_READY = S_READY + 2;       // [2] even CTA
constexpr int O_DONE = P_READY + 2;        // [2]
constexpr int DRAIN = O_DONE + 2;          // [3] one per MMA-issuing warp
constexpr int S_FREE = DRAIN + 3;          // [2] even CTA: the softmax has read S buffer sb
constexpr int RAW_V = S_FREE + 2;          // [kVStages] a last page's value stage landed (this CTA)
constexpr int SC_FULL = RAW_V + kVStages;  // [kScRing] token scales of a tile landed (this CTA)
constexpr int Q_STAGE = SC_FULL + kScRing; // this CTA's Q rows (bf16) landed in the staging areas
constexpr int Q_FREE = Q_STAGE + 1;        // the softmax warps have read them: the value ring is free
constexpr int NBARS = Q_FREE + 1;
// A scale slot is reloaded for tile u + kScRing only after the score stage of
// tile u + kScRing - kSStages was consumed; that score MMA waited for every
// softmax warp to release the S buffer of tile u + kScRing - kSStages - 2, which
// each does only after finishing tile u + kScRing - kSStages - 3.  Tile u must
// be among the finished ones.
static_assert(kScRing >= kSStages + 3, "scale ring too short");
constexpr int kSoftmaxWarps = 8;
constexpr int kPrefetchTiles = 2;          // L2 prefetch distance of the cache stream
constexpr uint32_t kMiscOff = kBarOff + 8 * NBARS;      // tmem slot, abort flag, issue counts
constexpr uint32_t kXmaxOff = kMiscOff + 32;            // float [2 tiles][2 column halves][128 lanes]
constexpr uint32_t kXlOff = kXmaxOff + 4 * 128 * 4;     // float [2][128]
// Q (bf16, the CTA's 64 head rows) is staged by TMA before it is split: K 0..383
// (the TMEM part, six 64-value chunks of 64 rows x 128 bytes, 128-byte swizzle) in
// the value ring, idle until the first value stage; K 384..575 (two latent chunks
// and q_pe) in an area of its own
constexpr uint32_t kQStChunk = 64 * 128;
constexpr uint32_t kQStOff = (kXlOff + 2 * 128 * 4 + 1023) / 1024 * 1024;
constexpr uint32_t kSmemUsed = kQStOff + 3 * kQStChunk;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;       // + alignment slack
static_assert(kVStages * kVStage >= 6 * kQStChunk, "Q staging in the value ring");
static_assert(kSmemBytes <= 232448, "shared memory budget");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 256;                        // S buffers at columns 256, 288
constexpr uint32_t kTmemQ = 320;                        // Q terms: hi 320..415, lo 416..511
constexpr uint32_t kTmemQTerm = kQTmemK / 4;            // 96 columns per term
static_assert(kTmemQ + 2 * kTmemQTerm <= kTmemCols, "TMEM budget");
constexpr uint64_t kDrainLimitNs = 100000000ull;        // 100 ms for copies already in flight
constexpr float kRescaleThreshold = 8.0f;               // log2 units

constexpr uint32_t kIdescS = idesc_e4m3_f32(128, 64, false, false);
constexpr uint32_t kIdescPV = idesc_e4m3_f32(128, 256, false, true);

struct F8Params {
  const __nv_bfloat16* q_lat;
  const __nv_bfloat16* q_pe;
  const uint8_t* kv;
  const float* kv_scale;
  const int32_t* block_table;
  const int32_t* seq_lens;
  float* lse;
  float* o_part;
  float* lse_part;
  uint32_t* status;
  int B, s_q, H, num_pages, max_pages, causal, splits;
  float scale_log2;
  uint64_t wait_ns;
};

// Two values -> their e4m3 codes (nearest even, saturating) and the values those
// codes hold.
MLA_DEVI uint16_t e4m3x2(float a, float b, float2& held) {
  const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(c, __NV_E4M3);
  held = __half22float2(*reinterpret_cast<const __half2*>(&h));
  return (uint16_t)c;
}
// Two-term split of four values: the e4m3 codes and the codes of the residuals,
// four codes per word, the lowest K in the lowest byte.
MLA_DEVI void split4(const float (&x)[4], uint32_t& hi, uint32_t& lo) {
  float2 h01, h23, unused;
  const uint16_t a = e4m3x2(x[0], x[1], h01), b = e4m3x2(x[2], x[3], h23);
  hi = (uint32_t)a | ((uint32_t)b << 16);
  const uint16_t c = e4m3x2(x[0] - h01.x, x[1] - h01.y, unused);
  const uint16_t d = e4m3x2(x[2] - h23.x, x[3] - h23.y, unused);
  lo = (uint32_t)c | ((uint32_t)d << 16);
}

MLA_DEVI float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
MLA_DEVI float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_f8_kernel(const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_kv,
                     const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_qpe, const F8Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
  uint8_t* sm = smem_raw + pad;
  const uint32_t sa = raw_addr + pad;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t r = cluster_ctarank();
  const int split = blockIdx.x >> 1, g = blockIdx.y, b = blockIdx.z;

  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kMiscOff + 4);
  // producer's issue counts, read by the teardown: score tiles, full value pages,
  // last (partial) value page issued, Q staged
  uint32_t* issued = reinterpret_cast<uint32_t*>(sm + kMiscOff + 8);
  float* xmax = reinterpret_cast<float*>(sm + kXmaxOff);
  float* xl = reinterpret_cast<float*>(sm + kXlOff);
  auto own_bar = [&](int i) -> uint32_t { return sa + kBarOff + 8u * i; };
  auto lead_bar = [&](int i) -> uint32_t { return mapa(sa + kBarOff + 8u * i, 0); };

  const int L_in = p.seq_lens[b];
  const int32_t* bt = p.block_table + (size_t)b * p.max_pages;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < 4; ++i) issued[i] = 0;
    for (int i = 0; i < kSStages; ++i) {
      mbar_init(own_bar(S_FULL + i), 1);
      mbar_init(own_bar(S_EMPTY + i), 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      // a full value stage: the even CTA's expect_tx and the odd CTA's arrival (a
      // last, partial page instead one arrival per CTA after its tail is zeroed)
      mbar_init(own_bar(V_FULL + i), 2);
      mbar_init(own_bar(V_EMPTY + i), 1);
      mbar_init(own_bar(RAW_V + i), 1);
    }
    for (int i = 0; i < kScRing; ++i) mbar_init(own_bar(SC_FULL + i), 1);
    mbar_init(own_bar(Q_STAGE), 1);
    mbar_init(own_bar(Q_FREE), kSoftmaxWarps);
    mbar_init(own_bar(Q_TMEM), 2 * kSoftmaxWarps);
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
  // tokens this query sees: a causal query stops at its own position
  const int vis = p.causal ? max(0, L - p.s_q + g + 1) : L;
  const int n_tiles = (vis + kPage - 1) / kPage;
  const int per = (n_tiles + p.splits - 1) / p.splits;
  const int t0 = min(n_tiles, split * per);
  const int t1 = min(n_tiles, t0 + per);
  const int n = t1 - t0;
  const int j_end = min(vis, t1 * kPage);
  const uint64_t wait_ns = p.wait_ns;

  if (warp == 0) {
    // =========================== TMA producer ===========================
    int n_s = 0, n_v = 0, v_part = 0, q_iss = 0;
    if (n > 0) {
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
        if (lane == 0) prefetch_l2_bulk(p.kv + ((size_t)pg * kPage + 32 * r) * kRow, 32 * kRow);
      };
      auto load_s = [&](int u) -> bool {
        const int st = u % kSStages;
        const uint32_t ph = ((u / kSStages) & 1) ^ 1;
        if (!mbar_wait_converged(own_bar(S_EMPTY + st), ph, abort_flag, p.status, wait_ns)) return false;
        const int pg = page_of(u, blk_s, pg_s);
        // one box: (64 codes, 32 rows, 9 chunks), 9 x 2 KB, 64-byte swizzle
        const uint32_t fb = lead_bar(S_FULL + st);
        if (r == 0) mbar_arrive_expect_tx_local_elect(own_bar(S_FULL + st), 2 * kSStage);
        tma_load_3d_pair_elect(sa + kSOff + st * kSStage, &tm_ks, fb, 0, pg * kPage + 32 * (int)r, 0);
        // the page's 64 token scales, into this CTA's ring
        if (lane == 0) {
          const int e = u % kScRing;
          mbar_arrive_expect_tx_local(own_bar(SC_FULL + e), 256);
          bulk_load_cta(sa + kScOff + 256 * e, p.kv_scale + (size_t)pg * kPage, 256, own_bar(SC_FULL + e));
        }
        __syncwarp();
        n_s = u + 1;
        if (u > 0 && u + kPrefetchTiles < n) prefetch(u + kPrefetchTiles);
        return true;
      };
      auto load_v = [&](int u) -> bool {
        const int st = u % kVStages;
        const uint32_t ph = ((u / kVStages) & 1) ^ 1;
        if (!mbar_wait_converged(own_bar(V_EMPTY + st), ph, abort_flag, p.status, wait_ns)) return false;
        const int pg = page_of(u, blk_v, pg_v);
        const uint32_t dst = sa + kVOff + st * kVStage;
        const int nvalid = j_end - (t0 + u) * kPage;  // rows of this page inside the sequence
        if (nvalid >= kPage) {
          // one box: (128 codes, 64 rows, group r, both N tiles): 2 x 8 KB
          const uint32_t fb = lead_bar(V_FULL + st);
          if (r == 0) mbar_arrive_expect_tx_local_elect(own_bar(V_FULL + st), 2 * kVStage);
          else if (lane == 0) mbar_arrive_remote_relaxed(fb);
          tma_load_4d_pair_elect(dst, &tm_kv, fb, 0, pg * kPage, (int)r, 0);
          n_v = u + 1;
        } else {
          // The last page of the sequence: P is 0 past the end, but 0 * NaN is not,
          // so whatever those rows hold is replaced by zeros before the MMA.  The
          // stage lands on this CTA's own barrier (once per work unit).
          if (lane == 0) {
            mbar_arrive_expect_tx_local(own_bar(RAW_V + st), kVStage);
            tma_load_4d_cta(dst, &tm_kv, own_bar(RAW_V + st), 0, pg * kPage, (int)r, 0);
          }
          __syncwarp();
          v_part = 1;
          if (!mbar_wait_converged(own_bar(RAW_V + st), 0, abort_flag, p.status, wait_ns)) return false;
          const int units = (kPage - nvalid) * 8;  // 16-byte units past the end, per N tile
          for (int q = lane; q < 2 * units; q += 32) {
            const int h = q / units, rem = q - h * units;
            *reinterpret_cast<uint4*>(sm + kVOff + st * kVStage + h * kVHalf + (nvalid + (rem >> 3)) * 128 +
                                      (rem & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(lead_bar(V_FULL + st));
        }
        return true;
      };
      // The cache, block table and lengths are not written by any kernel this one
      // may overlap with (the cache write lets nothing after it start early); Q is,
      // so it is requested after the wait for the previous kernel.
      bool ok = load_s(0);
      pdl_wait();
      if (lane == 0) {
        // this CTA's 64 head rows of Q (3-D maps: heads >= H read as zeros): K 0..383
        // into the value ring, K 384..575 into the Q staging area
        const int qtok = b * p.s_q + g, h0 = 64 * (int)r;
        mbar_arrive_expect_tx_local(own_bar(Q_STAGE), 9 * kQStChunk);
        for (int c = 0; c < 6; ++c)
          tma_load_3d_cta(sa + kVOff + c * kQStChunk, &tm_q, own_bar(Q_STAGE), 64 * c, h0, qtok);
        for (int c = 6; c < 8; ++c)
          tma_load_3d_cta(sa + kQStOff + (c - 6) * kQStChunk, &tm_q, own_bar(Q_STAGE), 64 * c, h0, qtok);
        tma_load_3d_cta(sa + kQStOff + 2 * kQStChunk, &tm_qpe, own_bar(Q_STAGE), 0, h0, qtok);
      }
      __syncwarp();
      q_iss = 1;
      for (int u = 1; u < n && u <= kPrefetchTiles; ++u) prefetch(u);
      // score stages two tiles ahead of value stages; the first value stage waits
      // until the softmax warps have read Q out of the value ring
      if (ok && n > 1) ok = load_s(1);
      for (int u = 0; ok && u < n; ++u) {
        if (u + 2 < n) ok = load_s(u + 2);
        if (u == 0 && ok) ok = mbar_wait_converged(own_bar(Q_FREE), 0, abort_flag, p.status, wait_ns);
        if (ok) ok = load_v(u);
      }
    }
    if (lane == 0) {
      issued[0] = n_s;
      issued[1] = n_v;
      issued[2] = v_part;
      issued[3] = q_iss;
    }
  } else if (warp >= 1 && warp <= 3) {
    // ==== MMA issuers (even CTA): warps 1 and 3 scores (even / odd pages), warp 2 P.V ====
    if (r == 0 && n > 0) {
      bool ok = true;
      if (warp != 2) {
        ok = mbar_wait_converged(own_bar(Q_TMEM), 0, abort_flag, p.status, wait_ns);
        // Each page's waits (S buffer free, then stage full) imply that the stage's
        // previous phase has completed, so the parity waits stay exact with two issuers.
        for (int u = warp == 3 ? 1 : 0; ok && u < n; u += 2) {
          const int st = u % kSStages, sb = u & 1;
          if (u >= 2 && !mbar_wait_converged(own_bar(S_FREE + sb), ((u - 2) >> 1) & 1, abort_flag, p.status,
                                             wait_ns))
            break;
          if (!mbar_wait_converged(own_bar(S_FULL + st), (u / kSStages) & 1, abort_flag, p.status, wait_ns))
            break;
          tc_fence_after();
          const uint32_t d = tmem + kTmemS + 32u * sb;
          const uint32_t sbase = sa + kSOff + st * kSStage;
          // K chunks 0..5 (64 codes, two K = 32 steps each): A from TMEM, both terms
#pragma unroll
          for (int c = 0; c < 6; ++c) {
            const uint64_t bs = desc_swz(sbase + c * kChunkS, 16, 512, kLayoutSw64);
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)
#pragma unroll
              for (int t = 0; t < 2; ++t)
                mma_pair_f8_ts_elect(d, tmem + kTmemQ + kTmemQTerm * t + 8u * (2 * c + kk), bs + 2 * kk, kIdescS,
                                     (c | kk | t) != 0);
          }
          // K chunks 6..8: A from shared memory
#pragma unroll
          for (int c = 6; c < 9; ++c) {
            const uint64_t bs = desc_swz(sbase + c * kChunkS, 16, 512, kLayoutSw64);
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              const uint64_t aq =
                  desc_swz(sa + kQOff + (t * kQSmemChunks + (c - 6)) * kQChunk, 16, 512, kLayoutSw64);
#pragma unroll
              for (int kk = 0; kk < 2; ++kk) mma_pair_f8_elect(d, aq + 2 * kk, bs + 2 * kk, kIdescS, 1u);
            }
          }
          commit_pair_mc_elect(own_bar(S_EMPTY + st), 0x3);
          commit_pair_mc_elect(own_bar(S_READY + sb), 0x3);
        }
      } else {
        for (int t = 0; t < n; ++t) {
          const int pb = t & 1, st = t % kVStages;
          if (!mbar_wait_converged(own_bar(P_READY + pb), (t >> 1) & 1, abort_flag, p.status, wait_ns)) break;
          if (!mbar_wait_converged(own_bar(V_FULL + st), (t / kVStages) & 1, abort_flag, p.status, wait_ns))
            break;
          tc_fence_after();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            // MN-major B: 128-byte rows (tokens) of one N tile, 8 K-rows per 1024-byte atom
            const uint64_t bv = desc_swz(sa + kVOff + st * kVStage + h * kVHalf, kVHalf, 1024, kLayoutSw128);
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)
#pragma unroll
              for (int tm = 0; tm < 2; ++tm) {
                const uint64_t ap = desc_swz(sa + kPOff + (pb * 2 + tm) * kPTerm, 16, 512, kLayoutSw64);
                mma_pair_f8_elect(tmem + 128u * h, ap + 2 * kk, bv + ((kk * 32 * 128) >> 4), kIdescPV,
                                  (t > 0 || kk > 0 || tm > 0) ? 1u : 0u);
              }
          }
          commit_pair_mc_elect(own_bar(V_EMPTY + st), 0x3);
          commit_pair_mc_elect(own_bar(O_DONE + pb), 0x3);
        }
      }
      // every MMA this warp issued has completed before TMEM and shared memory are released
      const int db = DRAIN + warp - 1;
      commit_pair_mc_elect(own_bar(db), 0x1);
      int keep_waiting = 0;
      mbar_wait_converged(own_bar(db), 0, &keep_waiting, p.status, kDrainLimitNs);
    }
  } else {
    // ====================== softmax / correction / epilogue ======================
    // Thread = (TMEM lane lt, column half ch).  Lane lt holds head row m = lt % 64
    // for tokens 32*half .. 32*half+31 of the page (half = lt / 64); the two warps
    // of a lane quadrant take 16 of those scores each, and half of the row's O
    // columns each.  A row's four threads agree on maxima through shared memory.
    const int wq = warp & 3;
    const int ch = (warp - 4) >> 2;
    const int lt = wq * 32 + lane;
    const int m = lt & 63, half = lt >> 6;
    const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t grp_bar = 3 + (wq & 1);  // the 4 warps of quadrants {q, q^2}
    pdl_wait();
    const int head = 64 * (int)r + m;       // rows beyond H pad the 128-row MMA tile
    const bool row_ok = head < p.H;
    const size_t qr = ((size_t)b * p.s_q + g) * p.H + (row_ok ? head : 0);
    float s_h = 1.f;                        // the Q row's power-of-two scale
    if (n > 0) {
      // This thread's Q values, read from the staging areas (64 head rows, 64-value
      // chunks of 128-byte rows, 128-byte swizzle): K [192 ch, 192 ch + 192) of the
      // TMEM part (chunks 3 ch .. 3 ch + 2, in the value ring), and 48 of the
      // shared-memory part (K 384 + 48 qi .., chunks 6..8), qi = 2 half + ch.
      const int qi = 2 * half + ch;
      auto q_unit = [&](int kv) -> uint32_t {  // 16-byte unit holding K values kv .. kv+7 of row m
        const int c = kv >> 6, u = (kv & 63) >> 3;
        const uint32_t base = c < 6 ? sa + kVOff + c * kQStChunk : sa + kQStOff + (c - 6) * kQStChunk;
        return base + m * 128 + ((u ^ (m & 7)) << 4);
      };
      auto absmax8 = [](const uint4 v) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) a = fmaxf(a, fmaxf(fabsf(bf16_lo(w[e])), fabsf(bf16_hi(w[e]))));
        return a;
      };
      mbar_wait(own_bar(Q_STAGE), 0, abort_flag, p.status, wait_ns);
      __syncwarp();
      // pass 1: the largest magnitude of this thread's values (rows past H are zeros)
      float amax = 0.f;
#pragma unroll 8
      for (int k = 0; k < 24; ++k) amax = fmaxf(amax, absmax8(lds128(q_unit(192 * ch + 8 * k))));
#pragma unroll
      for (int k = 0; k < 6; ++k) amax = fmaxf(amax, absmax8(lds128(q_unit(384 + 48 * qi + 8 * k))));
      // the row's maximum over its four threads
      xmax[ch * 128 + lt] = amax;
      named_bar_sync(grp_bar, 128);
      const float rmax = fmaxf(fmaxf(xmax[lt], xmax[lt ^ 64]), fmaxf(xmax[128 + lt], xmax[128 + (lt ^ 64)]));
      named_bar_sync(grp_bar, 128);  // xmax is reused by the first tile
      const float e = rmax > 0.f ? ceilf(log2f(rmax / 448.f)) : 0.f;
      s_h = exp2f(e);
      const float inv = exp2f(-e);
      // TMEM part: 192 values -> 48 columns per term, in three groups of 16 columns
#pragma unroll 1
      for (int grp = 0; grp < 3; ++grp) {
        uint4 raw[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) raw[k] = lds128(q_unit(192 * ch + 64 * grp + 8 * k));
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          // column c of the group holds K values 4c .. 4c+3 of the group's 64
          const uint4 v = raw[c >> 1];
          const uint32_t w0 = (c & 1) ? v.z : v.x, w1 = (c & 1) ? v.w : v.y;
          const float x[4] = {bf16_lo(w0) * inv, bf16_hi(w0) * inv, bf16_lo(w1) * inv, bf16_hi(w1) * inv};
          split4(x, hi[c], lo[c]);
        }
        const uint32_t col = kTmemQ + 48u * ch + 16u * grp;
        tmem_st16(tl + col, hi);
        tmem_st16(tl + col + kTmemQTerm, lo);
      }
      // shared-memory part: 48 values = three 16-byte units per term
#pragma unroll 1
      for (int k = 0; k < 3; ++k) {
        const uint4 raw2[2] = {lds128(q_unit(384 + 48 * qi + 16 * k)), lds128(q_unit(384 + 48 * qi + 16 * k + 8))};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const uint4 v = raw2[q4 >> 1];
          const uint32_t w0 = (q4 & 1) ? v.z : v.x, w1 = (q4 & 1) ? v.w : v.y;
          const float x[4] = {bf16_lo(w0) * inv, bf16_hi(w0) * inv, bf16_lo(w1) * inv, bf16_hi(w1) * inv};
          split4(x, hi[q4], lo[q4]);
        }
        // unit gu (16 codes) of the 12 units of K 384..575: chunk cs, unit w of its 64-byte row
        const int gu = 3 * qi + k, cs = gu >> 2, w = gu & 3;
        const uint32_t off = m * 64 + ((w ^ ((m >> 1) & 3)) << 4);
        sts128(sa + kQOff + (0 * kQSmemChunks + cs) * kQChunk + off, make_uint4(hi[0], hi[1], hi[2], hi[3]));
        sts128(sa + kQOff + (1 * kQSmemChunks + cs) * kQChunk + off, make_uint4(lo[0], lo[1], lo[2], lo[3]));
      }
      // the staging areas have been read: the value ring may take its first stage
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive_local(own_bar(Q_FREE));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(lead_bar(Q_TMEM));
    }
    const float row_scale_log2 = p.scale_log2 * s_h;
    float m_used = -CUDART_INF_F, l = 0.f;
    // Control flow stays uniform even if a wait gives up (the kernel is then
    // aborting and every later wait returns at once): no barrier is skipped.
    for (int t = 0; t < n; ++t) {
      const int sb = t & 1;
      mbar_wait(own_bar(S_READY + sb), (t >> 1) & 1, abort_flag, p.status, wait_ns);
      tc_fence_after();
      uint32_t sv[16];
      tmem_ld16(tl + kTmemS + 32u * sb + 16u * ch, sv);
      tmem_wait_ld();
      // the scores are in registers: S buffer sb may take S(t+2)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(lead_bar(S_FREE + sb));
      const int j0 = (t0 + t) * kPage + 32 * half + 16 * ch;
      const int nv = max(0, min(16, j_end - j0));
      // token scales of these 16 columns (0 where masked, so that nothing a masked
      // row holds reaches P)
      float sc[16];
      mbar_wait(own_bar(SC_FULL + t % kScRing), (t / kScRing) & 1, abort_flag, p.status, wait_ns);
      {
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
      for (int j = 0; j < 16; ++j) s[j] = j < nv ? __uint_as_float(sv[j]) * sc[j] : -CUDART_INF_F;
      float mx[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) mx[k] = fmaxf(fmaxf(s[k], s[k + 4]), fmaxf(s[k + 8], s[k + 12]));
      // the softmax scale and s_h are positive: scaling commutes with the maximum.
      // The reference bounds x_j + log2(scale_j) rather than x_j, so that every
      // P~ entry p_j * scale_j stays at or below 2^8 whatever the scales.
      float lmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * row_scale_log2;
      {
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
          m_used = tmax;  // nothing accumulated yet: O and l are zero
        } else if (tmax > m_used + kRescaleThreshold) {
          alpha = ex2_approx(m_used - tmax);
          m_used = tmax;
          resc = true;
          l *= alpha;
        }
      }
      // p = 2^(x - ref); a row with nothing visible yet keeps ref = 0 so that no
      // (-inf) - (-inf) appears
      const float nref = m_used == -CUDART_INF_F ? 0.f : -m_used;
      uint32_t phi[4], plo[4];
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float x[4];
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          const int j = 4 * k + e2;
          const float pj = ex2_approx(fmaf(s[j], row_scale_log2, nref));
          ls[k] += pj;
          x[e2] = pj * sc[j];  // <= 2^8 by the choice of reference
        }
        split4(x, phi[k], plo[k]);
      }
      l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      // P buffer sb was last read by PV(t-2)
      if (t >= 2) mbar_wait(own_bar(O_DONE + sb), ((t - 2) >> 1) & 1, abort_flag, p.status, wait_ns);
      // this warp's O columns may only be rescaled once PV(t-1) has accumulated into them
      if (__any_sync(0xffffffffu, resc)) {
        if (t >= 1) {
          mbar_wait(own_bar(O_DONE + (sb ^ 1)), ((t - 1) >> 1) & 1, abort_flag, p.status, wait_ns);
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
      // P row m, tokens 32 half + 16 ch .. +15: one 16-byte unit per term
      {
        const int u = 2 * half + ch;
        const uint32_t off = m * 64 + ((u ^ ((m >> 1) & 3)) << 4);
        sts128(sa + kPOff + (sb * 2 + 0) * kPTerm + off, make_uint4(phi[0], phi[1], phi[2], phi[3]));
        sts128(sa + kPOff + (sb * 2 + 1) * kPTerm + off, make_uint4(plo[0], plo[1], plo[2], plo[3]));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(lead_bar(P_READY + sb));
    }
    if (n > 0) {
      mbar_wait(own_bar(O_DONE + ((n - 1) & 1)), ((n - 1) >> 1) & 1, abort_flag, p.status, wait_ns);
      tc_fence_after();
    }
    xl[ch * 128 + lt] = l;
    named_bar_sync(1, 256);
    const bool alive = *abort_flag == 0;
    const float ltot = (xl[lt] + xl[lt ^ 64]) + (xl[128 + lt] + xl[128 + (lt ^ 64)]);
    const bool empty = !(ltot > 0.f) || !alive;
    const float inv = empty ? 0.f : 1.f / ltot;
    const float lse = empty ? -CUDART_INF_F : (m_used + log2f(ltot)) * 0.6931471805599453f;
    const bool read_o = alive && n > 0;
    // TMEM columns 128*ch .. +127 of this lane: latent half*128 + 256*ch + 0..127
#pragma unroll 1
    for (int c0 = 0; c0 < 4; c0 += 2) {
      uint32_t ovs[2][32];
      if (read_o) {
        tmem_ld32(tl + 128u * ch + 32u * c0, ovs[0]);
        tmem_ld32(tl + 128u * ch + 32u * (c0 + 1), ovs[1]);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int j = 0; j < 32; ++j) ovs[i][j] = 0u;
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint32_t (&ov)[32] = ovs[i];
        const int col = 256 * ch + half * 128 + 32 * (c0 + i);
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
            const int uu = ((col & 63) >> 3) + k;
            sts128(base + ((uu ^ (m & 7)) << 4), v);
          }
        } else {
          if (!row_ok) continue;
          float4* dst = reinterpret_cast<float4*>(p.o_part + (qr * p.splits + split) * kDc + col);
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
        bulk_wait_read<0>();  // the staging area may be released; the writes finish with the grid
      }
    }
    if (half == 0 && ch == 0 && row_ok) {
      if (p.splits == 1) {
        if (p.lse) p.lse[qr] = lse;
      } else {
        p.lse_part[qr * p.splits + split] = lse;
      }
    }
    tc_fence_before();
  }

  // ---- teardown: both CTAs are done with TMEM and shared memory
  __syncthreads();
  cluster_arrive();
  cluster_wait();
  const bool any_abort = threadIdx.x == 0 && (ld_shared_cluster_u32(mapa(sa + kMiscOff + 4, 0)) |
                                              ld_shared_cluster_u32(mapa(sa + kMiscOff + 4, 1))) != 0;
  if (any_abort) {
    // After a wait ran out in either CTA, copies either CTA issued may still be in flight, and
    // the two producers may have stopped at different tiles.  The even CTA owns
    // the barriers that count both CTAs' score and full value stages: for a tile
    // only one CTA issued it stands in for the other CTA's part (its bytes with
    // complete_tx, its arrival with an arrive), so that each stage's last phase
    // completes once the bytes really issued have landed, and waits for it.
    // Each CTA then waits for the copies counted on its own barriers.
    const int ns0 = (int)ld_shared_cluster_u32(mapa(sa + kMiscOff + 8, 0));
    const int nv0 = (int)ld_shared_cluster_u32(mapa(sa + kMiscOff + 12, 0));
    const int ns1 = (int)ld_shared_cluster_u32(mapa(sa + kMiscOff + 8, 1));
    const int nv1 = (int)ld_shared_cluster_u32(mapa(sa + kMiscOff + 12, 1));
    int give_up = 0;
    if (r == 0) {
      for (int u = min(ns0, ns1); u < max(ns0, ns1); ++u) {
        if (ns0 > ns1) mbar_complete_tx_local(own_bar(S_FULL + u % kSStages), kSStage);
        else mbar_arrive_expect_tx_local(own_bar(S_FULL + u % kSStages), kSStage);
      }
      for (int u = min(nv0, nv1); u < max(nv0, nv1); ++u) {
        if (nv0 > nv1) {
          mbar_complete_tx_local(own_bar(V_FULL + u % kVStages), kVStage);
          mbar_arrive_local(own_bar(V_FULL + u % kVStages));
        } else {
          mbar_arrive_expect_tx_local(own_bar(V_FULL + u % kVStages), kVStage);
        }
      }
      const int ns = max(ns0, ns1), nv = max(nv0, nv1);
      for (int u = max(0, ns - kSStages); u < ns; ++u)
        mbar_wait(own_bar(S_FULL + u % kSStages), (u / kSStages) & 1, &give_up, nullptr, kDrainLimitNs);
      for (int u = max(0, nv - kVStages); u < nv; ++u)
        mbar_wait(own_bar(V_FULL + u % kVStages), (u / kVStages) & 1, &give_up, nullptr, kDrainLimitNs);
    }
    const int ns_own = r == 0 ? ns0 : ns1;
    for (int u = max(0, ns_own - kScRing); u < ns_own; ++u)
      mbar_wait(own_bar(SC_FULL + u % kScRing), (u / kScRing) & 1, &give_up, nullptr, kDrainLimitNs);
    if (issued[2]) mbar_wait(own_bar(RAW_V + (n - 1) % kVStages), 0, &give_up, nullptr, kDrainLimitNs);
    if (issued[3]) mbar_wait(own_bar(Q_STAGE), 0, &give_up, nullptr, kDrainLimitNs);
  }
  cluster_arrive();
  cluster_wait();
  if (warp == 1) tmem_dealloc_pair(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_decode_f8(const mla_decode_args_t* a, int splits, cudaStream_t stream) {
  CUtensorMap tm_ks, tm_kv, tm_o, tm_q, tm_qpe;
  const uint64_t rows_kv = (uint64_t)a->num_pages * kPage;
  const int n_tok = a->B * a->s_q;
  // query maps (values, heads, tokens), boxes of 64 values x 64 heads x 1 token:
  // a box past H reads zeros
  if (!tma_map_3d(&tm_q, a->q_lat, kDc, a->H, n_tok, kDc * 2, (uint64_t)a->H * kDc * 2, 64, 64, 1) ||
      !tma_map_3d(&tm_qpe, a->q_pe, kDr, a->H, n_tok, kDr * 2, (uint64_t)a->H * kDr * 2, 64, 64, 1))
    return cudaErrorInvalidValue;
  // score operand: (64 codes, rows, 9 chunks 64 bytes apart), 64-byte swizzle;
  // value operand: (128 codes, rows, column group 128 bytes apart, N tile 256
  // bytes apart), 128-byte swizzle
  const uint64_t dks[3] = {64, rows_kv, 9}, sks[2] = {kRow, 64};
  const uint32_t bks[3] = {64, 32, 9};
  const uint64_t dkv[4] = {128, rows_kv, 2, 2}, skv[3] = {kRow, 128, 256};
  const uint32_t bkv[4] = {128, 64, 1, 2};
  if (!tma_map_nd(&tm_ks, a->kv_cache, 3, dks, sks, bks, true, 64) ||
      !tma_map_nd(&tm_kv, a->kv_cache, 4, dkv, skv, bkv, true, 128) ||
      !tma_map_3d(&tm_o, a->o_lat, kDc, a->H, n_tok, kDc * 2, (uint64_t)a->H * kDc * 2, 64, 64, 1))
    return cudaErrorInvalidValue;
  F8Params p;
  p.q_lat = static_cast<const __nv_bfloat16*>(a->q_lat);
  p.q_pe = static_cast<const __nv_bfloat16*>(a->q_pe);
  p.kv = static_cast<const uint8_t*>(a->kv_cache);
  p.kv_scale = static_cast<const float*>(a->kv_scale);
  p.block_table = a->block_table;
  p.seq_lens = a->seq_lens;
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
  p.wait_ns = device_wait_limit_ns();
  static PerDeviceOnce attrs;
  cudaError_t e = once_per_device(attrs, [&]() {
    return cudaFuncSetAttribute(decode_f8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  });
  if (e != cudaSuccess) return e;
  dim3 grid(2 * splits, a->s_q, a->B);
  return launch_pdl(decode_f8_kernel, grid, dim3(kThreads), kSmemBytes, stream, tm_ks, tm_kv, tm_o, tm_q, tm_qpe,
                    p);
}

}  // namespace mla
