// Paged latent-attention decode over a bf16, q8_0 or q4_0 cache on the 5th-generation
// tensor cores (sm_100a): tcgen05 MMAs over a CTA pair, accumulators in tensor
// memory (TMEM), cache pages streamed by TMA.  16 to 128 heads (fewer heads pad
// the 128-row tile with zero rows: the step stays bound by the cache stream, so
// the idle rows cost tensor work only).  An e4m3 cache runs on decode_f8.cu.
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
// 36 KB) and one for the value operand (V stages of 32 KB); score stages are
// requested two tiles ahead of value stages.  Only the even CTA posts the
// expected byte count of a stage (both CTAs' bytes) on its own barrier; the odd
// CTA's TMA completes its bytes there without arriving; each slot is released by
// the commit of the MMAs that read it, so the producer refills it at once.  Each
// CTA also prefetches its half of the page two tiles ahead into L2.
// Q: latent chunks 0..5 are the A operand from TMEM; they are staged by TMA in the
// value ring (idle until page 0's value operand) and moved into TMEM by the
// softmax warps; chunks 6..7 and q_pe stay in shared memory.
// TMEM per CTA (2x2 datapath layout of the paired M = 128 MMA): O takes 256
// columns, each S buffer 32 columns (two buffers).  Lane l < 64 holds head row l
// for the first half of every N tile, lane 64 + l the same row for the second.
//
// Warp roles (384 threads): warp 0 TMA producer, warp 1 TMEM allocator and (in
// the even CTA) issuer of the score MMAs of even pages, warp 3 of odd ones, warp
// 2 (even CTA) issuer of the P.V MMAs, warps 4..11 softmax / correction /
// epilogue, two warps per TMEM lane quadrant, each thread 16 scores of a row
// half per page.
// Two S buffers: each softmax warp releases its S buffer as soon as its scores
// are in registers, so S(t+2) is issued while the softmax of t is still running
// and the tensor pipe does not wait on it; each softmax warp signals its own P
// rows to the P.V issuer.
// P is double-buffered in shared memory, so the softmax of t+1 never waits for
// P.V of t.  The output rescale is lazy: the reference maximum moves only when
// the tile maximum exceeds it by more than 2^8, so O in TMEM is rarely touched.
//
// q8_0 and q4_0 caches (ik_llama.cpp docs "FlashMLA", section "KV cache with
// MLA": int8 or 4-bit codes with one fp16 scale per 32 values): the same MMAs on
// bf16 operands.  The
// producer brings the CTA's raw codes (and their block scales) into the back half
// of its score slot; four converter warps (12..15, 512 threads in all) read them
// into registers, meet at a named barrier, and write the values code * scale
// (fp32 product, exact, rounded once to bf16) over the whole slot in the layout
// TMA gives a bf16 cache, zeros for rows past the sequence end; then they arrive
// on the even CTA's full barrier of that slot.  The value operand is not
// converted again: the converted latent chunks of the CTA's 32 rows go by eight
// 4 KB shared-memory bulk copies into rows 32r .. 32r+31 of the value slot of the
// CTA that holds their columns (four to itself, four to the peer; the 128-byte
// swizzle depends on the row mod 8 only, so the layout survives the move), and a
// converter thread relays the landing of its CTA's value slot to the even CTA.
// q4_0 rows are 288 bytes (two codes a byte, 9 KB of raw codes per slot); a
// converter splits each byte into its low half (value 2j) and high half (2j + 1).
//
// Every mbarrier wait is bounded (MLA_ERR_DEVICE_TIMEOUT in the status word);
// after one runs out every role leaves its loop, issued MMAs are drained, the
// even CTA reconciles and waits for every copy either CTA issued, and TMEM is
// freed (see the teardown).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include "proj_tile.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace mla {
uint64_t device_wait_limit_ns();

namespace {

using namespace sm100;

constexpr int kThreads = 384;                // warps 0..11
constexpr int kConvWarps = 4;                // q8_0: converter warps 12..15
constexpr int kThreadsQ8 = kThreads + 32 * kConvWarps;
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
constexpr int DRAIN = O_DONE + 2;        // [3] one per MMA-issuing warp
constexpr int S_FREE = DRAIN + 3;         // [2] in the even CTA: the softmax has read S buffer sb
constexpr int RAW_V = S_FREE + 2;         // [kVStages] a last page's value stage landed here
constexpr int Q_STAGE = RAW_V + kVStages; // Q chunks 0..5 landed in the value ring (this CTA)
constexpr int Q_MOVED = Q_STAGE + 1;      // the softmax warps have moved them into TMEM
constexpr int RAW_QS = Q_MOVED + 1;       // [kSStages] q8_0: raw codes of a score slot landed (this CTA)
constexpr int VQ_LAND = RAW_QS + kSStages; // [kVStages] q8_0: both CTAs' copies into this value slot landed
constexpr int SRC_FREE = VQ_LAND + kVStages;  // [kSStages] q8_0: the copies out of this score slot are done
constexpr int NBARS = SRC_FREE + kSStages;
constexpr int kSoftmaxWarps = 8;          // warps 4..11: two per TMEM lane quadrant
constexpr int kPrefetchTiles = MLA_TC_PREFETCH;      // L2 prefetch distance of the cache stream
constexpr uint32_t kMiscOff = kBarOff + 8 * NBARS;
constexpr uint32_t kXmaxOff = kMiscOff + 32;         // float [2 tiles][2 column halves][128 lanes]
constexpr uint32_t kXlOff = kXmaxOff + 4 * 128 * 4;  // float [2][128]
constexpr uint32_t kSmemUsed = kXlOff + 2 * 128 * 4;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;    // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget");
// q8_0: fp16 block scales beside the ring (32 rows x 18 per score slot); raw
// codes in the back half of each score slot
constexpr uint32_t kQ8RowBytes = kRow;                  // 576 int8 codes
constexpr uint32_t kQ4RowBytes = kRow / 2;              // q4_0: 576 codes, two per byte
constexpr uint32_t kQ8ScRow = 18 * 2;                   // 36 bytes of scales per row
constexpr uint32_t kQ8RawS = 32 * kQ8RowBytes;          // 18432: the CTA's 32 rows
constexpr uint32_t kQ8ScS = 32 * kQ8ScRow;              // 1152
constexpr uint32_t kQ8ScOff = (kSmemUsed + 127) / 128 * 128;  // bulk-copy destination: 16-byte aligned
constexpr uint32_t kSmemBytesQ8 = kQ8ScOff + kSStages * kQ8ScS + 1024;
static_assert(kSmemBytesQ8 <= 232448, "shared memory budget (q8_0)");
static_assert(kQ8ScOff % 16 == 0 && kQ8ScS % 16 == 0, "bulk copies into the scale area start on 16 bytes");
static_assert(kSStage == 2 * kQ8RawS, "raw codes fill the back half of a score slot");
static_assert(kQ4RowBytes % 16 == 0, "q4_0 rows start on 16 bytes");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 256;                     // S buffers at columns 256, 288
constexpr uint32_t kTmemQ = 320;                     // Q chunks 0..5: columns 320..511 (2 bf16 each)
static_assert(kTmemQ + kQTmemChunks * 32 <= kTmemCols, "TMEM budget");
constexpr uint64_t kDrainLimitNs = 100000000ull;     // 100 ms for copies already in flight
constexpr float kRescaleThreshold = 8.0f;            // log2 units

constexpr uint32_t kIdescS = idesc_bf16_f32(128, 64, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 256, false, true);

struct TcParams {
  const __nv_bfloat16* q_lat;
  const __nv_bfloat16* q_pe;
  const uint8_t* kv;
  const uint8_t* kv_scale;  // q8_0, q4_0: fp16 [pages][64][18], 16-byte aligned
  const int32_t* block_table;
  const int32_t* seq_lens;
  __nv_bfloat16* o_lat;
  float* lse;
  float* o_part;
  float* lse_part;
  uint32_t* status;
  int B, s_q, H, num_pages, max_pages, causal, splits;
  float scale_log2;
  uint64_t wait_ns;
  // fused step only: the absorption's output (q_lat, read back through tm_q),
  // the up-projection's output, and the flags between the phases (workspace)
  __nv_bfloat16* q_lat_out;
  __nv_bfloat16* out;
  uint32_t* ready;       // [token blocks]: absorption tiles done
  uint32_t* done;        // [token blocks]: decode CTAs whose o_lat rows are written
  uint32_t* exit_count;  // CTAs that have finished
  int n_tok;
};

// ---------------------------------------------------------------- fused step
// The decode step in one launch (every CTA of the grid resident at once: the
// host launches it only when the grid fits the SMs): each CTA first takes a
// share of the query absorption (tiles of 64 tokens x one head x 128 latent
// columns, three groups of four warps per CTA), then decodes its work unit as
// the standalone kernel does, its producer waiting until every absorption tile
// of its token block is written before it requests Q; after its epilogue each
// CTA counts its o_lat rows as written, and finally takes a share of the value
// up-projection (tiles of 64 tokens x one head x 32 output columns), each tile
// waiting until every decode CTA of its token block has counted.  The weights
// are read once per token block, not once per query token.  The last CTA to
// finish clears the flags for the next launch.
constexpr int kPhaseGroups = 3;                 // groups of four warps (warps 0..11)
constexpr uint32_t kPhaseRing = 48 * 1024;      // shared memory of one group
constexpr int kMaxStepBlocks = 16;              // token blocks of 64 the flags hold
static_assert(kPhaseGroups * kPhaseRing <= kPOff, "projection rings below the P buffers");
static_assert(proj::Cfg<kDn, kDc, 128, true, 2>::RING <= kPhaseRing &&
                  proj::Cfg<kDc, kDv, 32, false, 4>::RING <= kPhaseRing,
              "a projection tile fits its group's ring");

MLA_DEVI bool group_any(int bar_id, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(bar_id)
      : "memory");
  return r != 0;
}

// One projection phase of the fused step (ABSORB: q_lat = W_UK^T q_nope; else
// out = W_UV o_lat) over all CTAs of the grid.  Every thread of the CTA calls it.
template <bool ABSORB>
MLA_DEVI void step_phase(const CUtensorMap* tm_x, const CUtensorMap* tm_w, const TcParams& p, uint32_t sa,
                         uint8_t* sm) {
  const int warp = threadIdx.x >> 5;
  const int group = warp / 4;
  const uint32_t bars = sa + kPOff;  // per group: 4 stage barriers
  if (threadIdx.x == 0) {
    for (int g = 0; g < kPhaseGroups; ++g)
      for (int s = 0; s < 4; ++s) mbar_init(bars + 64 * g + 8 * s, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (group < kPhaseGroups) {
    const int gtid = threadIdx.x - 128 * group, bar_id = 13 + group;
    const int cta = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
    const int n_ctas = gridDim.x * gridDim.y * gridDim.z;
    const int n_blocks = (p.n_tok + 63) / 64;
    const int n_tiles = n_blocks * p.H * 4;  // 4 column slices: 512 / 128 or 128 / 32
    const uint32_t ring = sa + group * kPhaseRing;
    uint8_t* ring_g = sm + group * kPhaseRing;
    const uint32_t bar0 = bars + 64 * group;
    int abort = 0;
    uint32_t iter = 0;
    for (int tau = cta * kPhaseGroups + group; tau < n_tiles; tau += n_ctas * kPhaseGroups, ++iter) {
      const int tb = tau / (p.H * 4), rem = tau - tb * (p.H * 4), h = rem >> 2, sl = rem & 3;
      if constexpr (ABSORB) {
        proj::tile<kDn, kDc, 128, true, 2>(tm_x, tm_w, p.q_lat_out, p.n_tok, p.H, 64 * tb, h, 128 * sl, ring,
                                           ring_g, bar0, iter, gtid, bar_id, []() {}, abort, p.status);
        // the tile's stores (every thread of the group, ordered by the tile's last
        // group barrier) are published before the count
        if (gtid == 0) {
          fence_proxy_async_all();
          __threadfence();
          red_release_gpu_add(p.ready + tb, 1u);
        }
      } else {
        const uint32_t need = 2u * (uint32_t)min(64, p.n_tok - 64 * tb);
        // a wait that runs out is recorded and the tile goes on (on rows that may
        // not be written yet): every copy it requests still lands before the CTA
        // moves on, as on the normal path
        proj::tile<kDc, kDv, 32, false, 4>(tm_x, tm_w, p.out, p.n_tok, p.H, 64 * tb, h, 32 * sl, ring, ring_g,
                                           bar0, iter, gtid, bar_id,
                                           [&]() {
                                             if (!wait_counter_geq(p.done + tb, need, p.wait_ns))
                                               set_status(p.status, MLA_ERR_DEVICE_TIMEOUT);
                                             fence_proxy_async_all();
                                           },
                                           abort, p.status);
      }
      // a group that gave up leaves together (its stage barriers are out of step)
      if (group_any(bar_id, abort != 0)) break;
    }
  }
  // generic stores into shared memory before the asynchronous proxy writes there again
  fence_proxy_async_smem();
  __syncthreads();
  if (threadIdx.x == 0)
    for (int g = 0; g < kPhaseGroups; ++g)
      for (int s = 0; s < 4; ++s) mbar_inval(bars + 64 * g + 8 * s);
  __syncthreads();
}

// q8_0 value of one code: the byte with its sign bit flipped, put under the
// exponent of 2^23, is 2^23 + 128 + code exactly; subtracting gives the code,
// and code * scale (8 x 11 significant bits) is exact in fp32.
MLA_DEVI float q8_code(uint32_t word_flipped, int k) {
  return __int_as_float((int)__byte_perm(word_flipped, 0x4B000000u, 0x7440u + k)) - 8388736.0f;
}
// q4_0 value of one code: byte k of a word of 4-bit numbers (code + 8, one per
// byte after the split into low and high halves) under the exponent of 2^23.
MLA_DEVI float q4_code(uint32_t nibbles, int k) {
  return __int_as_float((int)__byte_perm(nibbles, 0x4B000000u, 0x7440u + k)) - 8388616.0f;
}

// KV: 0 bf16 cache; 1 q8_0 and 2 q4_0 caches, expanded to bf16 by converter warps.
// FUSED: the whole decode step (absorption, decode, up-projection) in one launch;
// tm_qn, tm_wuk, tm_ol, tm_wuv are its projection operands (unused otherwise).
template <int KV, bool FUSED>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(KV != 0 ? kThreadsQ8 : kThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qpe,
                     const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_kv,
                     const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ CUtensorMap tm_qn,
                     const __grid_constant__ CUtensorMap tm_wuk, const __grid_constant__ CUtensorMap tm_ol,
                     const __grid_constant__ CUtensorMap tm_wuv, const TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
  uint8_t* sm = smem_raw + pad;
  const uint32_t sa = raw_addr + pad;
  constexpr bool Q8 = KV != 0;  // a blockwise cache (q8_0 or q4_0) through the converter warps
  constexpr bool Q4 = KV == 2;
  constexpr uint32_t kRawRow = Q4 ? kQ4RowBytes : kQ8RowBytes;  // stored bytes of a cache row
  constexpr uint32_t kRawS = 32 * kRawRow;                       // the CTA's 32 rows of a page

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t r = cluster_ctarank();
  const int split = blockIdx.x >> 1, g = blockIdx.y, b = blockIdx.z;

  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kMiscOff + 4);
  // producer's issue counts, read by the teardown: score tiles, full value pages,
  // last (partial) value page issued, Q issued
  uint32_t* issued = reinterpret_cast<uint32_t*>(sm + kMiscOff + 8);
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
    for (int i = 0; i < 4; ++i) issued[i] = 0;
    // a full score stage is the even CTA's expect_tx plus both CTAs' TMA bytes, a
    // full value stage that and the odd CTA's arrival (a last, partial page
    // instead takes one arrival per CTA after its tail rows are zeroed)
    // q8_0: a full stage is the arrival of both CTAs' converter warps instead
    for (int i = 0; i < kSStages; ++i) {
      mbar_init(own_bar(S_FULL + i), Q8 ? 2 * kConvWarps : 1);
      mbar_init(own_bar(S_EMPTY + i), 1);
      mbar_init(own_bar(RAW_QS + i), 1);
    }
    // (a full value stage: two arrivals either way; q8_0: one relay per CTA)
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(own_bar(V_FULL + i), 2);
      mbar_init(own_bar(V_EMPTY + i), 1);
      mbar_init(own_bar(RAW_V + i), 1);
      mbar_init(own_bar(VQ_LAND + i), 1);
    }
    for (int i = 0; i < kSStages; ++i) mbar_init(own_bar(SRC_FREE + i), 1);
    mbar_init(own_bar(Q_TMEM), 2 * kSoftmaxWarps);
    mbar_init(own_bar(Q_FULL), 1);
    mbar_init(own_bar(Q_STAGE), 1);
    // q8_0: the value ring of either CTA takes copies from both, so Q must have
    // left the ring in both CTAs
    mbar_init(own_bar(Q_MOVED), Q8 ? 2 * kSoftmaxWarps : kSoftmaxWarps);
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
  if constexpr (FUSED) {
    // q_nope, the weights and the workspace may come from or be read by the
    // kernels before this one
    pdl_wait();
    step_phase<true>(&tm_qn, &tm_wuk, p, sa, sm);
  }

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
  const uint64_t wait_ns = p.wait_ns;

  if (warp == 0) {
    // =========================== TMA producer ===========================
    // S(u) is the CTA's 32 tokens x 576 of page u (one 36 KB score stage), V(u)
    // the page's 64 tokens x the CTA's latent columns of both P.V halves (one
    // 32 KB value stage); requests go S(0), S(1), S(2), V(0), S(3), V(1), ...
    int n_s = 0, n_v = 0, v_part = 0, q_iss = 0;
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
      auto prefetch = [&](int u) {
        const int pg = page_of(u, blk_p, pg_p);
        constexpr uint32_t kRowBytes = Q8 ? kRawRow : kRow * 2;
        if (lane == 0) prefetch_l2_bulk(p.kv + ((size_t)pg * kPage + 32 * r) * kRowBytes, 32 * kRowBytes);
      };
      auto load_s = [&](int u) -> bool {
        const int st = u % kSStages;
        const uint32_t ph = ((u / kSStages) & 1) ^ 1;
        if (!mbar_wait_converged(own_bar(S_EMPTY + st), ph, abort_flag, p.status, wait_ns)) return false;
        const int pg = page_of(u, blk_s, pg_s);
        const uint32_t dst = sa + kSOff + st * kSStage;
        if constexpr (Q8) {
          // the CTA's 32 rows of codes (contiguous) into the back half of the slot,
          // their block scales beside the ring; the converters take it from there.
          // The slot's last page must also have been copied out to the value slots.
          if (!mbar_wait_converged(own_bar(SRC_FREE + st), ph, abort_flag, p.status, wait_ns)) return false;
          if (lane == 0) {
            const size_t row0 = (size_t)pg * kPage + 32 * r;
            mbar_arrive_expect_tx_local(own_bar(RAW_QS + st), kRawS + kQ8ScS);
            bulk_load_cta(dst + kQ8RawS, p.kv + row0 * kRawRow, kRawS, own_bar(RAW_QS + st));
            bulk_load_cta(sa + kQ8ScOff + st * kQ8ScS, p.kv_scale + row0 * kQ8ScRow, kQ8ScS,
                          own_bar(RAW_QS + st));
          }
          __syncwarp();
          n_s = u + 1;
          if (u > 0 && u + kPrefetchTiles < n) prefetch(u + kPrefetchTiles);
          return true;
        }
        // one box: (64 values, 32 rows, 9 chunks) lands chunk-major, 9 x 4 KB
        const uint32_t fb = lead_bar(S_FULL + st);
        if (r == 0) mbar_arrive_expect_tx_local_elect(own_bar(S_FULL + st), 2 * kSStage);
        tma_load_3d_pair_elect(dst, &tm_ks, fb, 0, pg * kPage + 32 * (int)r, 0);
        n_s = u + 1;
        if (u > 0 && u + kPrefetchTiles < n) prefetch(u + kPrefetchTiles);
        return true;
      };
      auto load_v = [&](int u) -> bool {
        if constexpr (Q8) {
          // the value slots are filled by the converters' copies
          n_v = u + 1;
          return true;
        }
        const int st = u % kVStages;
        const uint32_t ph = ((u / kVStages) & 1) ^ 1;
        if (!mbar_wait_converged(own_bar(V_EMPTY + st), ph, abort_flag, p.status, wait_ns)) return false;
        const int pg = page_of(u, blk_v, pg_v);
        const uint32_t dst = sa + kVOff + st * kVStage;
        const int nvalid = j_end - (t0 + u) * kPage;  // cached rows of this page inside the sequence
        if (nvalid >= kPage) {
          // one box: (64 values, 64 rows, chunks 2r and 2r+1, groups 0 and 1): latent
          // chunks {2r, 2r+1, 4+2r, 5+2r} of the page, 4 x 8 KB
          const uint32_t fb = lead_bar(V_FULL + st);
          if (r == 0) mbar_arrive_expect_tx_local_elect(own_bar(V_FULL + st), 2 * kVStage);
          else if (lane == 0) mbar_arrive_remote_relaxed(fb);
          tma_load_4d_pair_elect(dst, &tm_kv, fb, 0, pg * kPage, 2 * (int)r, 0);
          n_v = u + 1;
        } else {
          // The last page of the sequence: P is 0 past the end, but 0 * NaN is
          // not, so whatever those rows hold is replaced by zeros before the MMA.
          // The stage lands on this CTA's own barrier (once per work unit).
          if (lane == 0) {
            mbar_arrive_expect_tx_local(own_bar(RAW_V + st), kVStage);
            tma_load_4d_cta(dst, &tm_kv, own_bar(RAW_V + st), 0, pg * kPage, 2 * (int)r, 0);
          }
          __syncwarp();
          v_part = 1;
          if (!mbar_wait_converged(own_bar(RAW_V + st), 0, abort_flag, p.status, wait_ns)) return false;
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
      if constexpr (FUSED) {
        // every absorption tile of this token's block written (by any CTA).  A wait
        // that runs out is recorded and Q is requested all the same (both CTAs of
        // the pair then keep the same count of copies on the pair's barriers).
        if (lane == 0) {
          if (!wait_counter_geq(p.ready + (b * p.s_q + g) / 64, 4u * (uint32_t)p.H, wait_ns))
            set_status(p.status, MLA_ERR_DEVICE_TIMEOUT);
          fence_proxy_async_all();
        }
        __syncwarp();
      } else {
        pdl_wait();
      }
      if (lane == 0) {
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
      q_iss = 1;
      // nothing else is requested until Q has landed: at start-up every CTA asks
      // for its first bytes at once, and Q and page 0 gate the first MMA
      if (ok) ok = mbar_wait_converged(own_bar(Q_STAGE), 0, abort_flag, p.status, wait_ns);
      for (int u = 1; u < n && u <= kPrefetchTiles; ++u) prefetch(u);
      // score stages are requested two tiles ahead of value stages (the third
      // score stage allows it), so that a score stage's load latency is not on
      // the score MMA -> softmax -> P.V chain (V3 decode 75.6 -> 71.7 us)
      if (ok && n > 1) ok = load_s(1);
      for (int u = 0; ok && u < n; ++u) {
        if (u + 2 < n) ok = load_s(u + 2);
        if (!Q8 && u == 0 && ok) ok = mbar_wait_converged(own_bar(Q_MOVED), 0, abort_flag, p.status, wait_ns);
        if (ok) ok = load_v(u);
      }
    }
    if (lane == 0) {
      issued[0] = n_s;
      issued[1] = n_v;
      if (!Q8) issued[2] = v_part;  // q8_0: the converters' copy count
      issued[3] = q_iss;
    }
  } else if (warp >= 1 && warp <= 3) {
    // ==== MMA issuers (even CTA): warps 1 and 3 scores, warp 2 P.V ====
    // The two streams touch disjoint TMEM (S buffers / O) and shared memory
    // (Q and the S ring / P and the V ring), so they are issued independently.
    if (r == 0 && n > 0) {
      const uint64_t dq = desc_sw128(sa + kQOff, 16, 1024);
      const uint64_t ds = desc_sw128(sa + kSOff, 16, 1024);
      const uint64_t dv = desc_sw128(sa + kVOff, kChunkV, 1024);
      const uint64_t dp = desc_sw128(sa + kPOff, 16, 1024);
      bool ok = true;
      if (warp != 2) {
        ok = mbar_wait_converged(own_bar(Q_FULL), 0, abort_flag, p.status, wait_ns) &&
             mbar_wait_converged(own_bar(Q_TMEM), 0, abort_flag, p.status, wait_ns);
        // Warp 1 issues the even pages, warp 3 the odd ones.  Issuing 36 MMAs takes
        // the issue slots of the warp's SM sub-partition, whose softmax warps then
        // fall behind; two issuers halve that.  Each page's waits (S buffer free,
        // then stage full) imply that the stage's previous phase has completed, so
        // that parity waits stay exact with two issuers.
        for (int u = warp == 3 ? 1 : 0; ok && u < n; u += 2) {
          const int st = u % kSStages, sb = u & 1;
          // S buffer sb was last read by the softmax of tile u-2 (released as soon as
          // its scores are in registers)
          if (u >= 2 && !mbar_wait_converged(own_bar(S_FREE + sb), ((u - 2) >> 1) & 1, abort_flag, p.status,
                                             wait_ns))
            break;
          if (!mbar_wait_converged<Q8>(own_bar(S_FULL + st), (u / kSStages) & 1, abort_flag, p.status, wait_ns))
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
          if (!mbar_wait_converged(own_bar(P_READY + pb), (t >> 1) & 1, abort_flag, p.status, wait_ns))
            break;
          if (!mbar_wait_converged<Q8>(own_bar(V_FULL + st), (t / kVStages) & 1, abort_flag, p.status, wait_ns))
            break;
          tc_fence_after();
          if constexpr (Q8) {
            // every copy out of page t's score slots has landed: both producers may
            // refill them (once the score MMAs are done with them too)
            if (lane == 0) {
              mbar_arrive_remote(own_bar(SRC_FREE + t % kSStages));
              mbar_arrive_remote(mapa(own_bar(SRC_FREE + t % kSStages), 1));
            }
          }
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
      // every MMA this warp issued has completed before TMEM and shared memory are released
      const int db = DRAIN + warp - 1;
      commit_pair_mc_elect(own_bar(db), 0x1);
      int keep_waiting = 0;
      mbar_wait_converged(own_bar(db), 0, &keep_waiting, p.status, kDrainLimitNs);
    }
  } else if (warp < 12) {
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
      static_assert(kQTmemChunks % 2 == 0, "Q chunks split evenly between the column halves");
      constexpr int kPerWarp = kQTmemChunks / 2;
      // the chunks were staged by TMA (128-byte swizzled rows of 64 heads); read
      // this row's, store them into TMEM, then free the staging area
      mbar_wait(own_bar(Q_STAGE), 0, abort_flag, p.status, wait_ns);
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
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_remote(lead_bar(Q_TMEM));
        mbar_arrive_remote(own_bar(Q_MOVED));
        if (Q8) mbar_arrive_remote(mapa(own_bar(Q_MOVED), r ^ 1));
      }
    }
    float m_used = -CUDART_INF_F, l = 0.f;
    const int lim = min(vis, j_end);
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
    const size_t orow = ((size_t)b * p.s_q + g) * p.H + (row_ok ? head : 0);
    const bool read_o = alive && n > 0;
    // TMEM columns 128*ch .. +127 of this lane: latent half*128 + 256*ch + 0..127,
    // loaded kEpi x 32 columns at a time (one wait per group)
    constexpr int kEpi = 2;
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
        if constexpr (FUSED) {
          // the rows are read by other CTAs of this grid: written, then counted
          bulk_wait_all();
          fence_proxy_async_all();
          __threadfence();
          red_release_gpu_add(p.done + qtok / 64, 1u);
        } else {
          bulk_wait_read<0>();  // the staging area may be released; the writes finish with the grid
        }
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
  } else if constexpr (Q8) {
    // ================= q8_0 / q4_0 converters (warps 12..15) =================
    // Per page: the score slot (this CTA's 32 rows x 576 values, 9 chunks of
    // 32 rows x 128 bytes, 128-byte swizzle) and the value slot (64 rows x the
    // CTA's latent chunks 2r, 2r+1, 4+2r, 5+2r, 4 chunks of 64 rows x 128 bytes).
    // The raw codes sit in the back half of the slot they expand into, so every
    // thread reads its share into registers before any thread writes.  The four
    // warps meet at named barriers, so they leave the loop together: the
    // outcome of each wait is combined over the group first.
    const int ct = threadIdx.x - kThreads;  // 0 .. 127
    const __half* scs = reinterpret_cast<const __half*>(sm + kQ8ScOff);
    auto conv_s = [&](int u) -> bool {
      const int tok0 = (t0 + u) * kPage;  // first token of the page
      {
        const int st = u % kSStages;
        const bool got = mbar_wait_converged(own_bar(RAW_QS + st), (u / kSStages) & 1, abort_flag, p.status, wait_ns);
        if (!named_bar_and(6, 32 * kConvWarps, got)) return false;
        const uint32_t slot = sa + kSOff + st * kSStage;
        // unit i of a thread: values k0 .. k0+15 of one row (16 bytes of q8_0
        // codes, 8 bytes of q4_0 codes)
        uint4 raw[9];
#pragma unroll
        for (int i = 0; i < 9; ++i) {
          const int q = ct + 128 * i, row = q / 36, k0 = 16 * (q % 36);
          if constexpr (Q4) {
            const uint2 h = lds64(slot + kQ8RawS + row * kRawRow + (k0 >> 1));
            raw[i] = make_uint4(h.x, h.y, 0u, 0u);
          } else {
            raw[i] = lds128(slot + kQ8RawS + row * kRawRow + k0);
          }
        }
        named_bar_sync(6, 32 * kConvWarps);
#pragma unroll
        for (int i = 0; i < 9; ++i) {
          const int q = ct + 128 * i, row = q / 36, k0 = 16 * (q % 36);
          const bool live = tok0 + 32 * (int)r + row < j_end;
          const float d = live ? __half2float(scs[(st * 32 + row) * 18 + (k0 >> 5)]) : 0.f;
          uint32_t o[8];
          if constexpr (Q4) {
            // byte m of a word holds values 2m (low half) and 2m + 1 (high half)
            const uint32_t lo[2] = {raw[i].x & 0x0F0F0F0Fu, raw[i].y & 0x0F0F0F0Fu};
            const uint32_t hi[2] = {(raw[i].x >> 4) & 0x0F0F0F0Fu, (raw[i].y >> 4) & 0x0F0F0F0Fu};
#pragma unroll
            for (int k = 0; k < 8; ++k)
              o[k] = pack_bf16(q4_code(lo[k >> 2], k & 3) * d, q4_code(hi[k >> 2], k & 3) * d);
          } else {
            const uint32_t w[4] = {raw[i].x ^ 0x80808080u, raw[i].y ^ 0x80808080u, raw[i].z ^ 0x80808080u,
                                   raw[i].w ^ 0x80808080u};
#pragma unroll
            for (int k = 0; k < 8; ++k)
              o[k] = pack_bf16(q8_code(w[k >> 1], 2 * (k & 1)) * d, q8_code(w[k >> 1], 2 * (k & 1) + 1) * d);
          }
          const int c = k0 >> 6, unit = (k0 & 63) >> 3;
          const uint32_t base = slot + c * kChunkS + row * 128;
          sts128(base + (((unit) ^ (row & 7)) << 4), make_uint4(o[0], o[1], o[2], o[3]));
          sts128(base + (((unit + 1) ^ (row & 7)) << 4), make_uint4(o[4], o[5], o[6], o[7]));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote_release_cluster(lead_bar(S_FULL + st));
        // every converter warp's stores are visible to the bulk copies below
        named_bar_sync(6, 32 * kConvWarps);
      }
      return true;
    };
    // Warp 12 copies the converted latent chunks of page u out of the score slot:
    // latent chunk c (32 rows x 128 bytes) of this CTA's rows goes to rows
    // 32r .. 32r+31 of value chunk j of the CTA that holds chunk c's columns
    // (chunks 0, 1, 4, 5 to the even CTA, 2, 3, 6, 7 to the odd one, j = 2 (c / 4)
    // + c % 2), landing on that CTA's value-slot barrier.  A wait that gives up
    // here sets the abort flag; the group leaves at its next reduction barrier.
    int copied = 0;
    auto copy_v = [&](int u) {
      if (warp != 12) return;
      const int vs = u % kVStages;
      bool got = u > 0 || mbar_wait_converged<true>(own_bar(Q_MOVED), 0, abort_flag, p.status, wait_ns);
      if (got) got = mbar_wait_converged(own_bar(V_EMPTY + vs), ((u / kVStages) & 1) ^ 1, abort_flag, p.status, wait_ns);
      if (!got) return;
      if (lane == 0) {
        mbar_arrive_expect_tx_local(own_bar(VQ_LAND + vs), kVStage);  // 4 chunks from each CTA
        const uint32_t src = sa + kSOff + (u % kSStages) * kSStage;
        for (int c = 0; c < 8; ++c) {
          const uint32_t to = (c >> 1) & 1, j = 2 * (c >> 2) + (c & 1);
          bulk_copy_s2s(mapa(sa + kVOff + vs * kVStage + j * kChunkV + 32 * r * 128, to), src + c * kChunkS,
                        kChunkS, mapa(own_bar(VQ_LAND + vs), to));
        }
      }
      __syncwarp();
      copied = u + 1;
    };
    // ... and tells the even CTA once both CTAs' copies into this value slot landed
    auto relay = [&](int u) {
      if (warp != 12) return;
      const int vs = u % kVStages;
      if (!mbar_wait_converged<true>(own_bar(VQ_LAND + vs), (u / kVStages) & 1, abort_flag, p.status, wait_ns))
        return;
      if (lane == 0) mbar_arrive_remote_release_cluster(lead_bar(V_FULL + vs));
    };
    // score slots one page ahead of the value slots' relay; control flow stays
    // uniform across the four warps (only conv_s ends the loop)
    bool ok = n > 0 ? conv_s(0) : true;
    if (ok && n > 0) copy_v(0);
    for (int u = 0; ok && u < n; ++u) {
      if (u + 1 < n) {
        ok = conv_s(u + 1);
        if (ok) copy_v(u + 1);
      }
      if (ok) relay(u);
    }
    if (warp == 12 && lane == 0) issued[2] = copied;
  }

  // ---- teardown: both CTAs are done with TMEM and shared memory
  __syncthreads();
  cluster_arrive();
  cluster_wait();
  const bool any_abort = threadIdx.x == 0 && (ld_shared_cluster_u32(mapa(sa + kMiscOff + 4, 0)) |
                                              ld_shared_cluster_u32(mapa(sa + kMiscOff + 4, 1))) != 0;
  if (any_abort) {
    // After a wait ran out in either CTA, copies either CTA issued may still be
    // in flight, and the two producers may have stopped at different tiles.  The
    // even CTA owns the barriers that count both CTAs' score stages, full value
    // stages and Q: for a tile only one CTA issued it stands in for the other
    // CTA's part (its bytes with complete_tx, its arrival with an arrive), so that
    // each stage's last phase completes once the bytes really issued have landed,
    // and waits for it.  Each CTA then waits for the copies counted on its own
    // barriers (Q's TMEM part, a last partial value page).
    const int ns0 = (int)ld_shared_cluster_u32(mapa(sa + kMiscOff + 8, 0));
    const int nv0 = (int)ld_shared_cluster_u32(mapa(sa + kMiscOff + 12, 0));
    const int ns1 = (int)ld_shared_cluster_u32(mapa(sa + kMiscOff + 8, 1));
    const int nv1 = (int)ld_shared_cluster_u32(mapa(sa + kMiscOff + 12, 1));
    int give_up = 0;
    if constexpr (Q8) {
      // q8_0: the raw codes of every slot land on this CTA's own barriers; the
      // full barriers count the converters' arrivals only (no bytes in flight)
      const int ns = r == 0 ? ns0 : ns1;
      for (int u = max(0, ns - kSStages); u < ns; ++u)
        mbar_wait(own_bar(RAW_QS + u % kSStages), (u / kSStages) & 1, &give_up, nullptr, kDrainLimitNs);
      // copies into this CTA's value slots: for a page only one CTA copied, stand in
      // for the other CTA's half (its arrival, or its 16 KB), then wait for the
      // pages still open
      const int own = (int)issued[2], peer = (int)ld_shared_cluster_u32(mapa(sa + kMiscOff + 16, r ^ 1));
      for (int u = min(own, peer); u < max(own, peer); ++u) {
        if (own > peer) mbar_complete_tx_local(own_bar(VQ_LAND + u % kVStages), kVStage / 2);
        else mbar_arrive_expect_tx_local(own_bar(VQ_LAND + u % kVStages), kVStage / 2);
      }
      const int nc = max(own, peer);
      for (int u = max(0, nc - kVStages); u < nc; ++u)
        mbar_wait(own_bar(VQ_LAND + u % kVStages), (u / kVStages) & 1, &give_up, nullptr, kDrainLimitNs);
      if (r == 0 && issued[3]) mbar_wait(own_bar(Q_FULL), 0, &give_up, nullptr, kDrainLimitNs);
    } else if (r == 0) {
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
      // both CTAs request Q whenever their (common) work unit is not empty
      if (issued[3]) mbar_wait(own_bar(Q_FULL), 0, &give_up, nullptr, kDrainLimitNs);
    }
    if (issued[3]) mbar_wait(own_bar(Q_STAGE), 0, &give_up, nullptr, kDrainLimitNs);
    if (!Q8 && issued[2]) mbar_wait(own_bar(RAW_V + (n - 1) % kVStages), 0, &give_up, nullptr, kDrainLimitNs);
  }
  cluster_arrive();
  cluster_wait();
  if (warp == 1) tmem_dealloc_pair(tmem, kTmemCols);
  if constexpr (FUSED) {
    __syncthreads();
    step_phase<false>(&tm_ol, &tm_wuv, p, sa, sm);
    // the last CTA out clears the flags for the next launch (every CTA is past
    // its last use of them once it has counted itself here)
    if (threadIdx.x == 0) {
      __threadfence();
      const uint32_t n_ctas = gridDim.x * gridDim.y * gridDim.z;
      if (atomicAdd(p.exit_count, 1u) == n_ctas - 1) {
        const int n_blocks = (p.n_tok + 63) / 64;
        for (int i = 0; i < n_blocks; ++i) {
          p.ready[i] = 0u;
          p.done[i] = 0u;
        }
        *p.exit_count = 0u;
        __threadfence();
      }
    }
  }
}

// ---------------------------------------------------------------- host side
// One instance's launch: the kernel attributes once per device, then the launch.
template <int KV, bool F>
cudaError_t launch_inst(dim3 grid, const CUtensorMap (&m)[9], const TcParams& p, cudaStream_t stream) {
  constexpr uint32_t threads = KV != 0 ? kThreadsQ8 : kThreads;
  constexpr uint32_t smem = KV != 0 ? kSmemBytesQ8 : kSmemBytes;
  static PerDeviceOnce attrs;
  cudaError_t e = once_per_device(attrs, [&]() {
    cudaError_t e2 = cudaFuncSetAttribute(decode_tc_kernel<KV, F>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)smem);
    if (e2 != cudaSuccess) return e2;
    return cudaFuncSetAttribute(decode_tc_kernel<KV, F>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  });
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_tc_kernel<KV, F>, grid, dim3(threads), smem, stream, m[0], m[1], m[2], m[3], m[4], m[5],
                    m[6], m[7], m[8], p);
}

// fx: the fused step's extra operands (nullptr: the decode alone)
cudaError_t launch_tc(const mla_decode_args_t* a, int splits, cudaStream_t stream,
                      const StepOperands* fx = nullptr) {
  CUtensorMap tm_q, tm_qpe, tm_ks, tm_kv, tm_o;  // tm_o: o_lat, the single-split result
  const uint64_t rows_kv = (uint64_t)a->num_pages * kPage;
  const int n_tok = a->B * a->s_q;
  // query maps are 3-D (values, heads, tokens) so that a 64-head box past H reads zeros
  if (!tma_map_3d(&tm_q, a->q_lat, kDc, a->H, n_tok, kDc * 2, (uint64_t)a->H * kDc * 2, 64, 64, 1) ||
      !tma_map_3d(&tm_qpe, a->q_pe, kDr, a->H, n_tok, kDr * 2, (uint64_t)a->H * kDr * 2, 64, 64, 1) ||
      !tma_map_3d(&tm_o, a->o_lat, kDc, a->H, n_tok, kDc * 2, (uint64_t)a->H * kDc * 2, 64, 64, 1))
    return cudaErrorInvalidValue;
  // score operand: (64 values, rows, 9 chunks 128 bytes apart), one box per stage;
  // value operand: (64 values, rows, 4 chunks 128 bytes apart, 2 groups 512 bytes
  // apart), one box of 2 x 2 chunks per stage
  const bool q8 = a->kv_dtype == MLA_KV_Q8_0, q4 = a->kv_dtype == MLA_KV_Q4_0;
  if (q8 || q4) {
    // q8_0, q4_0: the raw codes come by bulk copies and the value operand from the
    // converted score slots; the cache maps are not read (any valid map will do)
    const uint64_t rb = q4 ? kQ4RowBytes : kQ8RowBytes;
    const uint64_t dq[2] = {rb, rows_kv}, sq[1] = {rb};
    const uint32_t bq[2] = {128, 64};
    if (!tma_map_nd(&tm_kv, a->kv_cache, 2, dq, sq, bq, true, 0)) return cudaErrorInvalidValue;
    tm_ks = tm_kv;
  } else {
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
  p.kv_scale = static_cast<const uint8_t*>(a->kv_scale);
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
  p.wait_ns = device_wait_limit_ns();
  p.n_tok = n_tok;
  p.q_lat_out = nullptr;
  p.out = nullptr;
  p.ready = p.done = p.exit_count = nullptr;
  // the fused step's projection operands: absorption X = q_nope (values, heads,
  // tokens; 64-token boxes) and W_UK (512 columns, H x 128 rows); up-projection
  // X = o_lat and W_UV (512 columns, H x 128 rows, 32-row boxes)
  CUtensorMap m[9] = {tm_q, tm_qpe, tm_ks, tm_kv, tm_o, tm_q, tm_q, tm_q, tm_q};
  if (fx) {
    if (!tma_map_3d(&m[5], fx->q_nope, kDn, a->H, n_tok, kDn * 2, (uint64_t)a->H * kDn * 2, 64, 1, proj::TM) ||
        !tma_map_2d(&m[6], fx->w_uk, kDc, (uint64_t)a->H * kDn, kDc * 2, 64, proj::TK) ||
        !tma_map_3d(&m[7], a->o_lat, kDc, a->H, n_tok, kDc * 2, (uint64_t)a->H * kDc * 2, 64, 1, proj::TM) ||
        !tma_map_2d(&m[8], fx->w_uv, kDc, (uint64_t)a->H * kDv, kDc * 2, 64, 32))
      return cudaErrorInvalidValue;
    p.q_lat_out = static_cast<__nv_bfloat16*>(const_cast<void*>(a->q_lat));
    p.out = static_cast<__nv_bfloat16*>(fx->out);
    p.ready = fx->flags;
    p.done = fx->flags + kMaxStepBlocks;
    p.exit_count = fx->flags + 2 * kMaxStepBlocks;
  }
  const dim3 grid(2 * splits, a->s_q, a->B);
  if (fx) {
    if (q8) return launch_inst<1, true>(grid, m, p, stream);
    if (q4) return launch_inst<2, true>(grid, m, p, stream);
    return launch_inst<0, true>(grid, m, p, stream);
  }
  if (q8) return launch_inst<1, false>(grid, m, p, stream);
  if (q4) return launch_inst<2, false>(grid, m, p, stream);
  return launch_inst<0, false>(grid, m, p, stream);
}

}  // namespace

// Whether the tensor-memory kernels (this one for a bf16 cache, decode_f8.cu for
// an e4m3 cache) take these arguments.
bool decode_tc_supported(const mla_decode_args_t* a) {
  // any head count up to 128 (rows beyond H pad the 128-row tile); a bf16 cache,
  // or an e4m3, q8_0 or q4_0 cache whose scale array starts on 16 bytes (bulk copies)
  if (a->H % 16 != 0 || a->H > 128) return false;
  if (a->kv_dtype == MLA_KV_BF16) return true;
  return (a->kv_dtype == MLA_KV_FP8_E4M3 || a->kv_dtype == MLA_KV_Q8_0 || a->kv_dtype == MLA_KV_Q4_0) &&
         (reinterpret_cast<uintptr_t>(a->kv_scale) & 15u) == 0;
}

int decode_tc_clusters_per_split(const mla_decode_args_t* a) { return a->B * a->s_q; }

cudaError_t launch_decode_tc(const mla_decode_args_t* a, int splits, cudaStream_t stream) {
  return launch_tc(a, splits, stream);
}

// CTA pairs of the fused kernel the current device holds at once (0 if unknown),
// queried once per device: the GPCs decide how many pairs fit, not the SM count.
int fused_cluster_capacity(bool coded) {
  static PerDeviceOnce once[2];
  static std::atomic<int> cap[2][PerDeviceOnce::kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= PerDeviceOnce::kMaxDevices) return 0;
  once_per_device(once[coded], [&]() {
    auto kern = coded ? decode_tc_kernel<1, true> : decode_tc_kernel<0, true>;
    const uint32_t smem = coded ? kSmemBytesQ8 : kSmemBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(coded ? kThreadsQ8 : kThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
    if (e == cudaSuccess) cap[coded][dev].store(n, std::memory_order_relaxed);
    return e;
  });
  return cap[coded][dev].load(std::memory_order_relaxed);
}

// The fused step takes one split, a cache this kernel reads, a grid whose CTA
// pairs the device holds all at once (one pair per query token) and token
// blocks the flags hold.
bool decode_step_fusable(const mla_decode_args_t* a, int splits) {
  const int n_tok = a->B * a->s_q;
  if (!(splits == 1 && a->kv_dtype != MLA_KV_FP8_E4M3 && decode_tc_supported(a) && n_tok > 0 &&
        (n_tok + 63) / 64 <= kMaxStepBlocks))
    return false;
  return n_tok <= fused_cluster_capacity(a->kv_dtype != MLA_KV_BF16);
}

size_t decode_step_flag_bytes() { return 3 * kMaxStepBlocks * sizeof(uint32_t); }

cudaError_t launch_decode_step_fused(const mla_decode_args_t* a, const StepOperands* fx, cudaStream_t stream) {
  return launch_tc(a, 1, stream, fx);
}

}  // namespace mla
