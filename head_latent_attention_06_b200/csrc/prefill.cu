// Prefill (chunks of many new tokens) in the explicit form of the attention,
// on the tcgen05 tensor cores (sm_100a).
//
// The architecture ("MLA: Multi-Head Latent Attention — DeepSeek-AI Explained",
// section "Architecture") defines keys and values as up-projections of the
// cached latent, k_t = [W_UK c_t ; k_pe_t] and v_t = W_UV c_t per head; the
// absorbed form of the decode kernels avoids forming them, which pays while few
// queries share the cache (snowgate thread 35: decode is bound by the cache,
// prefill by compute).  Per (query, cached token, head) the absorbed form costs
// 2 (576 + 512) = 2176 FLOPs, the explicit one 2 (192 + 128) = 640 plus, once per
// cached token and head, the two up-projections 2 * 2 * 128 * 512 = 262144; so
// beyond about 170 queries per sequence the explicit form does less work.
//
// Two kernels:
//   kv_up:   Kn[b][h][t] = W_UK[h] c_t and V[b][h][t] = W_UV[h] c_t (bf16, 128 each)
//            for every cached token t of every sequence: per CTA two GEMMs with
//            M = 128 tokens (two pages each, TMA from the paged cache), sharing
//            the B operand N = 256 (the head's W_UK and W_UV rows), K = 512 in
//            chunks of 64, accumulated in two TMEM accumulators (256 columns
//            each).  Sharing the weight chunk between 256 tokens cuts the
//            operand bytes per MMA by a third against one 128-token tile.
//   attn:    FlashAttention forward per (sequence, head, 2 x 128 queries): S = Q K^T
//            with Q = [q_nope | q_pe] (192), K = [Kn | k_pe] (k_pe from the cache,
//            shared by all heads), M = 128 queries, N = 128 keys; online softmax
//            (exp2, lazy rescale of O by more than 2^8); O += P V with P in TMEM
//            (it replaces S in place, each thread owning one query row) and V
//            from shared memory.  The output is o = sum_j p_j v_j directly, with
//            lse: no up-projection follows.
// Causal: new token i of a sequence of length L sits at position L - s_q + i and
// sees the cached tokens 0 .. L - s_q + i.
#include <cuda.h>
#include <math_constants.h>

#include "sm100.cuh"
#include "tma_host.cuh"

namespace mla {
uint64_t device_wait_limit_ns();

namespace {

using namespace sm100;

constexpr uint64_t kDrainNs = 100000000ull;

// ---------------------------------------------------------------- kv_up
constexpr int kUpThreads = 128;
constexpr int kUpStages = 3;
constexpr int kUpTok = 256;                  // tokens per CTA: two M = 128 tiles
constexpr uint32_t kUpA = 128 * 128;         // one tile: 128 tokens x 64 latent values (bf16)
constexpr uint32_t kUpB = 256 * 128;         // 256 weight rows x 64 values
constexpr uint32_t kUpStage = 2 * kUpA + kUpB;  // 64 KB
constexpr uint32_t kUpBarOff = kUpStages * kUpStage;
constexpr uint32_t kUpSmem = kUpBarOff + 128 + 1024;
constexpr uint32_t kUpIdesc = idesc_bf16_f32(128, 256, false, false);

struct UpParams {
  const int32_t* block_table;
  const int32_t* seq_lens;
  __nv_bfloat16* kn;   // [B][H][Lmax][128], Lmax a multiple of 256
  __nv_bfloat16* v;    // [B][H][Lmax][128]
  uint32_t* status;
  int H, max_pages, num_pages, Lmax, max_len;
  uint64_t wait_ns;
};

__global__ void __launch_bounds__(kUpThreads, 1)
    kv_up_kernel(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_wuk,
                 const __grid_constant__ CUtensorMap tm_wuv, const UpParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sa = (raw + 1023u) & ~1023u;
  uint8_t* sm = smem_raw + (sa - raw);
  const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t full0 = sa + kUpBarOff, empty0 = full0 + 8 * kUpStages, done = empty0 + 8 * kUpStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kUpBarOff + 64);
  int* abort_flag = reinterpret_cast<int*>(sm + kUpBarOff + 68);

  pdl_trigger();
  pdl_wait();  // whatever wrote the cache, the block table or the lengths
  int L = p.seq_lens[b];
  if (L < 0 || L > p.max_pages * kPage || L > p.max_len) L = 0;  // reported by the attention kernel
  const int t0 = tile * kUpTok;
  if (t0 >= L) return;  // whole CTA: nothing of this sequence here
  if (threadIdx.x == 0) {
    for (int s = 0; s < kUpStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_1(smem_u32(tmem_slot), 512);
    tmem_relinquish_1();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int32_t* bt = p.block_table + (size_t)b * p.max_pages;
  // the four pages of the 256 tokens; pages past the length stand in with the
  // first one (their rows are written as zeros)
  int pg[4];
  for (int k = 0; k < 4; ++k) {
    const int idx = t0 / kPage + k;
    int v = idx * kPage < L ? bt[idx] : bt[t0 / kPage];
    if (v < 0 || v >= p.num_pages) {
      if (threadIdx.x == 0 && idx * kPage < L) set_status(p.status, MLA_ERR_BAD_BLOCK_TABLE);
      v = 0;
    }
    pg[k] = v;
  }
  constexpr int kChunks = kDc / 64;
  if (warp == 0) {
    // ---- producer: chunk c of the 512 latent values, for both pages and both weights
    int issued = 0;
    for (int c = 0; c < kChunks; ++c) {
      const int s = c % kUpStages;
      if (!mbar_wait_converged(empty0 + 8 * s, ((c / kUpStages) & 1) ^ 1, abort_flag, p.status, p.wait_ns)) break;
      if (lane == 0) {
        const uint32_t dst = sa + s * kUpStage;
        mbar_arrive_expect_tx_local(full0 + 8 * s, kUpStage);
        for (int k = 0; k < 4; ++k) tma_load_2d_cta(dst + k * 64 * 128, &tm_c, full0 + 8 * s, 64 * c, pg[k] * kPage);
        tma_load_2d_cta(dst + 2 * kUpA, &tm_wuk, full0 + 8 * s, 64 * c, h * 128);
        tma_load_2d_cta(dst + 2 * kUpA + 128 * 128, &tm_wuv, full0 + 8 * s, 64 * c, h * 128);
      }
      __syncwarp();
      issued = c + 1;
    }
    // a wait that ran out may leave loads in flight
    if (lane == 0 && *reinterpret_cast<volatile int*>(abort_flag)) {
      int give_up = 0;
      for (int c = max(0, issued - kUpStages); c < issued; ++c)
        mbar_wait(full0 + 8 * (c % kUpStages), (c / kUpStages) & 1, &give_up, nullptr, kDrainNs);
    }
  } else if (warp == 1) {
    // ---- MMA issue: D[tokens][K | V] += C_chunk . [W_UK ; W_UV]_chunk^T
    for (int c = 0; c < kChunks; ++c) {
      const int s = c % kUpStages;
      if (!mbar_wait_converged(full0 + 8 * s, (c / kUpStages) & 1, abort_flag, p.status, p.wait_ns)) break;
      tc_fence_after();
      const uint64_t bd = desc_sw128(sa + s * kUpStage + 2 * kUpA, 16, 1024);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint64_t ad = desc_sw128(sa + s * kUpStage + i * kUpA, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_1_elect(tmem + 256u * i, ad + 2 * kk, bd + 2 * kk, kUpIdesc, (c | kk) != 0);
      }
      commit_1_elect(empty0 + 8 * s);
    }
    commit_1_elect(done);
  }
  // ---- epilogue: tile i in TMEM columns 256 i .. 256 i + 255, lane = token,
  // Kn in the first 128 columns, V in the next.  Rows past the length (and every
  // row after a wait ran out) get zeros: the attention multiplies them by zero
  // weights, which must not meet a NaN.
  int keep = 0;
  mbar_wait(done, 0, &keep, nullptr, kDrainNs);
  __syncwarp();  // the tensor-memory loads below are warp-collective
  tc_fence_after();
  const bool alive = __shfl_sync(0xffffffffu, *reinterpret_cast<volatile int*>(abort_flag), 0) == 0;
#pragma unroll 1
  for (int q = 0; q < 4; ++q) {
    const int i = q >> 1, half = q & 1;
    const int t = t0 + 128 * i + 32 * warp + lane;
    const bool ok = alive && t < L;
    __nv_bfloat16* dst = (half ? p.v : p.kn) + (((size_t)b * p.H + h) * p.Lmax + t) * 128;
#pragma unroll 1
    for (int c0 = 0; c0 < 128; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + 256 * i + 128 * half + c0, r);
      tmem_wait_ld();
      if (!ok) {
#pragma unroll
        for (int k = 0; k < 32; ++k) r[k] = 0u;
      }
      {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          reinterpret_cast<uint4*>(dst + c0)[k] =
              make_uint4(pack_bf16(__uint_as_float(r[8 * k]), __uint_as_float(r[8 * k + 1])),
                         pack_bf16(__uint_as_float(r[8 * k + 2]), __uint_as_float(r[8 * k + 3])),
                         pack_bf16(__uint_as_float(r[8 * k + 4]), __uint_as_float(r[8 * k + 5])),
                         pack_bf16(__uint_as_float(r[8 * k + 6]), __uint_as_float(r[8 * k + 7])));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc_1(tmem, 512);
}

// ---------------------------------------------------------------- attention
// One CTA per (sequence, head, 256 queries): two 128-query tiles A and B share
// every K and V tile, each with its own softmax warpgroup, S (P) and O in TMEM,
// so that the tensor pipe works on one tile while the other tile's softmax runs.
constexpr int kAtThreads = 384;             // warp 0 producer, warp 1 MMA, warps 4..7 tile A, 8..11 tile B
constexpr uint32_t kQChunk = 128 * 128;     // 128 rows x 64 bf16
constexpr uint32_t kQBytes = 3 * kQChunk;   // one tile's Q: q_nope (2 chunks) | q_pe
constexpr uint32_t kKBytes = 3 * kQChunk;   // Kn (2 chunks) | k_pe (two pages)
constexpr uint32_t kVBytes = 2 * kQChunk;   // V: 128 keys x 128 values, two 64-value chunks
constexpr int kVStagesAt = 2;
constexpr uint32_t kAtQOff = 0;                              // Q of tiles A and B
constexpr uint32_t kAtKOff = kAtQOff + 2 * kQBytes;          // one K stage
constexpr uint32_t kAtVOff = kAtKOff + kKBytes;              // two V stages
constexpr uint32_t kAtBarOff = kAtVOff + kVStagesAt * kVBytes;
constexpr uint32_t kAtSmem = kAtBarOff + 256 + 1024;
static_assert(kAtSmem <= 232448, "shared memory budget");
// TMEM: S (and P over it) of tile t at columns 128 t, O of tile t at 256 + 128 t
constexpr uint32_t kTmemO = 256;
constexpr uint32_t kAtIdescS = idesc_bf16_f32(128, 128, false, false);
constexpr uint32_t kAtIdescPV = idesc_bf16_f32(128, 128, false, true);
constexpr float kRescale = 8.0f;
// barriers ([2]: one per query tile or V stage)
constexpr int A_Q = 0, A_KFULL = 1, A_KEMPTY = 2, A_VFULL = 3, A_VEMPTY = 5, A_SREADY = 7, A_PREADY = 9,
              A_ODONE = 11, A_DRAIN = 13, A_NBARS = 14;

struct AtParams {
  const __nv_bfloat16* kn;
  const __nv_bfloat16* v;
  const int32_t* block_table;
  const int32_t* seq_lens;
  __nv_bfloat16* out;   // [B][s_q][H][128]
  float* lse;           // [B][s_q][H] or null
  uint32_t* status;
  int B, s_q, H, max_pages, num_pages, Lmax, max_len, causal;
  float scale_log2;
  uint64_t wait_ns;
};

__global__ void __launch_bounds__(kAtThreads, 1)
    prefill_attn_kernel(const __grid_constant__ CUtensorMap tm_qn, const __grid_constant__ CUtensorMap tm_qp,
                        const __grid_constant__ CUtensorMap tm_kn, const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_kpe, const AtParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sa = (raw + 1023u) & ~1023u;
  uint8_t* sm = smem_raw + (sa - raw);
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](int i) -> uint32_t { return sa + kAtBarOff + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kAtBarOff + 8 * A_NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kAtBarOff + 8 * A_NBARS + 4);
  uint32_t* issued = reinterpret_cast<uint32_t*>(sm + kAtBarOff + 8 * A_NBARS + 8);  // [0] K, [1] V tiles

  pdl_trigger();
  pdl_wait();  // the K / V up-projection is the previous kernel
  const int L_in = p.seq_lens[b];
  const bool bad_len = L_in < p.s_q || L_in > p.max_pages * kPage || L_in > p.max_len;
  const int L = bad_len ? 0 : L_in;
  const int q0 = qt * 256;                          // first query of tile A
  const int nq = max(0, min(256, p.s_q - q0));      // query rows of the two tiles
  // keys the CTA's last query sees (causal) or all of them; tile A runs the same
  // tiles (its last ones fully masked under the causal rule)
  const int kmax = L == 0 ? 0 : (p.causal ? min(L, L - p.s_q + q0 + nq) : L);
  const int n = nq > 0 ? (kmax + 127) / 128 : 0;
  const uint64_t wait_ns = p.wait_ns;

  if (threadIdx.x == 0) {
    if (bad_len && qt == 0 && h == 0) set_status(p.status, MLA_ERR_BAD_SEQ_LEN);
    *abort_flag = 0;
    issued[0] = issued[1] = 0;
    mbar_init(bar(A_Q), 1);
    mbar_init(bar(A_KFULL), 1);
    mbar_init(bar(A_KEMPTY), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(A_VFULL + i), 1);
      mbar_init(bar(A_VEMPTY + i), 1);
      mbar_init(bar(A_SREADY + i), 1);
      mbar_init(bar(A_PREADY + i), 4);
      mbar_init(bar(A_ODONE + i), 1);
    }
    mbar_init(bar(A_DRAIN), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_1(smem_u32(tmem_slot), 512);
    tmem_relinquish_1();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // =========================== TMA producer ===========================
    int n_k = 0, n_v = 0;
    if (n > 0) {
      const int32_t* bt = p.block_table + (size_t)b * p.max_pages;
      const size_t kv_row0 = ((size_t)b * p.H + h) * p.Lmax;
      if (lane == 0) {
        // Q of both tiles: 256 query rows (rows past s_q read as zeros or belong to
        // the next sequence; their outputs are not stored)
        const int tok = b * p.s_q + q0;
        mbar_arrive_expect_tx_local(bar(A_Q), 2 * kQBytes);
        for (int t = 0; t < 2; ++t) {
          const uint32_t dq = sa + kAtQOff + t * kQBytes;
          tma_load_3d_cta(dq, &tm_qn, bar(A_Q), 0, h, tok + 128 * t);
          tma_load_3d_cta(dq + kQChunk, &tm_qn, bar(A_Q), 64, h, tok + 128 * t);
          tma_load_3d_cta(dq + 2 * kQChunk, &tm_qp, bar(A_Q), 0, h, tok + 128 * t);
        }
      }
      auto page = [&](int idx) {
        int v = idx < p.max_pages ? bt[idx] : 0;
        if (v < 0 || v >= p.num_pages) v = 0;
        return v;
      };
      bool ok = true;
      for (int j = 0; ok && j < n; ++j) {
        // V(j) into its stage once P.V(j-2) is done, then K(j) into the one K stage
        // once both score MMAs of tile j-1 are done
        const int vs = j & 1;
        ok = mbar_wait_converged(bar(A_VEMPTY + vs), ((j >> 1) & 1) ^ 1, abort_flag, p.status, wait_ns);
        if (!ok) break;
        if (lane == 0) {
          const uint32_t dst = sa + kAtVOff + vs * kVBytes;
          mbar_arrive_expect_tx_local(bar(A_VFULL + vs), kVBytes);
          tma_load_2d_cta(dst, &tm_v, bar(A_VFULL + vs), 0, (int)(kv_row0 + 128 * j));
          tma_load_2d_cta(dst + kQChunk, &tm_v, bar(A_VFULL + vs), 64, (int)(kv_row0 + 128 * j));
        }
        __syncwarp();
        n_v = j + 1;
        ok = mbar_wait_converged(bar(A_KEMPTY), (j & 1) ^ 1, abort_flag, p.status, wait_ns);
        if (!ok) break;
        if (lane == 0) {
          // K: Kn rows of keys 128 j .. (rows past the length are zeros), k_pe of the two pages
          const uint32_t dst = sa + kAtKOff;
          mbar_arrive_expect_tx_local(bar(A_KFULL), kKBytes);
          tma_load_2d_cta(dst, &tm_kn, bar(A_KFULL), 0, (int)(kv_row0 + 128 * j));
          tma_load_2d_cta(dst + kQChunk, &tm_kn, bar(A_KFULL), 64, (int)(kv_row0 + 128 * j));
          tma_load_2d_cta(dst + 2 * kQChunk, &tm_kpe, bar(A_KFULL), kDc, page(2 * j) * kPage);
          tma_load_2d_cta(dst + 2 * kQChunk + 64 * 128, &tm_kpe, bar(A_KFULL), kDc, page(2 * j + 1) * kPage);
        }
        __syncwarp();
        n_k = j + 1;
      }
    }
    if (lane == 0) {
      issued[0] = n_k;
      issued[1] = n_v;
    }
  } else if (warp == 1) {
    // =========================== MMA issue ===========================
    // Per K/V tile j: P.V of tile A, then of tile B; then the scores of tile j + 1
    // for A and for B, each once P.V(j) of that tile has read its P out of the S
    // columns the new scores overwrite.
    if (n > 0) {
      bool ok = mbar_wait_converged(bar(A_Q), 0, abort_flag, p.status, wait_ns);
      // S_t(j) = Q_t K(j)^T into S columns of tile t; after both tiles, K is free
      auto issue_s = [&](int t, int j) -> bool {
        if (t == 0) {
          if (!mbar_wait_converged(bar(A_KFULL), j & 1, abort_flag, p.status, wait_ns)) return false;
          tc_fence_after();
        }
        const uint64_t dq = desc_sw128(sa + kAtQOff + t * kQBytes, 16, 1024);
        const uint64_t dk = desc_sw128(sa + kAtKOff, 16, 1024);
#pragma unroll
        for (int c = 0; c < 3; ++c)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_1_elect(tmem + 128u * t, dq + ((c * kQChunk) >> 4) + 2 * kk, dk + ((c * kQChunk) >> 4) + 2 * kk,
                        kAtIdescS, (c | kk) != 0);
        commit_1_elect(bar(A_SREADY + t));
        if (t == 1) commit_1_elect(bar(A_KEMPTY));
        return true;
      };
      if (ok) ok = issue_s(0, 0);
      if (ok) ok = issue_s(1, 0);
      for (int j = 0; ok && j < n; ++j) {
        const int vs = j & 1;
        for (int t = 0; ok && t < 2; ++t) {
          if (!mbar_wait_converged(bar(A_PREADY + t), j & 1, abort_flag, p.status, wait_ns)) { ok = false; break; }
          if (t == 0 && !mbar_wait_converged(bar(A_VFULL + vs), (j >> 1) & 1, abort_flag, p.status, wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t dv = desc_sw128(sa + kAtVOff + vs * kVBytes, kQChunk, 1024);
          // K = 128 keys in steps of 16: P columns 8 kk (2 bf16 each), V rows 16 kk
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_1_ts_elect(tmem + kTmemO + 128u * t, tmem + 128u * t + 8u * kk, dv + ((kk * 2048) >> 4),
                           kAtIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
          commit_1_elect(bar(A_ODONE + t));
          if (t == 1) commit_1_elect(bar(A_VEMPTY + vs));
        }
        if (ok && j + 1 < n) {
          for (int t = 0; ok && t < 2; ++t) {
            if (!mbar_wait_converged(bar(A_ODONE + t), j & 1, abort_flag, p.status, wait_ns)) { ok = false; break; }
            ok = issue_s(t, j + 1);
          }
        }
      }
      commit_1_elect(bar(A_DRAIN));
      int keep = 0;
      mbar_wait_converged(bar(A_DRAIN), 0, &keep, p.status, kDrainNs);
    }
  } else if (warp >= 4) {
    // ================ softmax / epilogue: thread = query row of tile t ================
    // S_t(j) is issued only after P.V_t(j-1) has completed, so O_t may be rescaled
    // as soon as the scores of tile j are there.
    const int t = (warp - 4) >> 2;
    const int row = 32 * (warp & 3) + lane;  // TMEM lane of this thread's query row
    const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    const uint32_t cs = 128u * t, co = kTmemO + 128u * t;
    const int qi = q0 + 128 * t + row;       // query index in the chunk
    const int vis = p.causal ? L - p.s_q + qi + 1 : L;  // keys this query sees
    float m_used = -CUDART_INF_F, l = 0.f;
    for (int j = 0; j < n; ++j) {
      if (!mbar_wait_converged(bar(A_SREADY + t), j & 1, abort_flag, p.status, wait_ns)) break;
      tc_fence_after();
      // the row's 128 raw scores: four loads in flight, one wait
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tl + cs + 32u * c, sr[c]);
      tmem_wait_ld();
      const int nv = max(0, min(128, vis - 128 * j));  // visible keys of this tile
      float s[128];
      // eight independent running maxima (the softmax scale is positive, so it
      // commutes with the maximum and is applied once)
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = -CUDART_INF_F;
#pragma unroll
      for (int k = 0; k < 128; ++k) {
        s[k] = k < nv ? __uint_as_float(sr[k >> 5][k & 31]) : -CUDART_INF_F;
        mx8[k & 7] = fmaxf(mx8[k & 7], s[k]);
      }
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * p.scale_log2;
      float alpha = 1.f;
      bool resc = false;
      if (mx > -CUDART_INF_F) {
        if (m_used == -CUDART_INF_F) {
          m_used = mx;
        } else if (mx > m_used + kRescale) {
          alpha = ex2_approx(m_used - mx);
          m_used = mx;
          resc = true;
          l *= alpha;
        }
      }
      const float nref = m_used == -CUDART_INF_F ? 0.f : -m_used;
      if (__any_sync(0xffffffffu, resc) && j >= 1) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tl + co + 32u * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tmem_st32(tl + co + 32u * c, o);
        }
        tmem_wait_st();
      }
      // P over S in place: 128 keys -> 64 columns of bf16 pairs; p = 2^(s * scale - m)
      float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float p0 = ex2_approx(fmaf(s[64 * c + 2 * k], p.scale_log2, nref));
          const float p1 = ex2_approx(fmaf(s[64 * c + 2 * k + 1], p.scale_log2, nref));
          l4[k & 3] += p0 + p1;
          pk[k] = pack_bf16(p0, p1);
        }
        tmem_st32(tl + cs + 32u * c, pk);
      }
      l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_local(bar(A_PREADY + t));
    }
    // ---- epilogue: o = O / l, lse
    if (n > 0) {
      mbar_wait_converged(bar(A_ODONE + t), (n - 1) & 1, abort_flag, p.status, wait_ns);
      tc_fence_after();
    }
    const bool alive = __shfl_sync(0xffffffffu, *abort_flag, 0) == 0;
    const bool empty = !(l > 0.f) || !alive;
    const float inv = empty ? 0.f : 1.f / l;
    // tcgen05.ld is a warp-collective instruction: every lane loads (the
    // condition is warp-uniform), only the rows of real queries are stored
    const bool live = n > 0 && alive;
    const bool mine = qi < p.s_q && nq > 0;
    const size_t orow = ((size_t)b * p.s_q + qi) * p.H + h;
    __nv_bfloat16* dst = p.out + orow * kDv;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t o[32];
      if (live) {
        tmem_ld32(tl + co + 32u * c, o);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) o[k] = 0u;
      }
      if (mine) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          reinterpret_cast<uint4*>(dst + 32 * c)[k] =
              make_uint4(pack_bf16(__uint_as_float(o[8 * k]) * inv, __uint_as_float(o[8 * k + 1]) * inv),
                         pack_bf16(__uint_as_float(o[8 * k + 2]) * inv, __uint_as_float(o[8 * k + 3]) * inv),
                         pack_bf16(__uint_as_float(o[8 * k + 4]) * inv, __uint_as_float(o[8 * k + 5]) * inv),
                         pack_bf16(__uint_as_float(o[8 * k + 6]) * inv, __uint_as_float(o[8 * k + 7]) * inv));
      }
    }
    if (mine && p.lse) p.lse[orow] = empty ? -CUDART_INF_F : (m_used + log2f(l)) * 0.6931471805599453f;
    tc_fence_before();
  }

  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    // a wait that ran out may leave loads in flight: wait (bounded) for Q and for
    // the last load of each ring
    int give_up = 0;
    if (n > 0) mbar_wait(bar(A_Q), 0, &give_up, nullptr, kDrainNs);
    if (issued[0] > 0) mbar_wait(bar(A_KFULL), (issued[0] - 1) & 1, &give_up, nullptr, kDrainNs);
    for (int j = max(0, (int)issued[1] - 2); j < (int)issued[1]; ++j)
      mbar_wait(bar(A_VFULL + (j & 1)), (j >> 1) & 1, &give_up, nullptr, kDrainNs);
  }
  __syncthreads();
  if (warp == 1) tmem_dealloc_1(tmem, 512);
}

}  // namespace

size_t prefill_workspace_bytes(int B, int H, int Lmax) {
  // status header, then Kn and V, each [B][H][Lmax rounded up to 256][128] bf16
  const size_t lpad = ((size_t)Lmax + kUpTok - 1) / kUpTok * kUpTok;
  return 256 + 2 * (size_t)B * H * lpad * 128 * 2;
}

cudaError_t launch_prefill(const mla_prefill_args_t* a, cudaStream_t stream) {
  const int Lmax = (a->max_seq_len + kUpTok - 1) / kUpTok * kUpTok;
  unsigned char* ws = static_cast<unsigned char*>(a->workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  __nv_bfloat16* kn = reinterpret_cast<__nv_bfloat16*>(ws + 256);
  __nv_bfloat16* v = kn + (size_t)a->B * a->H * Lmax * 128;
  const uint64_t rows_kv = (uint64_t)a->num_pages * kPage;
  const uint64_t kv_rows = (uint64_t)a->B * a->H * Lmax;
  CUtensorMap tm_c, tm_wuk, tm_wuv, tm_qn, tm_qp, tm_kn, tm_v;
  // cache rows (576 values, 1152 bytes apart): 64 values x 64 rows per box, for
  // the latent (kv_up) and the RoPE key (attention)
  if (!tma_map_2d(&tm_c, a->kv_cache, kRow, rows_kv, kRow * 2, 64, 64) ||
      !tma_map_2d(&tm_wuk, a->w_uk, kDc, (uint64_t)a->H * kDn, kDc * 2, 64, 128) ||
      !tma_map_2d(&tm_wuv, a->w_uv, kDc, (uint64_t)a->H * kDv, kDc * 2, 64, 128) ||
      !tma_map_3d(&tm_qn, a->q_nope, kDn, a->H, (uint64_t)a->B * a->s_q, kDn * 2, (uint64_t)a->H * kDn * 2, 64, 1,
                  128) ||
      !tma_map_3d(&tm_qp, a->q_pe, kDr, a->H, (uint64_t)a->B * a->s_q, kDr * 2, (uint64_t)a->H * kDr * 2, 64, 1,
                  128) ||
      !tma_map_2d(&tm_kn, kn, 128, kv_rows, 256, 64, 128) || !tma_map_2d(&tm_v, v, 128, kv_rows, 256, 64, 128))
    return cudaErrorInvalidValue;
  static PerDeviceOnce attrs;
  cudaError_t e = once_per_device(attrs, [&]() {
    cudaError_t e2 = cudaFuncSetAttribute(kv_up_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kUpSmem);
    if (e2 != cudaSuccess) return e2;
    return cudaFuncSetAttribute(prefill_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAtSmem);
  });
  if (e != cudaSuccess) return e;
  UpParams up;
  up.block_table = a->block_table;
  up.seq_lens = a->seq_lens;
  up.kn = kn;
  up.v = v;
  up.status = status;
  up.H = a->H;
  up.max_pages = a->max_pages_per_seq;
  up.num_pages = a->num_pages;
  up.Lmax = Lmax;
  up.max_len = a->max_seq_len;
  up.wait_ns = device_wait_limit_ns();
  e = launch_pdl(kv_up_kernel, dim3(Lmax / kUpTok, a->H, a->B), dim3(kUpThreads), kUpSmem, stream, tm_c, tm_wuk,
                 tm_wuv, up);
  if (e != cudaSuccess) return e;
  AtParams at;
  at.kn = kn;
  at.v = v;
  at.block_table = a->block_table;
  at.seq_lens = a->seq_lens;
  at.out = static_cast<__nv_bfloat16*>(a->out);
  at.lse = a->lse;
  at.status = status;
  at.B = a->B;
  at.s_q = a->s_q;
  at.H = a->H;
  at.max_pages = a->max_pages_per_seq;
  at.num_pages = a->num_pages;
  at.Lmax = Lmax;
  at.max_len = a->max_seq_len;
  at.causal = a->causal;
  at.scale_log2 = a->softmax_scale * kLog2e;
  at.wait_ns = device_wait_limit_ns();
  return launch_pdl(prefill_attn_kernel, dim3((a->s_q + 255) / 256, a->H, a->B), dim3(kAtThreads), kAtSmem, stream,
                    tm_qn, tm_qp, tm_kn, tm_v, tm_c, at);
}

}  // namespace mla
