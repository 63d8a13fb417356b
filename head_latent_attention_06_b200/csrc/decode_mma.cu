// Paged latent-attention decode, warp-level MMA formulation.
//
// This is the portable formulation of the decode step: legacy warp MMAs
// (mma.sync, fp32 accumulation) with cp.async staging.  It handles every
// supported shape (any H multiple of 16, any s_q, bf16, e4m3, q8_0 or q4_0
// cache) and is the path for shapes the tensor-memory kernels do not take: a
// scale array not on 16 bytes.
//
// Cache formats.  bf16: the rows as they are.  e4m3: codes converted exactly to
// bf16 in shared memory, the per-token scale folded into S and into P.  q8_0
// (ik_llama.cpp docs "FlashMLA", section "KV cache with MLA"): int8 codes with
// one fp16 scale per 32-value block; each value is formed as code * scale in
// fp32 and rounded to bf16 in shared memory (relative error 2^-9, against the
// format's own step of up to 1/254 of the block's largest value).  q4_0: the
// same with 4-bit codes, two a byte (value 2j in the low half of byte j).
//
// For one sequence b, the rows of the attention problem are the (query i,
// head h) pairs, r = i * H + h.  A CTA owns 64 rows and one split (a range of
// 32-token tiles) of the sequence.  Per tile:
//   S[64 x 32]  = Q[64 x 576] . C^T          (q_lat . c + q_pe . k_pe)
//   online softmax in the exp2 domain (running max m, running sum l)
//   O[64 x 512] = alpha * O + P[64 x 32] . C[32 x 512]
// (FlashAttention-style on-chip tiles, nnets.ru article, section
// "MLA и FlashAttention"; V is the latent itself, so the tile loaded for S is
// reused unchanged for P.C.)
#include <cuda_fp16.h>
#include <math_constants.h>

#include "common.cuh"

namespace mla {
namespace {

constexpr int ROWS = 64;            // attention rows per CTA
constexpr int TT = 32;              // tokens per tile
constexpr int NSTAGE = 3;           // cp.async ring depth
constexpr int CP = kRow + 8;        // padded smem row (elements): 1168 B, conflict-free ldmatrix
constexpr int PP = TT + 8;          // padded P row
constexpr int NTHREADS = 256;

struct DecodeParams {
  const __nv_bfloat16* q_lat;
  const __nv_bfloat16* q_pe;
  const uint8_t* kv;
  const void* kv_scale;  // e4m3: fp32 [pages][64]; q8_0, q4_0: fp16 [pages][64][18]
  const int32_t* block_table;
  const int32_t* seq_lens;
  __nv_bfloat16* o_lat;
  float* lse;
  float* o_part;
  float* lse_part;
  uint32_t* status;
  int B, s_q, H, num_pages, max_pages, causal, splits;
  float scale_log2;  // softmax_scale * log2(e)
};

// KIND: 0 bf16 cache, 1 e4m3 (+ fp32 token scales), 2 q8_0 (+ fp16 block
// scales), 3 q4_0 (+ fp16 block scales)
constexpr int kQ8Blocks = kRow / 32;  // 18 scale blocks per row
// stored bytes of one cache row
template <int KIND>
__host__ __device__ constexpr int row_bytes() { return KIND == 0 ? 2 * kRow : KIND == 3 ? kRow / 2 : kRow; }

template <int KIND>
struct Smem {
  static constexpr size_t q_bytes = (size_t)ROWS * CP * 2;
  static constexpr size_t stage_bytes = KIND ? (size_t)TT * row_bytes<KIND>() : (size_t)TT * CP * 2;
  static constexpr size_t conv_bytes = KIND ? (size_t)TT * CP * 2 : 0;
  static constexpr size_t p_bytes = (size_t)ROWS * PP * 2;
  static constexpr size_t red_bytes = 2 * ROWS * sizeof(float);
  static constexpr size_t sc_bytes = NSTAGE * TT * (KIND >= 2 ? kQ8Blocks * 2 : sizeof(float));
  static constexpr size_t q_off = 0;
  static constexpr size_t stage_off = q_off + q_bytes;
  static constexpr size_t conv_off = stage_off + NSTAGE * stage_bytes;
  static constexpr size_t p_off = conv_off + conv_bytes;
  static constexpr size_t red_off = p_off + p_bytes;
  static constexpr size_t sc_off = red_off + red_bytes;
  static constexpr size_t total = sc_off + sc_bytes;
};

template <int KIND>
__global__ void __launch_bounds__(NTHREADS, 1) decode_mma_kernel(DecodeParams p) {
  constexpr bool CODED = KIND != 0;  // the cache holds codes converted in shared memory
  using SM = Smem<KIND>;
  extern __shared__ __align__(16) unsigned char smem[];
  __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(smem + SM::q_off);
  unsigned char* stages = smem + SM::stage_off;
  __nv_bfloat16* ps = reinterpret_cast<__nv_bfloat16*>(smem + SM::p_off);
  float* red = reinterpret_cast<float*>(smem + SM::red_off);  // [2 halves][ROWS]
  float* scs = reinterpret_cast<float*>(smem + SM::sc_off);   // e4m3: [NSTAGE][TT]
  // q8_0: [NSTAGE][TT][18] fp16 block scales
  __half* qsc = reinterpret_cast<__half*>(smem + SM::sc_off);

  const int g = blockIdx.x, split = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_rows = p.s_q * p.H;
  const int row0 = g * ROWS;
  pdl_trigger();
  pdl_wait();

  int L = p.seq_lens[b];
  if (L < 0 || L > p.max_pages * kPage) {
    if (tid == 0) set_status(p.status, MLA_ERR_BAD_SEQ_LEN);
    L = 0;
  }
  const int n_tiles = (L + TT - 1) / TT;
  const int per = (n_tiles + p.splits - 1) / p.splits;
  const int tile_begin = min(n_tiles, split * per);
  const int tile_end = min(n_tiles, tile_begin + per);
  const int j_end = min(L, tile_end * TT);  // exclusive token end of this split
  const int32_t* bt = p.block_table + (size_t)b * p.max_pages;

  // ---- Q rows -> smem (zero rows beyond n_rows)
  for (int v = tid; v < ROWS * (kRow / 8); v += NTHREADS) {
    int r = v / (kRow / 8), c = (v % (kRow / 8)) * 8;
    int rr = row0 + r;
    __nv_bfloat16* dst = qs + r * CP + c;
    if (rr < n_rows) {
      int i = rr / p.H, h = rr % p.H;
      size_t qrow = ((size_t)b * p.s_q + i) * p.H + h;
      const __nv_bfloat16* src =
          c < kDc ? p.q_lat + qrow * kDc + c : p.q_pe + qrow * kDr + (c - kDc);
      cp_async16(dst, src);
    } else {
      *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
    }
  }
  cp_async_commit();

  // ---- cache tile loader: tokens [t*TT, t*TT+TT) of this sequence
  auto load_tile = [&](int t, int stage) {
    unsigned char* st = stages + stage * SM::stage_bytes;
    const int jb = t * TT;
    constexpr int RB = row_bytes<KIND>();
    constexpr int VPR = RB / 16;  // 16-byte vectors per token row
    for (int v = tid; v < TT * VPR; v += NTHREADS) {
      int r = v / VPR, c = v % VPR;
      int j = jb + r;
      unsigned char* dst = CODED ? st + r * RB + c * 16 : st + (r * CP + c * 8) * 2;
      bool ok = j < j_end;
      int page = ok ? bt[j / kPage] : 0;
      if (ok && (page < 0 || page >= p.num_pages)) {
        set_status(p.status, MLA_ERR_BAD_BLOCK_TABLE);
        ok = false;
      }
      if (ok) {
        size_t rowi = (size_t)page * kPage + (j % kPage);
        cp_async16(dst, p.kv + rowi * RB + c * 16);
      } else {
        *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      }
    }
    if (KIND == 1 && tid < TT) {
      int j = jb + tid;
      float s = 0.f;
      if (j < j_end) {
        int page = bt[j / kPage];
        if (page >= 0 && page < p.num_pages)
          s = static_cast<const float*>(p.kv_scale)[(size_t)page * kPage + (j % kPage)];
      }
      scs[stage * TT + tid] = s;
    }
    if (KIND >= 2) {
      // the 18 fp16 block scales of each row: nine 4-byte words (36 bytes)
      for (int v = tid; v < TT * (kQ8Blocks / 2); v += NTHREADS) {
        const int r = v / (kQ8Blocks / 2), w = v % (kQ8Blocks / 2);
        const int j = jb + r;
        uint32_t* dst = reinterpret_cast<uint32_t*>(qsc + ((size_t)stage * TT + r) * kQ8Blocks) + w;
        int page = j < j_end ? bt[j / kPage] : -1;
        if (page >= 0 && page < p.num_pages) {
          const size_t rowi = (size_t)page * kPage + (j % kPage);
          cp_async4(dst, static_cast<const __half*>(p.kv_scale) + rowi * kQ8Blocks + 2 * w);
        } else {
          *dst = 0u;
        }
      }
    }
    cp_async_commit();
  };

  const int mt = warp & 3;   // 16-row slice of the 64 rows
  const int hf = warp >> 2;  // S: token half of the tile; PV: column half of O
  // rows owned by this thread inside the CTA: r_lo = mt*16 + lane/4, r_hi = r_lo + 8
  const int r_lo = mt * 16 + (lane >> 2), r_hi = r_lo + 8;
  int vis_lo = 0, vis_hi = 0;  // visible token count of each row
  {
    int rr = row0 + r_lo;
    vis_lo = rr < n_rows ? (p.causal ? L - p.s_q + rr / p.H + 1 : L) : 0;
    rr = row0 + r_hi;
    vis_hi = rr < n_rows ? (p.causal ? L - p.s_q + rr / p.H + 1 : L) : 0;
  }

  float oacc[32][4];
#pragma unroll
  for (int j = 0; j < 32; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) oacc[j][e] = 0.f;
  float m_lo = -CUDART_INF_F, m_hi = -CUDART_INF_F;  // running max (log2 domain)
  float l_lo = 0.f, l_hi = 0.f;                      // this thread's part of the running sum

  const int n_my = tile_end - tile_begin;
#pragma unroll 1
  for (int s = 0; s < NSTAGE - 1; ++s) {
    if (s < n_my) load_tile(tile_begin + s, s);
    else cp_async_commit();
  }

#pragma unroll 1
  for (int it = 0; it < n_my; ++it) {
    const int stage = it % NSTAGE;
    cp_async_wait<NSTAGE - 2>();
    __syncthreads();
    {
      int nt = it + NSTAGE - 1;
      if (nt < n_my) load_tile(tile_begin + nt, nt % NSTAGE);
      else cp_async_commit();
    }
    const __nv_bfloat16* cs;
    if (CODED) {
      const uint8_t* raw = stages + stage * SM::stage_bytes;
      __nv_bfloat16* conv = reinterpret_cast<__nv_bfloat16*>(smem + SM::conv_off);
      for (int v = tid; v < TT * (kRow / 8); v += NTHREADS) {
        int r = v / (kRow / 8), c = (v % (kRow / 8)) * 8;
        uint4 o;
        if (KIND == 3) {
          // 8 four-bit codes (code + 8) of one 32-value block times its scale
          const float d = __half2float(qsc[((size_t)stage * TT + r) * kQ8Blocks + (c >> 5)]);
          const uint32_t w = *reinterpret_cast<const uint32_t*>(raw + r * (kRow / 2) + c / 2);
          uint32_t out[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int lo = (int)((w >> (8 * k)) & 15u) - 8, hi = (int)((w >> (8 * k + 4)) & 15u) - 8;
            out[k] = pack_bf16((float)lo * d, (float)hi * d);
          }
          o = make_uint4(out[0], out[1], out[2], out[3]);
          *reinterpret_cast<uint4*>(conv + r * CP + c) = o;
          continue;
        }
        uint2 in = *reinterpret_cast<const uint2*>(raw + r * kRow + c);
        if (KIND == 1) {
          o.x = e4m3x2_to_bf16x2((uint16_t)(in.x & 0xFFFF));
          o.y = e4m3x2_to_bf16x2((uint16_t)(in.x >> 16));
          o.z = e4m3x2_to_bf16x2((uint16_t)(in.y & 0xFFFF));
          o.w = e4m3x2_to_bf16x2((uint16_t)(in.y >> 16));
        } else {
          // 8 int8 codes of one 32-value block times its scale
          const float d = __half2float(qsc[((size_t)stage * TT + r) * kQ8Blocks + (c >> 5)]);
          const uint32_t w[2] = {in.x, in.y};
          uint32_t out[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int8_t lo = (int8_t)((w[k >> 1] >> (16 * (k & 1))) & 0xFF);
            const int8_t hi = (int8_t)((w[k >> 1] >> (16 * (k & 1) + 8)) & 0xFF);
            out[k] = pack_bf16((float)lo * d, (float)hi * d);
          }
          o = make_uint4(out[0], out[1], out[2], out[3]);
        }
        *reinterpret_cast<uint4*>(conv + r * CP + c) = o;
      }
      __syncthreads();
      cs = conv;
    } else {
      cs = reinterpret_cast<const __nv_bfloat16*>(stages + stage * SM::stage_bytes);
    }

    // ---- S = Q . C^T for rows [mt*16, +16) and tokens [hf*16, +16)
    float sacc[2][4];
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[n][e] = 0.f;
#pragma unroll 4
    for (int ks = 0; ks < kRow / 16; ++ks) {
      uint32_t a[4], b0, b1, b2, b3;
      ldmatrix_x4(a[0], a[1], a[2], a[3], qs + (mt * 16 + (lane & 15)) * CP + ks * 16 + (lane >> 4) * 8);
      ldmatrix_x4(b0, b1, b2, b3,
                  cs + (hf * 16 + (lane & 7) + 8 * (lane >> 4)) * CP + ks * 16 + 8 * ((lane >> 3) & 1));
      mma_bf16_16816(sacc[0], a, b0, b1);
      mma_bf16_16816(sacc[1], a, b2, b3);
    }

    // ---- scale, mask, tile max
    const int jb = (tile_begin + it) * TT;
    float tmax_lo = -CUDART_INF_F, tmax_hi = -CUDART_INF_F;
    float tsc[2][2];
#pragma unroll
    for (int n = 0; n < 2; ++n) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        int jl = hf * 16 + n * 8 + 2 * (lane & 3) + e;
        int j = jb + jl;
        float ksc = KIND == 1 ? scs[stage * TT + jl] : 1.f;
        tsc[n][e] = ksc;
        float f = p.scale_log2 * ksc;
        float vlo = (j < vis_lo && j < j_end) ? sacc[n][e] * f : -CUDART_INF_F;
        float vhi = (j < vis_hi && j < j_end) ? sacc[n][2 + e] * f : -CUDART_INF_F;
        sacc[n][e] = vlo;
        sacc[n][2 + e] = vhi;
        tmax_lo = fmaxf(tmax_lo, vlo);
        tmax_hi = fmaxf(tmax_hi, vhi);
      }
    }
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
      tmax_lo = fmaxf(tmax_lo, __shfl_xor_sync(0xffffffffu, tmax_lo, off));
      tmax_hi = fmaxf(tmax_hi, __shfl_xor_sync(0xffffffffu, tmax_hi, off));
    }
    if ((lane & 3) == 0) {
      red[hf * ROWS + r_lo] = tmax_lo;
      red[hf * ROWS + r_hi] = tmax_hi;
    }
    __syncthreads();
    tmax_lo = fmaxf(red[r_lo], red[ROWS + r_lo]);
    tmax_hi = fmaxf(red[r_hi], red[ROWS + r_hi]);
    const float mn_lo = fmaxf(m_lo, tmax_lo), mn_hi = fmaxf(m_hi, tmax_hi);
    // reference point for exp2: a fully masked row keeps 0 so that no inf - inf appears
    const float ref_lo = mn_lo == -CUDART_INF_F ? 0.f : mn_lo;
    const float ref_hi = mn_hi == -CUDART_INF_F ? 0.f : mn_hi;
    const float alpha_lo = exp2f(m_lo - ref_lo), alpha_hi = exp2f(m_hi - ref_hi);
    m_lo = mn_lo;
    m_hi = mn_hi;
    l_lo *= alpha_lo;
    l_hi *= alpha_hi;
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      float p0 = exp2f(sacc[n][0] - ref_lo), p1 = exp2f(sacc[n][1] - ref_lo);
      float p2 = exp2f(sacc[n][2] - ref_hi), p3 = exp2f(sacc[n][3] - ref_hi);
      l_lo += p0 + p1;
      l_hi += p2 + p3;
      // the PV product uses the undequantised e4m3 values: fold the token scale into P
      int col = hf * 16 + n * 8 + 2 * (lane & 3);
      *reinterpret_cast<uint32_t*>(ps + r_lo * PP + col) = pack_bf16(p0 * tsc[n][0], p1 * tsc[n][1]);
      *reinterpret_cast<uint32_t*>(ps + r_hi * PP + col) = pack_bf16(p2 * tsc[n][0], p3 * tsc[n][1]);
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      oacc[j][0] *= alpha_lo;
      oacc[j][1] *= alpha_lo;
      oacc[j][2] *= alpha_hi;
      oacc[j][3] *= alpha_hi;
    }
    __syncthreads();

    // ---- O[rows mt, cols hf*256 .. +256] += P . C
#pragma unroll
    for (int ks = 0; ks < TT / 16; ++ks) {
      uint32_t a[4];
      ldmatrix_x4(a[0], a[1], a[2], a[3], ps + (mt * 16 + (lane & 15)) * PP + ks * 16 + (lane >> 4) * 8);
#pragma unroll
      for (int np = 0; np < 16; ++np) {
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4_trans(b0, b1, b2, b3,
                          cs + (ks * 16 + (lane & 15)) * CP + hf * 256 + np * 16 + (lane >> 4) * 8);
        mma_bf16_16816(oacc[2 * np], a, b0, b1);
        mma_bf16_16816(oacc[2 * np + 1], a, b2, b3);
      }
    }
  }
  cp_async_wait<0>();

  // ---- finish: total l per row (quad, then the two token halves)
#pragma unroll
  for (int off = 1; off <= 2; off <<= 1) {
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, off);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, off);
  }
  __syncthreads();
  if ((lane & 3) == 0) {
    red[hf * ROWS + r_lo] = l_lo;
    red[hf * ROWS + r_hi] = l_hi;
  }
  __syncthreads();
  const float lt_lo = red[r_lo] + red[ROWS + r_lo];
  const float lt_hi = red[r_hi] + red[ROWS + r_hi];

#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = half ? r_hi : r_lo;
    const int rr = row0 + r;
    if (rr >= n_rows) continue;
    const float lt = half ? lt_hi : lt_lo;
    const float m = half ? m_hi : m_lo;
    const bool empty = !(lt > 0.f);
    const float inv = empty ? 0.f : 1.f / lt;
    const float lse = empty ? -CUDART_INF_F : (m + log2f(lt)) * 0.6931471805599453f;
    const int i = rr / p.H, h = rr % p.H;
    const size_t orow = ((size_t)b * p.s_q + i) * p.H + h;  // (token, head) row
    if (p.splits == 1) {
      __nv_bfloat16* dst = p.o_lat + orow * kDc + hf * 256 + 2 * (lane & 3);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        *reinterpret_cast<uint32_t*>(dst + j * 8) =
            pack_bf16(oacc[j][2 * half] * inv, oacc[j][2 * half + 1] * inv);
      if (p.lse && hf == 0 && (lane & 3) == 0) p.lse[orow] = lse;
    } else {
      const size_t prow = orow * p.splits + split;
      float* dst = p.o_part + prow * kDc + hf * 256 + 2 * (lane & 3);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        *reinterpret_cast<float2*>(dst + j * 8) =
            make_float2(oacc[j][2 * half] * inv, oacc[j][2 * half + 1] * inv);
      if (hf == 0 && (lane & 3) == 0) p.lse_part[prow] = lse;
    }
  }
}

}  // namespace

cudaError_t launch_decode_mma(const mla_decode_args_t* a, int splits, cudaStream_t stream) {
  DecodeParams p;
  p.q_lat = static_cast<const __nv_bfloat16*>(a->q_lat);
  p.q_pe = static_cast<const __nv_bfloat16*>(a->q_pe);
  p.kv = static_cast<const uint8_t*>(a->kv_cache);
  p.kv_scale = a->kv_scale;
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
  const int groups = (a->s_q * a->H + ROWS - 1) / ROWS;
  dim3 grid(groups, splits, a->B);
  static PerDeviceOnce attrs;
  cudaError_t e = once_per_device(attrs, [&]() {
    cudaError_t e2 = cudaFuncSetAttribute(decode_mma_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)Smem<0>::total);
    if (e2 != cudaSuccess) return e2;
    e2 = cudaFuncSetAttribute(decode_mma_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)Smem<1>::total);
    if (e2 != cudaSuccess) return e2;
    e2 = cudaFuncSetAttribute(decode_mma_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)Smem<2>::total);
    if (e2 != cudaSuccess) return e2;
    return cudaFuncSetAttribute(decode_mma_kernel<3>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)Smem<3>::total);
  });
  if (e != cudaSuccess) return e;
  if (a->kv_dtype == MLA_KV_FP8_E4M3)
    return launch_pdl(decode_mma_kernel<1>, grid, dim3(NTHREADS), Smem<1>::total, stream, p);
  if (a->kv_dtype == MLA_KV_Q8_0)
    return launch_pdl(decode_mma_kernel<2>, grid, dim3(NTHREADS), Smem<2>::total, stream, p);
  if (a->kv_dtype == MLA_KV_Q4_0)
    return launch_pdl(decode_mma_kernel<3>, grid, dim3(NTHREADS), Smem<3>::total, stream, p);
  return launch_pdl(decode_mma_kernel<0>, grid, dim3(NTHREADS), Smem<0>::total, stream, p);
}

int decode_mma_tiles(int len) { return (len + TT - 1) / TT; }
int decode_mma_ctas_per_split(int s_q, int H, int B) { return B * ((s_q * H + ROWS - 1) / ROWS); }

}  // namespace mla
