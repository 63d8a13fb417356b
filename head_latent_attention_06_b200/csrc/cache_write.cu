// Cache write: the s_q new tokens of every sequence go into the paged latent
// cache.  For token t = b * s_q + i at position pos = L_b - s_q + i:
//   c      = W_DKV h_t                     (512; "MLA: Multi-Head Latent Attention —
//                                           DeepSeek-AI Explained", "Architecture")
//   k_pe   = RoPE(W_KR h_t, pos)           (64; the decoupled RoPE key of the 576-value
//                                           record, snowgate thread 35)
//   row    = c || k_pe  -> row pos % 64 of page block_table[b][pos / 64], stored as
//            bf16 (round to nearest even) or as e4m3 codes with one fp32 scale per
//            row, scale = amax / 448 (ik_llama.cpp docs "FlashMLA", "KV cache with MLA":
//            the latent cache may be quantised), or blockwise q8_0 / q4_0 codes
//            with one fp16 scale per 32 values
// RoPE turns value pair (2i, 2i+1) by pos * base^(-2i/64).
//
// Two kernels.  The down-projection [n_tok x d_h] . [d_h x 576] is bound by
// reading the stacked weight (8.3 MB at d_h = 7168) at decode sizes, so it is
// split along d_h until the grid covers the SMs: each CTA owns 64 tokens, 64
// output columns and a range of 64-wide K chunks, streamed by TMA into
// 128-byte-swizzled shared memory, and writes fp32 partial sums.  The second
// kernel gives each token one warp: it adds the partials, rotates the RoPE
// slice (angle reduced in fp64: pos * theta reaches 1.3e5 radians at 128K
// tokens), takes the row maximum with warp shuffles, quantises with IEEE fp32
// division and stores the row.  Lane l holds values 64j + 2l, 64j + 2l + 1
// (j = 0..8): every load and store of the warp is contiguous, and RoPE pair l
// is lane l's ninth pair.
#include <cuda_fp8.h>
#include <math_constants.h>

#include <cuda_fp16.h>

#include "sm100.cuh"
#include "tma_host.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kWTok = 64;       // tokens per down-projection CTA, 16 per warp
constexpr int kWCols = 64;      // output columns per CTA (9 column tiles of the 576)
constexpr int kWK = 64;         // K per chunk: one 128-byte swizzled row per matrix row
constexpr int kWStages = 4;
constexpr int kWThreads = 128;
constexpr uint32_t kWChunk = 64 * 128;               // 64 rows x 64 bf16
constexpr uint32_t kWStage = 2 * kWChunk;            // activations + weight
constexpr size_t kWSmem = kWStages * kWStage + 1024 + 64;
constexpr int kMaxKSplit = 16;
constexpr uint64_t kWriteWaitNs = 2000000000ull;

MLA_DEVI void tma_load_2d_local(uint32_t dst, const void* tmap, uint32_t mbar, int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(tmap), "r"(mbar), "r"(x), "r"(y)
      : "memory");
}

// 16-byte unit holding columns c0 .. c0+7 of row r of a 128-byte-swizzled block
MLA_DEVI uint32_t swz(uint32_t base, int r, int c0) { return base + r * 128 + ((((c0 >> 3) ^ (r & 7)) & 7) << 4); }

// part[ks][t][n] = sum over the CTA's K chunks of h[t][k] * w[n][k]
__global__ void __launch_bounds__(kWThreads) kv_down_proj_kernel(const __grid_constant__ CUtensorMap tm_h,
                                                                 const __grid_constant__ CUtensorMap tm_w,
                                                                 float* __restrict__ part, int n_tok,
                                                                 int n_chunks, uint32_t* status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t sa = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t bar0 = sa + kWStages * kWStage;
  const int t0 = blockIdx.x * kWTok, ks = blockIdx.y, n0 = blockIdx.z * kWCols;
  const int c_begin = (int)(((long)ks * n_chunks) / gridDim.y);
  const int c_end = (int)(((long)(ks + 1) * n_chunks) / gridDim.y);
  const int nk = c_end - c_begin;  // >= 1: the split count never exceeds the chunk count
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_trigger();
  if (tid == 0) {
    for (int s = 0; s < kWStages; ++s) mbar_init(bar0 + 8 * s, 1);
    fence_mbar_init();
  }
  __syncthreads();

  // the weight is never written by a kernel this one may overlap with; the
  // hidden states may be, so their loads wait for the previous kernel
  auto load_w = [&](int kc, int s) {
    tma_load_2d_local(sa + s * kWStage + kWChunk, &tm_w, bar0 + 8 * s, (c_begin + kc) * kWK, n0);
  };
  auto load_h = [&](int kc, int s) {
    tma_load_2d_local(sa + s * kWStage, &tm_h, bar0 + 8 * s, (c_begin + kc) * kWK, t0);
  };
  int issued = 0;  // chunks whose loads thread 0 has issued
  if (tid == 0) {
    for (int s = 0; s < kWStages && s < nk; ++s) {
      mbar_arrive_expect_tx_local(bar0 + 8 * s, kWStage);
      load_w(s, s);
    }
    issued = min(kWStages, nk);
  }
  pdl_wait();
  if (tid == 0)
    for (int s = 0; s < kWStages && s < nk; ++s) load_h(s, s);

  float acc[kWCols / 8][4];
#pragma unroll
  for (int j = 0; j < kWCols / 8; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;

  int aborted = 0;
#pragma unroll 1
  for (int kc = 0; kc < nk; ++kc) {
    const int s = kc % kWStages;
    mbar_wait(bar0 + 8 * s, (kc / kWStages) & 1, &aborted, status, kWriteWaitNs);
    const uint32_t hb = sa + s * kWStage, wb = hb + kWChunk;
#pragma unroll
    for (int kk = 0; kk < kWK / 16; ++kk) {
      uint32_t a[4];
      {
        const uint32_t ad = swz(hb, warp * 16 + (lane & 15), kk * 16 + (lane >> 4) * 8);
        asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                     : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                     : "r"(ad));
      }
#pragma unroll
      for (int np = 0; np < kWCols / 16; ++np) {
        uint32_t b0, b1, b2, b3;
        const uint32_t ad = swz(wb, np * 16 + (lane & 7) + 8 * (lane >> 4), kk * 16 + 8 * ((lane >> 3) & 1));
        asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                     : "=r"(b0), "=r"(b1), "=r"(b2), "=r"(b3)
                     : "r"(ad));
        mma_bf16_16816(acc[2 * np], a, b0, b1);
        mma_bf16_16816(acc[2 * np + 1], a, b2, b3);
      }
    }
    __syncthreads();  // every warp is done with stage s
    const int next = kc + kWStages;
    if (tid == 0 && next < nk && !aborted) {
      mbar_arrive_expect_tx_local(bar0 + 8 * s, kWStage);
      load_w(next, s);
      load_h(next, s);
      ++issued;
    }
  }
  // A wait that ran out may leave loads in flight.  Before the CTA exits (and its
  // shared memory goes to another CTA) the issuing thread waits, bounded again,
  // for the last load issued into every stage: a stage's phases complete in order.
  if (__syncthreads_or(aborted) && tid == 0) {
    for (int s = 0; s < kWStages && s < issued; ++s) {
      const int last = s + ((issued - 1 - s) / kWStages) * kWStages;
      int give_up = 0;
      mbar_wait(bar0 + 8 * s, (last / kWStages) & 1, &give_up, nullptr, kWriteWaitNs);
    }
  }

#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const int t = t0 + warp * 16 + (lane >> 2) + hf * 8;
    if (t >= n_tok) continue;
    float* prow = part + ((size_t)ks * n_tok + t) * kRow + n0 + 2 * (lane & 3);
#pragma unroll
    for (int j = 0; j < kWCols / 8; ++j)
      *reinterpret_cast<float2*>(prow + 8 * j) = make_float2(acc[j][2 * hf], acc[j][2 * hf + 1]);
  }
}

struct FinishParams {
  const float* part;
  uint8_t* kv;
  void* kv_scale;  // e4m3: fp32 [pages][64]; q8_0: fp16 [pages][64][18]
  const int32_t* block_table;
  const int32_t* seq_lens;
  uint32_t* status;
  int n_tok, k_split, s_q, max_pages, num_pages;
  double log2_base;
};

// One warp per new token: sum the partials, rotate, quantise, store.  KIND: 0
// bf16 cache, 1 e4m3 with a per-row scale, 2 q8_0 with per-block scales.
template <int KIND>
__global__ void __launch_bounds__(128) kv_finish_kernel(const FinishParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 4 + warp;
  // No early trigger: the kernels after this one may start only once it has
  // completed.  The decode reads its first cache page before waiting for its
  // predecessor, and with an early trigger here a decode two launches later could
  // start while these rows are still being written.
  pdl_wait();  // the partials come from the previous kernel
  if (t >= p.n_tok) return;
  const int b = t / p.s_q, i = t - b * p.s_q;
  const int L = p.seq_lens[b];
  if (L < p.s_q || L > p.max_pages * kPage) {
    if (lane == 0) set_status(p.status, MLA_ERR_BAD_SEQ_LEN);
    return;
  }
  const int pos = L - p.s_q + i;
  const int page = p.block_table[(size_t)b * p.max_pages + pos / kPage];
  if (page < 0 || page >= p.num_pages) {
    if (lane == 0) set_status(p.status, MLA_ERR_BAD_BLOCK_TABLE);
    return;
  }
  const size_t slot = (size_t)page * kPage + pos % kPage;

  float2 v[9];
#pragma unroll
  for (int j = 0; j < 9; ++j) v[j] = make_float2(0.f, 0.f);
  for (int ks = 0; ks < p.k_split; ++ks) {
    const float* src = p.part + ((size_t)ks * p.n_tok + t) * kRow + 2 * lane;
#pragma unroll
    for (int j = 0; j < 9; ++j) {
      const float2 x = *reinterpret_cast<const float2*>(src + 64 * j);
      v[j].x += x.x;
      v[j].y += x.y;
    }
  }
  {
    // RoPE pair `lane` of the 64-value key (values 512 + 2 lane, 513 + 2 lane)
    const double theta = exp2(-(2.0 * lane / kDr) * p.log2_base);
    double ang = (double)pos * theta;
    const double two_pi = 6.283185307179586476925286766559;
    ang -= two_pi * rint(ang / two_pi);
    double sn, cs;
    sincos(ang, &sn, &cs);
    const double x0 = v[8].x, x1 = v[8].y;
    v[8] = make_float2((float)(x0 * cs - x1 * sn), (float)(x0 * sn + x1 * cs));
  }
  if constexpr (KIND == 0) {
    __nv_bfloat16* row = reinterpret_cast<__nv_bfloat16*>(p.kv) + slot * kRow + 2 * lane;
#pragma unroll
    for (int j = 0; j < 9; ++j) *reinterpret_cast<uint32_t*>(row + 64 * j) = pack_bf16(v[j].x, v[j].y);
  } else if constexpr (KIND == 2 || KIND == 3) {
    // q8_0 / q4_0: block 2j + lane / 16 is values 64j + 32 (lane / 16) .. +31, two
    // per lane of its half-warp; scale d = amax / levels (127 or 7) rounded to
    // fp16, codes the fp32 quotients by d rounded to nearest even and clamped to
    // [-levels, levels].  q4_0 stores code + 8 in four bits: values 64j + 2 lane
    // and 64j + 2 lane + 1 share byte 32j + lane (low half, high half).
    constexpr float levels = KIND == 2 ? 127.f : 7.f;
    __half* sc = static_cast<__half*>(p.kv_scale) + slot * (kRow / 32);
#pragma unroll
    for (int j = 0; j < 9; ++j) {
      float amax = fmaxf(fabsf(v[j].x), fabsf(v[j].y));
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const __half d = __float2half_rn(__fdiv_rn(amax, levels));
      const float df = __half2float(d);
      int c0 = 0, c1 = 0;
      if (df > 0.f) {
        c0 = (int)fminf(fmaxf(rintf(__fdiv_rn(v[j].x, df)), -levels), levels);
        c1 = (int)fminf(fmaxf(rintf(__fdiv_rn(v[j].y, df)), -levels), levels);
      }
      if constexpr (KIND == 2) {
        int8_t* row = reinterpret_cast<int8_t*>(p.kv) + slot * kRow + 2 * lane;
        *reinterpret_cast<uint16_t*>(row + 64 * j) = (uint16_t)((uint8_t)c0 | ((uint16_t)(uint8_t)c1 << 8));
      } else {
        p.kv[slot * (kRow / 2) + 32 * j + lane] = (uint8_t)((c0 + 8) | ((c1 + 8) << 4));
      }
      if ((lane & 15) == 0) sc[2 * j + (lane >> 4)] = d;
    }
  } else {
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < 9; ++j) amax = fmaxf(amax, fmaxf(fabsf(v[j].x), fabsf(v[j].y)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    uint8_t* row = p.kv + slot * kRow + 2 * lane;
#pragma unroll
    for (int j = 0; j < 9; ++j) {
      float2 q = make_float2(__fdiv_rn(v[j].x, scale), __fdiv_rn(v[j].y, scale));
      q.x = fminf(fmaxf(q.x, -448.f), 448.f);
      q.y = fminf(fmaxf(q.y, -448.f), 448.f);
      const __nv_fp8x2_storage_t code = __nv_cvt_float2_to_fp8x2(q, __NV_SATFINITE, __NV_E4M3);
      *reinterpret_cast<uint16_t*>(row + 64 * j) = (uint16_t)code;
    }
    if (lane == 0) static_cast<float*>(p.kv_scale)[slot] = scale;
  }
}

}  // namespace

// Split count of the down-projection: enough CTAs to cover the 148 SMs, at most
// one per K chunk and kMaxKSplit in all.
int write_kv_k_split(int n_tok, int d_h) {
  const int m_tiles = n_tok > 0 ? (n_tok + kWTok - 1) / kWTok : 1;
  const int ctas = m_tiles * (kRow / kWCols);
  int ks = (148 + ctas - 1) / ctas;
  const int n_chunks = d_h / kWK;
  if (ks > n_chunks) ks = n_chunks;
  if (ks > kMaxKSplit) ks = kMaxKSplit;
  return ks < 1 ? 1 : ks;
}

cudaError_t launch_write_kv(const mla_write_kv_args_t* a, cudaStream_t stream) {
  const int n_tok = a->B * a->s_q;
  const int ks = write_kv_k_split(n_tok, a->d_h);
  CUtensorMap tm_h, tm_w;
  if (!tma_map_2d(&tm_h, a->h, a->d_h, n_tok, (uint64_t)a->d_h * 2, kWK, kWTok) ||
      !tma_map_2d(&tm_w, a->w_dkv, a->d_h, kRow, (uint64_t)a->d_h * 2, kWK, kWCols))
    return cudaErrorInvalidValue;
  unsigned char* ws = static_cast<unsigned char*>(a->workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  float* part = reinterpret_cast<float*>(ws + 256);
  static PerDeviceOnce attrs;
  cudaError_t e = once_per_device(attrs, [&]() {
    return cudaFuncSetAttribute(kv_down_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kWSmem);
  });
  if (e != cudaSuccess) return e;
  dim3 grid((n_tok + kWTok - 1) / kWTok, ks, kRow / kWCols);
  e = launch_pdl(kv_down_proj_kernel, grid, dim3(kWThreads), kWSmem, stream, tm_h, tm_w, part, n_tok,
                 a->d_h / kWK, status);
  if (e != cudaSuccess) return e;
  FinishParams p;
  p.part = part;
  p.kv = static_cast<uint8_t*>(a->kv_cache);
  p.kv_scale = a->kv_scale;
  p.block_table = a->block_table;
  p.seq_lens = a->seq_lens;
  p.status = status;
  p.n_tok = n_tok;
  p.k_split = ks;
  p.s_q = a->s_q;
  p.max_pages = a->max_pages_per_seq;
  p.num_pages = a->num_pages;
  p.log2_base = log2((double)a->rope_base);
  const dim3 fgrid((n_tok + 3) / 4);
  if (a->kv_dtype == MLA_KV_FP8_E4M3) return launch_pdl(kv_finish_kernel<1>, fgrid, dim3(128), 0, stream, p);
  if (a->kv_dtype == MLA_KV_Q8_0) return launch_pdl(kv_finish_kernel<2>, fgrid, dim3(128), 0, stream, p);
  if (a->kv_dtype == MLA_KV_Q4_0) return launch_pdl(kv_finish_kernel<3>, fgrid, dim3(128), 0, stream, p);
  return launch_pdl(kv_finish_kernel<0>, fgrid, dim3(128), 0, stream, p);
}

}  // namespace mla
