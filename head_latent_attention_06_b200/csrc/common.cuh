// Shared device helpers: bf16/e4m3 conversion, cp.async, ldmatrix and the
// legacy warp-level MMA used by the projection kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/mla.h"

#define MLA_DEVI __device__ __forceinline__

namespace mla {

constexpr int kDc = 512;
constexpr int kDr = 64;
constexpr int kRow = kDc + kDr;  // 576 values per cached token
constexpr int kPage = 64;
constexpr int kDn = 128;
constexpr int kDv = 128;
constexpr float kLog2e = 1.4426950408889634f;

// The fused decode step's operands beyond the decode's own (q_lat and o_lat are
// then buffers of the step's workspace): q_nope, W_UK, W_UV, the output, and the
// flags between the step's phases.
struct StepOperands {
  const void* q_nope;
  const void* w_uk;
  const void* w_uv;
  void* out;
  uint32_t* flags;
};

// Layout of the decode workspace: a 256-byte header holding the sticky status
// word, then fp32 partial outputs [n_tok][H][S][d_c] and partial lse
// [n_tok][H][S], each 256-byte aligned.
struct WorkspaceLayout {
  size_t status_off, o_part_off, lse_part_off, total;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline WorkspaceLayout workspace_layout(int n_tok, int H, int splits) {
  WorkspaceLayout w;
  w.status_off = 0;
  w.o_part_off = 256;
  size_t rows = (size_t)n_tok * H * (splits > 1 ? splits : 0);
  w.lse_part_off = align_up(w.o_part_off + rows * kDc * sizeof(float), 256);
  w.total = align_up(w.lse_part_off + rows * sizeof(float), 256);
  return w;
}

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialisation may start while the previous kernel of the stream still runs;
// pdl_wait() blocks until that kernel has completed and its writes are visible,
// so nothing the previous kernel writes may be read before it.  pdl_trigger()
// lets the next kernel of the stream be scheduled early (a scheduling hint only).
MLA_DEVI void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
MLA_DEVI void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launches `kern` on `stream` with programmatic stream serialisation allowed.
template <typename Kern, typename... Args>
inline cudaError_t launch_pdl(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// One-time host set-up per device (kernel attributes and the like): `fn` runs
// with the device current, under a lock, until it has succeeded once on that
// device; later calls return at once.  Safe to call from several host threads.
struct PerDeviceOnce {
  static constexpr int kMaxDevices = 64;
  std::mutex mu;
  std::atomic<bool> done[kMaxDevices] = {};
};

template <typename Fn>
inline cudaError_t once_per_device(PerDeviceOnce& once, Fn fn) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= PerDeviceOnce::kMaxDevices) return fn();  // not cached, still correct
  if (once.done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  std::lock_guard<std::mutex> lock(once.mu);
  if (once.done[dev].load(std::memory_order_relaxed)) return cudaSuccess;
  e = fn();
  if (e == cudaSuccess) once.done[dev].store(true, std::memory_order_release);
  return e;
}

// Number of SMs of the current device, queried once per device (148 on a B200).
inline int device_sm_count() {
  static PerDeviceOnce once;
  static std::atomic<int> count[PerDeviceOnce::kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= PerDeviceOnce::kMaxDevices) return 148;
  once_per_device(once, [&]() {
    int n = 0;
    cudaError_t e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess && n > 0) count[dev].store(n, std::memory_order_relaxed);
    return e;
  });
  const int n = count[dev].load(std::memory_order_relaxed);
  return n > 0 ? n : 148;
}

MLA_DEVI void set_status(uint32_t* status, uint32_t code) {
  if (status) atomicCAS(status, 0u, code);
}

MLA_DEVI uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

MLA_DEVI void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem)), "l"(gmem));
}
MLA_DEVI void cp_async4(void* smem, const void* gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(smem)), "l"(gmem));
}
MLA_DEVI void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
MLA_DEVI void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

MLA_DEVI void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(smem_u32(p)));
}
MLA_DEVI void ldmatrix_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(smem_u32(p)));
}

// D = A(16x16 bf16, row) * B(16x8 bf16, col) + D, fp32 accumulation.
MLA_DEVI void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

MLA_DEVI uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Two e4m3fn codes (low byte first) to two bf16 values, exactly: every finite
// e4m3 value is representable in bf16.  Built from the format's definition:
// normal codes move the 4-bit exponent (bias 7) to bf16's 8-bit exponent (bias
// 127) and the 3 mantissa bits to the top of bf16's 7; subnormal codes
// (exponent 0) are m * 2^-9, produced through an fp32 multiply.
MLA_DEVI uint32_t e4m3x2_to_bf16x2(uint16_t two) {
  uint32_t out = 0;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    uint32_t c = (two >> (8 * k)) & 0xFFu;
    uint32_t s = (c & 0x80u) << 8;
    uint32_t e = (c >> 3) & 0xFu;
    uint32_t m = c & 0x7u;
    uint32_t h;
    if (e != 0) {
      h = s | ((e + 120u) << 7) | (m << 4);
    } else {
      float f = (float)m * 0.001953125f;  // 2^-9
      h = s | (__float_as_uint(f) >> 16);
    }
    out |= h << (16 * k);
  }
  return out;
}

}  // namespace mla
