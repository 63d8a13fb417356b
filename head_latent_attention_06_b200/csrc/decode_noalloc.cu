// Decode entry point for callers that cannot allocate device memory.
//
// mla_decode_paged needs a caller-provided workspace (the status word and, when
// a sequence is split across CTAs, the fp32 partial outputs).  Some callers
// cannot call cudaMalloc to provide one: a plugin running inside an engine that
// owns all device memory and forbids allocations after start-up, or code on a
// latency-critical path where an allocation could synchronise the device.
// mla_decode_paged_noalloc runs the same decode (and the split merge when one is
// needed) with its scratch in a fixed array compiled into this library instead.
//
// The array lives in device global memory on every GPU that loads the library,
// for the lifetime of the process.  Every call shares it and it keeps the last
// call's contents: the status word is zeroed once at set-up and then only by
// mla_get_status_noalloc (it is sticky, like a workspace's), the partials are
// always written before they are read.  Two calls whose work overlaps on the GPU
// (different streams, no ordering between them) race on the array; order them on
// one stream or with events.
#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t kStaticScratchBytes = (size_t)16 << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device.  In host code the symbol
// name is only a host-side stand-in; the address must come from
// cudaGetSymbolAddress, once per device, with that device current.  The first
// lookup on a device also zeroes the status word (synchronously).
mla_status_t scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return MLA_ERR_CUDA;
    if (cudaMemset(p, 0, 16) != cudaSuccess) return MLA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MLA_OK;
}

}  // namespace

extern "C" mla_status_t mla_noalloc_init(void) {
  void* scratch = nullptr;
  return scratch_address(&scratch);
}

extern "C" mla_status_t mla_decode_paged_noalloc(const mla_decode_args_t* args, void* stream) {
  if (!args) return MLA_ERR_INVALID_VALUE;
  mla_decode_args_t a = *args;
  a.workspace = nullptr;
  a.workspace_bytes = 0;
  size_t need = 0;
  mla_status_t st = mla_decode_workspace_size(&a, &need);
  if (st != MLA_OK) return st;
  if (need > kStaticScratchBytes) return MLA_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != MLA_OK) return st;
  a.workspace = scratch;
  a.workspace_bytes = kStaticScratchBytes;
  st = mla_decode_paged(&a, stream);
  if (st != MLA_OK) return st;
  return mla_combine_splits(&a, stream);
}

extern "C" mla_status_t mla_get_status_noalloc(void* stream) {
  void* scratch = nullptr;
  mla_status_t st = scratch_address(&scratch);
  if (st != MLA_OK) return st;
  return mla_get_status(scratch, stream);
}
