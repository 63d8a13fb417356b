// Host-side TMA tensor-map encoding and its cache (see tma_host.cuh).
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "tma_host.cuh"

namespace mla {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

struct MapKey {
  const void* ptr;
  uint32_t rank;
  uint64_t dims[5], strides[4];
  uint32_t box[5];
  CUtensorMapDataType dtype;
  CUtensorMapSwizzle swizzle;
  bool operator==(const MapKey& o) const {
    if (ptr != o.ptr || rank != o.rank || dtype != o.dtype || swizzle != o.swizzle) return false;
    for (int i = 0; i < 5; ++i)
      if (dims[i] != o.dims[i] || box[i] != o.box[i]) return false;
    for (int i = 0; i < 4; ++i)
      if (strides[i] != o.strides[i]) return false;
    return true;
  }
};

constexpr int kCache = 64;
std::mutex g_mu;
MapKey g_keys[kCache];
CUtensorMap g_maps[kCache];
int g_count = 0, g_next = 0;

bool encode(CUtensorMap* m, const MapKey& k) {
  {
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < g_count; ++i)
      if (g_keys[i] == k) {
        *m = g_maps[i];
        return true;
      }
  }
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[5], strides[4];
  cuuint32_t box[5], estr[5];
  for (int i = 0; i < 5; ++i) {
    dims[i] = k.dims[i];
    box[i] = k.box[i];
    estr[i] = 1;
  }
  for (int i = 0; i < 4; ++i) strides[i] = k.strides[i];
  CUresult res = enc(m, k.dtype, k.rank, const_cast<void*>(k.ptr), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, k.swizzle,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (res != CUDA_SUCCESS) return false;
  std::lock_guard<std::mutex> lock(g_mu);
  const int slot = g_count < kCache ? g_count++ : (g_next++ % kCache);
  g_keys[slot] = k;
  g_maps[slot] = *m;
  return true;
}

}  // namespace

bool tma_map_2d(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint64_t row_bytes,
                uint32_t box_cols, uint32_t box_rows) {
  MapKey k{ptr, 2, {cols, rows, 1, 1, 1}, {row_bytes, 0, 0, 0}, {box_cols, box_rows, 1, 1, 1},
           CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, CU_TENSOR_MAP_SWIZZLE_128B};
  return encode(m, k);
}

bool tma_map_3d(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2) {
  MapKey k{ptr, 3, {d0, d1, d2, 1, 1}, {s1, s2, 0, 0}, {b0, b1, b2, 1, 1},
           CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, CU_TENSOR_MAP_SWIZZLE_128B};
  return encode(m, k);
}

bool tma_map_nd(CUtensorMap* m, const void* ptr, uint32_t rank, const uint64_t* dims, const uint64_t* strides,
                const uint32_t* box, bool bytes, int swizzle_bytes) {
  if (rank < 1 || rank > 5) return false;
  CUtensorMapSwizzle swz;
  switch (swizzle_bytes) {
    case 128: swz = CU_TENSOR_MAP_SWIZZLE_128B; break;
    case 64: swz = CU_TENSOR_MAP_SWIZZLE_64B; break;
    case 32: swz = CU_TENSOR_MAP_SWIZZLE_32B; break;
    case 0: swz = CU_TENSOR_MAP_SWIZZLE_NONE; break;
    default: return false;
  }
  MapKey k{ptr, rank, {1, 1, 1, 1, 1}, {0, 0, 0, 0}, {1, 1, 1, 1, 1},
           bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, swz};
  for (uint32_t i = 0; i < rank; ++i) {
    k.dims[i] = dims[i];
    k.box[i] = box[i];
    if (i > 0) k.strides[i - 1] = strides[i - 1];
  }
  return encode(m, k);
}

}  // namespace mla
