// C ABI of the MLA decode library (declared in include/mla.h): host-side
// argument validation, split selection, workspace sizing and kernel launches.
// Nothing here allocates device memory or synchronises, except mla_get_status.
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "common.cuh"

namespace mla {
cudaError_t launch_absorb_q(const void*, const void*, void*, int, int, cudaStream_t);
cudaError_t launch_up_proj_v(const void*, const void*, void*, int, int, cudaStream_t);
cudaError_t launch_decode_mma(const mla_decode_args_t*, int, cudaStream_t);
cudaError_t launch_combine(const mla_decode_args_t*, int, cudaStream_t);
cudaError_t launch_decode_tc(const mla_decode_args_t*, int, cudaStream_t);
cudaError_t launch_decode_f8(const mla_decode_args_t*, int, cudaStream_t);
bool decode_tc_supported(const mla_decode_args_t*);
int decode_tc_clusters_per_split(const mla_decode_args_t*);
int decode_mma_tiles(int len);
int decode_mma_ctas_per_split(int s_q, int H, int B);
int write_kv_k_split(int n_tok, int d_h);
cudaError_t launch_write_kv(const mla_write_kv_args_t*, cudaStream_t);
size_t prefill_workspace_bytes(int B, int H, int Lmax);
cudaError_t launch_prefill(const mla_prefill_args_t*, cudaStream_t);
cudaError_t launch_fold_hadamard(void*, int, void*, void*, int, cudaStream_t);
bool decode_step_fusable(const mla_decode_args_t*, int splits);
size_t decode_step_flag_bytes();
cudaError_t launch_decode_step_fused(const mla_decode_args_t*, const StepOperands*, cudaStream_t);
}  // namespace mla

using namespace mla;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

mla_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

mla_status_t check_proj(const void* x, const void* w, const void* y, int32_t n_tok, int32_t H,
                        int32_t d_small, int32_t d_c) {
  if (n_tok < 0 || H <= 0) return MLA_ERR_INVALID_VALUE;
  if (d_small != 128 || d_c != kDc) return MLA_ERR_UNSUPPORTED;
  if (n_tok == 0) return MLA_OK;
  if (!x || !w || !y) return MLA_ERR_INVALID_VALUE;
  if (!aligned16(x) || !aligned16(w) || !aligned16(y)) return MLA_ERR_MISALIGNED;
  return MLA_OK;
}

// Shape checks shared by the decode entry points (no pointer checks).
mla_status_t check_decode_shape(const mla_decode_args_t* a) {
  if (!a) return MLA_ERR_INVALID_VALUE;
  if (a->B < 0 || a->H <= 0 || a->s_q <= 0 || a->num_pages < 0 || a->max_pages_per_seq <= 0)
    return MLA_ERR_INVALID_VALUE;
  if (a->d_c != kDc || a->d_r != kDr || a->page_size != kPage) return MLA_ERR_UNSUPPORTED;
  if (a->H % 16 != 0 || a->H > 128 || a->s_q > MLA_MAX_S_Q) return MLA_ERR_UNSUPPORTED;
  if (a->kv_dtype != MLA_KV_BF16 && a->kv_dtype != MLA_KV_FP8_E4M3 && a->kv_dtype != MLA_KV_Q8_0 &&
      a->kv_dtype != MLA_KV_Q4_0)
    return MLA_ERR_UNSUPPORTED;
  if (a->num_splits < 0 || a->num_splits > MLA_MAX_SPLITS) return MLA_ERR_INVALID_VALUE;
  if (a->max_seq_len < 0) return MLA_ERR_INVALID_VALUE;
  if (!(a->softmax_scale == a->softmax_scale)) return MLA_ERR_INVALID_VALUE;
  return MLA_OK;
}

// Process-wide kernel choice (mla_set_decode_kernel) and device wait limit
// (mla_set_device_wait_limit).
std::atomic<int32_t> g_decode_kernel{MLA_DECODE_AUTO};
constexpr uint64_t kDefaultWaitNs = 2000000000ull;  // 2 s
std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};

bool forced_mma() { return g_decode_kernel.load(std::memory_order_relaxed) == MLA_DECODE_WARP_MMA; }

// Which decode kernel runs: the tensor-memory kernel for the shapes it takes,
// else the warp-MMA kernel.
bool use_tc(const mla_decode_args_t* a) { return !forced_mma() && decode_tc_supported(a); }

// Workspace bytes the chosen path needs.
size_t workspace_bytes(const mla_decode_args_t* a, int splits) {
  return workspace_layout(a->B * a->s_q, a->H, splits).total;
}

// Split count.  Tensor-memory kernel: the count that minimises the modelled
// makespan (waves of 74 CTA pairs x per-unit work), preferring fewer splits.  Warp-MMA
// kernel: enough CTAs to cover the SMs, never a split shorter than 8 tiles.
int choose_splits(const mla_decode_args_t* a) {
  if (a->num_splits > 0) return a->num_splits;
  const int max_len = a->max_seq_len > 0 ? a->max_seq_len : a->max_pages_per_seq * kPage;
  if (use_tc(a)) {
    const int tiles = (max_len + kPage - 1) / kPage;
    const int units = decode_tc_clusters_per_split(a) > 0 ? decode_tc_clusters_per_split(a) : 1;
    const int slots = device_sm_count() / 2;
    int best = 1;
    long best_cost = -1;
    for (int s = 1; s <= MLA_MAX_SPLITS && s <= (tiles > 0 ? tiles : 1); ++s) {
      const long waves = ((long)units * s + slots - 1) / slots;
      // a work unit costs its tiles plus about 8 tiles of start-up (Q load, first
      // pages, epilogue); more than one split adds the combine pass
      const long cost = waves * ((tiles + s - 1) / s + 8) * 100 + (s > 1 ? 400 : 0) + s;
      if (best_cost < 0 || cost < best_cost) {
        best_cost = cost;
        best = s;
      }
    }
    return best;
  }
  const int tiles = decode_mma_tiles(max_len);
  const int ctas = decode_mma_ctas_per_split(a->s_q, a->H, a->B > 0 ? a->B : 1);
  int s = (device_sm_count() + ctas - 1) / ctas;
  int cap = tiles / 8;
  if (cap < 1) cap = 1;
  if (s > cap) s = cap;
  if (s > MLA_MAX_SPLITS) s = MLA_MAX_SPLITS;
  if (s < 1) s = 1;
  return s;
}

mla_status_t check_write_kv_shape(const mla_write_kv_args_t* a) {
  if (!a) return MLA_ERR_INVALID_VALUE;
  if (a->B < 0 || a->s_q <= 0 || a->d_h <= 0 || a->num_pages < 0 || a->max_pages_per_seq <= 0)
    return MLA_ERR_INVALID_VALUE;
  if ((int64_t)a->B * a->s_q > (1 << 24)) return MLA_ERR_INVALID_VALUE;
  if (a->d_c != kDc || a->d_r != kDr || a->page_size != kPage || a->d_h % 64 != 0) return MLA_ERR_UNSUPPORTED;
  if (a->kv_dtype != MLA_KV_BF16 && a->kv_dtype != MLA_KV_FP8_E4M3 && a->kv_dtype != MLA_KV_Q8_0 &&
      a->kv_dtype != MLA_KV_Q4_0)
    return MLA_ERR_UNSUPPORTED;
  if (!(a->rope_base > 0.f) || !isfinite(a->rope_base)) return MLA_ERR_INVALID_VALUE;
  return MLA_OK;
}

mla_status_t check_prefill_shape(const mla_prefill_args_t* a) {
  if (!a) return MLA_ERR_INVALID_VALUE;
  if (a->B < 0 || a->H <= 0 || a->s_q <= 0 || a->num_pages < 0 || a->max_pages_per_seq <= 0)
    return MLA_ERR_INVALID_VALUE;
  if (a->d_c != kDc || a->d_r != kDr || a->page_size != kPage) return MLA_ERR_UNSUPPORTED;
  if (a->H > 128 || a->B > 65535 || a->kv_dtype != MLA_KV_BF16) return MLA_ERR_UNSUPPORTED;
  if (a->max_seq_len < a->s_q) return MLA_ERR_INVALID_VALUE;
  // TMA coordinates are 32-bit: rows of the per-head key / value arrays and
  // query tokens must stay below 2^31
  const int64_t lpad = ((int64_t)a->max_seq_len + 255) / 256 * 256;
  if ((int64_t)a->B * a->H * lpad >= (int64_t)1 << 31 || (int64_t)a->B * a->s_q >= (int64_t)1 << 31)
    return MLA_ERR_UNSUPPORTED;
  if (!(a->softmax_scale == a->softmax_scale)) return MLA_ERR_INVALID_VALUE;
  return MLA_OK;
}

size_t write_kv_workspace(const mla_write_kv_args_t* a) {
  const int n_tok = a->B * a->s_q;
  return align_up(256 + (size_t)write_kv_k_split(n_tok, a->d_h) * n_tok * kRow * sizeof(float), 256);
}

}  // namespace

namespace mla {
// Limit of every bounded wait in the decode kernels, as set for this process.
uint64_t device_wait_limit_ns() { return g_wait_ns.load(std::memory_order_relaxed); }
}  // namespace mla

// ---- the whole step: the decode's arguments with q_lat and o_lat in the step's
// workspace, laid out after the decode's own part and the step's flags
namespace {
struct StepLayout {
  size_t flags_off, q_lat_off, o_lat_off, total;
};

mla_decode_args_t step_decode_args(const mla_step_args_t* s) {
  mla_decode_args_t d;
  memset(&d, 0, sizeof(d));
  d.q_pe = s->q_pe;
  d.kv_cache = s->kv_cache;
  d.kv_scale = s->kv_scale;
  d.block_table = s->block_table;
  d.seq_lens = s->seq_lens;
  d.lse = s->lse;
  d.workspace = s->workspace;
  d.workspace_bytes = s->workspace_bytes;
  d.B = s->B;
  d.s_q = s->s_q;
  d.H = s->H;
  d.d_c = s->d_c;
  d.d_r = s->d_r;
  d.page_size = s->page_size;
  d.num_pages = s->num_pages;
  d.max_pages_per_seq = s->max_pages_per_seq;
  d.kv_dtype = s->kv_dtype;
  d.causal = s->causal;
  d.num_splits = s->num_splits;
  d.max_seq_len = s->max_seq_len;
  d.softmax_scale = s->softmax_scale;
  return d;
}

StepLayout step_layout(const mla_decode_args_t* d, int splits) {
  StepLayout L;
  const size_t lat = (size_t)d->B * d->s_q * d->H * kDc * 2;
  L.flags_off = align_up(workspace_bytes(d, splits), 256);
  L.q_lat_off = align_up(L.flags_off + decode_step_flag_bytes(), 256);
  L.o_lat_off = align_up(L.q_lat_off + lat, 256);
  L.total = align_up(L.o_lat_off + lat, 256);
  return L;
}

// One launch: forced (fuse = 1) wherever the fused kernel takes the shape; by
// default only where it measured faster than the four launches chained by
// programmatic dependent launch: the q8_0 and q4_0 caches, whose decode is
// bound by its converter warps, with a grid covering at least half the SMs
// (with fewer CTAs the projection tiles queue up on them).
bool step_fused(const mla_step_args_t* s, const mla_decode_args_t* d, int splits) {
  if (s->fuse < 0 || !use_tc(d) || !decode_step_fusable(d, splits)) return false;
  if (s->fuse > 0) return true;
  return d->kv_dtype != MLA_KV_BF16 && 4 * d->B * d->s_q >= device_sm_count();
}
}  // namespace

extern "C" {

mla_status_t mla_absorb_q(const void* q_nope, const void* w_uk, void* q_lat, int32_t n_tok,
                          int32_t H, int32_t d_n, int32_t d_c, void* stream) {
  mla_status_t st = check_proj(q_nope, w_uk, q_lat, n_tok, H, d_n, d_c);
  if (st != MLA_OK || n_tok == 0) return st;
  return from_cuda(launch_absorb_q(q_nope, w_uk, q_lat, n_tok, H, (cudaStream_t)stream));
}

mla_status_t mla_up_proj_v(const void* o_lat, const void* w_uv, void* out, int32_t n_tok, int32_t H,
                           int32_t d_v, int32_t d_c, void* stream) {
  mla_status_t st = check_proj(o_lat, w_uv, out, n_tok, H, d_v, d_c);
  if (st != MLA_OK || n_tok == 0) return st;
  return from_cuda(launch_up_proj_v(o_lat, w_uv, out, n_tok, H, (cudaStream_t)stream));
}

mla_status_t mla_decode_num_splits(const mla_decode_args_t* a, int32_t* num_splits) {
  mla_status_t st = check_decode_shape(a);
  if (st != MLA_OK) return st;
  if (!num_splits) return MLA_ERR_INVALID_VALUE;
  *num_splits = choose_splits(a);
  return MLA_OK;
}

mla_status_t mla_decode_workspace_size(const mla_decode_args_t* a, size_t* bytes) {
  mla_status_t st = check_decode_shape(a);
  if (st != MLA_OK) return st;
  if (!bytes) return MLA_ERR_INVALID_VALUE;
  *bytes = workspace_bytes(a, choose_splits(a));
  return MLA_OK;
}

static mla_status_t check_decode_ptrs(const mla_decode_args_t* a, int splits) {
  if (!a->workspace) return MLA_ERR_INVALID_VALUE;
  if (!aligned16(a->workspace)) return MLA_ERR_MISALIGNED;
  if (a->workspace_bytes < workspace_bytes(a, splits)) return MLA_ERR_WORKSPACE_TOO_SMALL;
  if (a->B == 0) return MLA_OK;
  if (!a->q_lat || !a->q_pe || !a->kv_cache || !a->block_table || !a->seq_lens || !a->o_lat)
    return MLA_ERR_INVALID_VALUE;
  if (a->kv_dtype != MLA_KV_BF16 && !a->kv_scale) return MLA_ERR_INVALID_VALUE;
  if (a->num_pages <= 0) return MLA_ERR_INVALID_VALUE;
  if (!aligned16(a->q_lat) || !aligned16(a->q_pe) || !aligned16(a->kv_cache) ||
      !aligned16(a->o_lat))
    return MLA_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(a->block_table) & 3u) ||
      (reinterpret_cast<uintptr_t>(a->seq_lens) & 3u) ||
      (reinterpret_cast<uintptr_t>(a->lse) & 3u) || (reinterpret_cast<uintptr_t>(a->kv_scale) & 3u))
    return MLA_ERR_MISALIGNED;
  return MLA_OK;
}

mla_status_t mla_decode_paged(const mla_decode_args_t* a, void* stream) {
  mla_status_t st = check_decode_shape(a);
  if (st != MLA_OK) return st;
  const int splits = choose_splits(a);
  st = check_decode_ptrs(a, splits);
  if (st != MLA_OK || a->B == 0) return st;
  if (use_tc(a))
    return from_cuda(a->kv_dtype == MLA_KV_FP8_E4M3 ? launch_decode_f8(a, splits, (cudaStream_t)stream)
                                                      : launch_decode_tc(a, splits, (cudaStream_t)stream));
  return from_cuda(launch_decode_mma(a, splits, (cudaStream_t)stream));
}

mla_status_t mla_combine_splits(const mla_decode_args_t* a, void* stream) {
  mla_status_t st = check_decode_shape(a);
  if (st != MLA_OK) return st;
  const int splits = choose_splits(a);
  st = check_decode_ptrs(a, splits);
  if (st != MLA_OK || a->B == 0) return st;
  if (splits == 1) return st;
  return from_cuda(launch_combine(a, splits, (cudaStream_t)stream));
}

mla_status_t mla_write_kv_workspace_size(const mla_write_kv_args_t* a, size_t* bytes) {
  mla_status_t st = check_write_kv_shape(a);
  if (st != MLA_OK) return st;
  if (!bytes) return MLA_ERR_INVALID_VALUE;
  *bytes = write_kv_workspace(a);
  return MLA_OK;
}

mla_status_t mla_write_kv(const mla_write_kv_args_t* a, void* stream) {
  mla_status_t st = check_write_kv_shape(a);
  if (st != MLA_OK) return st;
  if (!a->workspace) return MLA_ERR_INVALID_VALUE;
  if (!aligned16(a->workspace)) return MLA_ERR_MISALIGNED;
  if (a->workspace_bytes < write_kv_workspace(a)) return MLA_ERR_WORKSPACE_TOO_SMALL;
  if (a->B == 0) return MLA_OK;
  if (!a->h || !a->w_dkv || !a->kv_cache || !a->block_table || !a->seq_lens) return MLA_ERR_INVALID_VALUE;
  if (a->kv_dtype != MLA_KV_BF16 && !a->kv_scale) return MLA_ERR_INVALID_VALUE;
  if (a->num_pages <= 0) return MLA_ERR_INVALID_VALUE;
  if (!aligned16(a->h) || !aligned16(a->w_dkv) || !aligned16(a->kv_cache)) return MLA_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(a->block_table) & 3u) || (reinterpret_cast<uintptr_t>(a->seq_lens) & 3u) ||
      (reinterpret_cast<uintptr_t>(a->kv_scale) & 3u))
    return MLA_ERR_MISALIGNED;
  return from_cuda(launch_write_kv(a, (cudaStream_t)stream));
}

mla_status_t mla_decode_step_workspace_size(const mla_step_args_t* a, size_t* bytes) {
  if (!a) return MLA_ERR_INVALID_VALUE;
  const mla_decode_args_t d = step_decode_args(a);
  mla_status_t st = check_decode_shape(&d);
  if (st != MLA_OK) return st;
  if (!bytes) return MLA_ERR_INVALID_VALUE;
  *bytes = step_layout(&d, choose_splits(&d)).total;
  return MLA_OK;
}

mla_status_t mla_decode_step_launches(const mla_step_args_t* a, int32_t* launches) {
  if (!a) return MLA_ERR_INVALID_VALUE;
  const mla_decode_args_t d = step_decode_args(a);
  mla_status_t st = check_decode_shape(&d);
  if (st != MLA_OK) return st;
  if (!launches) return MLA_ERR_INVALID_VALUE;
  const int splits = choose_splits(&d);
  *launches = a->B == 0 ? 0 : step_fused(a, &d, splits) ? 1 : splits > 1 ? 4 : 3;
  return MLA_OK;
}

mla_status_t mla_decode_step(const mla_step_args_t* a, void* stream) {
  if (!a) return MLA_ERR_INVALID_VALUE;
  mla_decode_args_t d = step_decode_args(a);
  mla_status_t st = check_decode_shape(&d);
  if (st != MLA_OK) return st;
  const int splits = choose_splits(&d);
  const StepLayout L = step_layout(&d, splits);
  if (!a->workspace) return MLA_ERR_INVALID_VALUE;
  if (!aligned16(a->workspace)) return MLA_ERR_MISALIGNED;
  if (a->workspace_bytes < L.total) return MLA_ERR_WORKSPACE_TOO_SMALL;
  if (a->B == 0) return MLA_OK;
  if (!a->q_nope || !a->w_uk || !a->w_uv || !a->out) return MLA_ERR_INVALID_VALUE;
  if (!aligned16(a->q_nope) || !aligned16(a->w_uk) || !aligned16(a->w_uv) || !aligned16(a->out))
    return MLA_ERR_MISALIGNED;
  unsigned char* ws = static_cast<unsigned char*>(a->workspace);
  d.q_lat = ws + L.q_lat_off;
  d.o_lat = ws + L.o_lat_off;
  st = check_decode_ptrs(&d, splits);
  if (st != MLA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const int n_tok = a->B * a->s_q;
  if (step_fused(a, &d, splits)) {
    const StepOperands fx = {a->q_nope, a->w_uk, a->w_uv, a->out, reinterpret_cast<uint32_t*>(ws + L.flags_off)};
    return from_cuda(launch_decode_step_fused(&d, &fx, s));
  }
  cudaError_t e = launch_absorb_q(a->q_nope, a->w_uk, ws + L.q_lat_off, n_tok, a->H, s);
  if (e == cudaSuccess)
    e = use_tc(&d) ? (d.kv_dtype == MLA_KV_FP8_E4M3 ? launch_decode_f8(&d, splits, s) : launch_decode_tc(&d, splits, s))
                   : launch_decode_mma(&d, splits, s);
  if (e == cudaSuccess && splits > 1) e = launch_combine(&d, splits, s);
  if (e == cudaSuccess) e = launch_up_proj_v(d.o_lat, a->w_uv, a->out, n_tok, a->H, s);
  return from_cuda(e);
}

mla_status_t mla_fold_hadamard(void* w_dkv, int32_t d_h, void* w_uk, void* w_uv, int32_t H, void* stream) {
  if (H < 0 || (w_dkv && d_h <= 0)) return MLA_ERR_INVALID_VALUE;
  if (H > 128 || (w_dkv && d_h % 64 != 0)) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(w_dkv) || !aligned16(w_uk) || !aligned16(w_uv)) return MLA_ERR_MISALIGNED;
  return from_cuda(launch_fold_hadamard(w_dkv, d_h, w_uk, w_uv, H, (cudaStream_t)stream));
}

mla_status_t mla_prefill_workspace_size(const mla_prefill_args_t* a, size_t* bytes) {
  mla_status_t st = check_prefill_shape(a);
  if (st != MLA_OK) return st;
  if (!bytes) return MLA_ERR_INVALID_VALUE;
  *bytes = prefill_workspace_bytes(a->B, a->H, a->max_seq_len);
  return MLA_OK;
}

mla_status_t mla_prefill(const mla_prefill_args_t* a, void* stream) {
  mla_status_t st = check_prefill_shape(a);
  if (st != MLA_OK) return st;
  if (!a->workspace) return MLA_ERR_INVALID_VALUE;
  if (!aligned16(a->workspace)) return MLA_ERR_MISALIGNED;
  if (a->workspace_bytes < prefill_workspace_bytes(a->B, a->H, a->max_seq_len)) return MLA_ERR_WORKSPACE_TOO_SMALL;
  if (a->B == 0) return MLA_OK;
  if (!a->q_nope || !a->q_pe || !a->w_uk || !a->w_uv || !a->kv_cache || !a->block_table || !a->seq_lens ||
      !a->out)
    return MLA_ERR_INVALID_VALUE;
  if (a->num_pages <= 0) return MLA_ERR_INVALID_VALUE;
  if (!aligned16(a->q_nope) || !aligned16(a->q_pe) || !aligned16(a->w_uk) || !aligned16(a->w_uv) ||
      !aligned16(a->kv_cache) || !aligned16(a->out))
    return MLA_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(a->block_table) & 3u) || (reinterpret_cast<uintptr_t>(a->seq_lens) & 3u) ||
      (reinterpret_cast<uintptr_t>(a->lse) & 3u))
    return MLA_ERR_MISALIGNED;
  return from_cuda(launch_prefill(a, (cudaStream_t)stream));
}

mla_status_t mla_get_status(void* workspace, void* stream) {
  if (!workspace) return MLA_ERR_INVALID_VALUE;
  uint32_t word = 0;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MLA_ERR_CUDA;
  if (word != 0) {
    if (cudaMemsetAsync(workspace, 0, sizeof(word), s) != cudaSuccess) return MLA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MLA_ERR_CUDA;
  }
  return (mla_status_t)word;
}

mla_status_t mla_set_device_wait_limit(uint64_t ns) {
  g_wait_ns.store(ns == 0 ? kDefaultWaitNs : ns, std::memory_order_relaxed);
  return MLA_OK;
}

mla_status_t mla_set_decode_kernel(int32_t kernel) {
  if (kernel != MLA_DECODE_AUTO && kernel != MLA_DECODE_WARP_MMA) return MLA_ERR_INVALID_VALUE;
  g_decode_kernel.store(kernel, std::memory_order_relaxed);
  return MLA_OK;
}

const char* mla_status_string(mla_status_t s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_VALUE: return "MLA_ERR_INVALID_VALUE";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_MISALIGNED: return "MLA_ERR_MISALIGNED";
    case MLA_ERR_WORKSPACE_TOO_SMALL: return "MLA_ERR_WORKSPACE_TOO_SMALL";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_DEVICE_TIMEOUT: return "MLA_ERR_DEVICE_TIMEOUT";
    case MLA_ERR_BAD_BLOCK_TABLE: return "MLA_ERR_BAD_BLOCK_TABLE";
    case MLA_ERR_BAD_SEQ_LEN: return "MLA_ERR_BAD_SEQ_LEN";
  }
  return "MLA_ERR_UNKNOWN";
}

}  // extern "C"
