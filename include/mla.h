/*
 * mla.h — C ABI of the B200 (sm_100a) MLA decode library.
 *
 * Multi-Head Latent Attention decode over a paged latent KV cache.  Every cached
 * token holds one latent c (d_c = 512 values) followed by a decoupled RoPE key
 * k_pe (d_r = 64 values), shared by all heads: the 576-value record worked
 * out in snowgate forum thread 35 (replies on the KV-cache arithmetic).  Keys
 * and values are up-projections of the latent, k = W_UK c and
 * v = W_UV c ("MLA: Multi-Head Latent Attention — DeepSeek-AI Explained",
 * section "Architecture"); decode never forms them, it folds W_UK into the query
 * and W_UV into the output (nnets.ru article, section "Суть MLA", the weight
 * absorbing trick).  One decode step is four calls, in order:
 *
 *   mla_absorb_q       q_lat = W_UK^T q_nope                 (per head)
 *   mla_decode_paged   scores, online softmax, o_lat = P c   (split-KV partials)
 *   mla_combine_splits log-sum-exp merge of the partials     (no-op when none)
 *   mla_up_proj_v      o = W_UV o_lat                         (per head)
 * and mla_write_kv appends new tokens (latent, RoPE key, bf16 or e4m3) to the
 * cache before the decode that reads them.
 *
 * Conventions for every entry point:
 *  - Pointers are DEVICE pointers unless a field says otherwise; the caller owns
 *    every buffer.  The library allocates nothing, frees nothing and keeps no
 *    pointer after a call returns.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL means the legacy default
 *    stream) and the call returns without waiting, except mla_get_status.
 *  - Tensors are dense and row-major in the index order written; bf16 is
 *    bfloat16, e4m3 is OCP float8 e4m3fn.
 *  - Calls return a status and never throw or abort.  Argument errors are found
 *    on the host before anything is enqueued; problems that only the device can
 *    see (a page id outside the cache, a length beyond the block table) are
 *    recorded in the workspace's status word and read by mla_get_status.
 *  - The library is built for sm_100a only; on another device the launch fails
 *    and MLA_ERR_CUDA is returned.
 *  - Kernels are launched with programmatic dependent launch: one may start while
 *    the previous kernel on the stream is still running, and waits for it before
 *    reading anything that kernel may write.  mla_decode_paged reads the cache,
 *    block table and lengths before that wait, so these must not be written by a
 *    kernel that lets its dependents start early (no kernel of this library
 *    that writes them does; a kernel that never signals an early start, the
 *    default, and copies are safe).
 */
#ifndef MLA_B200_H
#define MLA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_VALUE = 1,        /* null pointer, negative or inconsistent size */
  MLA_ERR_UNSUPPORTED = 2,          /* a dimension the library does not handle */
  MLA_ERR_MISALIGNED = 3,           /* a pointer is not 16-byte aligned */
  MLA_ERR_WORKSPACE_TOO_SMALL = 4,  /* workspace_bytes below the matching *_workspace_size() */
  MLA_ERR_CUDA = 5,                 /* a CUDA runtime call or launch failed */
  MLA_ERR_DEVICE_TIMEOUT = 6,       /* a bounded device wait ran out (device-side) */
  MLA_ERR_BAD_BLOCK_TABLE = 7,      /* a block-table entry outside [0, num_pages) (device-side) */
  MLA_ERR_BAD_SEQ_LEN = 8           /* seq_lens[b] < 0 or > max_pages_per_seq*page_size (device-side) */
} mla_status_t;

/* Cache formats of a 576-value row: bf16 values; e4m3 codes with one fp32 scale
 * per row (value = code * scale); q8_0 int8 codes with one fp16 scale per block
 * of 32 consecutive values (value = code * block scale, 18 blocks a row); q4_0
 * the same with codes in [-7, 7], each stored as the 4-bit number code + 8, value
 * 2j of the row in the low four bits of byte j and value 2j + 1 in the high four
 * (288 bytes a row).  q8_0 and q4_0 follow ik_llama.cpp docs "FlashMLA", section
 * "KV cache with MLA" (q8_0 the recommended MLA cache; below 6 bits a Hadamard
 * rotation, see mla_fold_hadamard). */
typedef enum { MLA_KV_BF16 = 0, MLA_KV_FP8_E4M3 = 1, MLA_KV_Q8_0 = 2, MLA_KV_Q4_0 = 3 } mla_kv_dtype_t;

/* Supported dimensions: d_c = 512, d_r = 64, d_n = d_v = 128, page_size = 64,
 * H a multiple of 16 up to 128, 1 <= s_q <= MLA_MAX_S_Q.  s_q > 1 covers
 * speculative decoding and chunked prefill in the absorbed form: every query
 * token is computed like a decode query (causal among the new tokens when
 * `causal` is set). */
#define MLA_D_C 512
#define MLA_D_R 64
#define MLA_D_QK_NOPE 128
#define MLA_D_V 128
#define MLA_PAGE_SIZE 64
#define MLA_MAX_SPLITS 128
#define MLA_MAX_S_Q 1024

/*
 * mla_absorb_q — weight absorption of the query (nnets.ru article, section
 * "Суть MLA"; snowgate thread 35, the reply on folding W_UK into the query).
 *   q_lat[t][h][c] = sum_n q_nope[t][h][n] * w_uk[h][n][c]
 * q_nope : bf16 [n_tok][H][d_n]        (n_tok = B * s_q, token t = b * s_q + i)
 * w_uk   : bf16 [H][d_n][d_c]          (k = W_UK[h] c, so W_UK[h] is d_n x d_c)
 * q_lat  : bf16 [n_tok][H][d_c]        (written; fp32 accumulation, rounded once)
 * d_n must be 128 and d_c 512.  n_tok = 0 enqueues nothing and returns MLA_OK.
 */
mla_status_t mla_absorb_q(const void* q_nope, const void* w_uk, void* q_lat,
                          int32_t n_tok, int32_t H, int32_t d_n, int32_t d_c, void* stream);

/*
 * Arguments of mla_decode_paged / mla_combine_splits / mla_decode_workspace_size.
 * Zero-initialise the struct, then fill every field.
 */
typedef struct {
  const void* q_lat;              /* bf16 [B][s_q][H][d_c], output of mla_absorb_q */
  const void* q_pe;               /* bf16 [B][s_q][H][d_r], RoPE already applied */
  const void* kv_cache;           /* [num_pages][page_size][d_c + d_r]: row = c || k_pe,
                                     bf16 (MLA_KV_BF16), e4m3 (MLA_KV_FP8_E4M3) or int8
                                     (MLA_KV_Q8_0); q4_0: [num_pages][page_size][288] bytes */
  const void* kv_scale;           /* e4m3: fp32 [num_pages][page_size], the scale of the whole
                                     row; q8_0, q4_0: fp16 [num_pages][page_size][18], the scale
                                     of each 32-value block, 4-byte aligned (q4_0: 16-byte
                                     aligned); NULL for bf16 */
  const int32_t* block_table;     /* int32 [B][max_pages_per_seq]: physical page of each
                                     64-token logical page */
  const int32_t* seq_lens;        /* int32 [B], device: cached tokens of sequence b, including
                                     its s_q new tokens */
  void* o_lat;                    /* bf16 [B][s_q][H][d_c], written (latent-space output) */
  float* lse;                     /* fp32 [B][s_q][H], natural-log partition function,
                                     written; may be NULL */
  void* workspace;                /* device scratch, >= mla_decode_workspace_size() bytes,
                                     16-byte aligned; its first 16 bytes must be zero before the
                                     first use (they hold the sticky status word) */
  size_t workspace_bytes;
  int32_t B, s_q, H;
  int32_t d_c, d_r, page_size;
  int32_t num_pages;              /* physical pages in kv_cache */
  int32_t max_pages_per_seq;      /* row length of block_table */
  int32_t kv_dtype;               /* mla_kv_dtype_t */
  int32_t causal;                 /* 1: query i of sequence b sees tokens 0 .. L_b - s_q + i */
  int32_t num_splits;             /* 0 = choose automatically; else 1 .. MLA_MAX_SPLITS */
  int32_t max_seq_len;            /* host-known upper bound of seq_lens (0 = use
                                     max_pages_per_seq * page_size); only steers the split count */
  float softmax_scale;            /* e.g. 1/sqrt(d_n + d_r) */
} mla_decode_args_t;

/* Bytes of workspace mla_decode_paged needs for these arguments (host only, no
 * device access).  Depends on B, s_q, H and the split count that will be used. */
mla_status_t mla_decode_workspace_size(const mla_decode_args_t* args, size_t* bytes);

/* The split count mla_decode_paged will use for these arguments (host only):
 * args->num_splits when it is set, else the count that minimises a model of the
 * kernel's makespan on this device's SMs. */
mla_status_t mla_decode_num_splits(const mla_decode_args_t* args, int32_t* num_splits);

/*
 * mla_decode_paged — latent attention over the paged cache (the absorbed form of
 * softmax attention; FlashAttention-style on-chip tiles with an online softmax,
 * nnets.ru article, section "MLA и FlashAttention").  For query i of sequence b,
 * head h and visible token j (j < L_b, or j <= L_b - s_q + i when causal):
 *   s_j   = softmax_scale * (q_lat . c_j + q_pe . k_pe_j)
 *   o_lat = sum_j softmax(s)_j c_j ,   lse = log sum_j exp(s_j)
 * Token j is row j % page_size of page block_table[b][j / page_size].  Rows of a
 * last page at positions >= L_b are read but weigh nothing, whatever they hold.
 * With one split the results go straight to o_lat / lse; with more, fp32
 * partials go to the workspace.  Always follow with mla_combine_splits on the
 * same stream (it enqueues nothing when one split was used).  A query with no
 * visible token gets o_lat = 0 and lse = -inf.
 */
mla_status_t mla_decode_paged(const mla_decode_args_t* args, void* stream);

/*
 * mla_combine_splits — merges split-KV partials (flash-decoding):
 *   lse = log sum_s exp(lse_s),  o_lat = sum_s exp(lse_s - lse) o_s
 * Reads the workspace written by mla_decode_paged with the same args; writes
 * o_lat (bf16) and lse.  Returns MLA_OK without enqueuing work when one split
 * was used.
 */
mla_status_t mla_combine_splits(const mla_decode_args_t* args, void* stream);

/*
 * mla_up_proj_v — value up-projection on the output side ("Architecture":
 * v = W_UV c; absorbed, o = W_UV o_lat).
 *   out[t][h][v] = sum_c w_uv[h][v][c] * o_lat[t][h][c]
 * o_lat : bf16 [n_tok][H][d_c];  w_uv : bf16 [H][d_v][d_c];  out : bf16 [n_tok][H][d_v]
 * d_v must be 128 and d_c 512.
 */
mla_status_t mla_up_proj_v(const void* o_lat, const void* w_uv, void* out,
                           int32_t n_tok, int32_t H, int32_t d_v, int32_t d_c, void* stream);

/*
 * mla_decode_paged_noalloc — mla_decode_paged followed by mla_combine_splits,
 * for callers that cannot allocate device memory (for example a plugin inside
 * an engine that owns all device memory and forbids allocations after start-up,
 * or a latency-critical path where an allocation could synchronise the device).
 * The pages describe no such entry point; it is a deployment convenience.
 * It ignores args->workspace and uses a scratch array built into the library
 * instead: 16 MiB of device memory on every GPU that loads the library, held
 * until the process exits.  A problem needing more scratch than that (see
 * mla_decode_workspace_size) is rejected with MLA_ERR_WORKSPACE_TOO_SMALL
 * before anything is enqueued.  The first use on a device looks up the
 * array's device address (cudaGetSymbolAddress) and clears its status word;
 * under CUDA's lazy module loading that lookup may be the moment the driver
 * loads the library's device code and backs the array, so make it during
 * start-up, before any allocation freeze or stream capture: call
 * mla_noalloc_init once per device (or make a first decode call then).
 * Every call shares the array: calls that overlap on the GPU race, so order
 * them on one stream or with events.  The call allocates nothing.  Problems
 * only the device sees (a page id outside the cache, a length beyond the block
 * table, a wait that ran out) go to the array's sticky status word, read and
 * cleared by mla_get_status_noalloc.
 */
mla_status_t mla_decode_paged_noalloc(const mla_decode_args_t* args, void* stream);

/* Set-up of mla_decode_paged_noalloc's built-in scratch on the current device:
 * looks up its device address and zeroes its status word (synchronously).
 * Idempotent; call it at start-up on every device that will decode without a
 * workspace. */
mla_status_t mla_noalloc_init(void);

/* Waits for `stream`, returns the sticky device status word of the built-in
 * scratch of the current device (MLA_OK if mla_decode_paged_noalloc recorded no
 * device-side problem since the last read) and clears it. */
mla_status_t mla_get_status_noalloc(void* stream);

/*
 * Arguments of mla_write_kv / mla_write_kv_workspace_size.
 * Zero-initialise the struct, then fill every field.
 */
typedef struct {
  const void* h;                  /* bf16 [n_tok][d_h]: hidden states of the new tokens,
                                     n_tok = B * s_q, token t = b * s_q + i */
  const void* w_dkv;              /* bf16 [d_c + d_r][d_h]: rows 0 .. d_c-1 are W_DKV, rows
                                     d_c .. d_c+d_r-1 the RoPE key's projection W_KR */
  void* kv_cache;                 /* [num_pages][page_size][d_c + d_r], bf16, e4m3 or q8_0
                                     codes, or [num_pages][page_size][288] q4_0 bytes; only the
                                     new tokens' rows are written */
  void* kv_scale;                 /* written at the new rows: e4m3: fp32 [num_pages][page_size];
                                     q8_0, q4_0: fp16 [num_pages][page_size][18]; NULL for bf16 */
  const int32_t* block_table;     /* int32 [B][max_pages_per_seq]: physical page of each
                                     64-token logical page */
  const int32_t* seq_lens;        /* int32 [B], device: lengths including the s_q new tokens */
  void* workspace;                /* device scratch, >= mla_write_kv_workspace_size() bytes,
                                     16-byte aligned; its first 16 bytes must be zero before the
                                     first use (they hold the sticky status word) */
  size_t workspace_bytes;
  int32_t B, s_q;
  int32_t d_h;                    /* hidden width, a positive multiple of 64 */
  int32_t d_c, d_r, page_size;
  int32_t num_pages;              /* physical pages in kv_cache */
  int32_t max_pages_per_seq;      /* row length of block_table */
  int32_t kv_dtype;               /* mla_kv_dtype_t */
  float rope_base;                /* RoPE frequency base, e.g. 10000 */
} mla_write_kv_args_t;

/* Bytes of workspace mla_write_kv needs for these arguments (host only). */
mla_status_t mla_write_kv_workspace_size(const mla_write_kv_args_t* args, size_t* bytes);

/*
 * mla_write_kv — appends the s_q new tokens of every sequence to the paged
 * cache.  The latent is the down-projection c = W_DKV h ("MLA: Multi-Head Latent
 * Attention — DeepSeek-AI Explained", section "Architecture"); beside it goes the
 * decoupled RoPE key k_pe = RoPE(W_KR h, pos) of the 576-value record (snowgate
 * thread 35).  RoPE turns value pair (2i, 2i+1) of the key by the angle
 * pos * rope_base^(-2i/d_r).  New token i of sequence b sits at position
 * pos = L_b - s_q + i: row pos % page_size of page block_table[b][pos / page_size].
 * bf16 cache: each value rounded to nearest even.  e4m3 cache (ik_llama.cpp docs
 * "FlashMLA", "KV cache with MLA": the latent cache may be quantised): one fp32
 * scale per 576-value row, scale = amax / 448 (1 for an all-zero row), codes =
 * the fp32 quotients value / scale rounded to nearest even, saturated at +-448.
 * q8_0 cache (the format those docs recommend): per block of 32 values, d =
 * amax / 127 (computed in fp32) rounded to fp16, codes = the fp32 quotients
 * value / d rounded to nearest even, clamped to +-127 (0 for an all-zero block).
 * q4_0 cache: the same with d = amax / 7 and codes clamped to +-7, packed two
 * to a byte as the cache format above states.
 * The projections accumulate in fp32.  No other cache row is touched.  A length
 * below s_q or beyond the block table (MLA_ERR_BAD_SEQ_LEN) or a page id outside
 * the cache (MLA_ERR_BAD_BLOCK_TABLE) is recorded in the workspace's status word
 * and that token is skipped.  Order this call before the decode that reads the
 * rows, on the same stream: kernels enqueued after it start only once it has
 * completed (it gives no early start to programmatic dependent launches).
 */
mla_status_t mla_write_kv(const mla_write_kv_args_t* args, void* stream);

/*
 * Arguments of mla_prefill / mla_prefill_workspace_size.
 * Zero-initialise the struct, then fill every field.
 */
typedef struct {
  const void* q_nope;             /* bf16 [B][s_q][H][d_n] */
  const void* q_pe;               /* bf16 [B][s_q][H][d_r], RoPE already applied */
  const void* w_uk;               /* bf16 [H][d_n][d_c] (k = W_UK[h] c) */
  const void* w_uv;               /* bf16 [H][d_v][d_c] (v = W_UV[h] c) */
  const void* kv_cache;           /* bf16 [num_pages][page_size][d_c + d_r]: row = c || k_pe */
  const int32_t* block_table;     /* int32 [B][max_pages_per_seq] */
  const int32_t* seq_lens;        /* int32 [B], device: cached tokens including the s_q new ones */
  void* out;                      /* bf16 [B][s_q][H][d_v], written */
  float* lse;                     /* fp32 [B][s_q][H], natural log, written; may be NULL */
  void* workspace;                /* device scratch, >= mla_prefill_workspace_size() bytes,
                                     16-byte aligned; its first 16 bytes must be zero before the
                                     first use (they hold the sticky status word) */
  size_t workspace_bytes;
  int32_t B, s_q, H;
  int32_t d_c, d_r, page_size;
  int32_t num_pages;              /* physical pages in kv_cache */
  int32_t max_pages_per_seq;      /* row length of block_table */
  int32_t kv_dtype;               /* MLA_KV_BF16 only */
  int32_t causal;                 /* 1: query i of sequence b sees tokens 0 .. L_b - s_q + i */
  int32_t max_seq_len;            /* host-known upper bound of seq_lens, >= s_q (sizes the
                                     workspace; a longer sequence is MLA_ERR_BAD_SEQ_LEN) */
  float softmax_scale;
} mla_prefill_args_t;

/* Bytes of workspace mla_prefill needs (host only): 256 plus the per-head keys
 * and values of every sequence, 2 * B * H * roundup(max_seq_len, 256) * 128 bf16. */
mla_status_t mla_prefill_workspace_size(const mla_prefill_args_t* args, size_t* bytes);

/*
 * mla_prefill — attention of many new tokens per sequence in the explicit form
 * ("MLA: Multi-Head Latent Attention — DeepSeek-AI Explained", section
 * "Architecture": k = [W_UK c ; k_pe], v = W_UV c per head).  Prefill is bound
 * by compute, not by the cache (snowgate thread 35, the reply on prefill), and
 * beyond about 170 queries per sequence forming K and V once costs fewer FLOPs
 * than the absorbed form's 576 + 512 products per query and token.  Two kernels:
 * the per-head keys and values of every cached token (bf16, into the
 * workspace), then a FlashAttention forward with an online softmax over them.
 * For query i of sequence b, head h and visible token j:
 *   s_j = softmax_scale * ([q_nope ; q_pe] . [W_UK[h] c_j ; k_pe_j])
 *   out = sum_j softmax(s)_j W_UV[h] c_j ,   lse = log sum_j exp(s_j)
 * The result equals mla_absorb_q + mla_decode_paged + mla_combine_splits +
 * mla_up_proj_v up to rounding (K and V are rounded to bf16 here, q_lat and
 * o_lat there).  H 1 .. 128, 1 <= s_q <= max_seq_len, bf16 cache only.  A
 * length below s_q or above max_seq_len or the block table (MLA_ERR_BAD_SEQ_LEN;
 * that sequence's outputs are zero, lse -inf) or a page id outside the cache
 * (MLA_ERR_BAD_BLOCK_TABLE) goes to the workspace's status word.
 */
mla_status_t mla_prefill(const mla_prefill_args_t* args, void* stream);

/*
 * Arguments of mla_decode_step / mla_decode_step_workspace_size /
 * mla_decode_step_launches: the whole decode step from the query's two parts to
 * the output.  Zero-initialise the struct, then fill every field.
 */
typedef struct {
  const void* q_nope;             /* bf16 [B][s_q][H][d_n] */
  const void* q_pe;               /* bf16 [B][s_q][H][d_r], RoPE already applied */
  const void* w_uk;               /* bf16 [H][d_n][d_c] */
  const void* w_uv;               /* bf16 [H][d_v][d_c] */
  const void* kv_cache;           /* as in mla_decode_args_t */
  const void* kv_scale;           /* as in mla_decode_args_t */
  const int32_t* block_table;     /* int32 [B][max_pages_per_seq] */
  const int32_t* seq_lens;        /* int32 [B], device, including the s_q new tokens */
  void* out;                      /* bf16 [B][s_q][H][d_v], written */
  float* lse;                     /* fp32 [B][s_q][H], natural log, written; may be NULL */
  void* workspace;                /* device scratch, >= mla_decode_step_workspace_size() bytes,
                                     16-byte aligned, zero before the first use (its first 16
                                     bytes hold the sticky status word; it also holds q_lat,
                                     o_lat and the step's flags) */
  size_t workspace_bytes;
  int32_t B, s_q, H;
  int32_t d_c, d_r, page_size;
  int32_t num_pages;
  int32_t max_pages_per_seq;
  int32_t kv_dtype;               /* mla_kv_dtype_t */
  int32_t causal;
  int32_t num_splits;             /* 0 = automatic, as for mla_decode_paged */
  int32_t max_seq_len;
  float softmax_scale;
  int32_t fuse;                   /* 0: one launch where it measured faster (a q8_0 or q4_0
                                     cache whose grid covers at least half the SMs); 1: one
                                     launch wherever the shape allows it; -1: never */
} mla_step_args_t;

/* Bytes of workspace mla_decode_step needs (host only). */
mla_status_t mla_decode_step_workspace_size(const mla_step_args_t* args, size_t* bytes);

/* Kernel launches mla_decode_step makes for these arguments (host only): 1 when
 * the step runs fused, else 3 (one split) or 4. */
mla_status_t mla_decode_step_launches(const mla_step_args_t* args, int32_t* launches);

/*
 * mla_decode_step — the decode step in one call: o = W_UV attention(W_UK^T
 * q_nope, q_pe; cache), the same function as mla_absorb_q, mla_decode_paged,
 * mla_combine_splits and mla_up_proj_v in sequence (snowgate thread 35: a
 * fused dequantise-and-multiply decode; nnets.ru article, section "Суть MLA",
 * for the absorbed form).  With a bf16, q8_0 or q4_0 cache, one split and at
 * most one query token per CTA pair the device holds at once, it can be one
 * launch (see `fuse`): every CTA first takes a
 * share of the query absorption (so W_UK is read once per 64 query tokens,
 * not once per token), decodes its unit once the absorption tiles of its
 * tokens are written, then takes a share of the up-projection once the decode
 * rows it needs are written (flags in the workspace; every wait bounded, a
 * wait that runs out records MLA_ERR_DEVICE_TIMEOUT).  Otherwise it enqueues
 * the four kernels above on `stream`.  Results are identical either way.  After
 * a recorded device timeout, zero the workspace before the next call.
 */
mla_status_t mla_decode_step(const mla_step_args_t* args, void* stream);

/*
 * mla_fold_hadamard — folds the Hadamard rotation of the latent space into the
 * weights, in place (ik_llama.cpp docs "FlashMLA", section "KV cache with MLA":
 * below 6 bits a Hadamard transform of the cache before quantisation recovers
 * quality).  With H the orthonormal Sylvester-Hadamard matrix of size d_c = 512
 * (entries +-2^-4.5, symmetric, H H = I):
 *   w_dkv : bf16 [d_c + d_r][d_h]; its first 512 rows W_DKV become H W_DKV (each
 *           column transformed), so mla_write_kv stores the rotated latent H c;
 *           the d_r RoPE rows are left as they are
 *   w_uk  : bf16 [H_heads][d_n][d_c]; every row becomes row * H (W_UK[h] H)
 *   w_uv  : bf16 [H_heads][d_v][d_c]; every row becomes row * H (W_UV[h] H)
 * Attention over the rotated cache with the folded weights equals attention
 * over the plain cache with the plain weights (H is orthonormal), and the
 * rotation spreads a large latent channel over every block of 32, which is
 * what a blockwise 4-bit cache needs.  Each vector is transformed in fp32 and
 * rounded once to bf16.  Any of the three pointers may be NULL (skipped);
 * pointers 16-byte aligned; d_h a positive multiple of 64 when w_dkv is given;
 * H_heads 0 .. 128 (d_n = d_v = 128).  Folding twice restores the weights up
 * to bf16 rounding.  Apply it once, before the weights are used.
 */
mla_status_t mla_fold_hadamard(void* w_dkv, int32_t d_h, void* w_uk, void* w_uv, int32_t H, void* stream);

/* Waits for `stream`, returns the sticky device status word of `workspace`
 * (MLA_OK if no device-side problem was recorded) and clears it. */
mla_status_t mla_get_status(void* workspace, void* stream);

/* Which decode kernel mla_decode_paged runs, process-wide.  MLA_DECODE_AUTO
 * (the default) picks the tensor-memory (tcgen05) kernel for every shape it
 * takes and the warp-MMA kernel otherwise; MLA_DECODE_WARP_MMA forces the
 * latter (a cross-check for tests and diagnosis).  Takes effect for calls made
 * after it returns; a CUDA graph keeps the kernels it captured. */
typedef enum { MLA_DECODE_AUTO = 0, MLA_DECODE_WARP_MMA = 1 } mla_decode_kernel_t;
mla_status_t mla_set_decode_kernel(int32_t kernel);

/* Limit, in nanoseconds, of every bounded wait inside the decode kernels
 * (process-wide; 0 restores the default of 2 s).  A wait that runs out records
 * MLA_ERR_DEVICE_TIMEOUT in the status word, and the kernel waits for its copies
 * in flight, frees its tensor memory and returns, leaving the context usable.
 * Takes effect for launches after it returns (a CUDA graph keeps the limit it
 * captured).  A limit of 1 ns gives up at the first wait that a non-blocking
 * test finds unsatisfied (the device clock may advance in steps much coarser
 * than 1 ns).
 * Meant for tests and diagnosis; the default suits every workload. */
mla_status_t mla_set_device_wait_limit(uint64_t ns);

/* Human-readable name of a status code (static storage). */
const char* mla_status_string(mla_status_t status);

#ifdef __cplusplus
}
#endif
#endif /* MLA_B200_H */
