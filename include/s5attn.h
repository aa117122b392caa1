/*
 * s5attn.h - C ABI of the B200 (sm_100a) sparse / sliding-window GQA library.
 *
 * The library computes the attention hot path of the Step 5 Preview hybrid
 * attention layers:
 *
 *   sparse full-attention layer  (SGLang day-0 blog "Step 5 Preview: Day-0
 *     Inference and RL Support with SGLang and Miles", section "Hybrid
 *     Attention"; StepFun open-weights blog, section "What the config says"):
 *     every block of 8 history tokens carries a 256-wide key that an
 *     indexer rates against the query; the 512 best-rated blocks and the
 *     block holding the query are the only tokens its grouped-query
 *     attention (64 query heads over 4 KV groups, dimension 192) reads;
 *   sliding-window layer (same sections): causal GQA limited to a window of
 *     512 positions ending at the query.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers.  Every tensor pointer is DEVICE memory owned by the caller; the
 *   library never allocates, frees or takes ownership, and never keeps a
 *   pointer after the call returns.  Descriptors are HOST structs read during
 *   the call only.
 * Streams.  Work is enqueued on `stream` (a cudaStream_t; NULL = legacy
 *   default stream) and the call returns without synchronising, except
 *   s5_get_device_error.  No entry point allocates or synchronises, so the
 *   compute calls can be captured into a CUDA graph.
 * Layouts.  All layouts are dense, row-major, little-endian; bf16 is IEEE
 *   bfloat16.
 *     K / V pool      bf16 [num_pages][4 kv groups][64 tokens][192]
 *                     (one 8-token block of one group = 3,072 contiguous bytes)
 *     index-key pool  bf16 [num_pages][8 blocks][256]: slot j of the page that
 *                     holds logical page P of a sequence is the key of block
 *                     8P + j (shares the sparse layer's page table)
 *     page table      int32 [batch][max_pages]; logical page P of sequence s
 *                     lives in physical page page_table[s][P]
 *     q               bf16 [total_q][64][192]; head h reads KV group h / 16
 *     q_index         bf16 [total_q][256]
 *     sel             int32 [total_q][topk]
 *     out             bf16 [total_q][64][192];  lse fp32 [total_q][64]
 * Batches.  Sequence s has ctx_lens[s] cached tokens followed by
 *   cu_q[s+1] - cu_q[s] new query tokens whose K/V are ALREADY in the pools;
 *   query row r of sequence s sits at absolute position
 *   t = ctx_lens[s] + (r - cu_q[s]).  Its current block is c = t / 8 and its
 *   history blocks are 0 .. c-1.
 * Errors.  Argument checks run on the host before anything is enqueued and
 *   return S5_ERR_INVALID_ARG / S5_ERR_UNSUPPORTED / S5_ERR_WORKSPACE with
 *   nothing enqueued.  Launch failures return S5_ERR_CUDA.  Faults in device
 *   data (a page id, block id, length or count out of range) never trap: the
 *   kernel records the first one in the workspace error record, skips the
 *   offending access and continues; read it with s5_get_device_error.  Every
 *   wait inside a kernel is bounded; a wait that runs out records
 *   S5_ERR_TIMEOUT.
 * Determinism.  Results are bit-identical run to run for identical inputs
 *   and launch configuration (fixed reduction orders, no atomics on data).
 */
#ifndef S5ATTN_H
#define S5ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *s5_stream_t; /* identical to cudaStream_t */

typedef enum {
  S5_OK = 0,
  S5_ERR_INVALID_ARG = 1,   /* bad pointer, size or descriptor field            */
  S5_ERR_UNSUPPORTED = 2,   /* valid request outside what this build implements */
  S5_ERR_CUDA = 3,          /* a CUDA launch or runtime call failed             */
  S5_ERR_DEVICE_BOUNDS = 4, /* device data out of range (recorded by a kernel)  */
  S5_ERR_TIMEOUT = 5,       /* a bounded in-kernel wait expired                 */
  S5_ERR_WORKSPACE = 6      /* workspace missing or smaller than required       */
} s5_status;

/* Geometry compiled into this build (StepFun open-weights blog, "What the
 * config says"; SGLang day-0 blog, "Get Started": --page-size 64). */
#define S5_N_HEADS 64
#define S5_N_KV_HEADS 4
#define S5_HEAD_DIM 192
#define S5_PAGE_SIZE 64
#define S5_BLOCK_SIZE 8
#define S5_INDEX_DIM 256
#define S5_MAX_TOPK 512
#define S5_MAX_LEN (1 << 21) /* longest sequence (cached + new tokens) */

/* ABI version (major * 100 + minor): 1.01 added the cache append, the
 * per-KV-group entry points and the one-byte-key indexer; 1.02 the sparse
 * attention over one-byte KV and its cache append. */
#define S5_ABI_VERSION 102

/* One attention layer's paged KV cache. */
typedef struct {
  const void *k_pool;  /* device bf16 [num_pages][4][64][192], 16-byte aligned */
  const void *v_pool;  /* device bf16, same shape                               */
  int32_t num_pages;   /* >= 1                                                  */
  int32_t page_size;   /* must be S5_PAGE_SIZE                                  */
  int32_t n_kv_heads;  /* must be S5_N_KV_HEADS                                 */
  int32_t head_dim;    /* must be S5_HEAD_DIM                                   */
} s5_kv_desc;

/* The sparse layer's block-key pool (same pages as its KV pool). */
typedef struct {
  const void *key_pool; /* device bf16 [num_pages][8][256], 16-byte aligned */
  int32_t num_pages;
  int32_t index_dim;    /* must be S5_INDEX_DIM */
} s5_index_desc;

/* A varlen batch and its page table. */
typedef struct {
  const int32_t *page_table; /* device int32 [batch][max_pages]                      */
  const int32_t *ctx_lens;   /* device int32 [batch]: cached tokens before new queries */
  const int32_t *cu_q;       /* device int32 [batch+1]: query-row offsets, cu_q[0]=0   */
  int32_t batch;             /* >= 1                                                  */
  int32_t max_pages;         /* row stride of page_table                              */
  int32_t total_q;           /* cu_q[batch]; 0 is allowed (nothing is enqueued)       */
  int32_t max_q;             /* upper bound on new tokens of any sequence             */
  int32_t max_len;           /* upper bound on ctx_lens[s] + new tokens, <= S5_MAX_LEN */
} s5_batch_desc;

/* Bytes of device workspace any of the calls below may use for this batch
 * (window: the largest sliding window that will be requested, or 0).  The
 * first S5_WS_FIXED_BYTES bytes hold the device error record and the
 * attention partition counters: zero them once before first use (or call
 * s5_reset_device_error); every call leaves the counters at zero again.  The
 * rest is per-call scratch with no state between calls.  Calls that share a
 * workspace must be ordered (one stream). */
#define S5_WS_FIXED_BYTES (256 + 16384)
/* Test hook for the bounded waits (not for normal use): a nonzero unsigned
 * 64-bit count of nanoseconds stored at this byte offset of a workspace makes
 * every CTA of the per-row attention kernel (s5_sparse_gqa_attn decode rows,
 * s5_sparse_gqa_attn_grouped, s5_sparse_gqa_attn_fp8kv, s5_swa_gqa_attn)
 * wait that long, after its first block copies land, on a barrier that nothing
 * arrives on, and then take the expired-wait path: it records S5_ERR_TIMEOUT,
 * waits (bounded) for its copies still in flight and returns with zero output
 * for its unit.  Zeroing the workspace or s5_reset_device_error clears it. */
#define S5_WS_TEST_STALL_OFFSET 64
s5_status s5_workspace_size(const s5_batch_desc *batch, int32_t window, size_t *bytes);

/* Indexer: score every history block of every query row and keep the best
 * `topk` (SGLang day-0 blog, "Kernels from StepFun": indexer scoring against
 * the compressed history in the paged cache; "Hybrid Attention": up to 512
 * historical blocks).
 *   score(r, b) = sum_d q_index[r][d] * key(s, b)[d]  for b < c(r), in fp32
 *   (exact for integer-valued inputs; otherwise a fixed summation order).
 * The indexer query is a per-token 256-dim input shared by all heads: the
 * pages fix only the key side, so this is an assumption of the API.
 * Selection: the `topk` best blocks by (score descending, block index
 * ascending); all c blocks when c <= topk.  Written to sel[r][0..n-1] in
 * ascending block order, sel[r][n..topk-1] = -1, sel_count[r] = n.
 * topk in [1, 512].  sel / sel_count are device int32.  At most 65,535
 * sequences per batch (S5_ERR_UNSUPPORTED otherwise; also for the sparse
 * attention of multi-token batches). */
s5_status s5_index_score_topk(const s5_index_desc *index, const s5_batch_desc *batch,
                              const void *q_index, int32_t topk, int32_t *sel,
                              int32_t *sel_count, void *workspace, size_t workspace_bytes,
                              s5_stream_t stream);

/* Sparse gathered GQA (SGLang day-0 blog, "Hybrid Attention" and "Kernels
 * from StepFun": attention over the selected blocks plus the current block;
 * long selections are split into partitions whose partial results are
 * merged).  For row r at position t and head h (group g = h / 16):
 *   T   = union of tokens 8b..8b+7 over b in sel[r][0..sel_count[r]-1],
 *         plus tokens 8c..t of the current block c = t / 8
 *   out = sum_{j in T} softmax_j(sm_scale * q[r][h] . K[j][g]) V[j][g]
 *   lse = log sum_{j in T} exp(sm_scale * q[r][h] . K[j][g])   (may be NULL)
 * sel entries may come in any order; -1 entries past sel_count are ignored.
 * sel_count[r] <= min(topk, c); entries must be distinct blocks < c. */
s5_status s5_sparse_gqa_attn(const s5_kv_desc *kv, const s5_batch_desc *batch,
                             const void *q, const int32_t *sel, const int32_t *sel_count,
                             int32_t topk, float sm_scale, void *out, float *lse,
                             void *workspace, size_t workspace_bytes, s5_stream_t stream);

/* Sliding-window GQA (SGLang day-0 blog, "Hybrid Attention": the layers
 * between sparse layers see a 512-token window).  T = positions
 * max(0, t - window + 1) .. t; otherwise as s5_sparse_gqa_attn.  Pages that
 * hold no position of any window are never read, so a sliding-window pool
 * may leave them unmapped (-1). */
s5_status s5_swa_gqa_attn(const s5_kv_desc *kv, const s5_batch_desc *batch, const void *q,
                          int32_t window, float sm_scale, void *out, float *lse,
                          void *workspace, size_t workspace_bytes, s5_stream_t stream);

/* s5_index_score_topk with one-byte block keys (StepFun open-weights blog,
 * "What sparse attention does and doesn't save": the indexer read at one or
 * two bytes per key value).  index->key_pool holds E4M3 codes, uint8
 * [num_pages][8][256] (the 8-bit float of the OCP FP8 specification: bias 7,
 * 3 mantissa bits, no infinities), 16-byte aligned; each code stands for its
 * exact value, and scores, selection and results are defined as for
 * s5_index_score_topk on those values (the same for keys that are exactly
 * representable in E4M3).  The indexer reads half the bytes.  The workspace
 * of s5_workspace_size covers this call. */
s5_status s5_index_score_topk_fp8(const s5_index_desc *index, const s5_batch_desc *batch, const void *q_index,
                                  int32_t topk, int32_t *sel, int32_t *sel_count, void *workspace,
                                  size_t workspace_bytes, s5_stream_t stream);

/* Sparse gathered GQA over one-byte KV (StepFun open-weights blog, "Fitting
 * it on a node": the full-attention layers' KV cache can be held in FP8, a
 * lossy format to be re-checked).  kv->k_pool / kv->v_pool hold E4M3 codes,
 * uint8 [num_pages][4][64][192] (one block of one group = 1,536 contiguous
 * bytes), 16-byte aligned; a K code stands for k_scale * E4M3(code) and a V
 * code for v_scale * E4M3(code) (E4M3: the 8-bit float of the OCP FP8
 * specification, bias 7, 3 mantissa bits, no infinities).  With those values
 * the result is defined exactly as for s5_sparse_gqa_attn; every row takes
 * the per-row kernel.  Products run on f16 tensor cores: every E4M3 value is
 * an f16 value, and q is rounded to f16 (exact for bf16 values of magnitude
 * 2^-14 .. 65,504; larger magnitudes overflow).  k_scale, v_scale and
 * sm_scale * k_scale must be finite (S5_ERR_INVALID_ARG).  The workspace of
 * s5_workspace_size covers this call. */
s5_status s5_sparse_gqa_attn_fp8kv(const s5_kv_desc *kv, const s5_batch_desc *batch, const void *q,
                                   const int32_t *sel, const int32_t *sel_count, int32_t topk, float sm_scale,
                                   float k_scale, float v_scale, void *out, float *lse, void *workspace,
                                   size_t workspace_bytes, s5_stream_t stream);

/* Per-KV-group selection (StepFun open-weights blog, "What sparse attention
 * does and doesn't save": each KV group picks its own blocks).  The block
 * keys stay shared (the configuration gives one 256-wide key per block); the
 * indexer query differs per group, so each token carries 4 queries and gets
 * 4 selections, and the heads of group g attend over group g's blocks.
 *
 * s5_index_score_topk_grouped: as s5_index_score_topk for every (token,
 * group) pair, each key read once for all four.
 *   q_index    device bf16 [total_q][4][256]: the query of token r, group g
 *   sel        device int32 [total_q][4][topk], sel_count [total_q][4]
 * s5_sparse_gqa_attn_grouped: as s5_sparse_gqa_attn, with head h (group
 * g = h / 16) reading sel[r][g][0 .. sel_count[r][g] - 1] plus the current
 * block.  Every row takes the per-row kernel (the shared-set tiles assume one
 * selection per token).
 * s5_workspace_size_grouped: a workspace size that covers these two calls as
 * well as every call s5_workspace_size covers.
 * Limits: selections of more than 16,384 history blocks need
 * 4 * total_q <= 65,535 (else S5_ERR_UNSUPPORTED). */
s5_status s5_workspace_size_grouped(const s5_batch_desc *batch, int32_t window, size_t *bytes);
s5_status s5_index_score_topk_grouped(const s5_index_desc *index, const s5_batch_desc *batch,
                                      const void *q_index, int32_t topk, int32_t *sel, int32_t *sel_count,
                                      void *workspace, size_t workspace_bytes, s5_stream_t stream);
s5_status s5_sparse_gqa_attn_grouped(const s5_kv_desc *kv, const s5_batch_desc *batch, const void *q,
                                     const int32_t *sel, const int32_t *sel_count, int32_t topk, float sm_scale,
                                     void *out, float *lse, void *workspace, size_t workspace_bytes,
                                     s5_stream_t stream);

/* s5_index_score_topk without a workspace.  The pages have no counterpart to
 * this entry point: it exists for callers that cannot allocate device memory
 * at all, such as code embedded in a host framework that owns every device
 * allocation and hands over only inputs and outputs, or a process whose
 * device-memory budget is fixed at start-up.  Results are those of
 * s5_index_score_topk for the same arguments.
 *   Scratch: a library-owned 8 MiB device array (file scope), which every GPU
 *   that loads the library keeps until the process exits.  Limits: at most
 *   16,384 history blocks per row (max_len <= 131,080) and
 *   256 + 4 * total_q * S bytes <= 8 MiB, S = (max_len - 1) / 8 rounded up to a
 *   multiple of 4; larger requests
 *   return S5_ERR_WORKSPACE with nothing enqueued.  batch <= 65,535 and
 *   max_q <= 262,140 (the scoring grid); larger ones return
 *   S5_ERR_UNSUPPORTED with nothing enqueued.
 *   The call allocates nothing: no cudaMalloc, no cudaFree, no allocating
 *   library routine.  The first call on a device (with that device current)
 *   looks up the array's device address once; make that first call before
 *   any stream capture.  The address is kept for the life of the process: a
 *   device reset (cudaDeviceReset) makes it stale, so do not call this entry
 *   point again in a process after resetting the device.
 *   Every call shares the one array and leaves its contents behind; each call
 *   clears the part that must start at zero.  Calls that can overlap on the
 *   GPU (other streams, other host threads) race on the array: serialise them.
 *   Device-data faults are recorded in the array's own error record, which
 *   this entry point does not expose; diagnose bad inputs with
 *   s5_index_score_topk and a workspace. */
s5_status s5_index_score_topk_noalloc(const s5_index_desc *index, const s5_batch_desc *batch,
                                      const void *q_index, int32_t topk, int32_t *sel, int32_t *sel_count,
                                      s5_stream_t stream);

/* Cache append: store the batch's new tokens, and the keys of the blocks
 * they complete, in the paged cache before the layer's attention reads them
 * (SGLang day-0 blog, "Kernels from StepFun": the indexer scores the
 * per-block history kept in the paged cache; "Get Started": 64-token pages,
 * bf16 cache).  For row r of sequence s at position t = ctx_lens[s] + j:
 *   K/V   k_new[r][g] / v_new[r][g] -> slot t % 64 of group g of physical page
 *         page_table[s][t / 64], for g = 0..3;
 *   key   if t % 8 == 7 (t completes block t / 8): key_new[r] -> slot
 *         (t % 64) / 8 of the same physical page of the index-key pool.
 * Only complete blocks are ever scored, so a block's key is stored once, with
 * its last token; key_new rows of other tokens are not read.
 *   kv       the pools to WRITE (the descriptor's const applies to the
 *            attention calls, which only read them)
 *   index    the bf16 block-key pool to write, or NULL for a cache without
 *            block keys (a sliding-window layer); key_new is then ignored
 *   k_new, v_new  device bf16 [total_q][4][192], 16-byte aligned
 *   key_new  device bf16 [total_q][256], 16-byte aligned (when index != NULL)
 *   workspace  at least S5_WS_FIXED_BYTES; only its error record is used
 * The pages of every new position must be mapped before the call.  An
 * unmapped page (-1), a page id outside the KV pool (or, with a key pool,
 * outside the key pool) or a position past the page table records
 * S5_ERR_DEVICE_BOUNDS (info = the first such row) and that row is skipped.  batch->max_q and batch->max_len are not used.  Rows are
 * independent: positions written by one call must be distinct. */
s5_status s5_append_kv(const s5_kv_desc *kv, const s5_index_desc *index, const s5_batch_desc *batch,
                       const void *k_new, const void *v_new, const void *key_new, void *workspace,
                       size_t workspace_bytes, s5_stream_t stream);

/* s5_append_kv for a cache whose K / V are one-byte E4M3 codes (the pools of
 * s5_sparse_gqa_attn_fp8kv; StepFun open-weights blog, "Fitting it on a
 * node": FP8 KV for the full-attention layers).  k_new / v_new are bf16 as in
 * s5_append_kv; value x of a K row is stored as the E4M3 code nearest to the
 * fp32 product x * (1 / k_scale) (1 / k_scale rounded to fp32; ties to an even
 * mantissa; magnitudes beyond 448 saturate to +-448), V likewise with v_scale,
 * so a stored code stands for about x / scale and s5_sparse_gqa_attn_fp8kv
 * with the same scales reads it back as scale * code.  kv->k_pool / v_pool
 * are uint8 [num_pages][4][64][192]; block keys (index, key_new) are bf16
 * exactly as in s5_append_kv.  k_scale and v_scale must be finite and nonzero
 * with finite reciprocals (S5_ERR_INVALID_ARG).  Otherwise as s5_append_kv. */
s5_status s5_append_kv_fp8(const s5_kv_desc *kv, const s5_index_desc *index, const s5_batch_desc *batch,
                           const void *k_new, const void *v_new, const void *key_new, float k_scale, float v_scale,
                           void *workspace, size_t workspace_bytes, s5_stream_t stream);

/* Zero the first S5_WS_FIXED_BYTES of a workspace: the device error record
 * and the partition counters (asynchronous, on `stream`). */
s5_status s5_reset_device_error(void *workspace, s5_stream_t stream);

/* Synchronise `stream` and read the device error record: *code is S5_OK or
 * the first recorded s5_status, *info the offending query row (or -1). */
s5_status s5_get_device_error(void *workspace, s5_stream_t stream, int32_t *code, int32_t *info);

/* Static English name of a status code. */
const char *s5_status_string(s5_status status);

/* S5_ABI_VERSION of the header the library was built with. */
int32_t s5_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* S5ATTN_H */
