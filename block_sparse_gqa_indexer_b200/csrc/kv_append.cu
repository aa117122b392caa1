// s5_append_kv: the cache-append step on either side of the attention path.
// Every new token's K and V rows go into their slot of the paged pools, and a
// token that completes its 8-token block stores that block's 256-wide key in
// the index-key pool, so the next indexer call scores it (SGLang day-0 blog,
// "Kernels from StepFun": the indexer reads the per-block history from the
// paged cache; "Get Started": 64-token pages, bf16 cache).
//
// Layout of one row's work: K and V of one token are 4 groups x 384 bytes
// each, scattered to 4 slots 24 KB apart in one physical page; the block key is
// 512 bytes.  The CTA has 7 warps, one 16-byte chunk of each row per thread:
// warps 0-2 copy K (96 chunks), warps 3-5 copy V, warp 6 the key.  Each warp
// covers 512 contiguous source bytes, and each group's 384-byte destination
// row is contiguous.  The kernel is a pure copy (about 3.6 KB read and
// written per token), so it is bound by latency at decode sizes and by HBM in
// prefill.
#include <cuda_runtime.h>

#include <cstdint>

#include "s5_common.cuh"

using namespace s5;

namespace {

constexpr int kAppendThreads = 224;                    // 7 warps
constexpr int kRowChunks = kD * 2 / 16;                // 24 chunks of 16 B per (token, group) row
constexpr int kKvChunks = kKv * kRowChunks;            // 96 per token, K or V
constexpr int kKeyChunks = kDx * 2 / 16;               // 32 per block key
constexpr int kAppendRows = 4;                         // rows per CTA pass
constexpr int kAppendMaxCtas = 148 * 32;

static_assert(2 * kKvChunks + kKeyChunks == kAppendThreads, "one chunk per thread");

struct AppendArgs {
  uint8_t *k_pool;
  uint8_t *v_pool;
  uint8_t *key_pool;  // null: no block keys
  int32_t kv_pages;
  int32_t key_pages;
  const int32_t *page_table;
  int32_t max_pages;
  const int32_t *ctx_lens;
  const int32_t *cu_q;
  int32_t batch;
  int32_t total_q;
  const uint8_t *k_new;
  const uint8_t *v_new;
  const uint8_t *key_new;
  int32_t *err;
};

// One pass of a CTA covers kAppendRows rows: first one thread per row finds
// its sequence, position and physical page (dependent lookups, all rows at
// once), then every thread issues its 16-byte loads for all rows before any
// store, so each thread keeps kAppendRows independent loads in flight.
__global__ void __launch_bounds__(kAppendThreads) kv_append_kernel(const AppendArgs a) {
  __shared__ int s_page[kAppendRows];
  __shared__ int s_pos[kAppendRows];
  const int tid = threadIdx.x;
  const bool is_key = tid >= 2 * kKvChunks;
  const bool is_v = tid >= kKvChunks && !is_key;
  const int c = is_key ? tid - 2 * kKvChunks : (is_v ? tid - kKvChunks : tid);
  const int g = c / kRowChunks, w = c % kRowChunks;
  for (int r0 = blockIdx.x * kAppendRows; r0 < a.total_q; r0 += gridDim.x * kAppendRows) {
    if (tid < kAppendRows) {
      const int r = r0 + tid;
      int page = -1, t = -1;
      if (r < a.total_q) {
        int s = 0;
        if (locate_row(a.cu_q, a.ctx_lens, a.batch, r, row_guess(r, a.batch, a.total_q), s, t) && t >= 0) {
          const int logical = t / kPage;
          page = logical < a.max_pages ? ld_cg(a.page_table + (size_t)s * a.max_pages + logical) : -1;
        }
        if (page < 0 || page >= a.kv_pages || (a.key_pool != nullptr && page >= a.key_pages)) {
          record_error(a.err, S5_ERR_DEVICE_BOUNDS, r);
          page = -1;
        }
      }
      s_page[tid] = page;
      s_pos[tid] = t;
    }
    __syncthreads();
    uint4 v[kAppendRows];
    bool on[kAppendRows];
#pragma unroll
    for (int i = 0; i < kAppendRows; ++i) {
      const int t = s_pos[i];
      // a key moves only for the token that completes its block
      on[i] = s_page[i] >= 0 && (!is_key || (a.key_pool != nullptr && t % kBlk == kBlk - 1));
      if (on[i]) {
        const size_t r = (size_t)(r0 + i);
        const uint8_t *src = is_key ? a.key_new + (r * kKeyChunks + c) * 16
                                    : (is_v ? a.v_new : a.k_new) + (r * kKvChunks + c) * 16;
        v[i] = *reinterpret_cast<const uint4 *>(src);
      }
    }
#pragma unroll
    for (int i = 0; i < kAppendRows; ++i) {
      if (!on[i]) continue;
      const size_t page = (size_t)s_page[i];
      const int slot = s_pos[i] % kPage;
      uint8_t *dst = is_key ? a.key_pool + ((page * kBpp + slot / kBlk) * kKeyChunks + c) * 16
                            : (is_v ? a.v_pool : a.k_pool) + (((page * kKv + g) * kPage + slot) * kRowChunks + w) * 16;
      *reinterpret_cast<uint4 *>(dst) = v[i];
    }
    __syncthreads();  // s_page / s_pos are rewritten by the next pass
  }
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" s5_status s5_append_kv(const s5_kv_desc *kv, const s5_index_desc *index, const s5_batch_desc *batch,
                                  const void *k_new, const void *v_new, const void *key_new, void *workspace,
                                  size_t workspace_bytes, s5_stream_t stream) {
  if (batch == nullptr || kv == nullptr) return S5_ERR_INVALID_ARG;
  if (batch->batch < 1 || batch->max_pages < 1 || batch->total_q < 0) return S5_ERR_INVALID_ARG;
  if (batch->page_table == nullptr || batch->ctx_lens == nullptr || batch->cu_q == nullptr)
    return S5_ERR_INVALID_ARG;
  if (kv->k_pool == nullptr || kv->v_pool == nullptr || kv->num_pages < 1) return S5_ERR_INVALID_ARG;
  if (kv->page_size != kPage || kv->n_kv_heads != kKv || kv->head_dim != kD) return S5_ERR_UNSUPPORTED;
  if (!aligned16(kv->k_pool) || !aligned16(kv->v_pool)) return S5_ERR_INVALID_ARG;
  if (index != nullptr) {
    if (index->key_pool == nullptr || index->num_pages < 1 || !aligned16(index->key_pool))
      return S5_ERR_INVALID_ARG;
    if (index->index_dim != kDx) return S5_ERR_UNSUPPORTED;
  }
  if (workspace == nullptr || workspace_bytes < S5_WS_FIXED_BYTES) return S5_ERR_WORKSPACE;
  if (batch->total_q == 0) return S5_OK;
  if (k_new == nullptr || v_new == nullptr || !aligned16(k_new) || !aligned16(v_new)) return S5_ERR_INVALID_ARG;
  if (index != nullptr && (key_new == nullptr || !aligned16(key_new))) return S5_ERR_INVALID_ARG;

  AppendArgs a{};
  // the pools are written: the descriptors' const covers the read-only calls
  a.k_pool = static_cast<uint8_t *>(const_cast<void *>(kv->k_pool));
  a.v_pool = static_cast<uint8_t *>(const_cast<void *>(kv->v_pool));
  a.key_pool = index != nullptr ? static_cast<uint8_t *>(const_cast<void *>(index->key_pool)) : nullptr;
  a.kv_pages = kv->num_pages;
  a.key_pages = index != nullptr ? index->num_pages : 0;
  a.page_table = batch->page_table;
  a.max_pages = batch->max_pages;
  a.ctx_lens = batch->ctx_lens;
  a.cu_q = batch->cu_q;
  a.batch = batch->batch;
  a.total_q = batch->total_q;
  a.k_new = static_cast<const uint8_t *>(k_new);
  a.v_new = static_cast<const uint8_t *>(v_new);
  a.key_new = index != nullptr ? static_cast<const uint8_t *>(key_new) : nullptr;
  a.err = static_cast<int32_t *>(workspace);
  const int passes = (batch->total_q + kAppendRows - 1) / kAppendRows;
  const int grid = passes < kAppendMaxCtas ? passes : kAppendMaxCtas;
  kv_append_kernel<<<grid, kAppendThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(a);
  return cudaGetLastError() == cudaSuccess ? S5_OK : S5_ERR_CUDA;
}
