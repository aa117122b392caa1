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
//
// s5_append_kv_fp8 is the same kernel for a cache whose K / V are one-byte
// E4M3 codes (StepFun open-weights blog, "Fitting it on a node": FP8 KV for
// the full-attention layers): each thread's 8 bf16 values are multiplied in
// fp32 by the reciprocal of the layer's scale and rounded to the nearest E4M3
// value (ties to even, saturating at 448), and 8 code bytes are stored; block
// keys stay bf16.
#include <cuda_runtime.h>

#include <cmath>
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
  float k_inv, v_inv;  // one-byte K / V: fp32 reciprocals of the scales
};

// Two fp32 values to their E4M3 codes (round to nearest even, saturating at
// 448), first value in the low byte.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  uint32_t d;
  asm("{\n\t.reg .b16 c;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 c, %2, %1;\n\t"
      "cvt.u32.u16 %0, c;\n\t}"
      : "=r"(d)
      : "f"(lo), "f"(hi));
  return d;
}

// Eight bf16 values (16 bytes) times `inv` in fp32, as eight E4M3 code bytes.
__device__ __forceinline__ uint2 bf16x8_to_e4m3x8(uint4 v, float inv) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) c[i] = f32x2_to_e4m3x2(__fmul_rn(bf16lo(w[i]), inv), __fmul_rn(bf16hi(w[i]), inv));
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// One pass of a CTA covers kAppendRows rows: first one thread per row finds
// its sequence, position and physical page (dependent lookups, all rows at
// once), then every thread issues its 16-byte loads for all rows before any
// store, so each thread keeps kAppendRows independent loads in flight.
template <bool KV8>
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
      if (is_key) {
        *reinterpret_cast<uint4 *>(a.key_pool + ((page * kBpp + slot / kBlk) * kKeyChunks + c) * 16) = v[i];
      } else if (KV8) {  // 8 code bytes per chunk of 8 values
        *reinterpret_cast<uint2 *>((is_v ? a.v_pool : a.k_pool) + (((page * kKv + g) * kPage + slot) * kRowChunks + w) * 8) =
            bf16x8_to_e4m3x8(v[i], is_v ? a.v_inv : a.k_inv);
      } else {
        *reinterpret_cast<uint4 *>((is_v ? a.v_pool : a.k_pool) + (((page * kKv + g) * kPage + slot) * kRowChunks + w) * 16) =
            v[i];
      }
    }
    __syncthreads();  // s_page / s_pos are rewritten by the next pass
  }
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// kv8: the K / V pools hold one-byte E4M3 codes (k_scale, v_scale used);
// otherwise bf16.
s5_status append_common(const s5_kv_desc *kv, const s5_index_desc *index, const s5_batch_desc *batch,
                        const void *k_new, const void *v_new, const void *key_new, void *workspace,
                        size_t workspace_bytes, s5_stream_t stream, bool kv8, float k_scale, float v_scale) {
  if (batch == nullptr || kv == nullptr) return S5_ERR_INVALID_ARG;
  if (kv8 && (!(std::isfinite(k_scale) && std::isfinite(v_scale)) || k_scale == 0.f || v_scale == 0.f ||
              !std::isfinite(1.f / k_scale) || !std::isfinite(1.f / v_scale)))
    return S5_ERR_INVALID_ARG;
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
  a.k_inv = kv8 ? 1.f / k_scale : 1.f;
  a.v_inv = kv8 ? 1.f / v_scale : 1.f;
  const int passes = (batch->total_q + kAppendRows - 1) / kAppendRows;
  const int grid = passes < kAppendMaxCtas ? passes : kAppendMaxCtas;
  if (kv8)
    kv_append_kernel<true><<<grid, kAppendThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(a);
  else
    kv_append_kernel<false><<<grid, kAppendThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(a);
  return cudaGetLastError() == cudaSuccess ? S5_OK : S5_ERR_CUDA;
}

}  // namespace

extern "C" s5_status s5_append_kv(const s5_kv_desc *kv, const s5_index_desc *index, const s5_batch_desc *batch,
                                  const void *k_new, const void *v_new, const void *key_new, void *workspace,
                                  size_t workspace_bytes, s5_stream_t stream) {
  return append_common(kv, index, batch, k_new, v_new, key_new, workspace, workspace_bytes, stream, false, 1.f, 1.f);
}

extern "C" s5_status s5_append_kv_fp8(const s5_kv_desc *kv, const s5_index_desc *index, const s5_batch_desc *batch,
                                      const void *k_new, const void *v_new, const void *key_new, float k_scale,
                                      float v_scale, void *workspace, size_t workspace_bytes, s5_stream_t stream) {
  return append_common(kv, index, batch, k_new, v_new, key_new, workspace, workspace_bytes, stream, true, k_scale,
                       v_scale);
}
