// s5_index_score_topk_noalloc: the indexer (block scores + top-k select) with
// its scratch in a fixed, library-owned device array instead of a caller
// workspace, for callers that cannot allocate device memory at all: code
// embedded in a host framework that owns every device allocation and hands a
// kernel only its inputs and outputs, or a process with a fixed device-memory
// budget that must not grow after start-up.
//
// The scratch array is a file-scope __device__ variable.  Every GPU that
// loads this library keeps its copy (kNoAllocScratchBytes) until the process
// exits.  In host code its name is only a host-side stand-in, so the device
// address is looked up once per device with cudaGetSymbolAddress (with that
// device current) and passed to the kernels.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "s5_common.cuh"
#include "s5_kernels.h"

using namespace s5;

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
constexpr int kNoAllocMaxHistory = 16384;  // blocks per row: the one-stage select only
constexpr int kNoAllocPagesPerCta = 64;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device (looked up on the
// first call made with that device current and kept for the life of the
// process; a device reset unloads the module and leaves the kept address
// stale, so after cudaDeviceReset this entry point must not be called again
// in that process).
cudaError_t scratch_address(void **out) {
  static std::mutex mu;
  static void *addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *out = addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" s5_status s5_index_score_topk_noalloc(const s5_index_desc *index, const s5_batch_desc *batch,
                                                 const void *q_index, int32_t topk, int32_t *sel,
                                                 int32_t *sel_count, s5_stream_t stream) {
  if (batch == nullptr || index == nullptr) return S5_ERR_INVALID_ARG;
  if (batch->batch < 1 || batch->max_pages < 1 || batch->total_q < 0 || batch->max_q < 0 || batch->max_len < 0)
    return S5_ERR_INVALID_ARG;
  if (batch->max_len > S5_MAX_LEN) return S5_ERR_UNSUPPORTED;
  if ((long long)batch->max_pages * kPage < (long long)batch->max_len) return S5_ERR_INVALID_ARG;
  if (batch->total_q > 0 && (batch->max_q < 1 || batch->max_len < 1)) return S5_ERR_INVALID_ARG;
  if (batch->page_table == nullptr || batch->ctx_lens == nullptr || batch->cu_q == nullptr)
    return S5_ERR_INVALID_ARG;
  if (index->key_pool == nullptr || index->num_pages < 1) return S5_ERR_INVALID_ARG;
  if (index->index_dim != kDx) return S5_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(index->key_pool) & 15u) != 0) return S5_ERR_INVALID_ARG;
  if (topk < 1 || topk > kMaxTopk) return S5_ERR_INVALID_ARG;
  if (batch->total_q == 0) return S5_OK;
  if (q_index == nullptr || sel == nullptr || sel_count == nullptr ||
      (reinterpret_cast<uintptr_t>(q_index) & 15u) != 0)
    return S5_ERR_INVALID_ARG;

  // scratch layout: error record (256 B), then fp32 scores [total_q][stride]
  const int hist = batch->max_len >= 1 ? (batch->max_len - 1) / kBlk : 0;
  const int stride = ((hist > 1 ? hist : 1) + 3) & ~3;  // rows start 16-byte aligned
  if (stride > kNoAllocMaxHistory) return S5_ERR_WORKSPACE;
  const size_t need = kWsHeader + (size_t)batch->total_q * stride * sizeof(float);
  if (need > kNoAllocScratchBytes) return S5_ERR_WORKSPACE;
  // launch limits of the scoring grid (sequences x 4-row tiles), checked
  // before anything is enqueued: short histories let the scratch hold more
  // rows than one sequence's tiles may span
  if (batch->batch > 65535 || (batch->max_q + 3) / 4 > 65535) return S5_ERR_UNSUPPORTED;

  void *scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return S5_ERR_CUDA;
  uint8_t *ws = static_cast<uint8_t *>(scratch);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  // the error record must start at zero; the scores are fully rewritten
  if (cudaMemsetAsync(ws, 0, kWsHeader, cs) != cudaSuccess) return S5_ERR_CUDA;
  int32_t *err = reinterpret_cast<int32_t *>(ws);

  IndexScoreArgs ia{};
  ia.key_pool = index->key_pool;
  ia.num_pages = index->num_pages;
  ia.page_table = batch->page_table;
  ia.max_pages = batch->max_pages;
  ia.ctx_lens = batch->ctx_lens;
  ia.cu_q = batch->cu_q;
  ia.batch = batch->batch;
  ia.total_q = batch->total_q;
  ia.q_index = q_index;
  ia.scores = reinterpret_cast<float *>(ws + kWsHeader);
  ia.score_stride = stride;
  ia.pages_per_cta = kNoAllocPagesPerCta;
  ia.topk = topk;
  ia.err = err;
  const int pages = (stride + kBpp - 1) / kBpp;
  const int grid_pages = (pages + kNoAllocPagesPerCta - 1) / kNoAllocPagesPerCta;
  if (launch_index_score(ia, batch->max_q, grid_pages, batch->batch, cs) != cudaSuccess) return S5_ERR_CUDA;

  SelectArgs sa{};
  sa.scores = ia.scores;
  sa.score_stride = stride;
  sa.ctx_lens = batch->ctx_lens;
  sa.cu_q = batch->cu_q;
  sa.batch = batch->batch;
  sa.total_q = batch->total_q;
  sa.topk = topk;
  sa.sel = sel;
  sa.sel_count = sel_count;
  sa.err = err;
  return launch_topk_select(sa, batch->total_q, false, cs) == cudaSuccess ? S5_OK : S5_ERR_CUDA;
}
