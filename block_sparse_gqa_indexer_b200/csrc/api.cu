// C ABI of the s5attn library: argument checks, workspace layout, TMA
// descriptors and launch selection.  Every entry point here is declared in
// include/s5attn.h, which states the semantics, layouts and error rules.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "s5_common.cuh"
#include "s5_kernels.h"

using namespace s5;

namespace {

constexpr int kAbiVersion = S5_ABI_VERSION;
constexpr int kSelCap = 16384;      // rows up to this many blocks: one CTA selects the whole row
constexpr int kSegShort = 4096;     // longer rows: top-k per segment of this many blocks, then a merge
constexpr int kSeg = 8192;          // ... segments of rows longer than 16,384 blocks
constexpr int kMaxSeg = 32;         // (kSeg * kMaxSeg >= S5_MAX_LEN / 8)
constexpr int kMaxSplit = 8;        // partitions per (row, group) beyond what kMaxList forces
constexpr int kScorePagesPerCta = 64;  // indexer CTA: 64 pages = 512 block keys = 256 KB
constexpr int kScoreMinPagesPerCta = 4;  // ... and at least 4 pages (two per warp pair in flight)
constexpr int kMaxGridYZ = 65535;      // CUDA limit on gridDim.y and gridDim.z

static_assert((long long)kSeg * kMaxSeg >= S5_MAX_LEN / S5_BLOCK_SIZE, "segments must cover the longest row");

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Longest history of any row: a query at t < max_len has c = t / 8 <= (max_len - 1) / 8 blocks.
int max_blocks(const s5_batch_desc *b) {
  const int h = b->max_len >= 1 ? (b->max_len - 1) / kBlk : 0;
  return h > 1 ? h : 1;
}

// ---------------------------------------------------------------- argument checks

s5_status check_batch(const s5_batch_desc *b) {
  if (b == nullptr) return S5_ERR_INVALID_ARG;
  if (b->batch < 1 || b->max_pages < 1 || b->total_q < 0 || b->max_q < 0 || b->max_len < 0)
    return S5_ERR_INVALID_ARG;
  if (b->max_len > S5_MAX_LEN) return S5_ERR_UNSUPPORTED;
  if ((long long)b->max_pages * kPage < (long long)b->max_len) return S5_ERR_INVALID_ARG;
  if (b->total_q > 0 && (b->max_q < 1 || b->max_len < 1)) return S5_ERR_INVALID_ARG;
  if (b->page_table == nullptr || b->ctx_lens == nullptr || b->cu_q == nullptr) return S5_ERR_INVALID_ARG;
  if ((long long)b->total_q * kHeads > 0x7fffffffLL) return S5_ERR_UNSUPPORTED;
  return S5_OK;
}

s5_status check_kv(const s5_kv_desc *kv) {
  if (kv == nullptr || kv->k_pool == nullptr || kv->v_pool == nullptr) return S5_ERR_INVALID_ARG;
  if (kv->page_size != kPage || kv->n_kv_heads != kKv || kv->head_dim != kD) return S5_ERR_UNSUPPORTED;
  if (kv->num_pages < 1) return S5_ERR_INVALID_ARG;
  if ((long long)kv->num_pages * kKv * kPage >= (1LL << 31)) return S5_ERR_UNSUPPORTED;
  if (!aligned16(kv->k_pool) || !aligned16(kv->v_pool)) return S5_ERR_INVALID_ARG;
  return S5_OK;
}

// ---------------------------------------------------------------- workspace layout

constexpr int kMaxHistRows = 1024;  // decode / verify batches: rows get a score histogram
constexpr int kGemmMinRows = 64;    // sequences with more query rows score on the tensor cores
constexpr int kGemmTilesPerCta = 16;  // 128-block N tiles per GEMM CTA: a 16K-row prefill is 1,024 CTAs (6.9 waves)

struct IndexWs {
  size_t scores, cand_key, cand_idx, hist, hist_bytes, kxs, kxs_bytes, end;
  int stride, seg, n_seg;
  bool two_stage;
};

// Indexer scratch for `groups` indexer queries per token (1, or one per KV
// group): every row below is one (token, group) pair.
IndexWs index_ws(const s5_batch_desc *b, int groups) {
  IndexWs w{};
  const size_t rows = (size_t)b->total_q * groups;
  w.stride = (max_blocks(b) + 3) & ~3;  // rows start 16-byte aligned
  w.two_stage = w.stride > kSelCap;
  w.seg = (w.stride <= 16384) ? kSegShort : kSeg;
  w.n_seg = w.two_stage ? (w.stride + w.seg - 1) / w.seg : 0;
  size_t off = kWsFixed;
  w.scores = off;
  off = align_up(off + rows * w.stride * sizeof(float), 256);
  w.cand_key = off;
  off = align_up(off + rows * w.n_seg * kMaxTopk * sizeof(uint32_t), 256);
  w.cand_idx = off;
  off = align_up(off + rows * w.n_seg * kMaxTopk * sizeof(int32_t), 256);
  w.hist = off;
  // the histograms are built by the CUDA-core scoring kernel (not by the tensor-core GEMM)
  const bool gemm = (long long)b->max_q * groups > kGemmMinRows;
  w.hist_bytes = (!gemm && !w.two_stage && rows <= (size_t)kMaxHistRows)
                     ? rows * kHistBins * sizeof(uint32_t) : 0;
  off = align_up(off + w.hist_bytes, 256);
  w.kxs = off;
  w.kxs_bytes = gemm ? (size_t)b->batch * w.stride * kDx * 2 : 0;
  off = align_up(off + w.kxs_bytes, 1024);
  w.end = off;
  return w;
}

// Partitions per (row, group).  The kernel is HBM-bound, so the aim is one
// wave of equal CTAs (2 resident per SM): as many partitions as fit in that
// wave, none when the batch alone fills it, each warp keeping at least two
// block pairs, and no CTA owning more than kMaxList blocks.  At most
// kMaxSplit partitions otherwise: for the smallest batches the last CTA's
// merge of every partition outweighs the shorter partitions (B=1 at 16K
// tokens, attention call: 32.8 us with a cap of 4, 28.7 us with 8, 30.7 us
// with 16; B=4 at 1M tokens: 34.8, 32.8 and 45.8 us).
int choose_split(int total_q, int blocks_per_row, int slots) {
  const int units = total_q * kKv;
  int n = units > 0 ? slots / units : 1;
  const int by_work = blocks_per_row / (4 * 4);  // 4 warps x 2 pairs x 2 blocks
  n = n < by_work ? n : by_work;
  n = n > kMaxSplit ? kMaxSplit : n;
  const int by_list = (blocks_per_row + kMaxList - 1) / kMaxList;
  if (n < by_list) n = by_list;
  return n < 1 ? 1 : n;
}

constexpr int kCtasPerSm = 2;
constexpr int kSizingSms = 256;  // workspace sizing assumes at most this many SMs

// Attention CTA slots of the current device (cached per device).
int device_slots() {
  static std::mutex mu;
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return kCtasPerSm * 148;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) sms = 148;
    if (sms > kSizingSms) sms = kSizingSms;
    cache[dev] = kCtasPerSm * sms;
  }
  return cache[dev];
}

}  // namespace

namespace s5 {
cudaError_t ensure_dynamic_smem(const void *kernel, int bytes) {
  struct Entry {
    int dev;
    const void *fn;
    int bytes;
  };
  static std::mutex mu;
  static Entry set[64];
  static int n_set = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n_set; ++i)
    if (set[i].dev == dev && set[i].fn == kernel && set[i].bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  for (int i = 0; i < n_set; ++i)
    if (set[i].dev == dev && set[i].fn == kernel) {
      set[i].bytes = bytes;
      return cudaSuccess;
    }
  if (n_set < 64) set[n_set++] = Entry{dev, kernel, bytes};
  return cudaSuccess;
}
}  // namespace s5

namespace {

struct AttnWs {
  size_t part_o, part_lse, end;
  int n_split;
};

AttnWs attn_ws(const s5_batch_desc *b, int blocks_per_row, int slots) {
  AttnWs w{};
  w.n_split = choose_split(b->total_q, blocks_per_row, slots);
  size_t off = kWsFixed;
  w.part_o = off;
  if (w.n_split > 1) {
    off = align_up(off + (size_t)b->total_q * kHeads * w.n_split * kD * sizeof(float), 256);
    w.part_lse = off;
    off = align_up(off + (size_t)b->total_q * kHeads * w.n_split * sizeof(float), 256);
  } else {
    w.part_lse = off;
  }
  w.end = off;
  return w;
}

// ---- multi-row tiles (verify / prefill) on the tensor cores ----

struct TileWs {
  size_t count, ent, tile_on, row_skip, part_o, part_lse, end;
  int tiles_per_seq, n_tiles, union_cap, map_words, n_split;
};

// Tile CTAs hold 215 KB of shared memory: one per SM.  With `sizing`, the
// partials are reserved for the largest partition count any device may pick.
// The region starts at `base`: below it lie the per-row kernel's partials,
// which that kernel writes while other CTAs still read the tile flags.
TileWs tile_ws(const s5_batch_desc *b, int topk, int slots_1cta, bool sizing, size_t base) {
  TileWs w{};
  w.tiles_per_seq = (b->max_q + kTileRows - 1) / kTileRows;
  w.n_tiles = b->batch * w.tiles_per_seq;
  w.union_cap = kTileRows * topk + kTileRows;
  const long long words = (long long)(b->max_len / kBlk) / 4 + 2;
  w.map_words = (int)(words < kUnionMapWords ? words : kUnionMapWords);
  // partitions: fewest waves of the persistent CTAs per unit of work
  // (ceil(n * units / slots) / n), n <= kMaxTileSplit, ties to fewer partitions; merge
  // counters cover 1,024 tiles
  const long long units = (long long)w.n_tiles * kKv;
  int best = 1;
  if (w.n_tiles <= kMaxMergeRows && units > 0 && slots_1cta > 0) {
    double best_cost = 1e30;
    for (int n = 1; n <= kMaxTileSplit; ++n) {
      const double cost = (double)((n * units + slots_1cta - 1) / slots_1cta) / n;
      if (cost < best_cost - 1e-9) {
        best_cost = cost;
        best = n;
      }
    }
  }
  w.n_split = best;
  size_t off = align_up(base, 256);
  w.count = off;
  off = align_up(off + (size_t)w.n_tiles * sizeof(int), 256);
  w.tile_on = off;
  off = align_up(off + (size_t)w.n_tiles * sizeof(int32_t), 256);
  w.row_skip = off;
  off = align_up(off + (size_t)b->total_q * sizeof(int32_t), 256);
  w.ent = off;
  off = align_up(off + (size_t)w.n_tiles * w.union_cap * sizeof(uint32_t), 256);
  w.part_o = w.part_lse = off;
  const int n_res = (sizing && w.n_tiles <= kMaxMergeRows) ? kMaxTileSplit : w.n_split;
  if (n_res > 1) {
    off = align_up(off + (size_t)b->total_q * kHeads * n_res * kD * sizeof(float), 256);
    w.part_lse = off;
    off = align_up(off + (size_t)b->total_q * kHeads * n_res * sizeof(float), 256);
  }
  w.end = off;
  return w;
}

// Multi-token batches go through the union kernel, which sends each 8-row
// tile to the shared-set tile kernel or to the per-row kernel.
bool use_tiles(const s5_batch_desc *b) { return b->max_q >= 2; }

// Crossover of the two paths: a tile takes the shared set when its union has
// at most this percentage of the blocks its rows read one by one.
constexpr int kTileUnionPct = 70;

int sparse_blocks_per_row(int topk) { return topk + 1; }
int swa_blocks_per_row(const s5_batch_desc *b, int window) {
  long long w = window < b->max_len ? window : b->max_len;
  return (int)((w + kBlk - 1) / kBlk + 1);
}

// ---------------------------------------------------------------- TMA descriptors

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A pool bf16 [num_pages][4][64][192] viewed as rows of 192 = 3 x 64 elements;
// one box is one 8-token block of one group: {64, 3, 8}, 128-byte swizzle.
bool make_kv_map(CUtensorMap *m, const void *pool, int num_pages) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {64, 3, (cuuint64_t)num_pages * kKv * kPage};
  cuuint64_t strides[2] = {128, (cuuint64_t)kD * 2};
  cuuint32_t box[3] = {64, 3, (cuuint32_t)kBlk};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(pool), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A one-byte (E4M3) K or V pool uint8 [num_pages][4][64][192] viewed as rows of
// 192 = 3 x 64 bytes; one box is one 8-token block of one group: {64, 3, 8},
// 1,536 bytes, 64-byte swizzle.
bool make_kv8_map(CUtensorMap *m, const void *pool, int num_pages) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {64, 3, (cuuint64_t)num_pages * kKv * kPage};
  cuuint64_t strides[2] = {64, (cuuint64_t)kD};
  cuuint32_t box[3] = {64, 3, (cuuint32_t)kBlk};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(pool), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A K or V pool as rows of 192 dims, each 8-row box landing plane-major: box
// {64 dims, 8 rows, 3 planes} with the planes (128 B apart in memory) as the
// outermost box dimension, so one copy places a whole 8-token block as three
// 1,024-byte swizzled planes [plane][token][64 dims].  The plane stride is
// smaller than the row stride; the box addresses stay inside the pool either
// way (every coordinate is range-checked against its own extent).
bool make_kv_plane_map(CUtensorMap *m, const void *pool, int num_pages) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)num_pages * kKv * kPage, 3};
  cuuint64_t strides[2] = {(cuuint64_t)kD * 2, 128};
  cuuint32_t box[3] = {64, (cuuint32_t)kBlk, 3};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(pool), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A bf16 matrix [rows][256] tiled as 64 x 128 boxes with the 128-byte swizzle
// (one K block of a K-major tcgen05 operand per box).
bool make_k256_map(CUtensorMap *m, const void *base, long long rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kDx, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kDx * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

s5_status cuda_status(cudaError_t e) { return e == cudaSuccess ? S5_OK : S5_ERR_CUDA; }

// kv8: the pools hold one-byte E4M3 codes (K value = k_scale * code value,
// V value = v_scale * code value); every row then takes the per-row kernel.
s5_status attn_common(int mode, const s5_kv_desc *kv, const s5_batch_desc *b, const void *q, const int32_t *sel,
                      const int32_t *sel_count, int32_t topk, int32_t window, float sm_scale, void *out,
                      float *lse, void *ws, size_t ws_bytes, cudaStream_t stream, int sel_groups = 1,
                      bool kv8 = false, float k_scale = 1.f, float v_scale = 1.f) {
  s5_status st = check_batch(b);
  if (st != S5_OK) return st;
  if ((st = check_kv(kv)) != S5_OK) return st;
  if (!std::isfinite(sm_scale)) return S5_ERR_INVALID_ARG;
  if (kv8 && (!std::isfinite(k_scale) || !std::isfinite(v_scale) || !std::isfinite(sm_scale * k_scale)))
    return S5_ERR_INVALID_ARG;
  if (mode == kModeSparse && (topk < 1 || topk > kMaxTopk)) return S5_ERR_INVALID_ARG;
  if (mode == kModeSwa && window < 1) return S5_ERR_INVALID_ARG;
  if (ws == nullptr) return S5_ERR_WORKSPACE;
  if (b->total_q == 0) return S5_OK;
  if (q == nullptr || out == nullptr || !aligned16(q) || !aligned16(out)) return S5_ERR_INVALID_ARG;
  if (mode == kModeSparse && (sel == nullptr || sel_count == nullptr)) return S5_ERR_INVALID_ARG;
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  const int bpr = (mode == kModeSparse) ? sparse_blocks_per_row(topk) : swa_blocks_per_row(b, window);
  const AttnWs w = attn_ws(b, bpr, device_slots());
  if (ws_bytes < w.end) return S5_ERR_WORKSPACE;
  CUtensorMap tk, tv;
  if (kv8) {
    if (!make_kv8_map(&tk, kv->k_pool, kv->num_pages) || !make_kv8_map(&tv, kv->v_pool, kv->num_pages))
      return S5_ERR_CUDA;
  } else if (!make_kv_map(&tk, kv->k_pool, kv->num_pages) || !make_kv_map(&tv, kv->v_pool, kv->num_pages)) {
    return S5_ERR_CUDA;
  }
  AttnArgs a{};
  a.q = q;
  a.sel = sel;
  a.sel_count = sel_count;
  a.sel_groups = sel_groups;
  a.topk = topk;
  a.window = window;
  a.page_table = b->page_table;
  a.max_pages = b->max_pages;
  a.ctx_lens = b->ctx_lens;
  a.cu_q = b->cu_q;
  a.batch = b->batch;
  a.total_q = b->total_q;
  a.max_len = b->max_len;
  a.num_pages = kv->num_pages;
  a.scale_log2 = (kv8 ? sm_scale * k_scale : sm_scale) * 1.4426950408889634f;
  a.kv8 = kv8 ? 1 : 0;
  a.v_scale = kv8 ? v_scale : 1.f;
  a.n_split = w.n_split;
  a.out = out;
  a.lse = lse;
  a.part_o = reinterpret_cast<float *>(wsb + w.part_o);
  a.part_lse = reinterpret_cast<float *>(wsb + w.part_lse);
  a.merge_cnt = (b->total_q <= kMaxMergeRows) ? reinterpret_cast<uint32_t *>(wsb + kWsHeader) : nullptr;
  a.row_skip = nullptr;
  a.err = reinterpret_cast<int32_t *>(ws);

  // (one selection per KV group, or one-byte KV: every row takes the per-row kernel)
  if (mode == kModeSparse && sel_groups == 1 && !kv8 && use_tiles(b)) {
    if (b->batch > kMaxGridYZ) return S5_ERR_UNSUPPORTED;  // the union kernel's grid.y
    // union lists and per-tile choice, then the shared-set tiles; the per-row
    // kernel below skips the rows those tiles computed
    const TileWs tw = tile_ws(b, topk, device_slots() / kCtasPerSm, false, w.end);
    if (ws_bytes < tw.end) return S5_ERR_WORKSPACE;
    CUtensorMap tpk, tpv;
    if (!make_kv_plane_map(&tpk, kv->k_pool, kv->num_pages) || !make_kv_plane_map(&tpv, kv->v_pool, kv->num_pages))
      return S5_ERR_CUDA;
    TileArgs t{};
    t.q = q;
    t.sel = sel;
    t.sel_count = sel_count;
    t.topk = topk;
    t.page_table = b->page_table;
    t.max_pages = b->max_pages;
    t.ctx_lens = b->ctx_lens;
    t.cu_q = b->cu_q;
    t.batch = b->batch;
    t.total_q = b->total_q;
    t.num_pages = kv->num_pages;
    t.scale_log2 = a.scale_log2;
    t.tiles_per_seq = tw.tiles_per_seq;
    t.n_tiles = tw.n_tiles;
    t.n_split = tw.n_split;
    t.map_words = tw.map_words;
    t.union_cap = tw.union_cap;
    t.union_count = reinterpret_cast<int *>(wsb + tw.count);
    t.union_ent = reinterpret_cast<uint32_t *>(wsb + tw.ent);
    t.out = out;
    t.lse = lse;
    t.part_o = reinterpret_cast<float *>(wsb + tw.part_o);
    t.part_lse = reinterpret_cast<float *>(wsb + tw.part_lse);
    t.merge_cnt = reinterpret_cast<uint32_t *>(wsb + kWsHeader);
    t.union_pct = kTileUnionPct;
    t.tile_on = reinterpret_cast<int32_t *>(wsb + tw.tile_on);
    t.row_skip = reinterpret_cast<int32_t *>(wsb + tw.row_skip);
    t.err = a.err;
    if (launch_tile_union(t, b->batch, stream) != cudaSuccess) return S5_ERR_CUDA;
    if (launch_gqa_tile(t, tpk, tpv, device_slots() / kCtasPerSm, stream) != cudaSuccess) return S5_ERR_CUDA;
    a.row_skip = t.row_skip;
  }
  // a grid of at most one CTA per SM takes the variant with the deeper ring
  const bool deep = (long long)a.n_split * b->total_q * kKv <= device_slots() / kCtasPerSm;
  return cuda_status(launch_gqa_decode(mode, a, tk, tv, b->total_q, deep, stream));
}

// Workspace of every call for this batch, with `groups` indexer queries and
// selections per token (1: shared; 4: one per KV group).
s5_status workspace_need(const s5_batch_desc *batch, int32_t window, int groups, size_t *bytes) {
  if (bytes == nullptr) return S5_ERR_INVALID_ARG;
  s5_status st = check_batch(batch);
  if (st != S5_OK) return st;
  if (window < 0) return S5_ERR_INVALID_ARG;
  size_t need = index_ws(batch, 1).end;
  if (groups > 1) {
    const size_t ng = index_ws(batch, groups).end;
    if (ng > need) need = ng;
  }
  const int slots = kCtasPerSm * kSizingSms;  // an upper bound: no device query here
  size_t sp = attn_ws(batch, sparse_blocks_per_row(kMaxTopk), slots).end;
  if (use_tiles(batch)) sp = tile_ws(batch, kMaxTopk, kSizingSms, true, sp).end;
  if (sp > need) need = sp;
  if (window > 0) {
    const size_t sw = attn_ws(batch, swa_blocks_per_row(batch, window), slots).end;
    if (sw > need) need = sw;
  }
  *bytes = need;
  return S5_OK;
}

// Block scores and top-k for `groups` indexer queries per token: q_index
// [total_q][groups][256], one selection per (token, group) row.
s5_status index_common(const s5_index_desc *index, const s5_batch_desc *batch, const void *q_index, int32_t topk,
                       int32_t *sel, int32_t *sel_count, void *workspace, size_t workspace_bytes,
                       s5_stream_t stream, int groups, bool key_fp8 = false) {
  s5_status st = check_batch(batch);
  if (st != S5_OK) return st;
  if (index == nullptr || index->key_pool == nullptr || index->num_pages < 1) return S5_ERR_INVALID_ARG;
  if (index->index_dim != kDx) return S5_ERR_UNSUPPORTED;
  if (!aligned16(index->key_pool)) return S5_ERR_INVALID_ARG;
  if (topk < 1 || topk > kMaxTopk) return S5_ERR_INVALID_ARG;
  if (workspace == nullptr) return S5_ERR_WORKSPACE;
  if (batch->total_q == 0) return S5_OK;
  if (q_index == nullptr || sel == nullptr || sel_count == nullptr || !aligned16(q_index))
    return S5_ERR_INVALID_ARG;
  if (batch->batch > kMaxGridYZ) return S5_ERR_UNSUPPORTED;  // sequences index grid.y / grid.z
  const long long rows = (long long)batch->total_q * groups;
  const IndexWs w = index_ws(batch, groups);
  if (w.two_stage && rows > 65535) return S5_ERR_UNSUPPORTED;  // stage 1 has one grid row per selection
  if (workspace_bytes < w.end) return S5_ERR_WORKSPACE;
  uint8_t *wsb = static_cast<uint8_t *>(workspace);
  int32_t *err = reinterpret_cast<int32_t *>(workspace);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

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
  ia.q_groups = groups;
  ia.key_fp8 = key_fp8 ? 1 : 0;
  ia.scores = reinterpret_cast<float *>(wsb + w.scores);
  ia.score_stride = w.stride;
  ia.pages_per_cta = kScorePagesPerCta;
  ia.topk = topk;
  ia.hist = w.hist_bytes ? reinterpret_cast<uint32_t *>(wsb + w.hist) : nullptr;
  ia.err = err;
  if (ia.hist != nullptr && cudaMemsetAsync(ia.hist, 0, w.hist_bytes, cs) != cudaSuccess) return S5_ERR_CUDA;
  if (w.kxs_bytes > 0) {
    // prefill-sized: gather each sequence's keys, then tensor-core GEMM
    GatherArgs ga{};
    ga.key_pool = index->key_pool;
    ga.num_pages = index->num_pages;
    ga.page_table = batch->page_table;
    ga.max_pages = batch->max_pages;
    ga.kxs = wsb + w.kxs;
    ga.max_blocks = w.stride;
    ga.key_fp8 = key_fp8 ? 1 : 0;
    if (launch_gather_keys(ga, batch->batch, cs) != cudaSuccess) return S5_ERR_CUDA;
    CUtensorMap tq, tk;
    if (!make_k256_map(&tq, q_index, rows) || !make_k256_map(&tk, ga.kxs, (long long)batch->batch * w.stride))
      return S5_ERR_CUDA;
    GemmArgs gm{};
    gm.ctx_lens = batch->ctx_lens;
    gm.cu_q = batch->cu_q;
    gm.batch = batch->batch;
    gm.total_q = batch->total_q;
    gm.q_groups = groups;
    gm.scores = ia.scores;
    gm.score_stride = w.stride;
    gm.max_blocks = w.stride;
    gm.tiles_per_cta = kGemmTilesPerCta;
    gm.err = err;
    if (launch_index_gemm(gm, tq, tk, batch->batch, batch->max_q * groups, cs) != cudaSuccess) return S5_ERR_CUDA;
  } else {
    const int pages = (w.stride + kBpp - 1) / kBpp;
    // 64 pages (256 KB of keys) per CTA, or fewer when that leaves the SMs
    // idle: a small batch is spread over at least two CTAs per SM
    const long long row_tiles = ((long long)batch->max_q * groups + 3) / 4;
    const long long want = 2LL * (device_slots() / kCtasPerSm);
    long long ppc = kScorePagesPerCta;
    const long long ctas64 = (long long)((pages + kScorePagesPerCta - 1) / kScorePagesPerCta) * batch->batch * row_tiles;
    if (ctas64 < want) {
      ppc = ((long long)pages * batch->batch * row_tiles + want - 1) / want;
      ppc = ppc < kScoreMinPagesPerCta ? kScoreMinPagesPerCta : (ppc > kScorePagesPerCta ? kScorePagesPerCta : ppc);
    }
    ia.pages_per_cta = (int)ppc;
    const int grid_pages = (int)((pages + ppc - 1) / ppc);
    if (launch_index_score(ia, batch->max_q * groups, grid_pages, batch->batch, cs) != cudaSuccess)
      return S5_ERR_CUDA;
  }

  SelectArgs sa{};
  sa.scores = ia.scores;
  sa.score_stride = w.stride;
  sa.ctx_lens = batch->ctx_lens;
  sa.cu_q = batch->cu_q;
  sa.batch = batch->batch;
  sa.total_q = batch->total_q;
  sa.q_groups = groups;
  sa.topk = topk;
  sa.sel = sel;
  sa.sel_count = sel_count;
  sa.seg = w.seg;
  sa.n_seg = w.n_seg;
  sa.cand_key = reinterpret_cast<uint32_t *>(wsb + w.cand_key);
  sa.cand_idx = reinterpret_cast<int32_t *>(wsb + w.cand_idx);
  sa.hist = ia.hist;
  sa.err = err;
  return cuda_status(launch_topk_select(sa, (int)rows, w.two_stage, cs));
}

}  // namespace

extern "C" {

s5_status s5_workspace_size(const s5_batch_desc *batch, int32_t window, size_t *bytes) {
  return workspace_need(batch, window, 1, bytes);
}

s5_status s5_workspace_size_grouped(const s5_batch_desc *batch, int32_t window, size_t *bytes) {
  return workspace_need(batch, window, kKv, bytes);
}

s5_status s5_index_score_topk(const s5_index_desc *index, const s5_batch_desc *batch, const void *q_index,
                              int32_t topk, int32_t *sel, int32_t *sel_count, void *workspace,
                              size_t workspace_bytes, s5_stream_t stream) {
  return index_common(index, batch, q_index, topk, sel, sel_count, workspace, workspace_bytes, stream, 1);
}

s5_status s5_index_score_topk_fp8(const s5_index_desc *index, const s5_batch_desc *batch, const void *q_index,
                                  int32_t topk, int32_t *sel, int32_t *sel_count, void *workspace,
                                  size_t workspace_bytes, s5_stream_t stream) {
  return index_common(index, batch, q_index, topk, sel, sel_count, workspace, workspace_bytes, stream, 1, true);
}

s5_status s5_index_score_topk_grouped(const s5_index_desc *index, const s5_batch_desc *batch, const void *q_index,
                                      int32_t topk, int32_t *sel, int32_t *sel_count, void *workspace,
                                      size_t workspace_bytes, s5_stream_t stream) {
  return index_common(index, batch, q_index, topk, sel, sel_count, workspace, workspace_bytes, stream, kKv);
}

s5_status s5_sparse_gqa_attn(const s5_kv_desc *kv, const s5_batch_desc *batch, const void *q, const int32_t *sel,
                             const int32_t *sel_count, int32_t topk, float sm_scale, void *out, float *lse,
                             void *workspace, size_t workspace_bytes, s5_stream_t stream) {
  return attn_common(kModeSparse, kv, batch, q, sel, sel_count, topk, 0, sm_scale, out, lse, workspace,
                     workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

s5_status s5_sparse_gqa_attn_grouped(const s5_kv_desc *kv, const s5_batch_desc *batch, const void *q,
                                     const int32_t *sel, const int32_t *sel_count, int32_t topk, float sm_scale,
                                     void *out, float *lse, void *workspace, size_t workspace_bytes,
                                     s5_stream_t stream) {
  return attn_common(kModeSparse, kv, batch, q, sel, sel_count, topk, 0, sm_scale, out, lse, workspace,
                     workspace_bytes, reinterpret_cast<cudaStream_t>(stream), kKv);
}

s5_status s5_sparse_gqa_attn_fp8kv(const s5_kv_desc *kv, const s5_batch_desc *batch, const void *q,
                                   const int32_t *sel, const int32_t *sel_count, int32_t topk, float sm_scale,
                                   float k_scale, float v_scale, void *out, float *lse, void *workspace,
                                   size_t workspace_bytes, s5_stream_t stream) {
  return attn_common(kModeSparse, kv, batch, q, sel, sel_count, topk, 0, sm_scale, out, lse, workspace,
                     workspace_bytes, reinterpret_cast<cudaStream_t>(stream), 1, true, k_scale, v_scale);
}

s5_status s5_swa_gqa_attn(const s5_kv_desc *kv, const s5_batch_desc *batch, const void *q, int32_t window,
                          float sm_scale, void *out, float *lse, void *workspace, size_t workspace_bytes,
                          s5_stream_t stream) {
  return attn_common(kModeSwa, kv, batch, q, nullptr, nullptr, 0, window, sm_scale, out, lse, workspace,
                     workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

s5_status s5_reset_device_error(void *workspace, s5_stream_t stream) {
  if (workspace == nullptr) return S5_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(workspace, 0, kWsFixed, reinterpret_cast<cudaStream_t>(stream)));
}

s5_status s5_get_device_error(void *workspace, s5_stream_t stream, int32_t *code, int32_t *info) {
  if (workspace == nullptr || code == nullptr || info == nullptr) return S5_ERR_INVALID_ARG;
  ErrRec rec{};
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(&rec, workspace, sizeof(rec), cudaMemcpyDeviceToHost, cs);
  if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
  if (e != cudaSuccess) return S5_ERR_CUDA;
  *code = rec.code;
  *info = rec.code ? rec.info : -1;
  return S5_OK;
}

const char *s5_status_string(s5_status status) {
  switch (status) {
    case S5_OK: return "S5_OK";
    case S5_ERR_INVALID_ARG: return "S5_ERR_INVALID_ARG: bad pointer, size or descriptor field";
    case S5_ERR_UNSUPPORTED: return "S5_ERR_UNSUPPORTED: outside what this build implements";
    case S5_ERR_CUDA: return "S5_ERR_CUDA: a CUDA launch or runtime call failed";
    case S5_ERR_DEVICE_BOUNDS: return "S5_ERR_DEVICE_BOUNDS: device data out of range";
    case S5_ERR_TIMEOUT: return "S5_ERR_TIMEOUT: a bounded in-kernel wait expired";
    case S5_ERR_WORKSPACE: return "S5_ERR_WORKSPACE: workspace missing or too small";
  }
  return "S5_ERR_UNKNOWN";
}

int32_t s5_abi_version(void) { return kAbiVersion; }

}  // extern "C"
