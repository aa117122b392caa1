// Internal interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace s5 {

constexpr int kModeSparse = 0;
constexpr int kModeSwa = 1;
constexpr int kMaxList = 544;  // blocks one attention CTA may own (>= 512 + 1)
constexpr int kMaxMergeRows = 1024;  // rows whose partitions merge inside the attention kernel

struct IndexScoreArgs {
  const void *key_pool;
  int num_pages;
  const int32_t *page_table;
  int max_pages;
  const int32_t *ctx_lens;
  const int32_t *cu_q;
  int batch;
  int total_q;
  const void *q_index;  // bf16 [total_q][q_groups][256]
  float *scores;     // [total_q * q_groups][score_stride]
  int score_stride;  // >= history blocks of any row
  int pages_per_cta;
  int topk;
  uint32_t *hist;  // [total_q * q_groups][4096] counts of score keys by their top 12 bits (zeroed before), or null
  int32_t *err;
  int q_groups;  // indexer queries per token (0 or 1: one shared query; 4: one per KV group)
  int key_fp8;   // nonzero: key_pool holds one-byte E4M3 codes [num_pages][8][256]
};

constexpr int kHistBins = 4096;  // row histogram of the top 12 bits of the score keys

struct SelectArgs {
  const float *scores;
  int score_stride;
  const int32_t *ctx_lens;
  const int32_t *cu_q;
  int batch;
  int total_q;
  int topk;
  int32_t *sel;        // [total_q * q_groups][topk]
  int32_t *sel_count;  // [total_q * q_groups]
  // two-stage select
  int seg;    // blocks per segment
  int n_seg;  // segments per row (stride of the candidate arrays)
  uint32_t *cand_key;
  int32_t *cand_idx;
  const uint32_t *hist;  // row histograms built by the scoring kernel, or null
  int32_t *err;
  int q_groups;  // selections per token: 0 or 1, or 4 (row r belongs to token r / 4)
};

struct AttnArgs {
  const void *q;
  const int32_t *sel;        // [total_q][sel_groups][topk]
  const int32_t *sel_count;  // [total_q][sel_groups]
  int sel_groups;            // 0 or 1: one selection per token; 4: one per KV group
  int topk;
  int window;
  const int32_t *page_table;
  int max_pages;
  const int32_t *ctx_lens;
  const int32_t *cu_q;
  int batch;
  int total_q;
  int max_len;
  int num_pages;
  float scale_log2;  // sm_scale * log2(e)
  int n_split;
  void *out;
  float *lse;
  float *part_o;    // [total_q * 64][n_split][192]
  float *part_lse;  // [total_q * 64][n_split]   (base-2)
  uint32_t *merge_cnt;  // [total_q * 4] arrival counters (zero between calls), or null: separate merge kernel
  const int32_t *row_skip;  // [total_q]: nonzero for rows the shared-set tile kernel computes, or null
  int32_t *err;
  int kv8;        // nonzero: K / V pools hold one-byte E4M3 codes (sparse mode only)
  float v_scale;  // one-byte KV: value of a V code = v_scale * E4M3(code) (k_scale is in scale_log2)
};

// Prefill-sized batches: block keys gathered per sequence, then a tcgen05 GEMM.
struct GatherArgs {
  const void *key_pool;
  int num_pages;
  const int32_t *page_table;
  int max_pages;
  void *kxs;       // bf16 [batch][max_blocks][256]
  int max_blocks;  // rows per sequence in kxs
  int key_fp8;     // nonzero: key_pool holds one-byte E4M3 codes, widened to bf16 in kxs
};

struct GemmArgs {
  const int32_t *ctx_lens;
  const int32_t *cu_q;
  int batch;
  int total_q;
  int q_groups;   // indexer queries per token (0 or 1, or 4); rows token-major, group-minor
  float *scores;  // [total_q * q_groups][score_stride]
  int score_stride;
  int max_blocks;     // rows per sequence of the gathered keys
  int tiles_per_cta;  // 128-block N tiles per CTA
  int32_t *err;
};

// Multi-row tiles (verify / prefill): shared-set attention on the tensor cores.
constexpr int kTileRows = 8;           // query rows per shared-set tile (8 rows x 16 heads = M 128)
constexpr int kMaxTileSplit = 8;      // partitions of one tile's block list
constexpr int kUnionMapWords = 49152;  // shared byte map of the union kernel: blocks < 196,608

struct TileArgs {
  const void *q;
  const int32_t *sel;
  const int32_t *sel_count;
  int topk;
  const int32_t *page_table;
  int max_pages;
  const int32_t *ctx_lens;
  const int32_t *cu_q;
  int batch;
  int total_q;
  int num_pages;
  float scale_log2;
  int tiles_per_seq;   // ceil(max_q / kTileRows)
  int n_tiles;         // batch * tiles_per_seq
  int n_split;         // partitions of a tile's block list
  int map_words;       // 32-bit words of the union kernel's byte map (one byte per block)
  int union_cap;       // entries per tile in the union lists
  int *union_count;    // [n_tiles]
  uint32_t *union_ent; // [n_tiles][union_cap]
  void *out;
  float *lse;
  float *part_o;
  float *part_lse;
  uint32_t *merge_cnt;
  int union_pct;       // a tile takes the shared-set path when 100 * |union| <= union_pct * sum of rows' blocks
  int32_t *tile_on;    // [n_tiles] written by the union kernel: 1 = shared-set path
  int32_t *row_skip;   // [total_q] written by the union kernel: 1 = row computed by the tile kernel
  int32_t *err;
};

// cudaFuncSetAttribute(kernel, MaxDynamicSharedMemorySize, bytes) on the
// current device, skipped when an equal or larger value is already set there
// (the host cost of a call stays off the launch path of small batches).
cudaError_t ensure_dynamic_smem(const void *kernel, int bytes);

cudaError_t launch_tile_union(const TileArgs &a, int batch, cudaStream_t st);
cudaError_t launch_gqa_tile(const TileArgs &a, const CUtensorMap &tk, const CUtensorMap &tv, int n_ctas,
                            cudaStream_t st);

cudaError_t launch_index_score(const IndexScoreArgs &a, int max_q, int grid_pages, int n_seq, cudaStream_t st);
cudaError_t launch_gather_keys(const GatherArgs &a, int batch, cudaStream_t st);
cudaError_t launch_index_gemm(const GemmArgs &a, const CUtensorMap &tq, const CUtensorMap &tk, int batch, int max_q,
                              cudaStream_t st);
cudaError_t launch_topk_select(const SelectArgs &a, int total_q, bool two_stage, cudaStream_t st);
// deep: the variant with twice the ring stages per warp (one CTA per SM), for
// grids that fit on the SMs one CTA each
cudaError_t launch_gqa_decode(int mode, const AttnArgs &a, const CUtensorMap &tk, const CUtensorMap &tv,
                              int total_q, bool deep, cudaStream_t st);

}  // namespace s5
