// Sparse attention for multi-token verify and chunked prefill on the
// 5th-generation tensor cores, over the shared set of selected blocks.
//
// SGLang day-0 blog ("Step 5 Preview: Day-0 Inference and RL Support with
// SGLang and Miles"), "Kernels from StepFun": sparse prefill gathers the blocks
// selected for a batch of queries into one shared set and runs attention over
// that set with per-query masks.  Here the batch is a tile of up to 4
// consecutive query rows of one sequence (the 4 tokens of a verify step, or 4
// neighbouring prefill tokens):
//
//   tile_union_kernel   builds, per tile, the ascending list of distinct blocks
//                       the tile's rows read (selected history blocks and the
//                       rows' current blocks), each entry carrying which rows
//                       read all 8 of its tokens and which read it causally;
//   gqa_tile_kernel     one CTA per (tile, KV group, partition of that list):
//                       the 4 rows x 16 heads of the group are the M = 64 rows
//                       of tcgen05 MMAs.  Warp 4 streams 8-block chunks of K
//                       and V by TMA; warp 5 issues S = Q K^T (M=64, N=64,
//                       K=192) into two tensor-memory buffers and
//                       O += P V (M=64, N=192, K=64) into a tensor-memory
//                       accumulator; warps 0-3 (warp w = row w of the tile)
//                       mask, run the online softmax with lazy rescaling of O,
//                       and write P as the bf16 A operand of the next MMA.
//
// Each shared block is read once for the tile instead of once per row; the
// masked-out products are the price of dense tiles.
#include <cuda.h>

#include "s5_common.cuh"
#include "s5_kernels.h"
#include "s5_tcgen05.cuh"

namespace s5 {

constexpr int kTRows = 4;                 // query rows per tile
constexpr int kTM = kTRows * kHpg;        // 64 MMA rows
constexpr int kTChunkBlocks = 8;          // blocks per chunk
constexpr int kTN = kTChunkBlocks * kBlk; // 64 tokens per chunk
constexpr int kTStages = 3;
constexpr int kTQBytes = 3 * kTM * 128;                       // [3 K-blocks][64 rows][128 B]
constexpr int kTKvBytes = kTChunkBlocks * kBlockBytes;        // K (or V) of one chunk
constexpr int kTStageBytes = 2 * kTKvBytes;                   // K then V
constexpr int kTPBytes = kTM * 128;                           // P: [64 rows][64 tokens] bf16
constexpr int kTPBufs = 3;                                    // P buffers (chunk c uses c % 3)
constexpr int kTThreads = 192;
constexpr uint32_t kTTmemCols = 512;                          // S0 [0,64), S1 [64,128), O [128,320)
constexpr uint64_t kTWaitNs = 2000000000ull;
constexpr float kLazyRescale = 8.0f;                          // log2 units

// ---------------------------------------------------------------- union lists

// Entry: block (bits 0..23) | rows reading all 8 tokens << 24 | rows reading it
// as their current block << 28.
__global__ void __launch_bounds__(256) tile_union_kernel(const TileArgs a) {
  extern __shared__ uint32_t bm[];  // [4 rows][words]
  __shared__ int cur_blk[kTRows];
  __shared__ int scan[32];
  const int s = blockIdx.y, k = blockIdx.x;
  const int tile = s * a.tiles_per_seq + k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int q_beg = ld_cg(a.cu_q + s);
  const int nq = ld_cg(a.cu_q + s + 1) - q_beg;
  const int ctx = ld_cg(a.ctx_lens + s);
  int *count = a.union_count + tile;
  uint32_t *ent = a.union_ent + (size_t)tile * a.union_cap;
  const int r0 = q_beg + k * kTRows;
  const int nr = min(kTRows, nq - k * kTRows);
  if (nr <= 0) {
    if (tid == 0) {
      *count = 0;
      a.tile_on[tile] = 0;
    }
    return;
  }
  const int c_last = (ctx + k * kTRows + nr - 1) / kBlk;  // largest current block of the tile
  const int words = c_last / 32 + 1;
  if (ctx < 0 || r0 + nr > a.total_q || words > a.bitmap_words) {
    if (tid == 0) {
      record_error(a.err, S5_ERR_DEVICE_BOUNDS, max(r0, 0));
      *count = 0;
      a.tile_on[tile] = 0;
      for (int j = 0; j < nr; ++j)
        if (r0 + j >= 0 && r0 + j < a.total_q) a.row_skip[r0 + j] = 0;
    }
    return;
  }
  for (int i = tid; i < kTRows * words; i += 256) bm[i] = 0;
  if (tid < kTRows) cur_blk[tid] = (tid < nr) ? (ctx + k * kTRows + tid) / kBlk : -1;
  __syncthreads();
  int row_blocks = 0;  // sum over the tile's rows of (selected blocks + current block)
  for (int j = 0; j < nr; ++j) {
    const int r = r0 + j;
    const int c = (ctx + k * kTRows + j) / kBlk;
    int n = ld_cg(a.sel_count + r);
    if (n < 0 || n > a.topk || n > c) {
      if (tid == 0) record_error(a.err, S5_ERR_DEVICE_BOUNDS, r);
      n = 0;
    }
    row_blocks += n + 1;
    for (int i = tid; i < n; i += 256) {
      const int b = ld_cg(a.sel + (size_t)r * a.topk + i);
      if (b >= 0 && b < c) atomicOr(bm + j * words + (b >> 5), 1u << (b & 31));
      else record_error(a.err, S5_ERR_DEVICE_BOUNDS, r);
    }
  }
  __syncthreads();
  // ascending compaction of the union of the 4 bitmaps and the current blocks
  const int per = (words + 255) / 256;  // words per thread, in order
  int cnt = 0;
  for (int w = tid * per; w < min(words, tid * per + per); ++w) {
    uint32_t u = 0;
    for (int j = 0; j < kTRows; ++j) u |= bm[j * words + w];
    for (int j = 0; j < nr; ++j)
      if ((cur_blk[j] >> 5) == w) u |= 1u << (cur_blk[j] & 31);
    cnt += __popc(u);
  }
  // exclusive scan of per-thread counts
  int incl = cnt;
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) scan[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int x = (lane < 8) ? scan[lane] : 0;
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += o;
    }
    if (lane < 8) scan[lane] = x;
  }
  __syncthreads();
  int pos = (warp > 0 ? scan[warp - 1] : 0) + incl - cnt;
  const int total = scan[7];
  for (int w = tid * per; w < min(words, tid * per + per); ++w) {
    uint32_t u = 0;
    for (int j = 0; j < kTRows; ++j) u |= bm[j * words + w];
    for (int j = 0; j < nr; ++j)
      if ((cur_blk[j] >> 5) == w) u |= 1u << (cur_blk[j] & 31);
    while (u != 0) {
      const int bit = __ffs(u) - 1;
      u &= u - 1;
      const int b = w * 32 + bit;
      uint32_t full = 0, cur = 0;
      for (int j = 0; j < nr; ++j) {
        if (bm[j * words + w] & (1u << bit)) full |= 1u << j;
        if (cur_blk[j] == b) cur |= 1u << j;
      }
      if (pos < a.union_cap) ent[pos] = (uint32_t)b | (full << 24) | (cur << 28);
      ++pos;
    }
  }
  if (tid == 0) {
    *count = min(total, a.union_cap);
    // per-tile crossover: the shared set pays when the rows' selections overlap
    const int on = (100LL * total <= (long long)a.union_pct * row_blocks) ? 1 : 0;
    a.tile_on[tile] = on;
    for (int j = 0; j < nr; ++j) a.row_skip[r0 + j] = on;
  }
}

// ---------------------------------------------------------------- attention tiles

// byte offset of element (row, col) of a K-major 128-byte-swizzled [rows][64] bf16 tile
__device__ __forceinline__ uint32_t sw128(int row, int col) {
  const uint32_t off = (uint32_t)(row * 128 + col * 2);
  return off ^ (((off >> 7) & 7u) << 4);
}

// Merge weights of the partitions of one (row, head): the same arithmetic as
// the decode kernel's merge, in partition order.
__device__ __forceinline__ void tile_partition_weights(const float *pl, int n, float *w, float &lse_nat) {
  float M = -INFINITY;
  for (int p = 0; p < n; ++p) M = fmaxf(M, ld_cg(pl + p));
  const float Mu = (M == -INFINITY) ? 0.f : M;
  float L = 0.f;
  for (int p = 0; p < n; ++p) {
    const float lp = ld_cg(pl + p);
    L += (lp == -INFINITY) ? 0.f : hw_exp2(lp - Mu);
  }
  const float inv = (L > 0.f) ? 1.f / L : 0.f;
  for (int p = 0; p < n; ++p) {
    const float lp = ld_cg(pl + p);
    w[p] = (lp == -INFINITY) ? 0.f : hw_exp2(lp - Mu) * inv;
  }
  lse_nat = (L > 0.f) ? (M + hw_log2(L)) * 0.69314718055994531f : -INFINITY;
}

__global__ void __launch_bounds__(kTThreads, 1)
    gqa_tile_kernel(const TileArgs a, const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sq = smem;                                   // Q tile
  uint8_t *skv = sq + kTQBytes;                         // K/V stages
  uint8_t *sp = skv + kTStages * kTStageBytes;          // P buffers [3]
  int32_t *erow = reinterpret_cast<int32_t *>(sp + kTPBufs * kTPBytes);  // TMA row per entry (-1: absent)
  uint32_t *eent = reinterpret_cast<uint32_t *>(erow + kMaxTileEntries);
  uint64_t *bars = reinterpret_cast<uint64_t *>(eent + kMaxTileEntries);
  uint64_t *bar_q = bars + 0;
  uint64_t *bar_kv_full = bars + 1;    // [3]
  uint64_t *bar_kv_empty = bars + 4;   // [3]
  uint64_t *bar_s_full = bars + 7;     // [2]
  uint64_t *bar_s_empty = bars + 9;    // [2]
  uint64_t *bar_p_full = bars + 11;    // [3] P_c written (chunk c uses buffer c % 3)
  uint64_t *bar_p_free = bars + 14;    // [3] PV_c done: P buffer c % 3 and O through chunk c
  uint64_t *bar_final = bars + 17;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 18);
  int *abort_flag = reinterpret_cast<int *>(bars + 19);
  int *is_last = abort_flag + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // flattened grid: partition fastest, then tile, then group
  const int p = blockIdx.x % a.n_split;
  const int tg = blockIdx.x / a.n_split;
  const int tile = tg % a.n_tiles;
  const int g = tg / a.n_tiles;
  pdl_wait();  // (no-op for an ordinary launch) every global read below follows it

  // ---- the tile ----
  const int s = tile / a.tiles_per_seq, k = tile % a.tiles_per_seq;
  const int q_beg = ld_cg(a.cu_q + s);
  const int nq = ld_cg(a.cu_q + s + 1) - q_beg;
  const int ctx = ld_cg(a.ctx_lens + s);
  const int r0 = q_beg + k * kTRows;
  const int nr = max(0, min(kTRows, nq - k * kTRows));
  if (nr == 0) return;  // a tile slot past this sequence's rows
  if (ld_cg(a.tile_on + tile) == 0) return;  // the per-row kernel computes this tile's rows
  const int n_ent = ld_cg(a.union_count + tile);

  if (warp == 0) tc::tmem_alloc(tmem_slot, kTTmemCols);
  if (tid == 0) {
    mbar_init(bar_q, 1);
    for (int i = 0; i < kTStages; ++i) {
      mbar_init(bar_kv_full + i, 1);
      mbar_init(bar_kv_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_s_full + i, 1);
      mbar_init(bar_s_empty + i, 4);
    }
    for (int i = 0; i < kTPBufs; ++i) {
      mbar_init(bar_p_full + i, 4);
      mbar_init(bar_p_free + i, 1);
    }
    mbar_init(bar_final, 1);
    *abort_flag = 0;
  }
  fence_mbar_init();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int chunk_e = ((n_ent + a.n_split - 1) / a.n_split + kTChunkBlocks - 1) / kTChunkBlocks * kTChunkBlocks;
  const int e0 = min(n_ent, p * chunk_e);
  const int ne = min(n_ent, e0 + chunk_e) - e0;  // this CTA's entries (<= kMaxTileEntries: host sizes n_split)
  const int n_chunks = (ne + kTChunkBlocks - 1) / kTChunkBlocks;
  const int32_t *pt = a.page_table + (size_t)s * a.max_pages;
  // resolve entries to TMA rows
  for (int i = tid; i < n_chunks * kTChunkBlocks; i += kTThreads) {
    int row = -1;
    uint32_t e = 0;
    if (i < ne) {
      e = ld_cg(a.union_ent + (size_t)tile * a.union_cap + e0 + i);
      const int b = (int)(e & 0xFFFFFFu);
      const int pg = b / kBpp;
      const int ph = (pg < a.max_pages) ? ld_cg(pt + pg) : -1;
      if (ph >= 0 && ph < a.num_pages) row = ((ph * kKv + g) * kPage) + (b % kBpp) * kBlk;
      else record_error(a.err, S5_ERR_DEVICE_BOUNDS, r0);
    }
    erow[i] = row;
    eent[i] = (row >= 0) ? e : 0u;
  }
  __syncthreads();

  auto wait = [&](uint64_t *bar, uint32_t parity) -> bool {
    if (*reinterpret_cast<volatile int *>(abort_flag)) return false;
    if (mbar_wait_bounded(bar, parity, kTWaitNs)) return true;
    *reinterpret_cast<volatile int *>(abort_flag) = 1;
    record_error(a.err, S5_ERR_TIMEOUT, max(r0, 0));
    return false;
  };

  if (warp == 4) {
    // ---------------- TMA producer ----------------
    // A chunk is 8 blocks x (K, V): 16 copies of one whole block (3 planes of
    // 1 KB), issued in parallel by lanes 0..15 (lane = 8 * tensor + block);
    // lane 0 keeps the barrier bookkeeping.
    if (n_chunks > 0) {
      if (lane == 0) {
        // Q: rows (query j, head 16g + h) -> smem row 16j + h; 3 K-blocks of 64 dims
        mbar_arrive_expect_tx(bar_q, kTQBytes);
        for (int j = 0; j < kTRows; ++j)
          for (int cb = 0; cb < 3; ++cb)
            tma_load_2d(sq + cb * kTM * 128 + j * kHpg * 128, &tm_q, cb * 64,
                        (min(r0 + j, a.total_q - 1)) * kHeads + g * kHpg, bar_q);
      }
      const uint64_t policy = policy_evict_normal();
      const int lb = lane & 7, lt = (lane >> 3) & 1;  // block and tensor (0 = K, 1 = V) of this lane
      int issued = 0;
      for (int c = 0; c < n_chunks; ++c) {
        const int st = c % kTStages;
        int go = 1;
        if (lane == 0 && c >= kTStages) go = wait(bar_kv_empty + st, ((c / kTStages) - 1) & 1) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, go, 0)) break;
        const int row = (lane < 16) ? erow[c * kTChunkBlocks + lb] : -1;
        uint32_t bytes = (row >= 0) ? (uint32_t)kBlockBytes : 0u;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) bytes += __shfl_xor_sync(0xffffffffu, bytes, off);
        if (lane == 0) mbar_arrive_expect_tx(bar_kv_full + st, bytes);
        __syncwarp();
        if (row >= 0)
          tma_load_3d(skv + st * kTStageBytes + lt * kTKvBytes + lb * kBlockBytes, lt ? &tm_v : &tm_k, 0, row, 0,
                      bar_kv_full + st, policy);
        ++issued;
      }
      if (lane == 0 && *reinterpret_cast<volatile int *>(abort_flag)) {  // drain copies still in flight
        mbar_wait_bounded(bar_q, 0, kTWaitNs);
        for (int c = max(0, issued - kTStages); c < issued; ++c)
          mbar_wait_bounded(bar_kv_full + c % kTStages, (c / kTStages) & 1, kTWaitNs);
      }
    }
  } else if (warp == 5) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && n_chunks > 0) {
      constexpr uint32_t idesc_s = tc::idesc_bf16_f32(kTM, kTN);
      constexpr uint32_t idesc_o = tc::idesc_bf16_f32_bmn(kTM, kD);  // B = V, MN-major
      const uint32_t q_base = smem_u32(sq), kv_base = smem_u32(skv), p_base = smem_u32(sp);
      const uint32_t t_o = tmem + 128;
      auto issue_pv = [&](int c) -> bool {  // O += P_c V_c
        const int pb = c % kTPBufs;
        if (!wait(bar_p_full + pb, (c / kTPBufs) & 1)) return false;
        tc::fence_after_sync();
        const int st = c % kTStages;
#pragma unroll
        for (int ks = 0; ks < kTN / 16; ++ks) {
          // A = P [64 rows][64 tokens], K-major; B = V, N = 192 dims MN-major over the chunk's 64 tokens:
          // 64-dim chunks 1,024 B apart (leading), 8-token groups 3,072 B apart (stride)
          const uint64_t ad = tc::smem_desc_k_sw128(p_base + pb * kTPBytes + ks * 32);
          const uint64_t bd = tc::smem_desc_mn_sw128(kv_base + st * kTStageBytes + kTKvBytes + ks * 2 * kBlockBytes,
                                                     1024, kBlockBytes);
          tc::mma_bf16(t_o, ad, bd, idesc_o, c > 0 || ks > 0);
        }
        tc::commit(bar_kv_empty + st);
        tc::commit(bar_p_free + pb);
        return true;
      };
      if (wait(bar_q, 0)) {
        bool ok = true;
        for (int c = 0; c < n_chunks && ok; ++c) {
          const int st = c % kTStages, sb = c & 1;
          if (!wait(bar_kv_full + st, (c / kTStages) & 1)) break;
          if (c >= 2 && !wait(bar_s_empty + sb, ((c >> 1) - 1) & 1)) break;
          tc::fence_after_sync();
          // S_c = Q K_c^T: K = 192 as 3 swizzle blocks of 64; the chunk's 8 blocks
          // are 8-token groups 3,072 B apart, each block's 64-dim chunk cb at cb * 1,024
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) {
            const int cb = ks >> 2, kk = ks & 3;
            const uint64_t ad = tc::smem_desc_k_sw128(q_base + cb * kTM * 128 + kk * 32);
            const uint64_t bd =
                tc::smem_desc_k_sw128_stride(kv_base + st * kTStageBytes + cb * 1024 + kk * 32, kBlockBytes);
            tc::mma_bf16(tmem + sb * kTN, ad, bd, idesc_s, ks > 0);
          }
          tc::commit(bar_s_full + sb);
          if (c > 0) ok = issue_pv(c - 1);
        }
        if (ok && !*reinterpret_cast<volatile int *>(abort_flag)) issue_pv(n_chunks - 1);
      }
      tc::commit(bar_final);  // arrives once every MMA issued above has completed
    }
  } else {
    // ---------------- softmax / epilogue: warp w = query row w of the tile ----------------
    // With the 16x256b tensor-memory shape, thread t holds heads h0 = t/4 and
    // h1 = t/4 + 8 of this query, columns 8i + 2(t%4) and +1 (i = 0..7) of a
    // 64-column tile: a head's row is spread over the 4 threads of a quad.
    const int j = warp;  // row of the tile handled by this warp
    const int h0 = lane >> 2, h1 = h0 + 8, cq = 2 * (lane & 3);
    const int t = ctx + k * kTRows + j;
    const bool row_ok = j < nr;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const float sl2 = a.scale_log2;
    const int t_max = ctx + k * kTRows + nr - 1;  // last position of the tile
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    bool ok = true;
    for (int c = 0; c < n_chunks; ++c) {
      const int st = c % kTStages, sb = c & 1;
      if (!wait(bar_s_full + sb, (c >> 1) & 1)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      uint32_t v[32];
      tc::ld_16x256b_x8(tmem + lane_base + sb * kTN, v);
      tc::wait_ld();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_s_empty + sb);
      // column i of this thread: 8 i + cq (+1) = token 8 i + cq (+1) of block i of the chunk
      float sv[2][16];
      float mx[2] = {-INFINITY, -INFINITY};
      bool need_zero = false;
#pragma unroll
      for (int i = 0; i < kTChunkBlocks; ++i) {
        const uint32_t e = eent[c * kTChunkBlocks + i];
        const int blk = (int)(e & 0xFFFFFFu);
        need_zero |= (erow[c * kTChunkBlocks + i] < 0) || (blk * kBlk + kBlk - 1 > t_max);
        bool vis0 = false, vis1 = false;
        if (row_ok) {
          if ((e >> (24 + j)) & 1u) {
            vis0 = vis1 = true;
          } else if ((e >> (28 + j)) & 1u) {
            vis0 = blk * kBlk + cq <= t;
            vis1 = blk * kBlk + cq + 1 <= t;
          }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const float s0 = vis0 ? __uint_as_float(v[4 * i + 2 * r]) * sl2 : -INFINITY;
          const float s1 = vis1 ? __uint_as_float(v[4 * i + 2 * r + 1]) * sl2 : -INFINITY;
          sv[r][2 * i] = s0;
          sv[r][2 * i + 1] = s1;
          mx[r] = fmaxf(mx[r], fmaxf(s0, s1));
        }
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {  // row max over the quad
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      }
      // lazy rescale: keep the reference max unless a row's max grows by more than 2^8
      float corr[2];
      bool any_rescale = false;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const bool grow = mx[r] > m[r] + kLazyRescale;
        const float m_new = grow ? mx[r] : m[r];
        corr[r] = (grow && m[r] != -INFINITY) ? hw_exp2(m[r] - m_new) : 1.f;
        any_rescale |= grow && m[r] != -INFINITY;
        m[r] = m_new;
      }
      if (__any_sync(0xffffffffu, any_rescale) && c > 0) {
        // O holds chunks 0 .. c-1: wait for PV_{c-1} (in-order completion covers the rest)
        if (!wait(bar_p_free + (c - 1) % kTPBufs, ((c - 1) / kTPBufs) & 1)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        for (int cb = 0; cb < kD / 64; ++cb) {
          uint32_t o[32];
          tc::ld_16x256b_x8(tmem + lane_base + 128 + cb * 64, o);
          tc::wait_ld();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            o[4 * i] = __float_as_uint(__uint_as_float(o[4 * i]) * corr[0]);
            o[4 * i + 1] = __float_as_uint(__uint_as_float(o[4 * i + 1]) * corr[0]);
            o[4 * i + 2] = __float_as_uint(__uint_as_float(o[4 * i + 2]) * corr[1]);
            o[4 * i + 3] = __float_as_uint(__uint_as_float(o[4 * i + 3]) * corr[1]);
          }
          tc::st_16x256b_x8(tmem + lane_base + 128 + cb * 64, o);
        }
        tc::wait_st();
      }
      // P (bf16) into P buffer c % 3, last read by PV_{c-3}
      const int pbi = c % kTPBufs;
      if (c >= kTPBufs && !wait(bar_p_free + pbi, ((c / kTPBufs) - 1) & 1)) {
        ok = false;
        break;
      }
      uint8_t *pb = sp + pbi * kTPBytes;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const float mu = (m[r] == -INFINITY) ? 0.f : m[r];
        const int row = j * kHpg + (r ? h1 : h0);
        float psum = 0.f;
#pragma unroll
        for (int i = 0; i < kTChunkBlocks; ++i) {
          const float p0 = hw_exp2(sv[r][2 * i] - mu);
          const float p1 = hw_exp2(sv[r][2 * i + 1] - mu);
          psum += p0 + p1;
          *reinterpret_cast<uint32_t *>(pb + sw128(row, 8 * i + cq)) = pack_bf16(p0, p1);
        }
        psum += __shfl_xor_sync(0xffffffffu, psum, 1);
        psum += __shfl_xor_sync(0xffffffffu, psum, 2);
        l[r] = l[r] * corr[r] + psum;
      }
      // V rows no row of the tile may read (absent blocks, tokens past the tile's
      // last position) must be finite: zero them (P is 0 there, but 0 * NaN is NaN)
      if (__any_sync(0xffffffffu, need_zero)) {
        uint8_t *vb = skv + st * kTStageBytes + kTKvBytes;
        for (int b = j; b < kTChunkBlocks; b += 4) {
          const int idx = c * kTChunkBlocks + b;
          const int blk = (int)(eent[idx] & 0xFFFFFFu);
          const bool absent = erow[idx] < 0;
          if (!absent && blk * kBlk + kBlk - 1 <= t_max) continue;
          for (int x = lane; x < 3 * kBlk * 8; x += 32) {  // 3 planes x 8 tokens x 8 16-byte chunks
            const int tok = (x >> 3) & 7;
            if (absent || blk * kBlk + tok > t_max)
              *reinterpret_cast<uint4 *>(vb + b * kBlockBytes + (x >> 6) * 1024 + tok * 128 + (x & 7) * 16) =
                  make_uint4(0, 0, 0, 0);
          }
        }
      }
      fence_proxy_async_smem();  // generic writes (P, zeroed V rows) before the tensor core reads them
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p_full + pbi);
    }
    // ---- epilogue: O / l ----
    if (!ok) *reinterpret_cast<volatile int *>(abort_flag) = 1;
    const bool have = ok && n_chunks > 0 &&
                      wait(bar_p_free + (n_chunks - 1) % kTPBufs, ((n_chunks - 1) / kTPBufs) & 1);
    if (have) tc::fence_after_sync();
    float inv[2], lse2[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float lr = have ? l[r] : 0.f;
      inv[r] = (lr > 0.f) ? 1.f / lr : 0.f;
      lse2[r] = (lr > 0.f) ? (m[r] + hw_log2(lr)) : -INFINITY;
    }
    for (int cb = 0; cb < kD / 64; ++cb) {
      uint32_t o[32];
      if (have) {
        tc::ld_16x256b_x8(tmem + lane_base + 128 + cb * 64, o);
        tc::wait_ld();
      } else {
#pragma unroll
        for (int x = 0; x < 32; ++x) o[x] = 0u;
      }
      if (row_ok) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const size_t rh = (size_t)(r0 + j) * kHeads + g * kHpg + (r ? h1 : h0);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int d = cb * 64 + 8 * i + cq;
            const float o0 = __uint_as_float(o[4 * i + 2 * r]) * inv[r];
            const float o1 = __uint_as_float(o[4 * i + 2 * r + 1]) * inv[r];
            if (a.n_split == 1) {
              *reinterpret_cast<uint32_t *>(reinterpret_cast<__nv_bfloat16 *>(a.out) + rh * kD + d) = pack_bf16(o0, o1);
            } else {
              *reinterpret_cast<float2 *>(a.part_o + (rh * a.n_split + p) * kD + d) = make_float2(o0, o1);
            }
          }
        }
      }
    }
    if (row_ok && (lane & 3) == 0) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const size_t rh = (size_t)(r0 + j) * kHeads + g * kHpg + (r ? h1 : h0);
        if (a.n_split == 1) {
          if (a.lse != nullptr) a.lse[rh] = lse2[r] * 0.69314718055994531f;
        } else {
          a.part_lse[rh * a.n_split + p] = lse2[r];
        }
      }
    }
  }
  // ---- teardown: no MMA may be writing tensor memory when it is released ----
  if (warp == 0 && n_chunks > 0) mbar_wait_bounded(bar_final, 0, kTWaitNs);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, kTTmemCols);
  if (a.n_split == 1 || a.merge_cnt == nullptr) return;

  // ---- the last partition CTA of (tile, group) merges every partition ----
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const uint32_t prev = atomicAdd(a.merge_cnt + (size_t)tile * kKv + g, 1u);
    *is_last = (prev == (uint32_t)a.n_split - 1);
  }
  __syncthreads();
  if (!*is_last) return;
  __threadfence();
  if (tid < kTM) {
    const int jj = tid / kHpg, hh = tid % kHpg;
    if (jj < nr) {
      const size_t rh = (size_t)(r0 + jj) * kHeads + g * kHpg + hh;
      float w[kMaxTileSplit];
      float lse;
      tile_partition_weights(a.part_lse + rh * a.n_split, a.n_split, w, lse);
      __nv_bfloat16 *out = reinterpret_cast<__nv_bfloat16 *>(a.out) + rh * kD;
      for (int x = 0; x < kD; x += 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int q = 0; q < a.n_split; ++q) {
          const float4 v = ld_cg(reinterpret_cast<const float4 *>(a.part_o + (rh * a.n_split + q) * kD + x));
          acc.x = fmaf(w[q], v.x, acc.x);
          acc.y = fmaf(w[q], v.y, acc.y);
          acc.z = fmaf(w[q], v.z, acc.z);
          acc.w = fmaf(w[q], v.w, acc.w);
        }
        uint2 w2;
        w2.x = pack_bf16(acc.x, acc.y);
        w2.y = pack_bf16(acc.z, acc.w);
        *reinterpret_cast<uint2 *>(out + x) = w2;
      }
      if (a.lse != nullptr) a.lse[rh] = lse;
    }
  }
  if (tid == 0) a.merge_cnt[(size_t)tile * kKv + g] = 0u;
}

constexpr int kTileSmem = kTQBytes + kTStages * kTStageBytes + kTPBufs * kTPBytes + 2 * kMaxTileEntries * 4 + 256 + 1024;

cudaError_t launch_tile_union(const TileArgs &a, int batch, cudaStream_t st) {
  const size_t smem = (size_t)kTRows * a.bitmap_words * sizeof(uint32_t);
  cudaError_t e = cudaFuncSetAttribute(tile_union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  tile_union_kernel<<<dim3(a.tiles_per_seq, batch), 256, smem, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_gqa_tile(const TileArgs &a, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                            cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(gqa_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTileSmem);
  if (e != cudaSuccess) return e;
  const long long n_cta = (long long)a.n_split * a.n_tiles * kKv;
  if (n_cta > 0x7fffffffLL) return cudaErrorInvalidValue;
  gqa_tile_kernel<<<(unsigned)n_cta, kTThreads, kTileSmem, st>>>(a, tq, tk, tv);
  return cudaGetLastError();
}

}  // namespace s5
