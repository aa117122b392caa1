// Indexer block scores for prefill-sized batches as a tensor-core GEMM.
//
// SGLang day-0 blog ("Step 5 Preview: Day-0 Inference and RL Support with
// SGLang and Miles"), "Kernels from StepFun": indexer scoring of each query
// against the compressed history in the paged cache, for prefill as well as
// decode.  With thousands of query rows per sequence the scores
// S[q][b] = QX[q] . KX[b] (K = 256) are a dense GEMM, so they run on the
// 5th-generation tensor cores:
//
//   * a sequence's block keys are first laid out contiguously (gather kernel),
//     so TMA can tile them;
//   * one CTA owns 128 query rows (MMA M = 128) and a range of 128-block N
//     tiles; TMA brings the 128 x 256 query tile once and streams key tiles
//     through two shared-memory stages (128-byte swizzle, K-major);
//   * one thread issues tcgen05.mma (bf16 x bf16 -> fp32) into two tensor-memory
//     accumulators of 128 columns, so the epilogue of one tile overlaps the
//     MMAs of the next;
//   * four epilogue warps read their 32 tensor-memory lanes each (a thread
//     holds one row) and store the causally visible scores (b < t / 8 of each
//     row) through a shared-memory staging tile, 8 lanes writing one row's
//     128 contiguous bytes at a time.
//
// Integer-valued inputs give exact fp32 scores in any summation order, so the
// selection downstream is the same as with the CUDA-core path.
#include <cuda.h>

#include "s5_common.cuh"
#include "s5_kernels.h"
#include "s5_tcgen05.cuh"

namespace s5 {

constexpr int kGM = 128;                   // query rows per CTA
constexpr int kGN = 128;                   // blocks per N tile
constexpr int kGKb = 4;                    // K = 256 as 4 swizzle blocks of 64
constexpr int kGTileBytes = kGM * 128;     // one 128-row x 64-element swizzled K block
constexpr int kGOperand = kGKb * kGTileBytes;  // 64 KB: a full 128 x 256 operand
constexpr int kGStages = 2;
constexpr int kGThreads = 192;             // warps 0-3 epilogue, 4 TMA, 5 MMA
constexpr int kGStRow = 36;                // floats per row of an epilogue staging tile (16-byte aligned, conflict-free)
constexpr int kGStageBytes = 4 * 32 * kGStRow * 4;  // 4 warps x 32 rows x 32 columns (padded)
constexpr int kGSmem = kGOperand * (1 + kGStages) + kGStageBytes + 256 + 1024;
constexpr uint32_t kGTmemCols = 2 * kGN;   // two fp32 accumulators
constexpr uint64_t kGWaitNs = 2000000000ull;

// Contiguous copy of each sequence's block keys: kxs[s][b] = key of block b.
__global__ void __launch_bounds__(256) gather_keys_kernel(GatherArgs a) {
  const int s = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pg = blockIdx.x * 8 + warp;  // one page (8 keys, 4 KB) per warp
  if (pg * kBpp >= a.max_blocks) return;
  const int ph = ld_cg(a.page_table + (size_t)s * a.max_pages + min(pg, a.max_pages - 1));
  uint4 *dst = reinterpret_cast<uint4 *>(a.kxs) + ((size_t)s * a.max_blocks + (size_t)pg * kBpp) * (kDx / 8);
  const int nb = min(kBpp, a.max_blocks - pg * kBpp);
  if (pg >= a.max_pages || ph < 0 || ph >= a.num_pages) {
    for (int i = lane; i < nb * (kDx / 8); i += 32) dst[i] = make_uint4(0, 0, 0, 0);
    return;
  }
  uint4 v[8];
  if (a.key_fp8) {
    // one-byte E4M3 keys: 8 bytes (8 dims) per 16-byte bf16 chunk, widened exactly
    const uint2 *src8 = reinterpret_cast<const uint2 *>(a.key_pool) + (size_t)ph * kBpp * (kDx / 8);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (lane + 32 * u < nb * (kDx / 8)) {
        const uint2 c = src8[lane + 32 * u];
        float f[8];
        e4m3x4_to_float(c.x, f[0], f[1], f[2], f[3]);
        e4m3x4_to_float(c.y, f[4], f[5], f[6], f[7]);
        v[u] = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
      }
    }
  } else {
    const uint4 *src = reinterpret_cast<const uint4 *>(a.key_pool) + (size_t)ph * kBpp * (kDx / 8);
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (lane + 32 * u < nb * (kDx / 8)) v[u] = ld_cg(src + lane + 32 * u);
  }
#pragma unroll
  for (int u = 0; u < 8; ++u)
    if (lane + 32 * u < nb * (kDx / 8)) dst[lane + 32 * u] = v[u];
}

__global__ void __launch_bounds__(kGThreads, 1)
    index_gemm_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sa = smem;                                 // query tile
  uint8_t *sb = smem + kGOperand;                     // key stages
  float *stage_all = reinterpret_cast<float *>(smem + kGOperand * (1 + kGStages));  // epilogue staging
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kGOperand * (1 + kGStages) + kGStageBytes);
  uint64_t *bar_a = bars + 0;
  uint64_t *bar_full = bars + 1;    // [2]
  uint64_t *bar_empty = bars + 3;   // [2]
  uint64_t *bar_dfull = bars + 5;   // [2]
  uint64_t *bar_dempty = bars + 7;  // [2]
  uint64_t *bar_final = bars + 9;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 10);
  int *abort_flag = reinterpret_cast<int *>(bars + 11);

  pdl_trigger();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int s = blockIdx.z;
  const int q_beg = ld_cg(a.cu_q + s);
  const int nq = ld_cg(a.cu_q + s + 1) - q_beg;
  const int ctx = ld_cg(a.ctx_lens + s);
  // indexer rows of the sequence: token-major, G queries per token (G = 1, or
  // one per KV group); row m of the sequence belongs to its token m / G
  const int G = a.q_groups > 1 ? a.q_groups : 1;
  const int m0 = blockIdx.y * kGM;
  if (nq <= 0 || m0 >= nq * G) return;
  const int rows = min(kGM, nq * G - m0);
  const int c_last = (ctx + (m0 + rows - 1) / G) / kBlk;  // history blocks of the tile's last row
  if (q_beg < 0 || q_beg + nq > a.total_q || ctx < 0 || c_last > a.score_stride || c_last > a.max_blocks) {
    if (tid == 0 && blockIdx.x == 0) record_error(a.err, S5_ERR_DEVICE_BOUNDS, max(q_beg, 0) + m0 / G);
    return;
  }
  const int row0 = q_beg * G + m0;  // first indexer row of the tile
  const int j_beg = blockIdx.x * a.tiles_per_cta;
  const int j_end = min(j_beg + a.tiles_per_cta, (c_last + kGN - 1) / kGN);
  const int nt = j_end - j_beg;
  if (nt <= 0) return;

  if (warp == 0) tc::tmem_alloc(tmem_slot, kGTmemCols);
  if (tid == 0) {
    mbar_init(bar_a, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_full + i, 1);
      mbar_init(bar_empty + i, 1);
      mbar_init(bar_dfull + i, 1);
      mbar_init(bar_dempty + i, 4);
    }
    mbar_init(bar_final, 1);
    *abort_flag = 0;
  }
  fence_mbar_init();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  auto wait = [&](uint64_t *bar, uint32_t parity) -> bool {
    if (*reinterpret_cast<volatile int *>(abort_flag)) return false;
    if (mbar_wait_bounded(bar, parity, kGWaitNs)) return true;
    *reinterpret_cast<volatile int *>(abort_flag) = 1;
    record_error(a.err, S5_ERR_TIMEOUT, q_beg + m0 / G);
    return false;
  };

  if (warp == 4) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_a, kGOperand);
      for (int kb = 0; kb < kGKb; ++kb) tma_load_2d(sa + kb * kGTileBytes, &tm_q, kb * 64, row0, bar_a);
      int issued = 0;
      for (int jj = 0; jj < nt; ++jj) {
        const int st = jj % kGStages;
        if (jj >= kGStages && !wait(bar_empty + st, ((jj / kGStages) - 1) & 1)) break;
        mbar_arrive_expect_tx(bar_full + st, kGOperand);
        const int n0 = (j_beg + jj) * kGN;
        for (int kb = 0; kb < kGKb; ++kb)
          tma_load_2d(sb + st * kGOperand + kb * kGTileBytes, &tm_k, kb * 64, s * a.max_blocks + n0, bar_full + st);
        ++issued;
      }
      // every issued stage is consumed by the MMA warp before it finishes; after
      // an abort, drain the stages that may still be in flight
      if (*reinterpret_cast<volatile int *>(abort_flag)) {
        mbar_wait_bounded(bar_a, 0, kGWaitNs);
        for (int jj = max(0, issued - kGStages); jj < issued; ++jj)
          mbar_wait_bounded(bar_full + jj % kGStages, (jj / kGStages) & 1, kGWaitNs);
      }
    }
  } else if (warp == 5) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16_f32(kGM, kGN);
      const uint32_t a_base = smem_u32(sa), b_base = smem_u32(sb);
      if (wait(bar_a, 0)) {
        for (int jj = 0; jj < nt; ++jj) {
          const int st = jj % kGStages, db = jj % 2;
          if (!wait(bar_full + st, (jj / kGStages) & 1)) break;
          if (jj >= 2 && !wait(bar_dempty + db, ((jj / 2) - 1) & 1)) break;
          tc::fence_after_sync();
          const uint32_t d = tmem + db * kGN;
#pragma unroll
          for (int ks = 0; ks < 16; ++ks) {
            const int kb = ks >> 2, k = ks & 3;
            const uint64_t ad = tc::smem_desc_k_sw128(a_base + kb * kGTileBytes + k * 32);
            const uint64_t bd = tc::smem_desc_k_sw128(b_base + st * kGOperand + kb * kGTileBytes + k * 32);
            tc::mma_bf16(d, ad, bd, idesc, ks > 0);
          }
          tc::commit(bar_empty + st);
          tc::commit(bar_dfull + db);
        }
      }
      tc::commit(bar_final);  // arrives once every MMA issued above has completed
    }
  } else {
    // ---------------- epilogue: warps 0-3, TMEM lanes 32w .. 32w+31 ----------------
    // Thread = row of the tile in tensor memory; stores go through a staging
    // tile so that 8 lanes write one row's 32 columns (128 bytes) together.
    const int row = warp * 32 + lane;
    const int c_row = (row < rows) ? (ctx + (m0 + row) / G) / kBlk : 0;  // visible blocks of this row
    float *stage = stage_all + warp * 32 * kGStRow;
    const int sub = lane >> 3, q4 = (lane & 7) * 4;  // row within a group of 4, first column of the lane
    for (int jj = 0; jj < nt; ++jj) {
      const int db = jj % 2;
      if (!wait(bar_dfull + db, (jj / 2) & 1)) break;
      tc::fence_after_sync();
      uint32_t v[4][32];
      const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16) + db * kGN;
#pragma unroll
      for (int c = 0; c < 4; ++c) tc::ld_32cols(taddr + c * 32, v[c]);
      tc::wait_ld();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_dempty + db);
      const int n0 = (j_beg + jj) * kGN;
      if (!__any_sync(0xffffffffu, row < rows && n0 < c_row)) continue;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4 *>(stage + lane * kGStRow + e) =
              make_float4(__uint_as_float(v[c][e]), __uint_as_float(v[c][e + 1]), __uint_as_float(v[c][e + 2]),
                          __uint_as_float(v[c][e + 3]));
        __syncwarp();
        const int b = n0 + c * 32 + q4;  // first of this lane's 4 blocks
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int r = it * 4 + sub;  // row of the warp's 32
          const int cr = __shfl_sync(0xffffffffu, c_row, r);
          if (warp * 32 + r < rows && b < cr) {
            const float4 x = *reinterpret_cast<const float4 *>(stage + r * kGStRow + q4);
            float *dst = a.scores + (size_t)(row0 + warp * 32 + r) * a.score_stride + b;
            if (b + 3 < cr) {
              *reinterpret_cast<float4 *>(dst) = x;
            } else {
              dst[0] = x.x;
              if (b + 1 < cr) dst[1] = x.y;
              if (b + 2 < cr) dst[2] = x.z;
            }
          }
        }
        __syncwarp();  // the staging tile is rewritten by the next column group
      }
    }
  }
  // ---- teardown: no MMA may be writing tensor memory when it is released ----
  if (warp == 0) mbar_wait_bounded(bar_final, 0, kGWaitNs);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, kGTmemCols);
}

cudaError_t launch_gather_keys(const GatherArgs &a, int batch, cudaStream_t st) {
  dim3 grid((a.max_blocks / kBpp + 8) / 8, batch);
  gather_keys_kernel<<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_index_gemm(const GemmArgs &a, const CUtensorMap &tq, const CUtensorMap &tk, int batch, int max_q,
                              cudaStream_t st) {
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void *>(index_gemm_kernel), kGSmem);
  if (e != cudaSuccess) return e;
  const int n_tiles = (a.max_blocks + kGN - 1) / kGN;
  dim3 grid((n_tiles + a.tiles_per_cta - 1) / a.tiles_per_cta, (max_q + kGM - 1) / kGM, batch);
  index_gemm_kernel<<<grid, kGThreads, kGSmem, st>>>(a, tq, tk);
  return cudaGetLastError();
}

}  // namespace s5
