// Indexer of the sparse layer: block scores and top-k block selection.
//
// SGLang day-0 blog ("Step 5 Preview: Day-0 Inference and RL Support with
// SGLang and Miles"), sections "Hybrid Attention" and "Kernels from StepFun":
// each query scores the 8-token block summaries kept in the paged cache and
// keeps up to 512 historical blocks.  StepFun open-weights blog, "What the
// config says": one 256-dim key per 8-token block, top 512 blocks.
//
// Decode / verify (a few query tokens per sequence) is an HBM-bound GEMV over
// the block keys: every key is read once per sequence and scored against all
// of that sequence's query tokens.  Scores go to the workspace (4 bytes per
// block, under 1% of the key bytes), and a CTA-wide radix select picks the
// top-k by the composite key (score descending, block index ascending).
#include "s5_common.cuh"
#include "s5_kernels.h"

namespace s5 {

// ============================================================================
// block scores (GEMV over the key pool)
// ============================================================================

// Butterfly reduce-scatter of V = 2^LOGV per-lane partial sums across the 32
// lanes.  Afterwards lane l holds the full sum of value index
// (l >> (5 - LOGV)) & (V - 1) in vals[0].
template <int LOGV>
__device__ __forceinline__ void warp_reduce_scatter(float (&vals)[1 << LOGV], int lane) {
  constexpr int V = 1 << LOGV;
#pragma unroll
  for (int step = 0; step < LOGV; ++step) {
    const int off = 16 >> step;
    const int n = V >> step;
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const float send = upper ? vals[i] : vals[i + n / 2];
      const float keep = upper ? vals[i + n / 2] : vals[i];
      vals[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
#pragma unroll
  for (int off = 16 >> LOGV; off >= 1; off >>= 1) vals[0] += __shfl_xor_sync(0xffffffffu, vals[0], off);
}

template <int QT, int UNROLL>
__global__ void __launch_bounds__(256) index_score_kernel(IndexScoreArgs a) {
  constexpr int LOGV = (QT == 1) ? 3 : (QT == 2) ? 4 : 5;
  constexpr int V = 1 << LOGV;  // 8 blocks x QT queries
  const int s = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int q_beg = __ldg(a.cu_q + s);
  const int nq_s = __ldg(a.cu_q + s + 1) - q_beg;
  const int tile0 = blockIdx.z * QT;
  if (nq_s < 0 || q_beg < 0 || q_beg + nq_s > a.total_q) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0) record_error(a.err, S5_ERR_DEVICE_BOUNDS, s);
    return;
  }
  if (tile0 >= nq_s) return;
  const int nq = min(QT, nq_s - tile0);
  const int ctx = __ldg(a.ctx_lens + s);
  const int t_last = ctx + tile0 + nq - 1;
  const int c_hi = t_last / kBlk;  // history blocks of the last query in the tile
  if (ctx < 0 || t_last >= a.max_pages * kPage || c_hi > a.score_stride) {
    if (threadIdx.x == 0 && blockIdx.x == 0) record_error(a.err, S5_ERR_DEVICE_BOUNDS, q_beg + tile0);
    return;
  }
  if (c_hi <= a.topk) return;  // every row of the tile keeps all its history blocks
  const int p_beg = blockIdx.x * a.pages_per_cta;
  const int p_end = min(p_beg + a.pages_per_cta, (c_hi + kBpp - 1) / kBpp);
  if (p_beg >= p_end) return;

  // indexer queries: lane l owns dims 8l .. 8l+7 of every query in the tile
  float qx[QT][8];
#pragma unroll
  for (int qi = 0; qi < QT; ++qi) {
    uint4 w = make_uint4(0, 0, 0, 0);
    if (qi < nq) w = __ldg(reinterpret_cast<const uint4 *>(a.q_index) + (size_t)(q_beg + tile0 + qi) * (kDx / 8) + lane);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      qx[qi][2 * e] = bf16lo(ww[e]);
      qx[qi][2 * e + 1] = bf16hi(ww[e]);
    }
  }

  const uint4 *keys = reinterpret_cast<const uint4 *>(a.key_pool);
  const int32_t *pt = a.page_table + (size_t)s * a.max_pages;
  const int nwarps = blockDim.x >> 5;

  for (int p = p_beg + warp * UNROLL; p < p_end; p += nwarps * UNROLL) {
    uint4 kv[UNROLL][kBpp];
    int phys[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int pp = p + u;
      phys[u] = -1;
      if (pp < p_end) {
        const int ph = __ldg(pt + pp);
        if (ph >= 0 && ph < a.num_pages) {
          phys[u] = ph;
        } else if (lane == 0) {
          record_error(a.err, S5_ERR_DEVICE_BOUNDS, q_beg + tile0);
        }
      }
#pragma unroll
      for (int j = 0; j < kBpp; ++j) {
        kv[u][j] = make_uint4(0, 0, 0, 0);
        if (phys[u] >= 0 && (pp * kBpp + j) < c_hi) {
          const uint4 *src = keys + ((size_t)phys[u] * kBpp + j) * (kDx / 8) + lane;
          asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(kv[u][j].x), "=r"(kv[u][j].y), "=r"(kv[u][j].z), "=r"(kv[u][j].w)
                       : "l"(src));
        }
      }
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int pp = p + u;
      float vals[V];
#pragma unroll
      for (int qi = 0; qi < QT; ++qi) {
#pragma unroll
        for (int j = 0; j < kBpp; ++j) {
          const uint32_t ww[4] = {kv[u][j].x, kv[u][j].y, kv[u][j].z, kv[u][j].w};
          float acc = 0.f;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc = fmaf(qx[qi][2 * e], bf16lo(ww[e]), acc);
            acc = fmaf(qx[qi][2 * e + 1], bf16hi(ww[e]), acc);
          }
          vals[qi * kBpp + j] = acc;
        }
      }
      warp_reduce_scatter<LOGV>(vals, lane);
      constexpr int kShift = 5 - LOGV;
      if (pp < p_end && (lane & ((1 << kShift) - 1)) == 0) {
        const int v = (lane >> kShift) & (V - 1);
        const int qi = v / kBpp;
        const int j = v % kBpp;
        const int b = pp * kBpp + j;
        if (qi < nq && b < (ctx + tile0 + qi) / kBlk) {
          a.scores[(size_t)(q_beg + tile0 + qi) * a.score_stride + b] =
              (phys[u] >= 0) ? vals[0] : __int_as_float(0xff800000);  // -inf for an unreadable page
        }
      }
    }
  }
}

// ============================================================================
// CTA-wide radix select: the k largest keys of a list, ties to the earlier
// list position, emitted in list order.
// ============================================================================

struct SelectSmem {
  uint32_t hist[256];
  int warp_a[32];
  int warp_b[32];
  uint32_t digit, above, bin_cnt;
};

// keys[0..n) in shared memory.  Calls emit(pos, i) for the k selected list
// positions i, pos = 0..k-1 in increasing i.  Requires n > k >= 1.
template <int NT, typename Emit>
__device__ void cta_select(const uint32_t *keys, int n, int k, SelectSmem &sm, Emit emit) {
  constexpr int NW = NT / 32;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  uint32_t prefix = 0, mask = 0;
  int kk = k;  // rank still to place among keys matching (prefix, mask)
  uint32_t t_lo = 0, t_hi = 0;
  bool done = false;
  for (int shift = 24; shift >= 0 && !done; shift -= 8) {
    for (int i = tid; i < 256; i += NT) sm.hist[i] = 0;
    __syncthreads();
    for (int base = warp * 32; base < n; base += NT) {
      const int i = base + lane;
      const uint32_t key = (i < n) ? keys[i] : 0u;
      const bool match = (i < n) && ((key & mask) == prefix);
      const unsigned act = __ballot_sync(0xffffffffu, match);
      if (match) {
        const uint32_t d = (key >> shift) & 255u;
        const unsigned peers = __match_any_sync(act, d);
        if (lane == __ffs(peers) - 1) atomicAdd(&sm.hist[d], (uint32_t)__popc(peers));
      }
    }
    __syncthreads();
    if (warp == 0) {
      // lane l scans bins 255-8l .. 248-8l (descending)
      uint32_t c8[8];
      uint32_t sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c8[i] = sm.hist[255 - (lane * 8 + i)];
        sum += c8[i];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      const uint32_t excl = incl - sum;
      if (excl < (uint32_t)kk && (uint32_t)kk <= incl) {
        uint32_t acc = excl;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (acc < (uint32_t)kk && (uint32_t)kk <= acc + c8[i]) {
            sm.digit = 255 - (lane * 8 + i);
            sm.above = acc;
            sm.bin_cnt = c8[i];
          }
          acc += c8[i];
        }
      }
    }
    __syncthreads();
    const uint32_t d = sm.digit;
    kk -= (int)sm.above;
    prefix |= d << shift;
    mask |= 255u << shift;
    if ((int)sm.bin_cnt == kk || shift == 0) {
      // either every key in this bin is taken, or the threshold is exact
      t_lo = prefix;
      t_hi = prefix | ~mask;
      done = true;
    }
    __syncthreads();
  }
  // keys > t_hi are taken; of the keys in [t_lo, t_hi] the first kk in list order
  const int per_warp = (((n + NW - 1) / NW) + 31) & ~31;
  const int wbeg = warp * per_warp;
  const int wend = min(n, wbeg + per_warp);
  const unsigned lt = (1u << lane) - 1u;
  int cnt_in = 0;
  for (int base = wbeg; base < wend; base += 32) {
    const int i = base + lane;
    const bool inr = (i < wend) && keys[i] >= t_lo && keys[i] <= t_hi;
    cnt_in += __popc(__ballot_sync(0xffffffffu, inr));
  }
  if (lane == 0) sm.warp_a[warp] = cnt_in;
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int w = 0; w < NW; ++w) {
      const int v = sm.warp_a[w];
      sm.warp_a[w] = acc;
      acc += v;
    }
  }
  __syncthreads();
  int rank = sm.warp_a[warp];
  int cnt_take = 0;
  for (int base = wbeg; base < wend; base += 32) {
    const int i = base + lane;
    const uint32_t key = (i < wend) ? keys[i] : 0u;
    const bool gt = (i < wend) && key > t_hi;
    const bool inr = (i < wend) && key >= t_lo && key <= t_hi;
    const unsigned bal = __ballot_sync(0xffffffffu, inr);
    const bool take = gt || (inr && (rank + __popc(bal & lt)) < kk);
    rank += __popc(bal);
    cnt_take += __popc(__ballot_sync(0xffffffffu, take));
  }
  if (lane == 0) sm.warp_b[warp] = cnt_take;
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int w = 0; w < NW; ++w) {
      const int v = sm.warp_b[w];
      sm.warp_b[w] = acc;
      acc += v;
    }
  }
  __syncthreads();
  rank = sm.warp_a[warp];
  int pos = sm.warp_b[warp];
  for (int base = wbeg; base < wend; base += 32) {
    const int i = base + lane;
    const uint32_t key = (i < wend) ? keys[i] : 0u;
    const bool gt = (i < wend) && key > t_hi;
    const bool inr = (i < wend) && key >= t_lo && key <= t_hi;
    const unsigned bal = __ballot_sync(0xffffffffu, inr);
    const bool take = gt || (inr && (rank + __popc(bal & lt)) < kk);
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    if (take) emit(pos + __popc(tb & lt), i);
    pos += __popc(tb);
    rank += __popc(bal);
  }
  __syncthreads();
}

// Query row -> (history blocks c).  Returns false (and records) on bad batch data.
__device__ __forceinline__ bool row_history(const SelectArgs &a, int r, int &c) {
  const int s = seq_of_row(a.cu_q, a.batch, r);
  if (s < 0) return false;
  const int t = __ldg(a.ctx_lens + s) + (r - __ldg(a.cu_q + s));
  if (t < 0 || t / kBlk > a.score_stride) return false;
  c = t / kBlk;
  return true;
}

// Single stage: one CTA per query row, the row's keys staged in shared memory.
template <int NT>
__global__ void __launch_bounds__(NT) topk_select_kernel(SelectArgs a) {
  extern __shared__ __align__(16) uint32_t keys_s[];
  __shared__ SelectSmem sm;
  const int r = blockIdx.x;
  int c = 0;
  if (!row_history(a, r, c)) {
    if (threadIdx.x == 0) {
      record_error(a.err, S5_ERR_DEVICE_BOUNDS, r);
      a.sel_count[r] = 0;
    }
    for (int i = threadIdx.x; i < a.topk; i += NT) a.sel[(size_t)r * a.topk + i] = -1;
    return;
  }
  int32_t *out = a.sel + (size_t)r * a.topk;
  if (c <= a.topk) {
    for (int i = threadIdx.x; i < a.topk; i += NT) out[i] = (i < c) ? i : -1;
    if (threadIdx.x == 0) a.sel_count[r] = c;
    return;
  }
  const float *sc = a.scores + (size_t)r * a.score_stride;
  for (int i = threadIdx.x; i < c; i += NT) keys_s[i] = score_key(__ldg(sc + i));
  __syncthreads();
  cta_select<NT>(keys_s, c, a.topk, sm, [&](int pos, int i) { out[pos] = i; });
  if (threadIdx.x == 0) a.sel_count[r] = a.topk;
}

// Two stages for long histories.  Stage 1: the top-k of each segment of
// `seg` blocks, as (key, block) candidates in block order.
template <int NT>
__global__ void __launch_bounds__(NT) topk_segment_kernel(SelectArgs a) {
  extern __shared__ __align__(16) uint32_t keys_s[];
  __shared__ SelectSmem sm;
  const int r = blockIdx.y;
  const int sg = blockIdx.x;
  int c = 0;
  if (!row_history(a, r, c)) return;  // recorded by the final stage
  if (c <= a.topk) return;
  const int b0 = sg * a.seg;
  const int n = min(a.seg, c - b0);
  if (n <= 0) return;
  const size_t cbase = ((size_t)r * a.n_seg + sg) * a.topk;
  const float *sc = a.scores + (size_t)r * a.score_stride + b0;
  if (n <= a.topk) {
    for (int i = threadIdx.x; i < n; i += NT) {
      a.cand_key[cbase + i] = score_key(__ldg(sc + i));
      a.cand_idx[cbase + i] = b0 + i;
    }
    return;
  }
  for (int i = threadIdx.x; i < n; i += NT) keys_s[i] = score_key(__ldg(sc + i));
  __syncthreads();
  cta_select<NT>(keys_s, n, a.topk, sm, [&](int pos, int i) {
    a.cand_key[cbase + pos] = keys_s[i];
    a.cand_idx[cbase + pos] = b0 + i;
  });
}

// Stage 2: the top-k of the concatenated candidates of every segment.
template <int NT>
__global__ void __launch_bounds__(NT) topk_merge_kernel(SelectArgs a) {
  extern __shared__ __align__(16) uint32_t smem[];
  __shared__ SelectSmem sm;
  const int r = blockIdx.x;
  int c = 0;
  if (!row_history(a, r, c)) {
    if (threadIdx.x == 0) {
      record_error(a.err, S5_ERR_DEVICE_BOUNDS, r);
      a.sel_count[r] = 0;
    }
    for (int i = threadIdx.x; i < a.topk; i += NT) a.sel[(size_t)r * a.topk + i] = -1;
    return;
  }
  int32_t *out = a.sel + (size_t)r * a.topk;
  if (c <= a.topk) {
    for (int i = threadIdx.x; i < a.topk; i += NT) out[i] = (i < c) ? i : -1;
    if (threadIdx.x == 0) a.sel_count[r] = c;
    return;
  }
  const int nseg = (c + a.seg - 1) / a.seg;
  uint32_t *keys_s = smem;
  int32_t *idx_s = reinterpret_cast<int32_t *>(smem + (size_t)a.n_seg * a.topk);
  int n = 0;
  for (int sg = 0; sg < nseg; ++sg) {
    const int m = min(a.topk, min(a.seg, c - sg * a.seg));
    const size_t cbase = ((size_t)r * a.n_seg + sg) * a.topk;
    for (int i = threadIdx.x; i < m; i += NT) {
      keys_s[n + i] = a.cand_key[cbase + i];
      idx_s[n + i] = a.cand_idx[cbase + i];
    }
    n += m;
  }
  __syncthreads();
  if (n <= a.topk) {  // a single segment whose candidates are all taken
    for (int i = threadIdx.x; i < a.topk; i += NT) out[i] = (i < n) ? idx_s[i] : -1;
    if (threadIdx.x == 0) a.sel_count[r] = n;
    return;
  }
  cta_select<NT>(keys_s, n, a.topk, sm, [&](int pos, int i) { out[pos] = idx_s[i]; });
  if (threadIdx.x == 0) a.sel_count[r] = a.topk;
}

// ============================================================================
// launchers
// ============================================================================

cudaError_t launch_index_score(const IndexScoreArgs &a, int max_q, int grid_pages, int n_seq, cudaStream_t st) {
  const int qt = (max_q <= 1) ? 1 : (max_q <= 2) ? 2 : 4;
  dim3 grid(grid_pages, n_seq, (max_q + qt - 1) / qt);
  if (qt == 1) index_score_kernel<1, 2><<<grid, 256, 0, st>>>(a);
  else if (qt == 2) index_score_kernel<2, 2><<<grid, 256, 0, st>>>(a);
  else index_score_kernel<4, 1><<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

constexpr int kSelThreads = 512;

cudaError_t launch_topk_select(const SelectArgs &a, int total_q, bool two_stage, cudaStream_t st) {
  if (!two_stage) {
    const size_t smem = (size_t)a.score_stride * sizeof(uint32_t);
    cudaError_t e = cudaFuncSetAttribute(topk_select_kernel<kSelThreads>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    topk_select_kernel<kSelThreads><<<total_q, kSelThreads, smem, st>>>(a);
    return cudaGetLastError();
  }
  const size_t smem1 = (size_t)a.seg * sizeof(uint32_t);
  cudaError_t e = cudaFuncSetAttribute(topk_segment_kernel<kSelThreads>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
  if (e != cudaSuccess) return e;
  topk_segment_kernel<kSelThreads><<<dim3(a.n_seg, total_q), kSelThreads, smem1, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem2 = (size_t)a.n_seg * a.topk * (sizeof(uint32_t) + sizeof(int32_t));
  e = cudaFuncSetAttribute(topk_merge_kernel<kSelThreads>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem2);
  if (e != cudaSuccess) return e;
  topk_merge_kernel<kSelThreads><<<total_q, kSelThreads, smem2, st>>>(a);
  return cudaGetLastError();
}

}  // namespace s5
