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

template <int NT>
struct SelectSmem {
  uint32_t whist[NT / 32][256];  // one private histogram per warp
  int wsum[32];
  int scan_a[32];
  int scan_b[32];
  uint32_t digit, above, bin_cnt;
};

// Exclusive prefix sum of v over threads in thread order.
template <int NT>
__device__ __forceinline__ int block_excl_scan(int v, int *buf) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) buf[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int x = (lane < NT / 32) ? buf[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += o;
    }
    if (lane < NT / 32) buf[lane] = x;  // inclusive warp totals
  }
  __syncthreads();
  return (warp > 0 ? buf[warp - 1] : 0) + incl - v;
}

// Top-k of a list of n keys (n > k >= 1).  Thread t owns list positions
// t*E .. t*E+E-1, held in shared memory as ks[j * NT + t].  Radix select on
// 8-bit digits from the top: each pass histograms the digit of the keys that
// still match the chosen prefix into per-warp histograms (no atomics shared
// between warps), sums them and picks the bin holding the kk-th largest; it
// stops early when that whole bin is taken.  Then the keys above the final
// range and the first kk keys inside it (list order) are emitted as
// emit(pos, list_position), pos = 0..k-1 in list order.
template <int NT, typename Emit>
__device__ void cta_select(const uint32_t *ks, int n, int E, int k, SelectSmem<NT> &sm, Emit emit) {
  constexpr int NW = NT / 32;
  static_assert(NT >= 256, "one thread per bin when summing histograms");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int first = tid * E;
  const int mine = max(0, min(E, n - first));
  uint32_t prefix = 0, mask = 0;
  int kk = k;
  uint32_t *wh = sm.whist[warp];
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = lane; i < 256; i += 32) wh[i] = 0;
    __syncwarp();
    for (int j = 0; j < mine; ++j) {
      const uint32_t key = ks[j * NT + tid];
      if ((key & mask) == prefix) atomicAdd(&wh[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    // thread i < 256 owns bin 255 - i: bins in descending order
    int cnt = 0;
    if (tid < 256) {
      const int b = 255 - tid;
#pragma unroll 8
      for (int w = 0; w < NW; ++w) cnt += (int)sm.whist[w][b];
    }
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    if (lane == 31 && warp < 8) sm.wsum[warp] = incl;
    __syncthreads();
    if (tid < 256) {
      int base = 0;
      for (int w = 0; w < warp; ++w) base += sm.wsum[w];
      const int excl = base + incl - cnt;
      if (excl < kk && kk <= excl + cnt) {
        sm.digit = (uint32_t)(255 - tid);
        sm.above = (uint32_t)excl;
        sm.bin_cnt = (uint32_t)cnt;
      }
    }
    __syncthreads();
    kk -= (int)sm.above;
    prefix |= sm.digit << shift;
    mask |= 255u << shift;
    const bool stop = ((int)sm.bin_cnt == kk);
    __syncthreads();  // sm.digit / above / bin_cnt are rewritten by the next pass
    if (stop) break;
  }
  const uint32_t t_lo = prefix, t_hi = prefix | ~mask;  // keys in [t_lo, t_hi] compete for the last kk places
  int in = 0, gt = 0;
  for (int j = 0; j < mine; ++j) {
    const uint32_t key = ks[j * NT + tid];
    gt += key > t_hi;
    in += (key >= t_lo) & (key <= t_hi);
  }
  const int in_before = block_excl_scan<NT>(in, sm.scan_a);
  const int take = gt + max(0, min(in, kk - in_before));
  int pos = block_excl_scan<NT>(take, sm.scan_b);
  int r = in_before;
  for (int j = 0; j < mine; ++j) {
    const uint32_t key = ks[j * NT + tid];
    const bool inr = (key >= t_lo) & (key <= t_hi);
    const bool tk = key > t_hi || (inr && r < kk);
    r += inr;
    if (tk) emit(pos++, first + j);
  }
  __syncthreads();
}

// Positions per thread for an n-long list: a multiple of 4 (whole float4 loads).
template <int NT>
__host__ __device__ constexpr int owned_per_thread(int n) {
  return (((n + NT - 1) / NT) + 3) & ~3;
}

// Stage the n scores row[0..n) as keys in the owner layout; a thread's loads
// are all in flight together.  row is 16-byte aligned and readable up to the
// next multiple of 4.
template <int NT>
__device__ __forceinline__ void load_keys(const float *row, int n, int E, uint32_t *ks) {
  const int t = threadIdx.x;
  const float4 *r4 = reinterpret_cast<const float4 *>(row + (size_t)t * E);
  constexpr int kMaxQ = 8;  // E <= 32
  float4 v[kMaxQ];
#pragma unroll
  for (int q = 0; q < kMaxQ; ++q)
    if (4 * q < E && t * E + 4 * q < n) v[q] = __ldcg(r4 + q);
#pragma unroll
  for (int q = 0; q < kMaxQ; ++q) {
    if (4 * q < E) {
      const int i0 = t * E + 4 * q;
      const float f[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) ks[(4 * q + e) * NT + t] = (i0 + e < n) ? score_key(f[e]) : 0u;
    }
  }
}

// Query row -> (history blocks c).  Returns false on bad batch data.
__device__ __forceinline__ bool row_history(const SelectArgs &a, int r, int &c) {
  const int s = seq_of_row(a.cu_q, a.batch, r);
  if (s < 0) return false;
  const int t = __ldg(a.ctx_lens + s) + (r - __ldg(a.cu_q + s));
  if (t < 0 || t / kBlk > a.score_stride) return false;
  c = t / kBlk;
  return true;
}

__device__ __forceinline__ void write_all(int32_t *out, int n, int topk, int nt) {
  for (int i = threadIdx.x; i < topk; i += nt) out[i] = (i < n) ? i : -1;
}

// Single stage: one CTA per query row.
template <int NT>
__global__ void __launch_bounds__(NT) topk_select_kernel(SelectArgs a) {
  extern __shared__ __align__(16) uint32_t ks[];
  __shared__ SelectSmem<NT> sm;
  const int r = blockIdx.x;
  int32_t *out = a.sel + (size_t)r * a.topk;
  int c = 0;
  if (!row_history(a, r, c)) {
    if (threadIdx.x == 0) {
      record_error(a.err, S5_ERR_DEVICE_BOUNDS, r);
      a.sel_count[r] = 0;
    }
    write_all(out, 0, a.topk, NT);
    return;
  }
  if (c <= a.topk) {
    write_all(out, c, a.topk, NT);
    if (threadIdx.x == 0) a.sel_count[r] = c;
    return;
  }
  const int E = owned_per_thread<NT>(c);
  load_keys<NT>(a.scores + (size_t)r * a.score_stride, c, E, ks);
  __syncthreads();
  cta_select<NT>(ks, c, E, a.topk, sm, [&](int pos, int i) { out[pos] = i; });
  if (threadIdx.x == 0) a.sel_count[r] = a.topk;
}

// Two stages for long histories.  Stage 1: the top-k of each segment of
// `seg` blocks, as (key, block) candidates in block order.
template <int NT>
__global__ void __launch_bounds__(NT) topk_segment_kernel(SelectArgs a) {
  extern __shared__ __align__(16) uint32_t ks[];
  __shared__ SelectSmem<NT> sm;
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
      a.cand_key[cbase + i] = score_key(__ldcg(sc + i));
      a.cand_idx[cbase + i] = b0 + i;
    }
    return;
  }
  const int E = owned_per_thread<NT>(n);
  load_keys<NT>(sc, n, E, ks);
  __syncthreads();
  cta_select<NT>(ks, n, E, a.topk, sm, [&](int pos, int i) {
    a.cand_key[cbase + pos] = ks[(i % E) * NT + i / E];
    a.cand_idx[cbase + pos] = b0 + i;
  });
}

// Stage 2: the top-k of the concatenated candidates of every segment.  Every
// segment but the last holds exactly topk candidates, so candidate L of the
// row sits at slot L % topk of segment L / topk.
template <int NT>
__global__ void __launch_bounds__(NT) topk_merge_kernel(SelectArgs a) {
  extern __shared__ __align__(16) uint32_t smem[];
  __shared__ SelectSmem<NT> sm;
  const int r = blockIdx.x;
  int32_t *out = a.sel + (size_t)r * a.topk;
  int c = 0;
  if (!row_history(a, r, c)) {
    if (threadIdx.x == 0) {
      record_error(a.err, S5_ERR_DEVICE_BOUNDS, r);
      a.sel_count[r] = 0;
    }
    write_all(out, 0, a.topk, NT);
    return;
  }
  if (c <= a.topk) {
    write_all(out, c, a.topk, NT);
    if (threadIdx.x == 0) a.sel_count[r] = c;
    return;
  }
  const int nseg = (c + a.seg - 1) / a.seg;
  const int last = c - (nseg - 1) * a.seg;
  const int n = (nseg - 1) * a.topk + min(a.topk, last);
  const int E = owned_per_thread<NT>(n);
  uint32_t *ks = smem;
  int32_t *is = reinterpret_cast<int32_t *>(smem + (size_t)E * NT);
  const size_t rbase = (size_t)r * a.n_seg * a.topk;
  for (int j = 0; j < E; ++j) {
    const int L = threadIdx.x * E + j;
    if (L < n) {
      const size_t src = rbase + (size_t)(L / a.topk) * a.topk + (L % a.topk);
      ks[j * NT + threadIdx.x] = __ldcg(a.cand_key + src);
      is[j * NT + threadIdx.x] = __ldcg(a.cand_idx + src);
    }
  }
  __syncthreads();
  if (n <= a.topk) {  // a single segment whose candidates are all taken
    for (int j = 0; j < E; ++j) {
      const int L = threadIdx.x * E + j;
      if (L < n) out[L] = is[j * NT + threadIdx.x];
    }
    for (int i = n + threadIdx.x; i < a.topk; i += NT) out[i] = -1;
    if (threadIdx.x == 0) a.sel_count[r] = n;
    return;
  }
  cta_select<NT>(ks, n, E, a.topk, sm, [&](int pos, int i) { out[pos] = is[(i % E) * NT + i / E]; });
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

constexpr int kSelThreads = 1024;  // one CTA per row (rows of up to 16,384 blocks)
constexpr int kSegThreads = 256;   // stage 1: one CTA per segment (E = seg / 256 <= 32)

template <int NT>
cudaError_t launch_merge(const SelectArgs &a, int total_q, cudaStream_t st) {
  const size_t smem = (size_t)owned_per_thread<NT>(a.n_seg * a.topk) * NT * (sizeof(uint32_t) + sizeof(int32_t));
  cudaError_t e = cudaFuncSetAttribute(topk_merge_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  topk_merge_kernel<NT><<<total_q, NT, smem, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_topk_select(const SelectArgs &a, int total_q, bool two_stage, cudaStream_t st) {
  if (!two_stage) {
    constexpr int NT = kSelThreads;
    const size_t smem = (size_t)owned_per_thread<NT>(a.score_stride) * NT * sizeof(uint32_t);
    cudaError_t e = cudaFuncSetAttribute(topk_select_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    topk_select_kernel<NT><<<total_q, NT, smem, st>>>(a);
    return cudaGetLastError();
  }
  constexpr int NS = kSegThreads;
  const size_t smem1 = (size_t)owned_per_thread<NS>(a.seg) * NS * sizeof(uint32_t);
  cudaError_t e = cudaFuncSetAttribute(topk_segment_kernel<NS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem1);
  if (e != cudaSuccess) return e;
  topk_segment_kernel<NS><<<dim3(a.n_seg, total_q), NS, smem1, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // stage 2: at most 32 owned candidates per thread
  if (a.n_seg * a.topk <= 32 * 512) return launch_merge<512>(a, total_q, st);
  return launch_merge<1024>(a, total_q, st);
}

}  // namespace s5
