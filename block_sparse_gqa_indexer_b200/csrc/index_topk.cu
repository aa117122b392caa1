// Indexer of the sparse layer: block scores and top-k block selection.
//
// SGLang day-0 blog ("Step 5 Preview: Day-0 Inference and RL Support with
// SGLang and Miles"), sections "Hybrid Attention" and "Kernels from StepFun":
// every query rates the per-block summaries held in the paged cache and keeps
// the best 512 blocks of its history.  StepFun open-weights blog, "What the
// config says": the key of each 8-token block is 256 wide; the selection
// size is 512.
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

// GROUPED: a.q_groups indexer queries per token (one per KV group), rows
// token-major; otherwise one query per token.  KEY8: block keys are one-byte
// E4M3 codes (a lane reads 8 bytes = 8 dims of a key), decoded exactly to
// fp32 before the same FMA chain as the bf16 keys.
template <int QT, int UNROLL, bool GROUPED, bool KEY8>
__device__ __forceinline__ void index_score_body(const IndexScoreArgs &a) {
  constexpr int LOGV = (QT == 1) ? 3 : (QT == 2) ? 4 : 5;
  constexpr int V = 1 << LOGV;  // 8 blocks x QT queries
  pdl_trigger();  // the select may launch now; it waits for these scores before reading them
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
  // indexer rows of the sequence: token-major, G queries per token (G = 1, or
  // one per KV group); row q of the sequence belongs to its token q / G
  const int G = GROUPED ? a.q_groups : 1;
  if (tile0 >= nq_s * G) return;
  const int nq = min(QT, nq_s * G - tile0);
  const int ctx = __ldg(a.ctx_lens + s);
  const int t_last = GROUPED ? ctx + (tile0 + nq - 1) / G : ctx + tile0 + nq - 1;
  const int c_hi = t_last / kBlk;  // history blocks of the last query in the tile
  if (ctx < 0 || t_last >= a.max_pages * kPage || c_hi > a.score_stride) {
    if (threadIdx.x == 0 && blockIdx.x == 0) record_error(a.err, S5_ERR_DEVICE_BOUNDS, q_beg + tile0 / G);
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
    if (qi < nq) w = __ldg(reinterpret_cast<const uint4 *>(a.q_index) + (size_t)(q_beg * G + tile0 + qi) * (kDx / 8) + lane);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      qx[qi][2 * e] = bf16lo(ww[e]);
      qx[qi][2 * e + 1] = bf16hi(ww[e]);
    }
  }

  const uint4 *keys = reinterpret_cast<const uint4 *>(a.key_pool);
  const uint2 *keys8 = reinterpret_cast<const uint2 *>(a.key_pool);
  const int32_t *pt = a.page_table + (size_t)s * a.max_pages;
  const int nwarps = blockDim.x >> 5;

  for (int p = p_beg + warp * UNROLL; p < p_end; p += nwarps * UNROLL) {
    // 4-row tiles (verify batches): the pages of this warp's next step, into L2
    // (0.1065 -> 0.1044 ms per 64 x 4-row index call; one-row decode tiles run
    // slower with it, 0.104 -> 0.114 ms)
    if (QT == 4 && !KEY8 && !GROUPED && lane < UNROLL) {
      const int pn = p + nwarps * UNROLL + lane;
      if (pn < p_end) {
        const int x = __ldg(pt + pn);
        if (x >= 0 && x < a.num_pages)
          bulk_prefetch_l2(reinterpret_cast<const uint8_t *>(a.key_pool) + (size_t)x * kBpp * kDx * (KEY8 ? 1 : 2),
                           kBpp * kDx * (KEY8 ? 1 : 2));
      }
    }
    uint4 kv[UNROLL][kBpp];
    uint2 kv8[UNROLL][kBpp];
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
          record_error(a.err, S5_ERR_DEVICE_BOUNDS, q_beg + tile0 / G);
        }
      }
#pragma unroll
      for (int j = 0; j < kBpp; ++j) {
        if constexpr (KEY8) {
          kv8[u][j] = make_uint2(0, 0);
          if (phys[u] >= 0 && (pp * kBpp + j) < c_hi) {
            const uint2 *src = keys8 + ((size_t)phys[u] * kBpp + j) * (kDx / 8) + lane;
            asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];"
                         : "=r"(kv8[u][j].x), "=r"(kv8[u][j].y)
                         : "l"(src));
          }
        } else {
          kv[u][j] = make_uint4(0, 0, 0, 0);
          if (phys[u] >= 0 && (pp * kBpp + j) < c_hi) {
            const uint4 *src = keys + ((size_t)phys[u] * kBpp + j) * (kDx / 8) + lane;
            asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(kv[u][j].x), "=r"(kv[u][j].y), "=r"(kv[u][j].z), "=r"(kv[u][j].w)
                         : "l"(src));
          }
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
          float acc = 0.f;
          if constexpr (KEY8) {
            float f[8];
            e4m3x4_to_float(kv8[u][j].x, f[0], f[1], f[2], f[3]);
            e4m3x4_to_float(kv8[u][j].y, f[4], f[5], f[6], f[7]);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc = fmaf(qx[qi][e], f[e], acc);
          } else {
            const uint32_t ww[4] = {kv[u][j].x, kv[u][j].y, kv[u][j].z, kv[u][j].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              acc = fmaf(qx[qi][2 * e], bf16lo(ww[e]), acc);
              acc = fmaf(qx[qi][2 * e + 1], bf16hi(ww[e]), acc);
            }
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
        const int t_q = GROUPED ? ctx + (tile0 + qi) / G : ctx + tile0 + qi;  // position of the row's token
        if (qi < nq && b < t_q / kBlk) {
          const size_t row = (size_t)(q_beg * G + tile0 + qi);
          const float sc = (phys[u] >= 0) ? vals[0] : __int_as_float(0xff800000);  // -inf: unreadable page
          a.scores[row * a.score_stride + b] = sc;
          if (a.hist != nullptr) atomicAdd(a.hist + row * kHistBins + (score_key(sc) >> 20), 1u);
        }
      }
    }
  }
}

template <int QT, int UNROLL, bool GROUPED, bool KEY8>
__global__ void __launch_bounds__(256) index_score_kernel(IndexScoreArgs a) {
  index_score_body<QT, UNROLL, GROUPED, KEY8>(a);
}

// 4-row bf16 tiles (the verify batches' shape) capped at 80 registers so that
// 3 CTAs share an SM: 64 x 4 rows at 32K-128K tokens in 0.106 ms per index
// call against 0.111 ms at 97 registers and 2 CTAs per SM.  (A minimum-blocks
// bound on the shared template would also change the other tiles' register
// allocation.)
__global__ void __launch_bounds__(256, 3) index_score_kernel_rows4(IndexScoreArgs a) {
  index_score_body<4, 1, false, false>(a);
}

// Per-KV-group rows (4 indexer queries per token) on the tensor cores: the
// FMA chain above scores every key against 4 queries, 4x the shared path's
// work, so the same HBM stream leaves it bound by instruction issue.  Here a
// warp scores two pages at a time as one bf16 mma.sync m16n8k16 tile: the 16
// keys (8 of page p, 8 of page p + 1) are the A rows, 8 * NT query rows of
// the sequence the B columns, 16 k-steps over the 256 dims.  Inside each
// k-step the dims are permuted identically for keys and queries (lane quad
// position q holds dims 8q .. 8q + 7 of each 32-dim group), so every
// fragment is one 16-byte load.  Products and sums of the integer-valued
// inputs are exact in the fp32 accumulators, so the scores equal the FMA
// path's.
template <int NT>
__global__ void __launch_bounds__(256) index_score_mma_kernel(IndexScoreArgs a) {
  constexpr int ROWS = 8 * NT;
  pdl_trigger();  // the select may launch now; it waits for these scores before reading them
  const int s = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g8 = lane >> 2, qd = lane & 3;
  const int q_beg = __ldg(a.cu_q + s);
  const int nq_s = __ldg(a.cu_q + s + 1) - q_beg;
  const int G = a.q_groups;
  const int tile0 = blockIdx.z * ROWS;
  if (nq_s < 0 || q_beg < 0 || q_beg + nq_s > a.total_q) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0) record_error(a.err, S5_ERR_DEVICE_BOUNDS, s);
    return;
  }
  if (tile0 >= nq_s * G) return;
  const int nq = min(ROWS, nq_s * G - tile0);
  const int ctx = __ldg(a.ctx_lens + s);
  const int t_last = ctx + (tile0 + nq - 1) / G;
  const int c_hi = t_last / kBlk;  // history blocks of the tile's last row
  if (ctx < 0 || t_last >= a.max_pages * kPage || c_hi > a.score_stride) {
    if (threadIdx.x == 0 && blockIdx.x == 0) record_error(a.err, S5_ERR_DEVICE_BOUNDS, q_beg + tile0 / G);
    return;
  }
  if (c_hi <= a.topk) return;  // every row of the tile keeps all its history blocks
  const int p_beg = blockIdx.x * a.pages_per_cta;
  const int p_end = min(p_beg + a.pages_per_cta, (c_hi + kBpp - 1) / kBpp);
  if (p_beg >= p_end) return;

  // B fragments: query row tile0 + 8 nt + g8, dims 32 sg + 8 qd .. + 7 (zeros past the tile)
  const uint4 *qx = reinterpret_cast<const uint4 *>(a.q_index) + (size_t)(q_beg * G + tile0) * (kDx / 8);
  uint4 qv[NT][kDx / 32];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int row = 8 * nt + g8;
#pragma unroll
    for (int sg = 0; sg < kDx / 32; ++sg)
      qv[nt][sg] = (row < nq) ? __ldg(qx + (size_t)row * (kDx / 8) + 4 * sg + qd) : make_uint4(0, 0, 0, 0);
  }
  const uint4 *keys = reinterpret_cast<const uint4 *>(a.key_pool);
  const int32_t *pt = a.page_table + (size_t)s * a.max_pages;
  const int nwarps = blockDim.x >> 5;
  for (int p = p_beg + 2 * warp; p < p_end; p += 2 * nwarps) {
    // 16-row tiles (4-token verify groups): the pages of this warp's next step,
    // into L2 (0.230 -> 0.199 ms per 64 x 16-row index call; 8-row decode tiles
    // run slower with it, 0.152 -> 0.160 ms)
    if (NT == 2 && lane < 2) {
      const int pn = p + 2 * nwarps + lane;
      if (pn < p_end) {
        const int x = __ldg(pt + pn);
        if (x >= 0 && x < a.num_pages) bulk_prefetch_l2(keys + (size_t)x * kBpp * (kDx / 8), kBpp * kDx * 2);
      }
    }
    int ph[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      ph[u] = -1;
      if (p + u < p_end) {
        const int x = __ldg(pt + p + u);
        if (x >= 0 && x < a.num_pages) ph[u] = x;
        else if (lane == 0) record_error(a.err, S5_ERR_DEVICE_BOUNDS, q_beg + tile0 / G);
      }
    }
    const int b0 = (p * kBpp) + g8, b1 = b0 + kBpp;  // A rows g8 (page p) and g8 + 8 (page p + 1)
    const bool ok0 = ph[0] >= 0 && b0 < c_hi, ok1 = ph[1] >= 0 && b1 < c_hi;
    uint4 xk[kDx / 32], yk[kDx / 32];
#pragma unroll
    for (int sg = 0; sg < kDx / 32; ++sg) {
      xk[sg] = make_uint4(0, 0, 0, 0);
      yk[sg] = make_uint4(0, 0, 0, 0);
      if (ok0) {
        const uint4 *src = keys + ((size_t)ph[0] * kBpp + g8) * (kDx / 8) + 4 * sg + qd;
        asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(xk[sg].x), "=r"(xk[sg].y), "=r"(xk[sg].z), "=r"(xk[sg].w)
                     : "l"(src));
      }
      if (ok1) {
        const uint4 *src = keys + ((size_t)ph[1] * kBpp + g8) * (kDx / 8) + 4 * sg + qd;
        asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(yk[sg].x), "=r"(yk[sg].y), "=r"(yk[sg].z), "=r"(yk[sg].w)
                     : "l"(src));
      }
    }
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
    for (int sg = 0; sg < kDx / 32; ++sg) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // k-step 2 sg + h: dims 32 sg + 8 qd + 4 h + {0,1} and {2,3}
        const uint32_t af[4] = {h ? xk[sg].z : xk[sg].x, h ? yk[sg].z : yk[sg].x, h ? xk[sg].w : xk[sg].y,
                                h ? yk[sg].w : yk[sg].y};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_bf16_16816(acc[nt], af, h ? qv[nt][sg].z : qv[nt][sg].x, h ? qv[nt][sg].w : qv[nt][sg].y);
      }
    }
    // acc[nt][e] = score of block b0, row 8 nt + 2 qd + e; acc[nt][2 + e]: block b1
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int row = 8 * nt + 2 * qd + e;
        if (row >= nq) continue;
        const int lim = (ctx + (tile0 + row) / G) / kBlk;  // history blocks of the row's token
        const size_t grow = (size_t)(q_beg * G + tile0 + row);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int b = u ? b1 : b0;
          if (p + u < p_end && b < lim) {
            const float sc = (ph[u] >= 0) ? acc[nt][2 * u + e] : __int_as_float(0xff800000);  // -inf: unreadable page
            a.scores[grow * a.score_stride + b] = sc;
            if (a.hist != nullptr) atomicAdd(a.hist + grow * kHistBins + (score_key(sc) >> 20), 1u);
          }
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

// Emission of a selection: keys > t_hi are taken, and of the keys in
// [t_lo, t_hi] the first kk in list order; emit(pos, list_position, key) in
// list order.  One scan of the packed per-thread counts (keys above in the
// high 16 bits, keys inside in the low 16) gives both prefixes: a thread's
// first output goes to above_before + min(inside_before, kk).
template <int NT, int EMAX, typename Emit>
__device__ __forceinline__ void emit_selected(const uint32_t (&key)[EMAX], int mine, int first, uint32_t t_lo,
                                              uint32_t t_hi, int kk, int k_out, int *scan_buf, Emit emit) {
  int in = 0, gt = 0;
#pragma unroll
  for (int j = 0; j < EMAX; ++j) {
    if (j < mine) {
      gt += key[j] > t_hi;
      in += (key[j] >= t_lo) & (key[j] <= t_hi);
    }
  }
  const int before = block_excl_scan<NT>((gt << 16) | in, scan_buf);  // list length <= 65535
  const int in_before = before & 0xFFFF;
  int pos = (before >> 16) + min(in_before, kk);
  int r = in_before;
#pragma unroll
  for (int j = 0; j < EMAX; ++j) {
    if (j < mine) {
      const bool inr = (key[j] >= t_lo) & (key[j] <= t_hi);
      const bool tk = key[j] > t_hi || (inr && r < kk);
      r += inr;
      if (tk && pos < k_out) emit(pos, first + j, key[j]);  // never past the k outputs
      pos += tk;
    }
  }
}

// Top-k of a list of n keys (n > k >= 1).  Thread t owns list positions
// t*E .. t*E+E-1 (E <= EMAX, a multiple of 4) and holds their keys in
// registers.  Radix select on 8-bit digits from the top: each pass histograms
// the digit of the keys still matching the chosen prefix into per-warp
// histograms (no atomics shared between warps), sums them and picks the bin
// holding the kk-th largest; it stops early when that whole bin is taken.
// Then the keys above the final range and the first kk keys inside it (list
// order) are emitted as emit(pos, list_position, key), pos = 0..k-1 in list
// order.
template <int NT, int EMAX, typename Emit>
__device__ void cta_select(const uint32_t (&key)[EMAX], int n, int E, int k, SelectSmem<NT> &sm, Emit emit) {
  constexpr int NW = NT / 32;
  static_assert(NT >= 256, "one thread per bin when summing histograms");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int first = tid * E;
  const int mine = max(0, min(E, n - first));
  uint32_t prefix = 0, mask = 0;
  int kk = k;
  uint32_t *wh = sm.whist[warp];
  for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
    for (int i = 0; i < 256 / 32; ++i) wh[lane + 32 * i] = 0;
    __syncwarp();
#pragma unroll
    for (int j = 0; j < EMAX; ++j)
      if (j < mine && (key[j] & mask) == prefix) atomicAdd(&wh[(key[j] >> shift) & 255u], 1u);
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
  emit_selected<NT, EMAX>(key, mine, first, prefix, prefix | ~mask, kk, k, sm.scan_a, emit);
}

// Positions per thread for an n-long list: a multiple of 4 (whole float4 loads).
template <int NT>
__host__ __device__ constexpr int owned_per_thread(int n) {
  return (((n + NT - 1) / NT) + 3) & ~3;
}

// The keys of scores row[0..n) owned by this thread (positions t*E ..), all
// loads in flight together.  row is 16-byte aligned and readable up to the
// next multiple of 4.
template <int NT, int EMAX>
__device__ __forceinline__ void load_keys(const float *row, int n, int E, uint32_t (&key)[EMAX]) {
  const int t = threadIdx.x;
  const float4 *r4 = reinterpret_cast<const float4 *>(row + (size_t)t * E);
  float4 v[EMAX / 4];
#pragma unroll
  for (int q = 0; q < EMAX / 4; ++q)
    v[q] = (4 * q < E && t * E + 4 * q < n) ? ld_cg(r4 + q) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int q = 0; q < EMAX / 4; ++q) {
    key[4 * q] = score_key(v[q].x);
    key[4 * q + 1] = score_key(v[q].y);
    key[4 * q + 2] = score_key(v[q].z);
    key[4 * q + 3] = score_key(v[q].w);
  }
}

// Selection row -> (history blocks c) of its token: r, or r / 4 with one
// selection per KV group (a.q_groups = 4; looked at only when GROUPED).
// Returns false on bad batch data.
template <bool GROUPED = true>
__device__ __forceinline__ bool row_history(const SelectArgs &a, int r, int &c) {
  static_assert(kKv == 4, "rows of per-group selections map to tokens by a shift");
  int s, t;
  const int tok = GROUPED ? r >> (a.q_groups > 1 ? 2 : 0) : r;
  if (!locate_row(a.cu_q, a.ctx_lens, a.batch, tok, row_guess(tok, a.batch, a.total_q), s, t)) return false;
  if (t < 0 || t / kBlk > a.score_stride) return false;
  c = t / kBlk;
  return true;
}

__device__ __forceinline__ void write_all(int32_t *out, int n, int topk, int nt) {
  for (int i = threadIdx.x; i < topk; i += nt) out[i] = (i < n) ? i : -1;
}

constexpr int kCandMax = 2048;  // threshold bins up to this size are refined over their gathered keys

struct HistSmem {
  uint32_t h1[kHistBins];       // row histogram of the top 12 key bits, when not given
  uint32_t h2[1024];            // 10-bit digits of the threshold bin's keys (refinement passes)
  uint32_t cand[kCandMax];      // keys of the threshold bin (any order)
  int scan_a[32];
  int ncand;
  uint32_t digit, above, bin_cnt;
};

// Bin of the kk-th largest key when thread t owns the NB consecutive bins
// counted from the top, starting at bin (top - t * NB); c[i] is the count of
// bin top - t * NB - i.  Results in sm.digit / above / bin_cnt.
template <int NT, int NB>
__device__ __forceinline__ void find_bin_desc(const uint32_t (&c)[NB], int top, int kk, HistSmem &sm) {
  if (threadIdx.x == 0) {  // defined results even if no bin holds the kk-th key
    sm.digit = 0;
    sm.above = 0;
    sm.bin_cnt = 0;
  }
  int cnt = 0;
#pragma unroll
  for (int i = 0; i < NB; ++i) cnt += (int)c[i];
  const int excl = block_excl_scan<NT>(cnt, sm.scan_a);
  if (excl < kk && kk <= excl + cnt) {
    int acc = excl;
#pragma unroll
    for (int i = 0; i < NB; ++i) {
      if (acc < kk && kk <= acc + (int)c[i]) {
        sm.digit = (uint32_t)(top - (int)threadIdx.x * NB - i);
        sm.above = (uint32_t)acc;
        sm.bin_cnt = c[i];
      }
      acc += (int)c[i];
    }
  }
  __syncthreads();
}

// Single stage from a row histogram of the top 12 key bits (built while the
// scores were produced, or here in shared memory from the keys when a.hist is
// null).  The histogram gives the threshold bin; its keys are then resolved
// by two block-wide radix passes of 10 bits over the bin's keys, gathered into
// shared memory (over all keys when the bin holds more than kCandMax), and the
// selection is written in list order through one bit per owned key.  MINB CTAs per SM: 1 keeps
// every key in registers (short launches: one CTA per row of a decode batch),
// 2 caps registers at 32 per thread so that batches of many rows (prefill)
// run twice as many rows at a time.
template <int NT, int EMAX, int MINB, bool GROUPED>
__global__ void __launch_bounds__(NT, MINB) topk_select_hist_kernel(SelectArgs a) {
  static_assert(NT == 512 || NT == 1024, "row-histogram and refinement bins are split evenly over threads");
  constexpr int NB1 = kHistBins / NT;  // row-histogram bins per thread
  constexpr int NB2 = 1024 / NT;       // refinement bins per thread
  __shared__ HistSmem sm;
  const int r = blockIdx.x;
  const int tid = threadIdx.x;
  int32_t *out = a.sel + (size_t)r * a.topk;
  pdl_trigger();
  pdl_wait();  // every input (batch data, scores, histograms) is read after this point
  int c = 0;
  const bool row_ok = row_history<GROUPED>(a, r, c) && c <= NT * EMAX;
  // this thread's row-histogram bins, top first: 4095 - NB1*t .. (loaded with the keys)
  uint32_t cc1[NB1];
  if (a.hist != nullptr) {
    const uint4 *h4 = reinterpret_cast<const uint4 *>(a.hist + (size_t)r * kHistBins);
#pragma unroll
    for (int q = 0; q < NB1 / 4; ++q) {
      const uint4 hv = ld_cg(h4 + (kHistBins / 4 - 1 - (NB1 / 4) * tid - q));
      cc1[4 * q] = hv.w;
      cc1[4 * q + 1] = hv.z;
      cc1[4 * q + 2] = hv.y;
      cc1[4 * q + 3] = hv.x;
    }
  }
  if (!row_ok) {
    if (tid == 0) {
      record_error(a.err, S5_ERR_DEVICE_BOUNDS, r);
      a.sel_count[r] = 0;
    }
    write_all(out, 0, a.topk, NT);
    return;
  }
  if (c <= a.topk) {
    write_all(out, c, a.topk, NT);
    if (tid == 0) a.sel_count[r] = c;
    return;
  }
  const int E = owned_per_thread<NT>(c);
  const int first = tid * E;
  const int mine = max(0, min(E, c - first));
  uint32_t key[EMAX];
  load_keys<NT, EMAX>(a.scores + (size_t)r * a.score_stride, c, E, key);
  if (a.hist == nullptr) {
#pragma unroll
    for (int i = 0; i < kHistBins / NT; ++i) sm.h1[tid + i * NT] = 0;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < EMAX; ++j)
      if (j < mine) atomicAdd(&sm.h1[key[j] >> 20], 1u);
    __syncthreads();
#pragma unroll
    for (int i = 0; i < NB1; ++i) cc1[i] = sm.h1[kHistBins - 1 - NB1 * tid - i];
  }
  if (tid == 0) sm.ncand = 0;
  find_bin_desc<NT, NB1>(cc1, kHistBins - 1, a.topk, sm);
  int kk = a.topk - (int)sm.above;
  const uint32_t b1 = sm.digit;
  const int nb = (int)sm.bin_cnt;
  uint32_t t_lo = b1 << 20, t_hi = t_lo | 0xFFFFFu;
  if (nb != kk) {
    // the threshold bin's keys are resolved by two more radix passes of 10
    // bits: over the bin's keys gathered into shared memory when they fit
    // (any order: the counts are the same), else over every key again
    bool gathered = nb <= kCandMax;
    if (gathered) {
#pragma unroll
      for (int j = 0; j < EMAX; ++j)
        if (j < mine && (key[j] >> 20) == b1) {
          const int slot = atomicAdd(&sm.ncand, 1);
          if (slot < kCandMax) sm.cand[slot] = key[j];
        }
      __syncthreads();
      gathered = sm.ncand <= kCandMax;  // (always, with a histogram of these keys)
    }
    const int ncand = gathered ? sm.ncand : 0;
    uint32_t prefix = b1 << 20, mask = 0xFFF00000u;
    for (int shift = 10; shift >= 0; shift -= 10) {
#pragma unroll
      for (int i = 0; i < NB2; ++i) sm.h2[tid + i * NT] = 0;
      __syncthreads();
      if (gathered) {
        for (int i = tid; i < ncand; i += NT) {
          const uint32_t x = sm.cand[i];
          if ((x & mask) == prefix) atomicAdd(&sm.h2[(x >> shift) & 1023u], 1u);
        }
      } else {
#pragma unroll
        for (int j = 0; j < EMAX; ++j)
          if (j < mine && (key[j] & mask) == prefix) atomicAdd(&sm.h2[(key[j] >> shift) & 1023u], 1u);
      }
      __syncthreads();
      uint32_t cc2[NB2];
#pragma unroll
      for (int i = 0; i < NB2; ++i) cc2[i] = sm.h2[1023 - NB2 * tid - i];
      find_bin_desc<NT, NB2>(cc2, 1023, kk, sm);
      kk -= (int)sm.above;
      prefix |= sm.digit << shift;
      mask |= 1023u << shift;
      const bool stop = ((int)sm.bin_cnt == kk);
      __syncthreads();  // sm.digit / above / bin_cnt and h2 are rewritten by the next pass
      if (stop) break;
    }
    t_lo = prefix;
    t_hi = prefix | ~mask;
  }
  // emission in list order: keys above the range, then the first kk keys in it
  // (one bit per owned key; the loop visits only the taken ones)
  static_assert(EMAX <= 32, "one mask bit per owned key");
  uint32_t above = 0u, ge = 0u;
#pragma unroll
  for (int j = 0; j < EMAX; ++j) {
    above |= (uint32_t)(key[j] > t_hi) << j;
    ge |= (uint32_t)(key[j] >= t_lo) << j;
  }
  const uint32_t owned = (mine >= 32) ? 0xFFFFFFFFu : ((1u << mine) - 1u);  // keys past mine are not the row's
  above &= owned;
  const uint32_t inside = ge & ~above & owned;
  const int before = block_excl_scan<NT>((__popc(above) << 16) | __popc(inside), sm.scan_a);  // list length <= 65535
  const int in_before = before & 0xFFFF;
  int pos = (before >> 16) + min(in_before, kk);
  int rin = in_before;
  for (uint32_t m = above | inside; m != 0u; m &= m - 1u) {
    const int j = __ffs(m) - 1;
    const bool inr = (inside >> j) & 1u;
    const bool tk = !inr || rin < kk;
    rin += inr;
    if (tk && pos < a.topk) out[pos] = first + j;  // never past the k outputs
    pos += tk;
  }
  if (tid == 0) a.sel_count[r] = a.topk;
}

// Two stages for long histories.  Stage 1: the top-k of each segment of
// `seg` blocks, as (key, block) candidates in block order.
template <int NT, int EMAX>
__global__ void __launch_bounds__(NT) topk_segment_kernel(SelectArgs a) {
  __shared__ SelectSmem<NT> sm;
  const int r = blockIdx.y;
  const int sg = blockIdx.x;
  pdl_trigger();
  pdl_wait();
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
      a.cand_key[cbase + i] = score_key(ld_cg(sc + i));
      a.cand_idx[cbase + i] = b0 + i;
    }
    return;
  }
  const int E = owned_per_thread<NT>(n);
  uint32_t key[EMAX];
  load_keys<NT, EMAX>(sc, n, E, key);
  cta_select<NT, EMAX>(key, n, E, a.topk, sm, [&](int pos, int i, uint32_t kv) {
    a.cand_key[cbase + pos] = kv;
    a.cand_idx[cbase + pos] = b0 + i;
  });
}

// Stage 2: the top-k of the concatenated candidates of every segment.  Every
// segment but the last holds exactly topk candidates, so candidate L of the
// row is entry L of the row's candidate arrays.
template <int NT, int EMAX>
__global__ void __launch_bounds__(NT) topk_merge_kernel(SelectArgs a) {
  __shared__ SelectSmem<NT> sm;
  const int r = blockIdx.x;
  int32_t *out = a.sel + (size_t)r * a.topk;
  pdl_trigger();
  pdl_wait();
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
  const size_t rbase = (size_t)r * a.n_seg * a.topk;
  if (n <= a.topk) {  // a single segment whose candidates are all taken
    for (int i = threadIdx.x; i < a.topk; i += NT) out[i] = (i < n) ? ld_cg(a.cand_idx + rbase + i) : -1;
    if (threadIdx.x == 0) a.sel_count[r] = n;
    return;
  }
  const int E = owned_per_thread<NT>(n);
  uint32_t key[EMAX];
#pragma unroll
  for (int j = 0; j < EMAX; ++j) {
    const int L = threadIdx.x * E + j;
    key[j] = (j < E && L < n) ? ld_cg(a.cand_key + rbase + L) : 0u;
  }
  cta_select<NT, EMAX>(key, n, E, a.topk, sm,
                       [&](int pos, int i, uint32_t) { out[pos] = ld_cg(a.cand_idx + rbase + i); });
  if (threadIdx.x == 0) a.sel_count[r] = a.topk;
}

// ============================================================================
// launchers
// ============================================================================

// max_q: indexer rows of the longest sequence (tokens x queries per token).
cudaError_t launch_index_score(const IndexScoreArgs &a, int max_q, int grid_pages, int n_seq, cudaStream_t st) {
  const int qt = (max_q <= 1) ? 1 : (max_q <= 2) ? 2 : 4;
  dim3 grid(grid_pages, n_seq, (max_q + qt - 1) / qt);
  if (a.q_groups > 1) {
    if (qt != 4) return cudaErrorInvalidValue;  // >= 4 rows per token
    if (a.key_fp8) {
      index_score_kernel<4, 2, true, true><<<grid, 256, 0, st>>>(a);
    } else if (max_q <= 8) {  // one token's 4 queries (8 MMA columns)
      index_score_mma_kernel<1><<<dim3(grid_pages, n_seq, (max_q + 7) / 8), 256, 0, st>>>(a);
    } else {  // 16 query rows per tile: the keys of a 4-token verify group are read once
      index_score_mma_kernel<2><<<dim3(grid_pages, n_seq, (max_q + 15) / 16), 256, 0, st>>>(a);
    }
  } else if (a.key_fp8) {
    // one-byte keys: half the bytes per page, so tiles of 2 and 4 rows keep twice
    // the pages in flight; one-row tiles keep 2 (48 registers, 5 CTAs per SM:
    // 64 rows x 16,384 blocks in 0.066 ms, against 0.078 ms with 4 pages in
    // flight at 2 CTAs per SM)
    if (qt == 1) index_score_kernel<1, 2, false, true><<<grid, 256, 0, st>>>(a);
    else if (qt == 2) index_score_kernel<2, 4, false, true><<<grid, 256, 0, st>>>(a);
    else index_score_kernel<4, 2, false, true><<<grid, 256, 0, st>>>(a);
  } else if (qt == 1) {
    index_score_kernel<1, 2, false, false><<<grid, 256, 0, st>>>(a);
  } else if (qt == 2) {
    index_score_kernel<2, 2, false, false><<<grid, 256, 0, st>>>(a);
  } else {
    index_score_kernel_rows4<<<grid, 256, 0, st>>>(a);
  }
  return cudaGetLastError();
}

constexpr int kSelThreads = 1024;  // one CTA per row: rows of up to 16,384 blocks
constexpr int kSegThreads = 256;   // stage 1: one CTA per segment of up to 8,192 blocks

// Launch with programmatic stream serialization: the kernel may begin while
// the previous kernel of the stream drains; it calls pdl_wait() before it
// reads any global memory.
template <typename... Args>
cudaError_t launch_pdl(void (*kernel)(Args...), dim3 grid, dim3 block, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

cudaError_t launch_topk_select(const SelectArgs &a, int total_q, bool two_stage, cudaStream_t st) {
  if (!two_stage) {  // with a row histogram from the scoring kernel, or one built in shared memory
    const dim3 grid(total_q), block(kSelThreads);
    if (a.q_groups > 1) {
      if (total_q > 1024)
        return launch_pdl(topk_select_hist_kernel<kSelThreads, 16, 2, true>, grid, block, st, a);
      return launch_pdl(topk_select_hist_kernel<kSelThreads, 16, 1, true>, grid, block, st, a);
    }
    if (total_q > 1024) return launch_pdl(topk_select_hist_kernel<kSelThreads, 16, 2, false>, grid, block, st, a);
    return launch_pdl(topk_select_hist_kernel<kSelThreads, 16, 1, false>, grid, block, st, a);
  }
  cudaError_t e = launch_pdl(topk_segment_kernel<kSegThreads, 32>, dim3(a.n_seg, total_q), dim3(kSegThreads), st, a);
  if (e != cudaSuccess) return e;
  if (a.n_seg * a.topk <= 512 * 16) return launch_pdl(topk_merge_kernel<512, 16>, dim3(total_q), dim3(512), st, a);
  return launch_pdl(topk_merge_kernel<1024, 20>, dim3(total_q), dim3(1024), st, a);
}

}  // namespace s5
