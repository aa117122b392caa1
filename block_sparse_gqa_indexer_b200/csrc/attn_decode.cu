// Gathered grouped-query attention for decode and multi-token verify, shared by
// the sparse layer (selected blocks + current block) and the sliding-window
// layer (the last `window` tokens).
//
// SGLang day-0 blog ("Step 5 Preview: Day-0 Inference and RL Support with
// SGLang and Miles"), "Hybrid Attention": a sparse-layer query attends to the
// tokens of at most 512 chosen 8-token blocks and of its own block; the
// sliding-window layers attend to a 512-token window.  "Kernels from
// StepFun": decode cuts long selections into partitions and combines their
// partial results.  StepFun open-weights blog, "What the config says": the
// head geometry (64 query heads over 4 KV groups of dimension 192).
//
// Work unit: (query row r, KV group g, partition p).  One CTA of 4 warps owns
// a unit; each warp streams its share of the unit's 8-token blocks through a
// private 2-stage shared-memory ring filled by TMA (one 3,072-byte tile of K
// and one of V per block, 128-byte swizzled so ldmatrix reads are
// conflict-free).  The 16 query heads of the group are the M=16 rows of
// mma.sync m16n8k16 tiles: S = Q K^T over one block is a 16x8 tile, P V over
// two blocks a 16x192 accumulation.  Softmax is online (base 2, running max
// per head).  The warps of a CTA merge through shared memory; the partitions
// of a (row, group) are merged in a fixed order by the last of their CTAs to
// finish (or, beyond 1,024 rows, by s5_combine_kernel), so results are
// deterministic.  In multi-token batches the kernel skips the rows whose tile
// the shared-set tile kernel computes.
//
// This path is HBM-bound (16 FLOPs per gathered byte); its QK^T / PV run on
// the tensor pipe only because the FP32 CUDA cores could not keep up with the
// bandwidth.
#include <cuda.h>

#include "s5_common.cuh"
#include "s5_kernels.h"

namespace s5 {

constexpr int kWarps = 4;
constexpr int kStages = 2;
constexpr int kStageBytes = 4 * kBlockBytes;  // K block A, K block B, V block A, V block B
constexpr int kQStride = kD * 2 + 16;         // padded q row (bytes): conflict-free ldmatrix
constexpr int kRingBytes = kWarps * kStages * kStageBytes;
constexpr int kQBytes = kHpg * kQStride;
constexpr int kListOff = kRingBytes + kQBytes;
constexpr int kBarOff = kListOff + 2 * kMaxList * 4;
constexpr int kAttnSmem = kBarOff + kWarps * kStages * 8 + 1024;  // + alignment slack
constexpr uint64_t kWaitNs = 2000000000ull;                       // 2 s per wait
constexpr int kMaxSplitMerge = 32;

// byte offset of (token row r, dim d) inside a 128B-swizzled [8][192] bf16 tile
__device__ __forceinline__ uint32_t swz(int r, int d) {
  const uint32_t off = (uint32_t)((r * 3 + (d >> 6)) * 128 + (d & 63) * 2);
  return off ^ (((off >> 7) & 7u) << 4);
}

// Merge weights of the partitions of one (row, head): w[p] = exp2(lse_p - M) / L
// in partition order, and the merged natural-log lse.  The same arithmetic
// wherever the merge runs, so results do not depend on which partition
// finished last.
__device__ __forceinline__ void partition_weights(const float *pl, int n, float *w, float &lse_nat) {
  float lv[kMaxSplitMerge];  // all loads in flight together (n <= kMaxSplitMerge)
#pragma unroll
  for (int p = 0; p < kMaxSplitMerge; ++p) lv[p] = (p < n) ? ld_cg(pl + p) : -INFINITY;
  float M = -INFINITY;
#pragma unroll
  for (int p = 0; p < kMaxSplitMerge; ++p) M = fmaxf(M, lv[p]);
  const float Mu = (M == -INFINITY) ? 0.f : M;
  float L = 0.f;
#pragma unroll
  for (int p = 0; p < kMaxSplitMerge; ++p) L += (lv[p] == -INFINITY) ? 0.f : hw_exp2(lv[p] - Mu);
  const float inv = (L > 0.f) ? 1.f / L : 0.f;
#pragma unroll
  for (int p = 0; p < kMaxSplitMerge; ++p)
    if (p < n) w[p] = (lv[p] == -INFINITY) ? 0.f : hw_exp2(lv[p] - Mu) * inv;
  lse_nat = (L > 0.f) ? (M + hw_log2(L)) * 0.69314718055994531f : -INFINITY;
}

__device__ __forceinline__ void store_bf16x4(__nv_bfloat16 *dst, float4 v) {
  uint2 w2;
  w2.x = pack_bf16(v.x, v.y);
  w2.y = pack_bf16(v.z, v.w);
  *reinterpret_cast<uint2 *>(dst) = w2;
}

// Standalone merge for batches whose partitions are not merged in place:
// one CTA per (row, head), one float4 of dims per thread.
__global__ void __launch_bounds__(kD / 4) s5_combine_kernel(const AttnArgs a) {
  const size_t rh = blockIdx.x;
  if (a.row_skip != nullptr && ld_cg(a.row_skip + rh / kHeads) != 0) return;  // row computed by the tile kernel
  const int n = a.n_split;
  float w[kMaxSplitMerge];
  float lse;
  partition_weights(a.part_lse + rh * n, n, w, lse);
  const int d = threadIdx.x * 4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int p0 = 0; p0 < n; p0 += 8) {  // eight partitions' loads in flight at a time
    float4 v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if (p0 + q < n) v[q] = ld_cg(reinterpret_cast<const float4 *>(a.part_o + (rh * n + p0 + q) * kD + d));
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (p0 + q < n) {
        acc.x = fmaf(w[p0 + q], v[q].x, acc.x);
        acc.y = fmaf(w[p0 + q], v[q].y, acc.y);
        acc.z = fmaf(w[p0 + q], v[q].z, acc.z);
        acc.w = fmaf(w[p0 + q], v[q].w, acc.w);
      }
    }
  }
  store_bf16x4(reinterpret_cast<__nv_bfloat16 *>(a.out) + rh * kD + d, acc);
  if (threadIdx.x == 0 && a.lse != nullptr) a.lse[rh] = lse;
}

template <int MODE>
__global__ void __launch_bounds__(kWarps * 32, 2)
    gqa_decode_kernel(const AttnArgs a, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *ring = smem;
  uint8_t *q_s = smem + kRingBytes;
  int32_t *blist = reinterpret_cast<int32_t *>(smem + kListOff);
  int32_t *brow = blist + kMaxList;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kBarOff);

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  // flattened grid, partition fastest, then row, then group: rows running
  // together share one group's KV (100 MB per 128K-token sequence, L2-sized)
  const int p = blockIdx.x % a.n_split;
  const int rg = blockIdx.x / a.n_split;
  const int r = rg % a.total_q;
  const int g = rg / a.total_q;

  // ---- the unit's token range -------------------------------------------------
  if (tid < kWarps * kStages) mbar_init(bars + tid, 1);
  fence_mbar_init();
  // programmatic launch: everything above touches shared memory only; every
  // global input (batch data, q, the selection) is read after this wait
  pdl_wait();
  if (a.row_skip != nullptr && ld_cg(a.row_skip + r) != 0) return;  // row computed by the tile kernel
  int s = -1, t = -1, lo_tok = 0, n_list = 0, b_first = 0, n_sel = 0;
  // the selection this unit reads: the row's, or its KV group's (sel_groups = 4)
  const int srow = a.sel_groups > 1 ? r * a.sel_groups + g : r;
  const int sel_cnt = (MODE == kModeSparse) ? ld_cg(a.sel_count + srow) : 0;
  bool bad = !locate_row(a.cu_q, a.ctx_lens, a.batch, r, row_guess(r, a.batch, a.total_q), s, t);
  if (!bad) bad = (t < 0) || (t >= a.max_pages * kPage) || (t >= a.max_len);
  const int c = bad ? 0 : t / kBlk;
  if (!bad) {
    if (MODE == kModeSparse) {
      n_sel = sel_cnt;
      if (n_sel < 0 || n_sel > a.topk || n_sel > c) {
        bad = true;
      } else {
        n_list = n_sel + 1;  // + the current block
      }
    } else {
      lo_tok = max(0, t - a.window + 1);
      b_first = lo_tok / kBlk;
      n_list = c - b_first + 1;
    }
  }
  if (bad) {
    if (tid == 0 && p == 0 && (g == 0 || a.sel_groups > 1)) record_error(a.err, S5_ERR_DEVICE_BOUNDS, r);
    n_list = 0;
  }
  int chunk = (n_list + a.n_split - 1) / a.n_split;
  if (chunk > kMaxList) {  // the host sizes n_split so this cannot happen for valid lengths
    if (tid == 0) record_error(a.err, S5_ERR_DEVICE_BOUNDS, r);
    n_list = chunk = 0;
  }
  const int i_beg = min(n_list, p * chunk);
  const int n_items = min(n_list, i_beg + chunk) - i_beg;

  // (block ids and TMA rows are resolved by each warp for its own items, below)
  const int32_t *pt = a.page_table + (size_t)max(s, 0) * a.max_pages;
  __syncthreads();

  // ---- this warp's share ----------------------------------------------------------
  const int per_w = (n_items + kWarps - 1) / kWarps;
  const int w_beg = min(n_items, warp * per_w);
  const int w_n = min(n_items, w_beg + per_w) - w_beg;
  const int n_pairs = (w_n + 1) / 2;
  uint8_t *wring = ring + warp * kStages * kStageBytes;
  uint64_t *wbar = bars + warp * kStages;
  const uint64_t policy = policy_evict_first();

  auto issue = [&](int j) {  // lane 0 only
    const int st = j % kStages;
    uint8_t *buf = wring + st * kStageBytes;
    uint32_t bytes = 0;
    int rows[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int it = 2 * j + h;
      rows[h] = (it < w_n) ? brow[w_beg + it] : -1;
      if (rows[h] >= 0) bytes += 2 * kBlockBytes;
    }
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(wbar + st, bytes);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (rows[h] >= 0) {
        tma_load_3d(buf + h * kBlockBytes, &tm_k, 0, 0, rows[h], wbar + st, policy);
        tma_load_3d(buf + (2 + h) * kBlockBytes, &tm_v, 0, 0, rows[h], wbar + st, policy);
      }
    }
  };
  // resolve this warp's items to block ids and TMA rows (lane k: items k, k+32, ...);
  // the first 32 are resolved before the first loads are issued
  auto resolve = [&](int k) {
    const int li = i_beg + w_beg + k;
    int b;
    bool ok = true;
    if (MODE == kModeSparse) {
      if (li < n_sel) {
        b = ld_cg(a.sel + (size_t)srow * a.topk + li);
        ok = (b >= 0) && (b < c);
      } else {
        b = c;
      }
    } else {
      b = b_first + li;
    }
    int row = -1;
    if (ok) {
      const int ph = ld_cg(pt + b / kBpp);
      if (ph >= 0 && ph < a.num_pages) row = ((ph * kKv + g) * kPage) + (b % kBpp) * kBlk;
      else ok = false;
    }
    if (!ok) record_error(a.err, S5_ERR_DEVICE_BOUNDS, r);
    blist[w_beg + k] = ok ? b : -1;
    brow[w_beg + k] = row;
  };
  if (lane < w_n) resolve(lane);
  __syncwarp();
  if (lane == 0) {
    for (int j = 0; j < kStages && j < n_pairs; ++j) issue(j);
  }
  // the query tile of the group (16 heads x 192, padded rows) is read while
  // the first blocks are in flight: every thread's loads issued together
  {
    constexpr int kQv = kHpg * (kD / 8) / (kWarps * 32);  // 16-byte pieces per thread
    static_assert(kHpg * (kD / 8) % (kWarps * 32) == 0, "query tile split evenly over the CTA");
    const uint4 *qg = reinterpret_cast<const uint4 *>(a.q) + ((size_t)r * kHeads + g * kHpg) * (kD / 8);
    uint4 qv[kQv];
#pragma unroll
    for (int x = 0; x < kQv; ++x) qv[x] = ld_cg(qg + tid + x * kWarps * 32);
#pragma unroll
    for (int x = 0; x < kQv; ++x) {
      const int i = tid + x * kWarps * 32;
      const int h = i / (kD / 8), cc = i % (kD / 8);
      *reinterpret_cast<uint4 *>(q_s + h * kQStride + cc * 16) = qv[x];
    }
  }
  for (int k = lane + 32; k < w_n; k += 32) resolve(k);
  __syncthreads();  // the query tile is complete

  // Q fragments (A operand) for the 12 k-steps of 16 dims
  uint32_t qa[kD / 16][4];
  {
    const int m = lane >> 3, rr = lane & 7;
    const uint32_t base = smem_u32(q_s) + ((m & 1) * 8 + rr) * kQStride + (m >> 1) * 16;
#pragma unroll
    for (int kk = 0; kk < kD / 16; ++kk) ldsm_x4(base + kk * 32, qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
  }

  float o[kD / 8][4];
#pragma unroll
  for (int i = 0; i < kD / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const float sl2 = a.scale_log2;
  const int tq = lane & 3;
  const int lm = lane >> 3, lr = lane & 7;
  bool timed_out = false;
  int j_fail = n_pairs;

  for (int j = 0; j < n_pairs; ++j) {
    const int st = j % kStages;
    uint8_t *buf = wring + st * kStageBytes;
    // warp-uniform outcome: every lane leaves together if any lane's wait expired
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(wbar + st, (j / kStages) & 1, kWaitNs))) {
      timed_out = true;
      j_fail = j;
      break;
    }
    int bk[2];
    bool full[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int it = 2 * j + h;
      const bool loaded = (it < w_n) && brow[w_beg + it] >= 0;
      bk[h] = loaded ? blist[w_beg + it] : -1;
      full[h] = loaded && (bk[h] * kBlk >= lo_tok) && (bk[h] * kBlk + kBlk - 1 <= t);
      if (!full[h]) {
        // zero V rows of tokens that are not read (absent block, or outside
        // [lo_tok, t]): masked P is 0, and 0 * (stale or non-finite) must not leak
        uint8_t *vb = buf + (2 + h) * kBlockBytes;
        for (int x = lane; x < kBlk * 3 * 8; x += 32) {  // 24 rows of 128 B, 8 x 16 B each
          const int row128 = x >> 3;
          const int tok = row128 / 3;
          const int pos = bk[h] * kBlk + tok;
          if (bk[h] < 0 || pos < lo_tok || pos > t)
            *reinterpret_cast<uint4 *>(vb + row128 * 128 + (x & 7) * 16) = make_uint4(0, 0, 0, 0);
        }
      }
    }
    __syncwarp();
    // ---- S = Q K^T for the two blocks ----
    float sa[2][4];
#pragma unroll
    for (int h = 0; h < 2; ++h) sa[h][0] = sa[h][1] = sa[h][2] = sa[h][3] = 0.f;
    const uint32_t kbase = smem_u32(buf);
#pragma unroll
    for (int kk = 0; kk < kD / 16; kk += 2) {
      const uint32_t off = swz(lr, 16 * kk + 8 * lm);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kbase + h * kBlockBytes + off, b0, b1, b2, b3);
        mma_bf16_16816(sa[h], qa[kk], b0, b1);
        mma_bf16_16816(sa[h], qa[kk + 1], b2, b3);
      }
    }
    // ---- online softmax (rows: head tq-quad row lane/4 and lane/4 + 8) ----
    float mx0 = m0, mx1 = m1;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int pos = bk[h] * kBlk + 2 * tq + e;
        const bool v = bk[h] >= 0 && pos >= lo_tok && pos <= t;
        sa[h][e] = v ? sa[h][e] * sl2 : -INFINITY;
        sa[h][2 + e] = v ? sa[h][2 + e] * sl2 : -INFINITY;
        mx0 = fmaxf(mx0, sa[h][e]);
        mx1 = fmaxf(mx1, sa[h][2 + e]);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float u0 = (mx0 == -INFINITY) ? 0.f : mx0;
    const float u1 = (mx1 == -INFINITY) ? 0.f : mx1;
    const float cr0 = hw_exp2(m0 - u0), cr1 = hw_exp2(m1 - u1);
    m0 = mx0;
    m1 = mx1;
    float pr[2][4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      pr[h][0] = hw_exp2(sa[h][0] - u0);
      pr[h][1] = hw_exp2(sa[h][1] - u0);
      pr[h][2] = hw_exp2(sa[h][2] - u1);
      pr[h][3] = hw_exp2(sa[h][3] - u1);
    }
    l0 = l0 * cr0 + (pr[0][0] + pr[0][1] + pr[1][0] + pr[1][1]);
    l1 = l1 * cr1 + (pr[0][2] + pr[0][3] + pr[1][2] + pr[1][3]);
#pragma unroll
    for (int i = 0; i < kD / 8; ++i) {
      o[i][0] *= cr0;
      o[i][1] *= cr0;
      o[i][2] *= cr1;
      o[i][3] *= cr1;
    }
    const uint32_t pa[4] = {pack_bf16(pr[0][0], pr[0][1]), pack_bf16(pr[0][2], pr[0][3]),
                            pack_bf16(pr[1][0], pr[1][1]), pack_bf16(pr[1][2], pr[1][3])};
    // ---- O += P V ----
    const uint32_t vbase = smem_u32(buf) + 2 * kBlockBytes + (lm & 1) * kBlockBytes;
#pragma unroll
    for (int np = 0; np < kD / 16; ++np) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(vbase + swz(lr, 16 * np + 8 * (lm >> 1)), b0, b1, b2, b3);
      mma_bf16_16816(o[2 * np], pa, b0, b1);
      mma_bf16_16816(o[2 * np + 1], pa, b2, b3);
    }
    // order this stage's generic reads / zero fills before the next async-proxy write into it
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && j + kStages < n_pairs) issue(j + kStages);
  }
  // a warp may leave the loop early only after a wait expired
  timed_out = __any_sync(0xffffffffu, timed_out);
  if (timed_out) {
    if (lane == 0) record_error(a.err, S5_ERR_TIMEOUT, r);
    // drain: wait (bounded) for the copies still in flight (issued, not consumed)
    for (int j2 = j_fail; j2 < n_pairs && j2 < j_fail + kStages; ++j2)
      mbar_wait_bounded(wbar + (j2 % kStages), (j2 / kStages) & 1, kWaitNs);
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.f;
  }
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

  // ---- merge the 4 warps (each writes into its own ring slice) ----
  float *ow = reinterpret_cast<float *>(wring);  // [16][192] fp32, then m[16], l[16]
  {
    const int r0 = lane >> 2;
#pragma unroll
    for (int i = 0; i < kD / 8; ++i) {
      const int col = i * 8 + 2 * tq;
      const float z = timed_out ? 0.f : 1.f;
      *reinterpret_cast<float2 *>(ow + r0 * kD + col) = make_float2(o[i][0] * z, o[i][1] * z);
      *reinterpret_cast<float2 *>(ow + (r0 + 8) * kD + col) = make_float2(o[i][2] * z, o[i][3] * z);
    }
    if (tq == 0) {
      ow[kHpg * kD + r0] = m0;
      ow[kHpg * kD + r0 + 8] = m1;
      ow[kHpg * kD + kHpg + r0] = l0;
      ow[kHpg * kD + kHpg + r0 + 8] = l1;
    }
  }
  __syncthreads();
  {
    const int h = tid >> 3;         // 16 heads x 8 threads
    const int d0 = (tid & 7) * 24;  // 24 dims each
    float mw[kWarps], lw[kWarps];
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float *oww = reinterpret_cast<const float *>(ring + w * kStages * kStageBytes);
      mw[w] = oww[kHpg * kD + h];
      lw[w] = oww[kHpg * kD + kHpg + h];
      M = fmaxf(M, mw[w]);
    }
    const float Mu = (M == -INFINITY) ? 0.f : M;
    float L = 0.f, sc[kWarps];
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      sc[w] = (lw[w] > 0.f) ? hw_exp2(mw[w] - Mu) : 0.f;
      L += lw[w] * sc[w];
    }
    const float inv = (L > 0.f) ? 1.f / L : 0.f;
    const int hg = g * kHpg + h;
    const size_t rh = (size_t)r * kHeads + hg;
    float acc[24];
#pragma unroll
    for (int e = 0; e < 24; ++e) acc[e] = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float *oww = reinterpret_cast<const float *>(ring + w * kStages * kStageBytes) + h * kD + d0;
#pragma unroll
      for (int e = 0; e < 24; e += 4) {
        const float4 v = *reinterpret_cast<const float4 *>(oww + e);
        acc[e] += v.x * sc[w];
        acc[e + 1] += v.y * sc[w];
        acc[e + 2] += v.z * sc[w];
        acc[e + 3] += v.w * sc[w];
      }
    }
    const float lse2 = (L > 0.f) ? (M + hw_log2(L)) : -INFINITY;
    if (a.n_split == 1) {
      __nv_bfloat16 *out = reinterpret_cast<__nv_bfloat16 *>(a.out) + rh * kD + d0;
#pragma unroll
      for (int e = 0; e < 24; e += 8) {
        uint4 w4;
        w4.x = pack_bf16(acc[e] * inv, acc[e + 1] * inv);
        w4.y = pack_bf16(acc[e + 2] * inv, acc[e + 3] * inv);
        w4.z = pack_bf16(acc[e + 4] * inv, acc[e + 5] * inv);
        w4.w = pack_bf16(acc[e + 6] * inv, acc[e + 7] * inv);
        *reinterpret_cast<uint4 *>(out + e) = w4;
      }
      if ((tid & 7) == 0 && a.lse != nullptr) a.lse[rh] = lse2 * 0.69314718055994531f;
    } else {
      float *po = a.part_o + (rh * a.n_split + p) * kD + d0;
#pragma unroll
      for (int e = 0; e < 24; e += 4)
        *reinterpret_cast<float4 *>(po + e) =
            make_float4(acc[e] * inv, acc[e + 1] * inv, acc[e + 2] * inv, acc[e + 3] * inv);
      if ((tid & 7) == 0) a.part_lse[rh * a.n_split + p] = lse2;
    }
  }
  if (a.n_split == 1 || a.merge_cnt == nullptr) return;

  // ---- the last partition CTA of (r, g) to arrive merges every partition ----
  __shared__ int is_last;
  __shared__ float w_s[kHpg][kMaxSplitMerge];
  __shared__ float lse_s[kHpg];
  __threadfence();  // publish this CTA's partial before counting it
  __syncthreads();
  if (tid == 0) {
    const uint32_t prev = atomicAdd(a.merge_cnt + (size_t)r * kKv + g, 1u);
    is_last = (prev == (uint32_t)a.n_split - 1);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  const int n = a.n_split;
  const size_t rh0 = (size_t)r * kHeads + g * kHpg;
  if (tid < kHpg) partition_weights(a.part_lse + (rh0 + tid) * n, n, w_s[tid], lse_s[tid]);
  __syncthreads();
  {
    const int h = tid >> 3;          // 16 heads x 8 threads
    const int c0 = (tid & 7) * 6;    // 6 float4 columns each
    const size_t rh = rh0 + h;
    const float4 *src = reinterpret_cast<const float4 *>(a.part_o + rh * n * kD) + c0;
    float4 acc[6];
#pragma unroll
    for (int c = 0; c < 6; ++c) acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p0 = 0; p0 < n; p0 += 4) {
      float4 v[4][6];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int c = 0; c < 6; ++c)
          if (p0 + q < n) v[q][c] = ld_cg(src + (size_t)(p0 + q) * (kD / 4) + c);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (p0 + q < n) {
          const float wp = w_s[h][p0 + q];
#pragma unroll
          for (int c = 0; c < 6; ++c) {
            acc[c].x = fmaf(wp, v[q][c].x, acc[c].x);
            acc[c].y = fmaf(wp, v[q][c].y, acc[c].y);
            acc[c].z = fmaf(wp, v[q][c].z, acc[c].z);
            acc[c].w = fmaf(wp, v[q][c].w, acc[c].w);
          }
        }
      }
    }
    __nv_bfloat16 *out = reinterpret_cast<__nv_bfloat16 *>(a.out) + rh * kD;
#pragma unroll
    for (int c = 0; c < 6; ++c) store_bf16x4(out + 4 * (c0 + c), acc[c]);
    if ((tid & 7) == 0 && a.lse != nullptr) a.lse[rh] = lse_s[h];
  }
  if (tid == 0) a.merge_cnt[(size_t)r * kKv + g] = 0u;  // ready for the next call
}

cudaError_t launch_gqa_decode(int mode, const AttnArgs &a, const CUtensorMap &tk, const CUtensorMap &tv,
                              int total_q, cudaStream_t st) {
  const long long n_cta = (long long)a.n_split * total_q * kKv;
  if (n_cta > 0x7fffffffLL) return cudaErrorInvalidValue;
  dim3 grid((unsigned)n_cta);
  cudaError_t e;
  auto kernel = (mode == kModeSparse) ? gqa_decode_kernel<kModeSparse> : gqa_decode_kernel<kModeSwa>;
  e = ensure_dynamic_smem(reinterpret_cast<const void *>(kernel), kAttnSmem);
  if (e != cudaSuccess) return e;
  // programmatic stream serialization: launch and barrier setup overlap the
  // previous kernel; the kernel reads no global memory before pdl_wait()
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kWarps * 32);
  cfg.dynamicSmemBytes = kAttnSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kernel, a, tk, tv);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess || a.n_split == 1 || a.merge_cnt != nullptr) return e;
  s5_combine_kernel<<<(unsigned)total_q * kHeads, kD / 4, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace s5
