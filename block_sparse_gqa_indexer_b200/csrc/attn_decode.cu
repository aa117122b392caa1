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
//
// One-byte KV (sparse layer; StepFun open-weights blog, "Fitting it on a
// node": FP8 KV for the full-attention layers): the same kernel with E4M3
// blocks of 1,536 bytes, four stages per warp in the same ring.  Each E4M3
// pair widens exactly to an f16 pair in registers (cvt), Q is staged as f16,
// and the MMAs are f16 m16n8k16 with fp32 accumulation; k_scale is folded into
// the softmax scale and v_scale into the final normalisation.  The blocks land
// through a 64-byte-swizzled TMA box; inside every 16-dim k-step the dims are
// permuted identically for Q and K, and the tokens of a block are taken in the
// order 0 1 3 2 4 5 7 6, which together make every fragment load from the
// swizzled tiles free of bank conflicts.
#include <cuda.h>

#include "s5_common.cuh"
#include "s5_kernels.h"

namespace s5 {

constexpr int kWarps = 4;
constexpr int kStages = 2;
constexpr int kStageBytes = 4 * kBlockBytes;  // K block A, K block B, V block A, V block B
constexpr int kBlockBytes8 = kBlk * kD;       // 1,536 bytes: one block of one group, one-byte KV
constexpr int kStages8 = 4;                   // one-byte KV: twice the stages in the same ring
constexpr int kStageBytes8 = 4 * kBlockBytes8;
static_assert(kStages8 * kStageBytes8 == kStages * kStageBytes, "both KV widths share one ring layout");
constexpr int kMaxStages = kStages8;
constexpr int kQStride = kD * 2 + 16;         // padded q row (bytes): conflict-free ldmatrix
constexpr int kQBytes = kHpg * kQStride;
// Grids that fit one CTA per SM (the smallest batches) run a deep variant with
// kDeep times the ring stages per warp: with one CTA on an SM the shared memory
// is there, and a warp's few block pairs are in flight together instead of one
// HBM round trip per pair.
constexpr int kDeep = 2;
template <bool DEEP>
__host__ __device__ constexpr int ring_bytes() {
  return kWarps * kStages * kStageBytes * (DEEP ? kDeep : 1);
}
template <bool DEEP>
__host__ __device__ constexpr int list_off() {
  return ring_bytes<DEEP>() + kQBytes;
}
template <bool DEEP>
__host__ __device__ constexpr int bar_off() {
  return list_off<DEEP>() + 2 * kMaxList * 4;
}
template <bool DEEP>  // + a stall barrier, alignment slack
__host__ __device__ constexpr int attn_smem() {
  return bar_off<DEEP>() + (kWarps * kMaxStages * (DEEP ? kDeep : 1) + 1) * 8 + 1024;
}
static_assert(attn_smem<true>() <= 227 * 1024, "deep variant: shared memory per CTA");
constexpr uint64_t kWaitNs = 2000000000ull;                       // 2 s per wait
constexpr float kLazyMax = 8.0f;  // log2 units: a softmax reference max moves only when exceeded by more
constexpr int kMaxSplitMerge = 32;

// byte offset of (token row r, dim d) inside a 128B-swizzled [8][192] bf16 tile
__device__ __forceinline__ uint32_t swz(int r, int d) {
  const uint32_t off = (uint32_t)((r * 3 + (d >> 6)) * 128 + (d & 63) * 2);
  return off ^ (((off >> 7) & 7u) << 4);
}

// byte offset of (token row r, dim d) inside a 64B-swizzled [8][192] one-byte
// tile: the 16-byte unit of every 64-byte segment is XORed with bits 7..8 of
// the offset (the TMA 64-byte swizzle)
__device__ __forceinline__ uint32_t swz8(int r, int d) {
  const uint32_t off = (uint32_t)(r * kD + d);
  return off ^ (((off >> 7) & 3u) << 4);
}

// token of a block behind mma column n in the one-byte path (0 1 3 2 4 5 7 6)
__device__ __forceinline__ int tok8(int n) { return n ^ ((n >> 1) & 1); }

// f16 m16n8k16 with fp32 accumulate (both operands f16)
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// four E4M3 codes (byte i = element i) to their exact values as two f16 pairs:
// lo = elements 0, 1 and hi = elements 2, 3 (first element in the low half);
// one conversion instruction per pair, straight into the MMA operand register
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t w, uint32_t &lo, uint32_t &hi) {
  asm("{\n\t.reg .b16 a, b;\n\t"
      "mov.b32 {a, b}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, a;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

// eight bf16 values to f16 (round to nearest; exact within the f16 normal range)
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 v) {
  return make_uint4(pack_f16(bf16lo(v.x), bf16hi(v.x)), pack_f16(bf16lo(v.y), bf16hi(v.y)),
                    pack_f16(bf16lo(v.z), bf16hi(v.z)), pack_f16(bf16lo(v.w), bf16hi(v.w)));
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

template <int MODE, bool KV8, bool DEEP>
__global__ void __launch_bounds__(kWarps * 32, 2)
    gqa_decode_kernel(const AttnArgs a, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v) {
  constexpr int NST = (KV8 ? kStages8 : kStages) * (DEEP ? kDeep : 1);  // ring stages per warp
  constexpr int BB = KV8 ? kBlockBytes8 : kBlockBytes;  // one block of one group (K or V)
  constexpr int SB = 4 * BB;                            // one stage: K A, K B, V A, V B
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *ring = smem;
  uint8_t *q_s = smem + ring_bytes<DEEP>();
  int32_t *blist = reinterpret_cast<int32_t *>(smem + list_off<DEEP>());
  int32_t *brow = blist + kMaxList;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + bar_off<DEEP>());

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
  uint64_t *stall_bar = bars + kWarps * NST;  // nothing ever arrives on it (expired-wait test hook)
  if (tid <= kWarps * NST) mbar_init(bars + tid, 1);
  fence_mbar_init();
  // programmatic launch: everything above touches shared memory only; every
  // global input (batch data, q, the selection) is read after this wait
  pdl_wait();
  if (a.row_skip != nullptr && ld_cg(a.row_skip + r) != 0) return;  // row computed by the tile kernel
  // the query tile of the group (16 heads x 192) is loaded first: its address
  // needs only the row and group, so it is in flight during the lookups below
  constexpr int kQv = kHpg * (kD / 8) / (kWarps * 32);  // 16-byte pieces per thread
  static_assert(kHpg * (kD / 8) % (kWarps * 32) == 0, "query tile split evenly over the CTA");
  uint4 qv[kQv];
  {
    const uint4 *qg = reinterpret_cast<const uint4 *>(a.q) + ((size_t)r * kHeads + g * kHpg) * (kD / 8);
#pragma unroll
    for (int x = 0; x < kQv; ++x) qv[x] = ld_cg(qg + tid + x * kWarps * 32);
  }
  // expired-wait test hook (workspace header, zero in normal use): a nonzero
  // count of nanoseconds makes each warp's first stage wait also wait that long
  // on stall_bar and then leave through the expired-wait path below
  const uint64_t stall_ns = (a.err != nullptr) ? ld_cg_u64(reinterpret_cast<const uint64_t *>(a.err) + kWsStallWord) : 0;
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
  uint8_t *wring = ring + warp * NST * SB;
  uint64_t *wbar = bars + warp * NST;
  const uint64_t policy = policy_evict_first();

  auto issue = [&](int j) {  // lane 0 only
    const int st = j % NST;
    uint8_t *buf = wring + st * SB;
    uint32_t bytes = 0;
    int rows[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int it = 2 * j + h;
      rows[h] = (it < w_n) ? brow[w_beg + it] : -1;
      if (rows[h] >= 0) bytes += 2 * BB;
    }
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(wbar + st, bytes);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (rows[h] >= 0) {
        tma_load_3d(buf + h * BB, &tm_k, 0, 0, rows[h], wbar + st, policy);
        tma_load_3d(buf + (2 + h) * BB, &tm_v, 0, 0, rows[h], wbar + st, policy);
      }
    }
  };
  // resolve this warp's items to block ids and TMA rows (lane k: items k, k+32,
  // ...) in two rounds of loads, every load of a round in flight together:
  // the selected blocks, then their pages
  {
    constexpr int kRes = ((kMaxList + kWarps - 1) / kWarps + 31) / 32;  // items per lane at most
    static_assert(kRes * 32 * kWarps >= kMaxList, "a warp owns at most ceil(kMaxList / kWarps) items");
    int bv[kRes], ph[kRes];
#pragma unroll
    for (int u = 0; u < kRes; ++u) {
      const int k = lane + 32 * u, li = i_beg + w_beg + k;
      bv[u] = (MODE == kModeSparse) ? c : b_first + li;
      if (MODE == kModeSparse && k < w_n && li < n_sel) bv[u] = ld_cg(a.sel + (size_t)srow * a.topk + li);
    }
#pragma unroll
    for (int u = 0; u < kRes; ++u) {
      const int k = lane + 32 * u, li = i_beg + w_beg + k;
      const bool ok = k < w_n && (MODE != kModeSparse || li >= n_sel || (bv[u] >= 0 && bv[u] < c));
      ph[u] = -1;
      if (ok) ph[u] = ld_cg(pt + bv[u] / kBpp);
      if (k < w_n && !ok) bv[u] = -1;
    }
#pragma unroll
    for (int u = 0; u < kRes; ++u) {
      const int k = lane + 32 * u;
      if (k < w_n) {
        const bool ok = bv[u] >= 0 && ph[u] >= 0 && ph[u] < a.num_pages;
        if (!ok) record_error(a.err, S5_ERR_DEVICE_BOUNDS, r);
        blist[w_beg + k] = ok ? bv[u] : -1;
        brow[w_beg + k] = ok ? ((ph[u] * kKv + g) * kPage) + (bv[u] % kBpp) * kBlk : -1;
      }
    }
  }
  __syncwarp();
  if (lane == 0) {
    for (int j = 0; j < NST && j < n_pairs; ++j) issue(j);
  }
  // the query tile into shared memory (one-byte KV: as f16, which its MMAs take)
#pragma unroll
  for (int x = 0; x < kQv; ++x) {
    const int i = tid + x * kWarps * 32;
    const int h = i / (kD / 8), cc = i % (kD / 8);
    *reinterpret_cast<uint4 *>(q_s + h * kQStride + cc * 16) = KV8 ? bf16x8_to_f16x8(qv[x]) : qv[x];
  }
  __syncthreads();  // the query tile is complete

  // Q fragments (A operand) for the 12 k-steps of 16 dims
  uint32_t qa[kD / 16][4];
  if constexpr (KV8) {
    // k-step 4c + j: lanes with lane % 4 == i hold dims 64c + 16i + 4j + {0,1} (k slots 2i, 2i+1)
    // and + {2,3} (k slots 2i+8, 2i+9); the K fragments below use the same map
    const int gq = lane >> 2, iq = lane & 3;
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      const uint4 *r0 = reinterpret_cast<const uint4 *>(q_s + gq * kQStride + (64 * c + 16 * iq) * 2);
      const uint4 *r1 = reinterpret_cast<const uint4 *>(q_s + (gq + 8) * kQStride + (64 * c + 16 * iq) * 2);
      const uint4 x0 = r0[0], x1 = r0[1], y0 = r1[0], y1 = r1[1];
      const uint32_t wa[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
      const uint32_t wb[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        qa[4 * c + j][0] = wa[2 * j];
        qa[4 * c + j][1] = wb[2 * j];
        qa[4 * c + j][2] = wa[2 * j + 1];
        qa[4 * c + j][3] = wb[2 * j + 1];
      }
    }
  } else {
    const int m = lane >> 3, rr = lane & 7;
    const uint32_t base = smem_u32(q_s) + ((m & 1) * 8 + rr) * kQStride + (m >> 1) * 16;
#pragma unroll
    for (int kk = 0; kk < kD / 16; ++kk) ldsm_x4(base + kk * 32, qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
  }
  // one-byte KV: swizzled byte offsets of this lane's fragment loads inside a block tile
  // (K: token tok8(lane/4), 16 dims per 64-dim chunk; V: tokens tok8(2i), tok8(2i+1), 8 dims)
  uint32_t koff[3], voff0[3], voff1[3];
  if constexpr (KV8) {
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      koff[c] = swz8(tok8(lane >> 2), 64 * c + 16 * (lane & 3));
      voff0[c] = swz8(tok8(2 * (lane & 3)), 64 * c + 8 * (lane >> 2));
      voff1[c] = swz8(tok8(2 * (lane & 3) + 1), 64 * c + 8 * (lane >> 2));
    }
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
    const int st = j % NST;
    uint8_t *buf = wring + st * SB;
    // warp-uniform outcome: every lane leaves together if any lane's wait expired
    // (each poll may suspend the warp for up to 1 us: one-byte KV at the
    // 64 x 131,072 headline shape 0.1044 -> 0.1024 ms; bf16 KV unchanged)
    bool landed = mbar_wait_bounded_hint(wbar + st, (j / NST) & 1, kWaitNs, 1000u);
    if (stall_ns != 0 && j == 0) landed = landed && mbar_wait_bounded(stall_bar, 0, stall_ns);
    if (!__all_sync(0xffffffffu, landed)) {
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
        uint8_t *vb = buf + (2 + h) * BB;
        if constexpr (KV8) {
          for (int x = lane; x < kBlk * (kD / 16); x += 32) {  // 8 token rows of 12 x 16 B
            const int tok = x / (kD / 16);                      // (the swizzle stays inside a row)
            const int pos = bk[h] * kBlk + tok;
            if (bk[h] < 0 || pos < lo_tok || pos > t)
              *reinterpret_cast<uint4 *>(vb + x * 16) = make_uint4(0, 0, 0, 0);
          }
        } else {
          for (int x = lane; x < kBlk * 3 * 8; x += 32) {  // 24 rows of 128 B, 8 x 16 B each
            const int row128 = x >> 3;
            const int tok = row128 / 3;
            const int pos = bk[h] * kBlk + tok;
            if (bk[h] < 0 || pos < lo_tok || pos > t)
              *reinterpret_cast<uint4 *>(vb + row128 * 128 + (x & 7) * 16) = make_uint4(0, 0, 0, 0);
          }
        }
      }
    }
    __syncwarp();
    // ---- S = Q K^T for the two blocks ----
    // two accumulators per block (even / odd k-steps) halve the dependent MMA chain
    float sa[2][4], sb[2][4];
#pragma unroll
    for (int h = 0; h < 2; ++h) sa[h][0] = sa[h][1] = sa[h][2] = sa[h][3] = sb[h][0] = sb[h][1] = sb[h][2] = sb[h][3] = 0.f;
    if constexpr (KV8) {
#pragma unroll
      for (int c = 0; c < 3; ++c) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint4 w = *reinterpret_cast<const uint4 *>(buf + h * BB + koff[c]);
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t b0, b1;
            e4m3x4_to_f16x2x2(ww[j], b0, b1);
            mma_f16_16816((j & 1) ? sb[h] : sa[h], qa[4 * c + j], b0, b1);
          }
        }
      }
    } else {
      const uint32_t kbase = smem_u32(buf);
#pragma unroll
      for (int kk = 0; kk < kD / 16; kk += 2) {
        const uint32_t off = swz(lr, 16 * kk + 8 * lm);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kbase + h * BB + off, b0, b1, b2, b3);
          mma_bf16_16816(sa[h], qa[kk], b0, b1);
          mma_bf16_16816(sb[h], qa[kk + 1], b2, b3);
        }
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int e = 0; e < 4; ++e) sa[h][e] += sb[h][e];
    // ---- online softmax (rows: head lane/4 and lane/4 + 8) ----
    // m0 / m1 are reference maxima: the weights are exp2(s - m), and a
    // reference moves (and O is rescaled) only when a row's maximum exceeds it
    // by more than kLazyMax, so weights stay below 2^8 and after the first
    // blocks O is almost never rescaled
    float mx0 = -INFINITY, mx1 = -INFINITY;
    if (full[0] && full[1]) {  // (warp-uniform) every token of both blocks is read: no masks
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          sa[h][e] *= sl2;
          sa[h][2 + e] *= sl2;
          mx0 = fmaxf(mx0, sa[h][e]);
          mx1 = fmaxf(mx1, sa[h][2 + e]);
        }
      }
    } else {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int pos = bk[h] * kBlk + (KV8 ? tok8(2 * tq + e) : 2 * tq + e);
          const bool v = bk[h] >= 0 && pos >= lo_tok && pos <= t;
          sa[h][e] = v ? sa[h][e] * sl2 : -INFINITY;
          sa[h][2 + e] = v ? sa[h][2 + e] * sl2 : -INFINITY;
          mx0 = fmaxf(mx0, sa[h][e]);
          mx1 = fmaxf(mx1, sa[h][2 + e]);
        }
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const bool grow0 = mx0 > m0 + kLazyMax, grow1 = mx1 > m1 + kLazyMax;  // any finite max grows a -inf reference
    const float cr0 = grow0 ? hw_exp2(m0 - mx0) : 1.f;  // (a -inf reference: 0, and O, l are still 0)
    const float cr1 = grow1 ? hw_exp2(m1 - mx1) : 1.f;
    if (grow0) m0 = mx0;
    if (grow1) m1 = mx1;
    const float u0 = (m0 == -INFINITY) ? 0.f : m0;  // still -inf: every score so far masked
    const float u1 = (m1 == -INFINITY) ? 0.f : m1;
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
    if (__any_sync(0xffffffffu, grow0 || grow1)) {
#pragma unroll
      for (int i = 0; i < kD / 8; ++i) {
        o[i][0] *= cr0;
        o[i][1] *= cr0;
        o[i][2] *= cr1;
        o[i][3] *= cr1;
      }
    }
    // ---- O += P V ----
    if constexpr (KV8) {
      const uint32_t pa[4] = {pack_f16(pr[0][0], pr[0][1]), pack_f16(pr[0][2], pr[0][3]),
                              pack_f16(pr[1][0], pr[1][1]), pack_f16(pr[1][2], pr[1][3])};
      // n-tile 8c + e, column n = lane / 4: dim 64c + 8n + e; k slots 2i, 2i+1 (+8 for
      // block B) are tokens tok8(2i), tok8(2i+1), as in S
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        uint32_t bv[2][8];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint8_t *vb = buf + (2 + h) * BB;
          const uint2 x0 = *reinterpret_cast<const uint2 *>(vb + voff0[c]);  // token tok8(2i), 8 dims
          const uint2 x1 = *reinterpret_cast<const uint2 *>(vb + voff1[c]);  // token tok8(2i+1)
          const uint32_t p01 = __byte_perm(x0.x, x1.x, 0x5140), p23 = __byte_perm(x0.x, x1.x, 0x7362);
          const uint32_t p45 = __byte_perm(x0.y, x1.y, 0x5140), p67 = __byte_perm(x0.y, x1.y, 0x7362);
          e4m3x4_to_f16x2x2(p01, bv[h][0], bv[h][1]);
          e4m3x4_to_f16x2x2(p23, bv[h][2], bv[h][3]);
          e4m3x4_to_f16x2x2(p45, bv[h][4], bv[h][5]);
          e4m3x4_to_f16x2x2(p67, bv[h][6], bv[h][7]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) mma_f16_16816(o[8 * c + e], pa, bv[0][e], bv[1][e]);
      }
    } else {
      const uint32_t pa[4] = {pack_bf16(pr[0][0], pr[0][1]), pack_bf16(pr[0][2], pr[0][3]),
                              pack_bf16(pr[1][0], pr[1][1]), pack_bf16(pr[1][2], pr[1][3])};
      const uint32_t vbase = smem_u32(buf) + 2 * BB + (lm & 1) * BB;
#pragma unroll
      for (int np = 0; np < kD / 16; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vbase + swz(lr, 16 * np + 8 * (lm >> 1)), b0, b1, b2, b3);
        mma_bf16_16816(o[2 * np], pa, b0, b1);
        mma_bf16_16816(o[2 * np + 1], pa, b2, b3);
      }
    }
    // order this stage's generic reads / zero fills before the next async-proxy write into it
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && j + NST < n_pairs) issue(j + NST);
  }
  // a warp may leave the loop early only after a wait expired
  timed_out = __any_sync(0xffffffffu, timed_out);
  if (timed_out) {
    if (lane == 0) record_error(a.err, S5_ERR_TIMEOUT, r);
    // drain: wait (bounded) for the copies still in flight (issued, not consumed)
    for (int j2 = j_fail; j2 < n_pairs && j2 < j_fail + NST; ++j2)
      mbar_wait_bounded(wbar + (j2 % NST), (j2 / NST) & 1, kWaitNs);
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
    const float z = timed_out ? 0.f : 1.f;
    if constexpr (KV8) {
      // n-tile 8c + e holds dims 64c + 16 tq + e (o[.][0], o[.][2]) and 64c + 16 tq + 8 + e ([1], [3])
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        float *d0 = ow + r0 * kD + 64 * c + 16 * tq;
        float *d1 = ow + (r0 + 8) * kD + 64 * c + 16 * tq;
#pragma unroll
        for (int e = 0; e < 8; e += 4) {
          *reinterpret_cast<float4 *>(d0 + e) = make_float4(o[8 * c + e][0] * z, o[8 * c + e + 1][0] * z,
                                                            o[8 * c + e + 2][0] * z, o[8 * c + e + 3][0] * z);
          *reinterpret_cast<float4 *>(d0 + 8 + e) = make_float4(o[8 * c + e][1] * z, o[8 * c + e + 1][1] * z,
                                                                o[8 * c + e + 2][1] * z, o[8 * c + e + 3][1] * z);
          *reinterpret_cast<float4 *>(d1 + e) = make_float4(o[8 * c + e][2] * z, o[8 * c + e + 1][2] * z,
                                                            o[8 * c + e + 2][2] * z, o[8 * c + e + 3][2] * z);
          *reinterpret_cast<float4 *>(d1 + 8 + e) = make_float4(o[8 * c + e][3] * z, o[8 * c + e + 1][3] * z,
                                                                o[8 * c + e + 2][3] * z, o[8 * c + e + 3][3] * z);
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < kD / 8; ++i) {
        const int col = i * 8 + 2 * tq;
        *reinterpret_cast<float2 *>(ow + r0 * kD + col) = make_float2(o[i][0] * z, o[i][1] * z);
        *reinterpret_cast<float2 *>(ow + (r0 + 8) * kD + col) = make_float2(o[i][2] * z, o[i][3] * z);
      }
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
      const float *oww = reinterpret_cast<const float *>(ring + w * NST * SB);
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
    // (one-byte KV: the values are v_scale times their codes)
    const float inv = (L > 0.f) ? (KV8 ? a.v_scale : 1.f) / L : 0.f;
    const int hg = g * kHpg + h;
    const size_t rh = (size_t)r * kHeads + hg;
    float acc[24];
#pragma unroll
    for (int e = 0; e < 24; ++e) acc[e] = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float *oww = reinterpret_cast<const float *>(ring + w * NST * SB) + h * kD + d0;
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
                              int total_q, bool deep, cudaStream_t st) {
  const long long n_cta = (long long)a.n_split * total_q * kKv;
  if (n_cta > 0x7fffffffLL) return cudaErrorInvalidValue;
  dim3 grid((unsigned)n_cta);
  cudaError_t e;
  auto kernel = (mode == kModeSparse)
                    ? (a.kv8 ? (deep ? gqa_decode_kernel<kModeSparse, true, true> : gqa_decode_kernel<kModeSparse, true, false>)
                             : (deep ? gqa_decode_kernel<kModeSparse, false, true>
                                     : gqa_decode_kernel<kModeSparse, false, false>))
                    : (deep ? gqa_decode_kernel<kModeSwa, false, true> : gqa_decode_kernel<kModeSwa, false, false>);
  const int smem = deep ? attn_smem<true>() : attn_smem<false>();
  e = ensure_dynamic_smem(reinterpret_cast<const void *>(kernel), smem);
  if (e != cudaSuccess) return e;
  // programmatic stream serialization: launch and barrier setup overlap the
  // previous kernel; the kernel reads no global memory before pdl_wait()
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kWarps * 32);
  cfg.dynamicSmemBytes = smem;
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
