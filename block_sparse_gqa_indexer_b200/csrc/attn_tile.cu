// Sparse attention for chunked prefill and multi-token verify on the
// 5th-generation tensor cores, over the shared set of selected blocks.
//
// SGLang day-0 blog ("Step 5 Preview: Day-0 Inference and RL Support with
// SGLang and Miles"), "Kernels from StepFun": for prefill, the union of the
// blocks chosen by every query of a batch is attended once, with a mask that
// keeps each query to its own blocks.  Here the batch is a tile of up to 8
// consecutive query rows of one sequence:
//
//   tile_union_kernel   builds, per tile, the ascending list of distinct blocks
//                       its rows read (selected history blocks and the rows'
//                       current blocks), each entry carrying which rows
//                       selected it, and decides per tile whether the shared
//                       set pays (its union is small next to the blocks the
//                       rows read one by one) or the rows go to the per-row
//                       kernel;
//   gqa_tile_kernel     a persistent kernel, one CTA per SM, walking work items
//                       (tile, KV group, partition of the tile's list).  The
//                       8 rows x 16 heads of a group are the M = 128 rows of
//                       the MMAs.  Warp 8 streams 8-block chunks of K and
//                       warp 9 of V by TMA (one 3 KB copy per block,
//                       plane-major, 128-byte swizzled) through 4-stage rings;
//                       warp 10 issues S = Q K^T (N = 64 tokens, K = 192) into
//                       two tensor-memory buffers and warp 11 O += P V, both
//                       with their A operand (Q, P) in tensor memory (two
//                       issuing threads, so S of a later chunk never waits
//                       behind the PV of an earlier one); warps 0-7 (two per
//                       tensor-memory lane quarter, one thread per tile row
//                       each, 32 of a chunk's 64 columns each, row maxima of
//                       the two halves exchanged through shared memory) load Q
//                       into tensor memory, run the masked online softmax,
//                       write P back to tensor memory as bf16 and finish each
//                       item.
//
// Each shared block is read once per tile instead of once per row; the
// masked-out products are the price of dense tiles.
#include <cuda.h>

#include <climits>

#include "s5_common.cuh"
#include "s5_kernels.h"
#include "s5_tcgen05.cuh"

namespace s5 {

// Packed fp32 pairs (one instruction for two lanes of work on sm_100):
// element-wise a * b + c and a + b, each rounded to nearest as fmaf / __fadd_rn.
__device__ __forceinline__ float2 fma_f32x2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(d)
      : "l"(*reinterpret_cast<uint64_t *>(&a)), "l"(*reinterpret_cast<uint64_t *>(&b)),
        "l"(*reinterpret_cast<uint64_t *>(&c)));
  return *reinterpret_cast<float2 *>(&d);
}
// max(a, b, c) in one instruction (sm_100 three-input max)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float2 add_f32x2(float2 a, float2 b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(*reinterpret_cast<uint64_t *>(&a)), "l"(*reinterpret_cast<uint64_t *>(&b)));
  return *reinterpret_cast<float2 *>(&d);
}

// 2^x for two values on the FMA and integer pipes (the multi-function unit that
// evaluates ex2 serves a quarter warp per cycle and the softmax warps of a lane
// quarter reach their exponentials together).  x = n + f: n, the nearest
// integer, is rounded by adding 1.5 * 2^23 (the sum's low mantissa bits then
// hold n) and |f| <= 1/2; 2^f is a cubic whose coefficients were fitted to
// minimise the relative error on [-1/2, 1/2] (at most 7.5e-5 evaluated in fp32,
// far below the bf16 rounding of P), and n is added to its exponent field.
// Arguments are at most 8 here; below -125 (masked: -inf) the result is 2^-125
// instead of 0, which no visible weight of a row notices.
__device__ __forceinline__ float2 exp2_fma_x2(float2 x) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  constexpr float c0 = 0.99992806f, c1 = 0.69326097f, c2 = 0.24261114f, c3 = 0.055171657f;
  x = make_float2(fmaxf(x.x, -125.f), fmaxf(x.y, -125.f));
  const float2 t = add_f32x2(x, make_float2(kRound, kRound));
  const float2 n = add_f32x2(t, make_float2(-kRound, -kRound));
  const float2 f = fma_f32x2(n, make_float2(-1.f, -1.f), x);  // exact
  float2 q = fma_f32x2(make_float2(c3, c3), f, make_float2(c2, c2));
  q = fma_f32x2(q, f, make_float2(c1, c1));
  q = fma_f32x2(q, f, make_float2(c0, c0));
  return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}

constexpr int kTRows = kTileRows;          // query rows per tile
constexpr int kTM = kTRows * kHpg;         // 128 MMA rows = tensor-memory lanes
constexpr int kTChunkBlocks = 8;           // blocks per chunk
constexpr int kTN = kTChunkBlocks * kBlk;  // 64 tokens per chunk
constexpr int kTStages = 4;                // depth of the K ring and of the V ring
constexpr int kTKvBytes = kTChunkBlocks * kBlockBytes;  // K (or V) of one chunk
constexpr int kTSoftWarps = 8;                 // softmax / epilogue warps: two threads per tile row
constexpr int kTSoftThreads = kTSoftWarps * 32;
constexpr int kTSplit = kTSoftWarps / 4;        // warps per tensor-memory lane quarter
constexpr int kTCols = kTN / kTSplit;           // S columns per softmax warp (16)
constexpr int kTBlocksW = kTCols / kBlk;        // blocks per softmax warp and chunk (2)
constexpr int kTOCols = kD / kTSplit;           // O columns (= Q dims) per softmax warp
static_assert(kTCols == 16 || kTCols % 32 == 0, "S columns per softmax thread: 16 or a multiple of 32");
constexpr int kTWarpK = kTSoftWarps, kTWarpV = kTSoftWarps + 1, kTWarpS = kTSoftWarps + 2,
              kTWarpPv = kTSoftWarps + 3;
constexpr int kTThreads = (kTSoftWarps + 4) * 32;
constexpr uint32_t kTTmemCols = 512;
constexpr uint32_t kTmemS = 0;    // 2 x 64 columns: S of chunk gc in buffer gc % 2
constexpr uint32_t kTmemP = 128;  // 2 x 32 columns: bf16 P of chunk gc in buffer gc % 2
constexpr uint32_t kTmemO = 192;  // 192 columns: O
constexpr uint32_t kTmemQ = 384;  // 96 columns: Q (two bf16 dims per column)
constexpr uint64_t kTWaitNs = 2000000000ull;
// Each poll of a wait may suspend the warp for up to this long (it resumes when
// the phase completes), so producers and issuers that wait take fewer issue
// slots from the softmax warps on their schedulers (16,384-token block-coherent
// prefill: 5.38 -> 5.34 ms for the attention call; 0.5 and 20 us hints gained
// nothing measurable).
constexpr uint32_t kTWaitHintNs = 4000;
constexpr float kLazyRescale = 8.0f;  // log2 units
// Every kTPolyEvery-th column pair takes its exponentials on the FMA pipe: a
// quarter of them (a 16,384-token prefill at 114,688 cached tokens with
// block-coherent indexer queries: 5.33 ms for the attention call against
// 5.45 ms with none, 5.36 ms with an eighth and 5.55 ms with half).
constexpr int kTPolyEvery = 4;
constexpr uint32_t kPadEntry = 0x00FFFFFFu;  // union entry of an empty slot: no rows, block id 2^24 - 1

// shared memory (offsets from a 1,024-byte aligned base)
constexpr int kOffK = 0;
constexpr int kOffV = kOffK + kTStages * kTKvBytes;
constexpr int kOffXm = kOffV + kTStages * kTKvBytes;  // float [2 buffers][kTSplit][128 rows]
constexpr int kOffXl = kOffXm + 2 * kTSplit * kTM * 4;  // float [kTSplit][128 rows]
constexpr int kOffBar = kOffXl + kTSplit * kTM * 4;
constexpr int kNumBars = 44;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kOffList = kOffMisc + 128;           // int [kMaxListTiles]: shared-set tiles, ascending
constexpr int kMaxListTiles = 4096;
constexpr int kTileSmem = kOffList + kMaxListTiles * 4 + 1024;  // + alignment slack

// barriers
constexpr int kBQFull = 0, kBQEmpty = 1;
constexpr int kBKFull = 2, kBKEmpty = kBKFull + kTStages;  // [kTStages] each
constexpr int kBVFull = kBKEmpty + kTStages, kBVEmpty = kBVFull + kTStages;
constexpr int kBSFull = kBVEmpty + kTStages, kBSEmpty = kBSFull + 2;  // [2] each
constexpr int kBPFull = kBSEmpty + 2, kBPFree = kBPFull + 2;
constexpr int kBOEmpty = kBPFree + 2;
constexpr int kBXm = kBOEmpty + 1;  // [4 lane quarters][2 buffers]
constexpr int kBXl = kBXm + 8;      // [4 lane quarters]
constexpr int kBMgAll = kBXl + 4, kBMgDec = kBMgAll + 1, kBFinal = kBMgDec + 1;
static_assert(kBFinal < kNumBars, "barrier slots");

// ---------------------------------------------------------------- union lists

// Entry: block (bits 0..23) | rows that selected it << 24 (bit j = row j).
__global__ void __launch_bounds__(256) tile_union_kernel(const TileArgs a) {
  extern __shared__ uint32_t bmap[];  // byte b: rows that selected block b
  __shared__ int scan[8];
  __shared__ int n_sel[kTRows];
  const int s = blockIdx.y, k = blockIdx.x;
  const int tile = s * a.tiles_per_seq + k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();  // (programmatic launch) the selection is read after this point
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
  const int words = c_last / 4 + 1;
  const bool bad = ctx < 0 || r0 < 0 || r0 + nr > a.total_q;
  if (bad || words > a.map_words) {
    // bad batch data (recorded; the per-row kernel reports it too), or a
    // history too long for the shared map: the rows go to the per-row kernel
    if (tid == 0) {
      if (bad) record_error(a.err, S5_ERR_DEVICE_BOUNDS, max(r0, 0));
      *count = 0;
      a.tile_on[tile] = 0;
      for (int j = 0; j < nr; ++j)
        if (r0 + j >= 0 && r0 + j < a.total_q) a.row_skip[r0 + j] = 0;
    }
    return;
  }
  for (int i = tid; i < words; i += 256) bmap[i] = 0;
  __syncthreads();
  // the rows' selection counts first, then every (row, entry) pair with eight
  // loads per thread in flight at a time
  if (tid < kTRows) {
    int n = 0;
    if (tid < nr) {
      const int c = (ctx + k * kTRows + tid) / kBlk;
      n = ld_cg(a.sel_count + r0 + tid);
      if (n < 0 || n > a.topk || n > c) {
        record_error(a.err, S5_ERR_DEVICE_BOUNDS, r0 + tid);
        n = 0;
      }
    }
    n_sel[tid] = n;
  }
  __syncthreads();
  int row_blocks = 0;  // sum over the tile's rows of (selected blocks + current block)
  for (int j = 0; j < nr; ++j) row_blocks += n_sel[j] + 1;
  const int pairs = nr * a.topk;
  for (int x0 = 0; x0 < pairs; x0 += 256 * 8) {
    int bv[8], jv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int x = x0 + u * 256 + tid;
      const int j = min(x / a.topk, kTRows - 1), i = x - j * a.topk;  // j is only used when x < pairs
      jv[u] = j;
      bv[u] = (x < pairs && i < n_sel[j]) ? ld_cg(a.sel + (size_t)(r0 + j) * a.topk + i) : INT_MIN;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (bv[u] == INT_MIN) continue;
      const int j = jv[u], b = bv[u];
      const int c = (ctx + k * kTRows + j) / kBlk;
      if (b >= 0 && b < c) atomicOr(bmap + (b >> 2), (1u << j) << ((b & 3) * 8));
      else record_error(a.err, S5_ERR_DEVICE_BOUNDS, r0 + j);
    }
  }
  __syncthreads();
  // ascending compaction of the selected blocks and the current blocks (the
  // rows' positions are consecutive, so their current blocks are exactly
  // c_first .. c_last)
  const int c_first = (ctx + k * kTRows) / kBlk;
  auto in_union = [&](int b, uint32_t byte) { return byte != 0 || (b >= c_first && b <= c_last); };
  const int per = (words + 255) / 256;  // words per thread, in order
  const int w_lo = min(words, tid * per), w_hi = min(words, tid * per + per);
  int cnt = 0;
  for (int w = w_lo; w < w_hi; ++w) {
    const uint32_t u = bmap[w];
    for (int q = 0; q < 4; ++q) cnt += in_union(4 * w + q, (u >> (8 * q)) & 0xFFu) ? 1 : 0;
  }
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
  for (int w = w_lo; w < w_hi; ++w) {
    const uint32_t u = bmap[w];
    for (int q = 0; q < 4; ++q) {
      const int b = 4 * w + q;
      const uint32_t byte = (u >> (8 * q)) & 0xFFu;
      if (!in_union(b, byte)) continue;
      if (pos < a.union_cap) ent[pos] = (uint32_t)b | (byte << 24);
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

struct TileItem {
  int tile, g, p, s, k, r0, nr, ctx, e0, ne, n_chunks;
  bool on;
};

// Work item idx: partition fastest, then tile, then KV group (CTAs working at
// the same time share one group's blocks of neighbouring tiles in L2).  The
// tiles are the n_list shared-set tiles in `list` (ascending), or all tiles
// when list is null.
__device__ __forceinline__ TileItem decode_item(const TileArgs &a, const int *list, int n_list, int idx) {
  TileItem it;
  it.p = idx % a.n_split;
  const int tg = idx / a.n_split;
  const int rank = tg % n_list;
  it.tile = (list != nullptr) ? list[rank] : rank;
  it.g = tg / n_list;
  it.s = it.tile / a.tiles_per_seq;
  it.k = it.tile % a.tiles_per_seq;
  const int q_beg = ld_cg(a.cu_q + it.s);
  const int nq = ld_cg(a.cu_q + it.s + 1) - q_beg;
  it.ctx = ld_cg(a.ctx_lens + it.s);
  it.r0 = q_beg + it.k * kTRows;
  it.nr = max(0, min(kTRows, nq - it.k * kTRows));
  it.on = it.nr > 0 && ld_cg(a.tile_on + it.tile) != 0;
  it.e0 = it.ne = it.n_chunks = 0;
  if (it.on) {
    const int n_ent = max(0, min(ld_cg(a.union_count + it.tile), a.union_cap));
    const int per = (n_ent + a.n_split - 1) / a.n_split;
    const int chunk_e = (per + kTChunkBlocks - 1) / kTChunkBlocks * kTChunkBlocks;
    it.e0 = min(n_ent, it.p * chunk_e);
    it.ne = min(n_ent, it.e0 + chunk_e) - it.e0;
    it.n_chunks = (it.ne + kTChunkBlocks - 1) / kTChunkBlocks;
  }
  return it;
}

// Merge weights of the partitions of one (row, head): the same arithmetic as
// the per-row kernel's merge, in partition order.
__device__ __forceinline__ void tile_partition_weights(const float *pl, int n, float *w, float &lse_nat) {
  constexpr int kMaxN = kMaxTileSplit;
  float lv[kMaxN];  // all loads in flight together
#pragma unroll
  for (int p = 0; p < kMaxN; ++p) lv[p] = (p < n) ? ld_cg(pl + p) : -INFINITY;
  float M = -INFINITY;
#pragma unroll
  for (int p = 0; p < kMaxN; ++p) M = fmaxf(M, lv[p]);
  const float Mu = (M == -INFINITY) ? 0.f : M;
  float L = 0.f;
#pragma unroll
  for (int p = 0; p < kMaxN; ++p) L += (lv[p] == -INFINITY) ? 0.f : hw_exp2(lv[p] - Mu);
  const float inv = (L > 0.f) ? 1.f / L : 0.f;
#pragma unroll
  for (int p = 0; p < kMaxN; ++p)
    if (p < n) w[p] = (lv[p] == -INFINITY) ? 0.f : hw_exp2(lv[p] - Mu) * inv;
  lse_nat = (L > 0.f) ? (M + hw_log2(L)) * 0.69314718055994531f : -INFINITY;
}

__global__ void __launch_bounds__(kTThreads, 1)
    gqa_tile_kernel(const TileArgs a, const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sk = smem + kOffK;
  uint8_t *sv = smem + kOffV;
  float *xm = reinterpret_cast<float *>(smem + kOffXm);
  float *xl = reinterpret_cast<float *>(smem + kOffXl);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffMisc);
  int *abort_flag = reinterpret_cast<int *>(smem + kOffMisc + 4);
  int *is_last = reinterpret_cast<int *>(smem + kOffMisc + 8);

  int *list_s = reinterpret_cast<int *>(smem + kOffList);
  int *wsum = reinterpret_cast<int *>(smem + kOffMisc + 16);  // [kTThreads / 32] per-warp counts

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_wait();  // (programmatic launch) the union kernel's outputs are read after this point

  // ---- the shared-set tiles, in order (most batches of independent queries have none) ----
  const int *list = nullptr;
  int n_list = a.n_tiles;
  if (a.n_tiles <= kMaxListTiles) {
    int base = 0;
    for (int i0 = 0; i0 < a.n_tiles; i0 += kTThreads) {
      const int i = i0 + tid;
      const bool on = i < a.n_tiles && ld_cg(a.tile_on + i) != 0;
      const uint32_t bal = __ballot_sync(0xffffffffu, on);
      if (lane == 0) wsum[warp] = __popc(bal);
      __syncthreads();
      int before = base;
      for (int w = 0; w < warp; ++w) before += wsum[w];
      if (on) list_s[before + __popc(bal & ((1u << lane) - 1u))] = i;
      int tot = 0;
      for (int w = 0; w < kTThreads / 32; ++w) tot += wsum[w];
      __syncthreads();
      base += tot;
    }
    list = list_s;
    n_list = base;
    if (n_list == 0) return;  // every tile goes to the per-row kernel
  }
  const int n_items = n_list * kKv * a.n_split;

  // K/V slots that no copy fills (padding, an unmapped page) must hold finite
  // values: start from zeros
  for (int i = tid; i < (2 * kTStages * kTKvBytes) / 16; i += kTThreads)
    reinterpret_cast<uint4 *>(sk)[i] = make_uint4(0, 0, 0, 0);
  if (warp == 0) tc::tmem_alloc(tmem_slot, kTTmemCols);
  if (tid == 0) {
    mbar_init(bars + kBQFull, kTSoftWarps);
    mbar_init(bars + kBQEmpty, 1);
    for (int i = 0; i < kTStages; ++i) {
      mbar_init(bars + kBKFull + i, 1);
      mbar_init(bars + kBKEmpty + i, 1);
      mbar_init(bars + kBVFull + i, 1);
      mbar_init(bars + kBVEmpty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bars + kBSFull + i, 1);
      mbar_init(bars + kBSEmpty + i, kTSoftWarps);
      mbar_init(bars + kBPFull + i, kTSoftWarps);
      mbar_init(bars + kBPFree + i, 1);
    }
    mbar_init(bars + kBOEmpty, kTSoftWarps);
    for (int i = 0; i < 8; ++i) mbar_init(bars + kBXm + i, 32 * kTSplit);
    for (int i = 0; i < 4; ++i) mbar_init(bars + kBXl + i, 32 * kTSplit);
    mbar_init(bars + kBMgAll, kTSoftThreads);
    mbar_init(bars + kBMgDec, 1);
    mbar_init(bars + kBFinal, 2);  // one commit from each MMA issuer
    *abort_flag = 0;
  }
  fence_mbar_init();
  fence_proxy_async_smem();  // the zero fill before any copy or MMA touches those bytes
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  auto wait = [&](uint64_t *bar, uint32_t parity) -> bool {
    if (*reinterpret_cast<volatile int *>(abort_flag)) return false;
    if (mbar_wait_bounded_hint(bar, parity, kTWaitNs, kTWaitHintNs)) return true;
    *reinterpret_cast<volatile int *>(abort_flag) = 1;
    record_error(a.err, S5_ERR_TIMEOUT, 0);
    return false;
  };

  if (warp == kTWarpK || warp == kTWarpV) {
    // ---------------- TMA producers: warp kTWarpK streams K, warp kTWarpV V ----------------
    // Lane b < 8 copies block b of each chunk (one 3 KB box: 3 planes x 8
    // tokens x 64 dims); lane 0 keeps the barrier bookkeeping.
    const bool is_k = warp == kTWarpK;
    uint8_t *ring = is_k ? sk : sv;
    const CUtensorMap *map = is_k ? &tm_k : &tm_v;
    uint64_t *full = bars + (is_k ? kBKFull : kBVFull);
    uint64_t *empty = bars + (is_k ? kBKEmpty : kBVEmpty);
    const uint64_t policy = policy_evict_normal();
    int gc = 0;
    bool ok = true;
    for (int idx = blockIdx.x; idx < n_items && ok; idx += gridDim.x) {
      const TileItem it = decode_item(a, list, n_list, idx);
      if (it.n_chunks == 0) continue;
      const uint32_t *ent = a.union_ent + (size_t)it.tile * a.union_cap + it.e0;
      const int32_t *pt = a.page_table + (size_t)it.s * a.max_pages;
      // lookups run two chunks ahead of the copies: the entry of chunk c + 2
      // and the page of chunk c + 1 are in flight while chunk c is issued
      auto load_block = [&](int c) -> int {  // this lane's block of chunk c, or -1
        const int i = c * kTChunkBlocks + lane;
        return (lane < kTChunkBlocks && c < it.n_chunks && i < it.ne) ? (int)(ld_cg(ent + i) & 0xFFFFFFu) : -1;
      };
      auto load_page = [&](int b) -> int {  // physical page of block b (-1: none or unmapped)
        const int pg = b / kBpp;
        return (b >= 0 && pg < a.max_pages) ? ld_cg(pt + pg) : -1;
      };
      int b0 = load_block(0);
      int ph0 = load_page(b0);
      int b1 = load_block(1);
      for (int c = 0; c < it.n_chunks; ++c, ++gc) {
        const int b2 = load_block(c + 2);
        const int ph1 = load_page(b1);
        const int st = gc % kTStages;
        int go = 1;
        if (lane == 0 && gc >= kTStages) go = wait(empty + st, ((gc / kTStages) - 1) & 1) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, go, 0)) {
          ok = false;
          break;
        }
        int row = -1;
        if (b0 >= 0) {
          if (ph0 >= 0 && ph0 < a.num_pages) row = ((ph0 * kKv + it.g) * kPage) + (b0 % kBpp) * kBlk;
          else record_error(a.err, S5_ERR_DEVICE_BOUNDS, it.r0);
        }
        b0 = b1;
        ph0 = ph1;
        b1 = b2;
        uint32_t bytes = (row >= 0) ? (uint32_t)kBlockBytes : 0u;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) bytes += __shfl_xor_sync(0xffffffffu, bytes, off);
        if (lane == 0) mbar_arrive_expect_tx(full + st, bytes);
        __syncwarp();
        if (row >= 0) tma_load_3d(ring + st * kTKvBytes + lane * kBlockBytes, map, 0, row, 0, full + st, policy);
      }
    }
    // no copy may still be writing shared memory when the CTA retires
    if (lane == 0) {
      for (int c = max(0, gc - kTStages); c < gc; ++c)
        mbar_wait_bounded(full + c % kTStages, (c / kTStages) & 1, kTWaitNs);
    }
  } else if (warp == kTWarpS) {
    // ---------------- S issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = tc::idesc_bf16_f32(kTM, kTN);
      const uint32_t k_base = smem_u32(sk);
      int gc = 0, qi = 0;
      bool ok = true;
      for (int idx = blockIdx.x; idx < n_items && ok; idx += gridDim.x) {
        const TileItem it = decode_item(a, list, n_list, idx);
        if (it.n_chunks == 0) continue;
        if (!wait(bars + kBQFull, qi & 1)) break;
        for (int c = 0; c < it.n_chunks; ++c, ++gc) {
          const int st = gc % kTStages, sb = gc & 1;
          if (!wait(bars + kBKFull + st, (gc / kTStages) & 1) ||
              (gc >= 2 && !wait(bars + kBSEmpty + sb, ((gc >> 1) - 1) & 1))) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          // S = Q K^T: Q from tensor memory (K-step kk = 8 columns); K = 192
          // as 3 swizzled planes of 64; the chunk's blocks are 8-token groups
          // 3,072 B apart, plane cb of a block at cb * 1,024
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const int cb = kk >> 2, k4 = kk & 3;
            const uint64_t bd =
                tc::smem_desc_k_sw128_stride(k_base + st * kTKvBytes + cb * 1024 + k4 * 32, kBlockBytes);
            tc::mma_bf16_ts(tmem + kTmemS + sb * kTN, tmem + kTmemQ + kk * 8, bd, idesc_s, kk > 0);
          }
          tc::commit(bars + kBKEmpty + st);
          tc::commit(bars + kBSFull + sb);
          if (c == it.n_chunks - 1) tc::commit(bars + kBQEmpty);
        }
        ++qi;
      }
      tc::commit(bars + kBFinal);  // arrives once every MMA issued above has completed
    }
  } else if (warp == kTWarpPv) {
    // ---------------- PV issuer ----------------
    // O += P_x V_x (P: tensor memory, 64 tokens = 4 K-steps of 8 columns; V:
    // 64-dim planes 1,024 B apart (leading), 8-token blocks 3,072 B apart (stride))
    if (lane == 0) {
      constexpr uint32_t idesc_o = tc::idesc_bf16_f32_bmn(kTM, kD);  // B = V, MN-major
      const uint32_t v_base = smem_u32(sv);
      int gc = 0, qi = 0;
      bool ok = true;
      for (int idx = blockIdx.x; idx < n_items && ok; idx += gridDim.x) {
        const TileItem it = decode_item(a, list, n_list, idx);
        if (it.n_chunks == 0) continue;
        for (int c = 0; c < it.n_chunks; ++c, ++gc) {
          const bool first = c == 0;
          if (!wait(bars + kBPFull + (gc & 1), (gc >> 1) & 1) ||
              !wait(bars + kBVFull + gc % kTStages, (gc / kTStages) & 1) ||
              (first && qi > 0 && !wait(bars + kBOEmpty, (qi - 1) & 1))) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const int vs = gc % kTStages;
#pragma unroll
          for (int ks = 0; ks < kTN / 16; ++ks) {
            const uint64_t bd =
                tc::smem_desc_mn_sw128(v_base + vs * kTKvBytes + ks * 2 * kBlockBytes, 1024, kBlockBytes);
            tc::mma_bf16_ts(tmem + kTmemO, tmem + kTmemP + (gc & 1) * 32 + ks * 8, bd, idesc_o, !first || ks > 0);
          }
          tc::commit(bars + kBVEmpty + vs);
          tc::commit(bars + kBPFree + (gc & 1));
        }
        ++qi;
      }
      tc::commit(bars + kBFinal);
    }
  } else {
    // ---------------- softmax / epilogue: warps 0 .. kTSoftWarps-1 ----------------
    // Warp w reads lanes 32 (w % 4) .. + 31 (tile rows m = lane index: query
    // j = m / 16, head h = m % 16) and columns kTCols (w / 4) .. + kTCols - 1
    // of each S (blocks kTBlocksW (w / 4) ..); it owns Q dims and O columns
    // kTOCols (w / 4) .. + kTOCols - 1 of its rows.  With four warps every
    // thread owns a whole row: all 64 columns of S, all 192 of Q and O.
    const int q4 = warp & 3, qq = warp >> 2;
    const int m = q4 * 32 + lane;
    const int j = m >> 4, h = m & 15;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const float sl2 = a.scale_log2;
    int gc = 0, qi = 0, mi = 0;
    bool ok = true;
    for (int idx = blockIdx.x; idx < n_items && ok; idx += gridDim.x) {
      const TileItem it = decode_item(a, list, n_list, idx);
      if (!it.on) continue;
      const bool row_ok = j < it.nr;
      const int t = it.ctx + it.k * kTRows + j;  // this row's position
      const int cj = t / kBlk;                    // and its current block
      const int tcur = t - cj * kBlk;             // last visible token of the current block
      // block id this row reads token by token (never an entry's 24-bit block id
      // for rows past the tile's end), and the entry bit of its selections
      const uint32_t cj_row = row_ok ? (uint32_t)cj : 0xFFFFFFFFu;
      const int sel_sh = 24 + j;
      const int t_max = it.ctx + it.k * kTRows + it.nr - 1;
      const uint32_t *ent = a.union_ent + (size_t)it.tile * a.union_cap + it.e0;
      float m_ref = -INFINITY, l = 0.f;
      if (it.n_chunks > 0) {
        // Q of the item into tensor memory: this thread's row (query j, head
        // 16g + h), its 48 dims (zeros past the tile's rows); the previous
        // item's last S must be done with the old Q
        if (qi > 0 && !wait(bars + kBQEmpty, (qi - 1) & 1)) {
          ok = false;
          break;
        }
        const uint4 *qs = reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(a.q) +
                                                          ((size_t)(it.r0 + j) * kHeads + it.g * kHpg + h) * kD +
                                                          qq * kTOCols);
#pragma unroll
        for (int x = 0; x < kTOCols / 16; ++x) {  // 16 dims = 8 columns per store
          const uint4 u0 = row_ok ? ld_cg(qs + 2 * x) : make_uint4(0, 0, 0, 0);
          const uint4 u1 = row_ok ? ld_cg(qs + 2 * x + 1) : make_uint4(0, 0, 0, 0);
          const uint32_t w8[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
          tc::st_8cols(tmem + lane_base + kTmemQ + qq * (kTOCols / 2) + x * 8, w8);
        }
        tc::wait_st();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + kBQFull);
      }
      // lanes 0..1 hold the entries of this warp's 2 blocks of the next chunk
      // (slots past the item's last entry read as kPadEntry: no row bits, and a
      // block id no row is in)
      uint32_t e_next = kPadEntry;
      if (lane < kTBlocksW && qq * kTBlocksW + lane < it.ne) e_next = ld_cg(ent + qq * kTBlocksW + lane);
      for (int c = 0; c < it.n_chunks; ++c, ++gc) {
        const uint32_t e_cur = e_next;
        {
          const int i = (c + 1) * kTChunkBlocks + qq * kTBlocksW + lane;
          e_next = (lane < kTBlocksW && c + 1 < it.n_chunks && i < it.ne) ? ld_cg(ent + i) : kPadEntry;
        }
        // mask of this chunk, before S arrives: column x = 8 ib + tok is token tok
        // of block (kTBlocksW qq + ib) of the chunk.  A row sees a block it
        // selected whole and its current block up to its own token (selected
        // blocks are all before the current one, so the two never coincide).
        // Scores are taken relative to the row's current reference max, so the
        // weights need no subtraction unless the reference moves (rare).
        const float mu0 = (m_ref == -INFINITY) ? 0.f : m_ref;
        int lim[kTBlocksW];  // tokens 0 .. lim of block ib are visible to this row
        bool cur_any = false;
#pragma unroll
        for (int ib = 0; ib < kTBlocksW; ++ib) {
          const uint32_t e = __shfl_sync(0xffffffffu, e_cur, ib);
          const bool cur = (e & 0xFFFFFFu) == cj_row;
          lim[ib] = cur ? tcur : (((e >> sel_sh) & 1u) ? kBlk - 1 : -1);
          cur_any |= cur;
        }
        const bool partial = cur_any && tcur < kBlk - 1;  // (a row's last chunk) token-by-token masks
        const int sb = gc & 1;
        if (!wait(bars + kBSFull + sb, (gc >> 1) & 1)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        uint32_t v[kTCols];
        if constexpr (kTCols % 32 == 0) {
#pragma unroll
          for (int x = 0; x < kTCols / 32; ++x)
            tc::ld_32cols(tmem + lane_base + kTmemS + sb * kTN + qq * kTCols + 32 * x,
                          *reinterpret_cast<uint32_t(*)[32]>(v + 32 * x));
        } else {
          tc::ld_16cols(tmem + lane_base + kTmemS + sb * kTN + qq * kTCols, *reinterpret_cast<uint32_t(*)[16]>(v));
        }
        tc::wait_ld();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + kBSEmpty + sb);
        float sc[kTCols];  // scaled, masked scores minus mu0
        float mxb[kTBlocksW];  // per-block maxima (independent chains), then a tree
#pragma unroll
        for (int ib = 0; ib < kTBlocksW; ++ib) mxb[ib] = -INFINITY;
        if (__any_sync(0xffffffffu, partial)) {
#pragma unroll
          for (int ib = 0; ib < kTBlocksW; ++ib) {
#pragma unroll
            for (int tok = 0; tok < kBlk; ++tok) {
              const float s = (tok <= lim[ib]) ? fmaf(__uint_as_float(v[ib * kBlk + tok]), sl2, -mu0) : -INFINITY;
              sc[ib * kBlk + tok] = s;
              mxb[ib] = fmaxf(mxb[ib], s);
            }
          }
        } else {  // every block is visible whole or not at all: one FMA with a -mu0 / -inf bias
          const float2 sl2x2 = make_float2(sl2, sl2);
#pragma unroll
          for (int ib = 0; ib < kTBlocksW; ++ib) {
            const float bias = (lim[ib] >= 0) ? -mu0 : -INFINITY;
            const float2 bias2 = make_float2(bias, bias);
#pragma unroll
            for (int tok = 0; tok < kBlk; tok += 2) {  // two columns per packed FMA
              const float2 s2 = fma_f32x2(
                  make_float2(__uint_as_float(v[ib * kBlk + tok]), __uint_as_float(v[ib * kBlk + tok + 1])), sl2x2, bias2);
              sc[ib * kBlk + tok] = s2.x;
              sc[ib * kBlk + tok + 1] = s2.y;
              mxb[ib] = fmax3(mxb[ib], s2.x, s2.y);
            }
          }
        }
#pragma unroll
        for (int w2 = kTBlocksW / 2; w2 > 0; w2 /= 2)
#pragma unroll
          for (int ib = 0; ib < w2; ++ib) mxb[ib] = fmaxf(mxb[ib], mxb[ib + w2]);
        const float mx = mxb[0];
        float rmax = mx;
        if constexpr (kTSplit > 1) {
          // row max over the column quarters of the row's kTSplit threads
          float *xmb = xm + sb * kTSplit * kTM;
          xmb[qq * kTM + m] = mx;
          mbar_arrive(bars + kBXm + q4 * 2 + sb);
          if (!wait(bars + kBXm + q4 * 2 + sb, (gc >> 1) & 1)) {
            ok = false;
            break;
          }
#pragma unroll
          for (int o = 1; o < kTSplit; ++o) rmax = fmaxf(rmax, xmb[((qq + o) % kTSplit) * kTM + m]);
        }
        // lazy rescale: keep the reference max unless the row max grows by more than
        // 2^8 (rmax is relative to mu0; a row without a reference takes its first max)
        const bool grow = (m_ref == -INFINITY) ? (rmax > -INFINITY) : (rmax > kLazyRescale);
        const bool resc = grow && m_ref != -INFINITY;
        const float corr = resc ? hw_exp2(-rmax) : 1.f;  // exp2(old reference - new)
        const float shift = grow ? rmax : 0.f;           // new reference - mu0
        if (grow) m_ref = mu0 + rmax;
        if (__any_sync(0xffffffffu, resc) && c > 0) {
          // O holds chunks up to gc - 1: wait for that PV (in-order completion covers the rest)
          if (!wait(bars + kBPFree + ((gc - 1) & 1), ((gc - 1) >> 1) & 1)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
#pragma unroll 1
          for (int cb = 0; cb < kTOCols / 16; ++cb) {
            uint32_t o[16];
            const uint32_t ta = tmem + lane_base + kTmemO + qq * kTOCols + cb * 16;
            tc::ld_16cols(ta, o);
            tc::wait_ld();
#pragma unroll
            for (int x = 0; x < 16; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * corr);
            tc::st_16cols(ta, o);
          }
          tc::wait_st();
        }
        l *= corr;
        // P (bf16) into tensor-memory buffer sb, last read by the PV of chunk gc - 2
        if (gc >= 2 && !wait(bars + kBPFree + sb, ((gc >> 1) - 1) & 1)) {
          ok = false;
          break;
        }
        if (__any_sync(0xffffffffu, grow)) {  // (rare) scores relative to the moved reference
          const float2 ns2 = make_float2(-shift, -shift);
#pragma unroll
          for (int x = 0; x < kTCols / 2; ++x) {
            const float2 d2 = add_f32x2(make_float2(sc[2 * x], sc[2 * x + 1]), ns2);
            sc[2 * x] = d2.x;
            sc[2 * x + 1] = d2.y;
          }
        }
        uint32_t pk[kTCols / 2];
        float2 psb[kTBlocksW];  // per-block sums of column pairs, then a tree
#pragma unroll
        for (int ib = 0; ib < kTBlocksW; ++ib) psb[ib] = make_float2(0.f, 0.f);
#pragma unroll
        for (int x = 0; x < kTCols / 2; ++x) {
          const float2 p2 = (kTPolyEvery > 0 && x % kTPolyEvery == kTPolyEvery - 1)
                                ? exp2_fma_x2(make_float2(sc[2 * x], sc[2 * x + 1]))
                                : make_float2(hw_exp2(sc[2 * x]), hw_exp2(sc[2 * x + 1]));
          psb[(2 * x) / kBlk] = add_f32x2(psb[(2 * x) / kBlk], p2);
          pk[x] = pack_bf16(p2.x, p2.y);
        }
#pragma unroll
        for (int w2 = kTBlocksW / 2; w2 > 0; w2 /= 2)
#pragma unroll
          for (int ib = 0; ib < w2; ++ib) psb[ib] = add_f32x2(psb[ib], psb[ib + w2]);
        l += psb[0].x + psb[0].y;
        if constexpr ((kTCols / 2) % 16 == 0) {
#pragma unroll
          for (int x = 0; x < kTCols / 32; ++x)
            tc::st_16cols(tmem + lane_base + kTmemP + sb * 32 + qq * (kTCols / 2) + 16 * x,
                          *reinterpret_cast<const uint32_t(*)[16]>(pk + 16 * x));
        } else {
          tc::st_8cols(tmem + lane_base + kTmemP + sb * 32 + qq * (kTCols / 2),
                       *reinterpret_cast<const uint32_t(*)[8]>(pk));
        }
        // V rows no row may read (padding slots, tokens past the tile's last
        // position, all in the item's last chunk) must be finite: zero them
        // (P is 0 there, but 0 * NaN is NaN).  Warp w checks blocks w, w + 4, ...
        if (c == it.n_chunks - 1) {
          for (int wb = warp; wb < kTChunkBlocks && ok; wb += kTSoftWarps) {
            const int ir = c * kTChunkBlocks + wb;
            const int blk = (ir < it.ne) ? (int)(ld_cg(ent + ir) & 0xFFFFFFu) : -1;
            const int first_bad = (blk < 0) ? 0 : t_max - blk * kBlk + 1;  // tokens >= first_bad are zeroed
            if (first_bad < kBlk) {
              if (!wait(bars + kBVFull + gc % kTStages, (gc / kTStages) & 1)) {
                ok = false;
                break;
              }
              uint8_t *vb = sv + (gc % kTStages) * kTKvBytes + wb * kBlockBytes;
              for (int x = lane; x < 3 * kBlk * 8; x += 32) {  // plane, token, 16-byte chunk
                const int tok = (x >> 3) & 7;
                if (tok >= first_bad)
                  *reinterpret_cast<uint4 *>(vb + (x >> 6) * 1024 + tok * 128 + (x & 7) * 16) = make_uint4(0, 0, 0, 0);
              }
              fence_proxy_async_smem();
            }
          }
          if (!ok) break;
        }
        tc::wait_st();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + kBPFull + sb);
      }
      if (!ok) break;
      // ---- epilogue: O / l of the item ----
      float lt = 0.f;
      const bool have = it.n_chunks > 0;
      if (have) {
        if constexpr (kTSplit > 1) {
          xl[qq * kTM + m] = l;
          mbar_arrive(bars + kBXl + q4);
          if (!wait(bars + kBXl + q4, qi & 1)) {
            ok = false;
            break;
          }
#pragma unroll
          for (int o = 0; o < kTSplit; ++o) lt += xl[o * kTM + m];
        } else {
          lt = l;
        }
        if (!wait(bars + kBPFree + ((gc - 1) & 1), ((gc - 1) >> 1) & 1)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
      }
      const float inv = (lt > 0.f) ? 1.f / lt : 0.f;
      const float lse2 = (lt > 0.f) ? m_ref + hw_log2(lt) : -INFINITY;
      const size_t rh = (size_t)(it.r0 + j) * kHeads + it.g * kHpg + h;
#pragma unroll 1
      for (int cb = 0; cb < kTOCols / 16; ++cb) {
        uint32_t o[16];
        if (have) {
          tc::ld_16cols(tmem + lane_base + kTmemO + qq * kTOCols + cb * 16, o);
          tc::wait_ld();
        } else {
#pragma unroll
          for (int x = 0; x < 16; ++x) o[x] = 0u;
        }
        if (row_ok) {
          const int d0 = qq * kTOCols + cb * 16;
          if (a.n_split == 1) {
            uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(a.out) + rh * kD + d0);
#pragma unroll
            for (int x = 0; x < 2; ++x)
              dst[x] = make_uint4(pack_bf16(__uint_as_float(o[8 * x]) * inv, __uint_as_float(o[8 * x + 1]) * inv),
                                  pack_bf16(__uint_as_float(o[8 * x + 2]) * inv, __uint_as_float(o[8 * x + 3]) * inv),
                                  pack_bf16(__uint_as_float(o[8 * x + 4]) * inv, __uint_as_float(o[8 * x + 5]) * inv),
                                  pack_bf16(__uint_as_float(o[8 * x + 6]) * inv, __uint_as_float(o[8 * x + 7]) * inv));
          } else {
            float4 *dst = reinterpret_cast<float4 *>(a.part_o + (rh * a.n_split + it.p) * kD + d0);
#pragma unroll
            for (int x = 0; x < 4; ++x)
              dst[x] = make_float4(__uint_as_float(o[4 * x]) * inv, __uint_as_float(o[4 * x + 1]) * inv,
                                   __uint_as_float(o[4 * x + 2]) * inv, __uint_as_float(o[4 * x + 3]) * inv);
          }
        }
      }
      if (have) {
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + kBOEmpty);
        ++qi;
      }
      if (row_ok && qq == 0) {
        if (a.n_split == 1) {
          if (a.lse != nullptr) a.lse[rh] = lse2 * 0.69314718055994531f;
        } else {
          a.part_lse[rh * a.n_split + it.p] = lse2;
        }
      }
      if (a.n_split == 1) continue;
      // ---- the last partition to finish (tile, group) merges every partition ----
      __threadfence();
      mbar_arrive(bars + kBMgAll);
      if (tid == 0) {
        int last = 0;
        if (wait(bars + kBMgAll, mi & 1)) {
          uint32_t *cnt = a.merge_cnt + (size_t)it.tile * kKv + it.g;
          const uint32_t prev = atomicAdd(cnt, 1u);
          last = (prev == (uint32_t)a.n_split - 1) ? 1 : 0;
          if (last) *cnt = 0u;  // every partition has arrived: ready for the next call
        }
        *is_last = last;
        mbar_arrive(bars + kBMgDec);
      }
      if (!wait(bars + kBMgDec, mi & 1)) {
        ok = false;
        break;
      }
      ++mi;
      if (*is_last) {
        __threadfence();
        const int mm = tid / kTSplit, dh = (tid % kTSplit) * kTOCols;
        const int jj = mm >> 4, hh = mm & 15;
        if (jj < it.nr) {
          const size_t rh2 = (size_t)(it.r0 + jj) * kHeads + it.g * kHpg + hh;
          float w[kMaxTileSplit];
          float lse;
          tile_partition_weights(a.part_lse + rh2 * a.n_split, a.n_split, w, lse);
          __nv_bfloat16 *out = reinterpret_cast<__nv_bfloat16 *>(a.out) + rh2 * kD + dh;
          for (int x = 0; x < kTOCols; x += 4) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int q = 0; q < a.n_split; ++q) {
              const float4 pv = ld_cg(reinterpret_cast<const float4 *>(a.part_o + (rh2 * a.n_split + q) * kD + dh + x));
              acc.x = fmaf(w[q], pv.x, acc.x);
              acc.y = fmaf(w[q], pv.y, acc.y);
              acc.z = fmaf(w[q], pv.z, acc.z);
              acc.w = fmaf(w[q], pv.w, acc.w);
            }
            uint2 w2;
            w2.x = pack_bf16(acc.x, acc.y);
            w2.y = pack_bf16(acc.z, acc.w);
            *reinterpret_cast<uint2 *>(out + x) = w2;
          }
          if ((tid % kTSplit) == 0 && a.lse != nullptr) a.lse[rh2] = lse;
        }
      }
    }
  }

  // ---- teardown: no MMA may be writing tensor memory when it is released ----
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) {
    mbar_wait_bounded(bars + kBFinal, 0, kTWaitNs);
    tc::tmem_dealloc(tmem, kTTmemCols);
  }
}

// Programmatic stream serialization: a kernel's launch overlaps the end of the
// previous one; every global read of these kernels follows pdl_wait().
template <typename K>
cudaError_t launch_after(K kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st, const TileArgs &a) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, a);
}

cudaError_t launch_tile_union(const TileArgs &a, int batch, cudaStream_t st) {
  const size_t smem = (size_t)a.map_words * sizeof(uint32_t);
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void *>(tile_union_kernel), (int)smem);
  if (e != cudaSuccess) return e;
  return launch_after(tile_union_kernel, dim3(a.tiles_per_seq, batch), dim3(256), smem, st, a);
}

cudaError_t launch_gqa_tile(const TileArgs &a, const CUtensorMap &tk, const CUtensorMap &tv, int n_ctas,
                            cudaStream_t st) {
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void *>(gqa_tile_kernel), kTileSmem);
  if (e != cudaSuccess) return e;
  const long long n_items = (long long)a.n_split * a.n_tiles * kKv;  // upper bound: every tile shared-set
  if (n_items > 0x7fffffffLL) return cudaErrorInvalidValue;
  const int grid = (int)(n_items < n_ctas ? n_items : n_ctas);
  if (grid < 1) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kTThreads);
  cfg.dynamicSmemBytes = kTileSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gqa_tile_kernel, a, tk, tv);
}

}  // namespace s5
