// Shared device helpers of the s5attn library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "s5attn.h"

namespace s5 {

constexpr int kHeads = S5_N_HEADS;          // 64 query heads
constexpr int kKv = S5_N_KV_HEADS;          // 4 KV groups
constexpr int kHpg = kHeads / kKv;          // 16 query heads share one group
constexpr int kD = S5_HEAD_DIM;             // 192
constexpr int kPage = S5_PAGE_SIZE;         // 64 tokens per page
constexpr int kBlk = S5_BLOCK_SIZE;         // 8 tokens per indexer block
constexpr int kBpp = kPage / kBlk;          // 8 blocks per page
constexpr int kDx = S5_INDEX_DIM;           // 256
constexpr int kMaxTopk = S5_MAX_TOPK;       // 512
constexpr int kBlockBytes = kBlk * kD * 2;  // 3,072 bytes: one block of one group (K or V)

// Workspace header: the device error record lives in the first 256 bytes,
// followed by the attention merge counters (4 per row for up to 1,024 rows).
constexpr size_t kWsHeader = 256;
constexpr size_t kWsCounterBytes = 16384;
constexpr size_t kWsFixed = kWsHeader + kWsCounterBytes;  // first byte of per-call scratch
// 64-bit word 8 of the header (bytes 64..71): the expired-wait test hook of
// the per-row attention kernel (S5_WS_TEST_STALL_OFFSET), zero in normal use
constexpr int kWsStallWord = S5_WS_TEST_STALL_OFFSET / 8;

// Loads that stay after a preceding wait or fence in program order (asm
// volatile, L2-coherent).  Used for every read of data another kernel or CTA
// may have just written: plain __ldg loads are treated as invariant and may be
// hoisted above griddepcontrol.wait or a fence.
__device__ __forceinline__ int32_t ld_cg(const int32_t *p) {
  int32_t v;
  asm volatile("ld.global.cg.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t ld_cg(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.global.cg.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint64_t ld_cg_u64(const uint64_t *p) {
  uint64_t v;
  asm volatile("ld.global.cg.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ float ld_cg(const float *p) {
  float v;
  asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint4 ld_cg(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ float4 ld_cg(const float4 *p) {
  float4 v;
  asm volatile("ld.global.cg.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p) : "memory");
  return v;
}

struct ErrRec {
  int32_t code;
  int32_t info;
};

__device__ __forceinline__ void record_error(int32_t *err, int code, int info) {
  if (err == nullptr) return;
  if (atomicCAS(err, 0, code) == 0) atomicExch(err + 1, info);
}

// ---------------------------------------------------------------- batch lookup

// Sequence owning query row r: the largest s with cu_q[s] <= r (cu_q is
// non-decreasing).  Returns -1 when r is outside [cu_q[0], cu_q[batch]).
__device__ __forceinline__ int seq_of_row(const int32_t *cu_q, int batch, int r) {
  int lo = 0, hi = batch;  // invariant: cu_q[lo] <= r < cu_q[hi]
  if (r < ld_cg(cu_q) || r >= ld_cg(cu_q + batch)) return -1;
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (ld_cg(cu_q + mid) <= r) lo = mid; else hi = mid;
  }
  return lo;
}

// Sequence s and absolute position t of query row r.  `guess` is tried
// first (one round trip: cu_q[g], cu_q[g+1], ctx_lens[g] are independent
// loads); a miss falls back to the binary search.  False on bad batch data.
__device__ __forceinline__ bool locate_row(const int32_t *cu_q, const int32_t *ctx_lens, int batch, int r,
                                           int guess, int &s, int &t) {
  const int g = min(max(guess, 0), batch - 1);
  const int lo = ld_cg(cu_q + g), hi = ld_cg(cu_q + g + 1), ctx = ld_cg(ctx_lens + g);
  if (lo <= r && r < hi) {
    s = g;
    t = ctx + (r - lo);
    return true;
  }
  s = seq_of_row(cu_q, batch, r);
  if (s < 0) return false;
  t = ld_cg(ctx_lens + s) + (r - ld_cg(cu_q + s));
  return true;
}

// Proportional guess of the sequence of row r (exact when every sequence has
// the same number of query rows).
__device__ __forceinline__ int row_guess(int r, int batch, int total_q) {
  return total_q > 0 ? (int)(((long long)r * batch) / total_q) : 0;
}

// ---------------------------------------------------------------- small PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start before the previous kernel in the stream finishes;
// pdl_wait() blocks until that kernel has completed and its writes are
// visible (a no-op for ordinary launches).  pdl_trigger() lets the next such
// kernel start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait on an mbarrier phase: gives up after `limit_ns` of wall time.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 63 && globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// try_wait with a suspend-time hint: a thread whose phase is not complete may
// be suspended for up to hint_ns (it resumes when the phase completes) instead
// of returning at once, so a waiting warp does not take issue slots.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t *bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Bounded wait that sleeps between polls (suspend hint of hint_ns per poll).
__device__ __forceinline__ bool mbar_wait_bounded_hint(uint64_t *bar, uint32_t parity, uint64_t limit_ns,
                                                       uint32_t hint_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait_hint(bar, parity, hint_ns)) return true;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// 3-D tiled TMA load (no multicast) into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(void *smem_dst, const void *tmap, int c0, int c1, int c2,
                                            uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// L2 prefetch of `bytes` contiguous global bytes (16-byte aligned, a multiple
// of 16): no data reaches the issuing thread and nothing is signalled.
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(src)), "r"(bytes)
               : "memory");
}

// 2-D tiled TMA load (no multicast) into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const void *tmap, int c0, int c1, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// For data other CTAs of the same launch will read again (blocks shared by
// neighbouring query tiles).
__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D = A (16x16 bf16, row) * B (16x8 bf16, col) + D, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// bf16 pair (packed in a 32-bit word) to two floats: exact (bf16 is the top half of fp32).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Order-preserving map of a float score to an unsigned key (larger score ->
// larger key); -0.0 is folded onto +0.0 so equal scores give equal keys.
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t u = __float_as_uint(s);
  if ((u & 0x7FFFFFFFu) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Four one-byte E4M3 codes (byte i of w is element i) to their exact values:
// every E4M3 value is a half-precision value, and every half a float.  The
// codes widen pairwise to f16 pairs (first element in the low half), then
// each half to fp32.
__device__ __forceinline__ void e4m3x4_to_float(uint32_t w, float &f0, float &f1, float &f2, float &f3) {
  asm("{\n\t.reg .b16 a, b, h0, h1, h2, h3;\n\t.reg .b32 p, q;\n\t"
      "mov.b32 {a, b}, %4;\n\t"
      "cvt.rn.f16x2.e4m3x2 p, a;\n\t"
      "cvt.rn.f16x2.e4m3x2 q, b;\n\t"
      "mov.b32 {h0, h1}, p;\n\t"
      "mov.b32 {h2, h3}, q;\n\t"
      "cvt.f32.f16 %0, h0;\n\t"
      "cvt.f32.f16 %1, h1;\n\t"
      "cvt.f32.f16 %2, h2;\n\t"
      "cvt.f32.f16 %3, h3;\n\t}"
      : "=f"(f0), "=f"(f1), "=f"(f2), "=f"(f3)
      : "r"(w));
}

// Hardware base-2 exponential / logarithm (PTX ex2.approx / lg2.approx).
__device__ __forceinline__ float hw_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float hw_log2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace s5
