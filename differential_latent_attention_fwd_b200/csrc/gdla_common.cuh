// Device-side building blocks shared by the GDLA kernels (sm_100a only).
//
// Thin inline-PTX wrappers for mbarriers, TMA tiled loads, the 5th-generation tensor core
// (tcgen05: TMEM allocation, MMA issue, commit, TMEM loads/stores) and bounded waits.
// Every wait on an mbarrier is bounded in wall-clock time: when the bound is hit the wait
// records a site code in the device error word and returns false, so that a kernel whose
// producer or consumer went missing exits with an error status instead of hanging.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "gdla kernels target sm_100a only"
#endif

namespace gdla {

// Per-launch control block: where to report a failed wait and how long a wait may last.
struct KernelCtl {
  int* err;                      // device error word (0 = ok); first failing site wins
  unsigned long long limit_ns;   // bound of one mbarrier wait
};

// Site codes written to the error word (the host maps them to GDLA_ERR_DEVICE_TIMEOUT).
enum : int {
  SITE_GEMM_PRODUCER = 0x101, SITE_GEMM_MMA = 0x102, SITE_GEMM_EPI = 0x103,
  SITE_ATTN_PRODUCER = 0x201, SITE_ATTN_MMA = 0x202, SITE_ATTN_SOFTMAX = 0x203,
  SITE_DRAIN = 0x301, SITE_SELFTEST = 0x401,
  SITE_DEC_PRODUCER = 0x501, SITE_DEC_MMA = 0x502, SITE_DEC_SOFTMAX = 0x503, SITE_DEC_CONVERT = 0x504,
  SITE_BWD_PRODUCER = 0x511, SITE_BWD_MMA = 0x512, SITE_BWD_SOFTMAX = 0x513,
  SITE_BAD_CACHE_LEN = 0x601,  // a cache_len entry outside [0, cap): that sequence is skipped
  SITE_BAD_CU_SEQLENS = 0x602, // document offsets not 0..total non-decreasing: bad documents skipped
  SITE_FP16_RANGE = 0x701,     // an fp16 attention operand was outside +-65504 (saturated) or NaN
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
               ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

// Non-blocking test: has the phase with the given parity completed?
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity has completed.  Returns false (after writing
// `site` to the error word) when the bound expires or another role already failed.
static __device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, const KernelCtl& ctl,
                                            int site) {
  const uint64_t t0 = global_timer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*reinterpret_cast<volatile int*>(ctl.err) != 0) return false;
    if (global_timer_ns() - t0 > ctl.limit_ns) {
      atomicCAS(ctl.err, 0, site);
      return false;
    }
  }
}
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const KernelCtl& ctl,
                                          int site) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, ctl, site);
}
// Used on exit paths to let our own in-flight copies / MMAs land before the CTA retires:
// a fixed generous bound that test knobs on `ctl.limit_ns` do not shorten.
static __device__ __noinline__ bool mbar_drain(uint64_t* bar, uint32_t parity, int* err) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > 2000000000ull) {
      atomicCAS(err, 0, SITE_DRAIN);
      return false;
    }
  }
  return true;
}

// ------------------------------------------------------------------ TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}
// 2-D tiled load of one box at (x = inner element index, y = row) into shared memory,
// completing `bytes` on the mbarrier.  x * element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y) : "memory");
}

// Bulk prefetch of [addr, addr + bytes) into L2 (16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void l2_prefetch_bulk(const void* addr, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(addr), "r"(bytes) : "memory");
}

// L2 cache policies for TMA loads: keep a line for an upcoming re-read, or let it go first.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
// tma_load_2d with an L2 cache policy.
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map, uint64_t* bar,
                                                 int x, int y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;"
      ::"r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy) : "memory");
}

// ------------------------------------------------------------------ tcgen05 / TMEM
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D(tmem) (+)= A(smem) * B(smem)
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                      uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}
// D(tmem) (+)= A(tmem) * B(smem)
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                      uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}
// The same two with shared-memory descriptors given as (low, high) 32-bit words: the low word
// holds the start address (and the leading offset), so an issuer steps through a buffer with
// one 32-bit add per operand instead of rebuilding 64-bit descriptors.
__device__ __forceinline__ void mma_ss_w(uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi, uint32_t b_lo,
                                        uint32_t b_hi, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\tsetp.ne.b32 p, %6, 0;\n\t"
      "mov.b64 da, {%1, %2};\n\tmov.b64 db, {%3, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %5, p;\n\t}"
      ::"r"(d_tmem), "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate) : "memory");
}
__device__ __forceinline__ void mma_ts_w(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t b_hi,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\tsetp.ne.b32 p, %5, 0;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate) : "memory");
}
// Arrive once on `bar` when every previously issued tcgen05.mma of this thread has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_u32(bar)) : "memory");
}

// Instruction descriptor of tcgen05.mma kind::f16 with an fp32 accumulator.
//   ab_bf16: 1 = both operands bf16, 0 = both fp16; *_mn: 1 = operand is M/N-major in smem.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N, int ab_bf16, int a_mn, int b_mn) {
  return (1u << 4) | (uint32_t(ab_bf16) << 7) | (uint32_t(ab_bf16) << 10) | (uint32_t(a_mn) << 15) |
         (uint32_t(b_mn) << 16) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand (version 1, sm_100).
//   K-major: rows of 64 16-bit elements along K; sbo = 1024 (8-row group stride).
//   MN-major: rows along K holding 64 M/N elements; lbo = stride between 64-element M/N
//   chunks, sbo = 1024 (stride between 8-row K groups).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= uint64_t((saddr & 0x3FFFFu) >> 4);
  d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
  d |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;
  return d;
}

// 32 lanes x 32 consecutive 32-bit TMEM columns -> 32 registers per thread.
#define GDLA_TMEM_LD32(taddr, r)                                                                   \
  asm volatile(                                                                                    \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14," \
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"              \
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),      \
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),  \
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),            \
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),            \
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])             \
      : "r"(taddr))

#define GDLA_TMEM_ST32(taddr, r)                                                                   \
  asm volatile(                                                                                    \
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"  \
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"             \
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), \
        "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),         \
        "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]),      \
        "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),      \
        "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])                                           \
      : "memory")

// 32 lanes x 16 consecutive 32-bit TMEM columns.
#define GDLA_TMEM_LD16(taddr, r)                                                                   \
  asm volatile(                                                                                    \
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14," \
      "%15}, [%16];"                                                                              \
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),      \
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),  \
        "=r"(r[14]), "=r"(r[15])                                                                 \
      : "r"(taddr))

#define GDLA_TMEM_ST16(taddr, r)                                                                   \
  asm volatile(                                                                                    \
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"  \
      "%14,%15,%16};"                                                                             \
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), \
        "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),         \
        "r"(r[14]), "r"(r[15])                                                                   \
      : "memory")

#define GDLA_TMEM_ST8(taddr, r)                                                                    \
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"            \
               ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),   \
                 "r"(r[6]), "r"(r[7])                                                            \
               : "memory")

// 16-byte asynchronous global -> shared copy (all of a thread's copies stay in flight).
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Make generic-proxy writes to shared memory visible to the async proxy (TMA, tensor core).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Named barrier among `count` threads (ids 1.. are free; 0 is __syncthreads).
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Named barrier that also ORs a predicate over the participating threads.
__device__ __forceinline__ bool named_bar_or(int id, int count, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out) : "r"(uint32_t(pred)), "r"(id), "r"(count) : "memory");
  return out != 0;
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------------ CTA pairs
// A cluster of two CTAs on one TPC that share tcgen05 MMAs of M = 256 (cta_group::2): the
// even-ranked CTA ("leader") issues the MMAs; A rows and the accumulator are split 128 / 128
// between the two CTAs, B columns N / 2 / N / 2.  Every tcgen05 instruction of such a kernel
// uses cta_group::2, and TMEM is allocated by the same warp of both CTAs.
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address, in the cluster shared window, of the variable at `saddr` in the CTA of rank `rank`.
__device__ __forceinline__ uint32_t smem_map_rank(uint32_t saddr, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(saddr), "r"(rank));
  return out;
}
// Every thread of both CTAs: release this CTA's prior writes, wait for the peer's.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
// Arrive on an mbarrier given by its cluster-window address (possibly in the peer CTA).  The
// release is CTA-scoped: what it publishes is TMEM state ordered by tcgen05 fences, and a
// cluster-scoped release costs about a microsecond per arrive.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cl_addr) {
  asm volatile("mbarrier.arrive.release.cta.shared::cluster.b64 _, [%0];" ::"r"(cl_addr)
               : "memory");
}
// 2-D tiled load into this CTA's shared memory whose completion is counted on an mbarrier of
// either CTA of the pair (`bar_cl`: cluster-window address); one destination only.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cl,
                                                 int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(dst)), "l"(map), "r"(bar_cl), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// M = 256 pair MMAs, issued by the leader: D (+)= A(smem) B(smem) and D (+)= A(tmem) B(smem).
// Shared-memory descriptors come as (low, high) words: the low word holds the start address,
// so a caller steps through a tile with one 32-bit add per operand.  acc != 0: accumulate.
__device__ __forceinline__ void mma_ss_pair(uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi,
                                           uint32_t b_lo, uint32_t b_hi, uint32_t idesc,
                                           uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\tsetp.ne.b32 p, %6, 0;\n\t"
      "mov.b64 da, {%1, %2};\n\tmov.b64 db, {%3, %4};\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], da, db, %5, p;\n\t}"
      ::"r"(d_tmem), "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(acc) : "memory");
}
__device__ __forceinline__ void mma_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo,
                                           uint32_t b_hi, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\tsetp.ne.b32 p, %5, 0;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], db, %4, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(acc) : "memory");
}
// When every pair MMA issued so far has completed, arrive once on the mbarrier at the same
// shared-memory offset in each CTA of `cta_mask` (bit r = rank r).
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)), "h"(cta_mask) : "memory");
}

// ------------------------------------------------------------------ math helpers
// cos/sin of pos * inv_freq: the angle is formed and reduced to [-pi, pi) in double precision,
// then evaluated with the hardware single-precision sin/cos (absolute error ~2^-21 on that range).
__device__ __forceinline__ void rope_cs(int pos, double inv_freq, float* c, float* s) {
  const double two_pi = 6.283185307179586476925286766559;
  double a = double(pos) * inv_freq;
  a -= two_pi * floor(a * (1.0 / two_pi) + 0.5);
  __sincosf(float(a), s, c);
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// ---- softmax arithmetic.  Packed f32x2 instructions halve the issue slots of the scale,
// subtract and sum steps; the attention kernels run part of their exponentials on the FMA pipe
// (exp2_poly2) instead of MUFU, whose 16 results per clock per SM bound a softmax.
__device__ __forceinline__ float fmax3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// (d0, d1) = (a0, a1) + (b0, b1)
__device__ __forceinline__ void fadd2v(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 d, a, b;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "add.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
// (d0, d1) = (a0, a1) * (b0, b1) + (c, c)
__device__ __forceinline__ void ffma2v(float& d0, float& d1, float a0, float a1, float b0, float b1, float c) {
  asm("{\n\t.reg .b64 d, a, b, c;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\tmov.b64 c, {%6, %6};\n\t"
      "fma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c));
}
// (d0, d1) = (a0, a1) * (b0, b1) + (c0, c1)
__device__ __forceinline__ void ffma2vv(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                        float c1) {
  asm("{\n\t.reg .b64 d, a, b, c;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\tmov.b64 c, {%6, %7};\n\t"
      "fma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
// (d0, d1) = (a0, a1) * (b0, b1)
__device__ __forceinline__ void fmul2v(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 d, a, b;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "mul.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
// (x0, x1) = (a0, a1) * b + c
__device__ __forceinline__ void ffma2(float& x0, float& x1, float a0, float a1, float b, float c) {
  ffma2v(x0, x1, a0, a1, b, b, c);
}
// (s0, s1) += (a0, a1)
__device__ __forceinline__ void fadd2(float& s0, float& s1, float a0, float a1) {
  fadd2v(s0, s1, s0, s1, a0, a1);
}
// 2^x for a pair on the FMA pipe.  x = j + f with j = round(x) (adding and subtracting
// 1.5 * 2^23 rounds to the nearest integer) and |f| <= 1/2; 2^f from a cubic fitted to 2^f
// on [-1/2, 1/2] (iteratively reweighted least squares towards the minimax fit, max relative
// error 7.5e-5, below the 2^-12 half-ulp of the fp16 or bf16 P it feeds; exp2_poly_fit.py beside this
// file reproduces the coefficients); j is added to the exponent field as an integer.  x is
// clamped at -126, where P is 0 either way in fp16 and ~2^-126 in bf16.
__device__ __forceinline__ void exp2_poly2(float x0, float x1, float& r0, float& r1) {
  x0 = fmaxf(x0, -126.f);
  x1 = fmaxf(x1, -126.f);
  float t0, t1, j0, j1, f0, f1;
  fadd2v(t0, t1, x0, x1, 12582912.f, 12582912.f);
  fadd2v(j0, j1, t0, t1, -12582912.f, -12582912.f);
  fadd2v(f0, f1, x0, x1, -j0, -j1);
  float q0 = 0.05517144128680229f, q1 = 0.05517144128680229f;
  ffma2v(q0, q1, q0, q1, f0, f1, 0.24261070787906647f);
  ffma2v(q0, q1, q0, q1, f0, f1, 0.6932609677314758f);
  ffma2v(q0, q1, q0, q1, f0, f1, 0.9999281167984009f);
  // the low 9 bits of t's bit pattern hold j mod 512; * 2^23 moves them into the exponent field
  r0 = __int_as_float(__float_as_int(t0) * 8388608 + __float_as_int(q0));
  r1 = __int_as_float(__float_as_int(t1) * 8388608 + __float_as_int(q1));
}

__device__ __forceinline__ float sigmoidf_fast(float z) {
  // 1 / (1 + 2^(-z log2 e)); the hardware exp2 has ~2 ulp relative error.
  return 1.0f / (1.0f + ex2_approx(-z * 1.4426950408889634f));
}
__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
// fp16 pair for the attention operands (q, K^C, V, k^R): a finite value beyond the fp16 range
// saturates to +-65504 instead of becoming Inf, and `bad` is set for it and for NaN, so that
// the caller can record SITE_FP16_RANGE.
__device__ __forceinline__ uint32_t pack_half2_sat(float lo, float hi, bool& bad) {
  constexpr float kMax = 65504.f;
  bad |= !(fabsf(lo) <= kMax) || !(fabsf(hi) <= kMax);
  lo = fabsf(lo) > kMax ? copysignf(kMax, lo) : lo;
  hi = fabsf(hi) > kMax ? copysignf(kMax, hi) : hi;
  return pack_half2(lo, hi);
}
__device__ __forceinline__ __half half_sat(float v, bool& bad) {
  constexpr float kMax = 65504.f;
  bad |= !(fabsf(v) <= kMax);
  return __float2half_rn(fabsf(v) > kMax ? copysignf(kMax, v) : v);
}
__device__ __forceinline__ uint32_t pack_bf162(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace gdla
