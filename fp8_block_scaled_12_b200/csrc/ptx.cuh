// ptx.cuh -- thin inline-PTX wrappers for sm_100a: mbarriers, TMA tensor loads,
// tcgen05 (tensor memory allocation, FP8 MMA, commit, loads) and bounded waits.
//
// Every spin-wait here is bounded: after FP8LIN_WAIT_NS of wall time (read from
// %globaltimer) or FP8LIN_WAIT_ITERS polls it records FP8_ERR_TIMEOUT in the
// library's device error word, raises the calling CTA's abort flag and returns
// false, so the kernel can skip its remaining work and exit instead of hanging.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#ifndef FP8LIN_WAIT_NS
#define FP8LIN_WAIT_NS 2000000000ull   // 2 s
#endif
#ifndef FP8LIN_WAIT_ITERS
#define FP8LIN_WAIT_ITERS (1u << 26)
#endif

namespace fp8lin {

// Device-side error word (one per device that loaded the library).  Bit 0:
// a bounded wait ran out.  Read and cleared by fp8_device_error().  The whole
// library is one translation unit, so this definition is the only one.
__device__ unsigned int g_device_error;
// Limit of the pipeline waits in ns (FP8LIN_WAIT_NS unless a diagnostic call lowers it
// to exercise the timeout and abort path).
__device__ unsigned long long g_wait_limit_ns = FP8LIN_WAIT_NS;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity of `bar` has completed.  Returns
// false (and raises *abort) when the wait runs out or another thread of the CTA
// has already aborted.
// One failed try_wait already suspends the thread for a hardware-defined time, so a
// limit under 1 us gives up at the first poll that fails.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort, uint64_t limit_ns = 0) {
  if (mbar_try_wait(bar, parity)) return true;
  if (limit_ns == 0) limit_ns = *reinterpret_cast<volatile unsigned long long*>(&g_wait_limit_ns);
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = limit_ns < 1000 ? FP8LIN_WAIT_ITERS : 1u; i < FP8LIN_WAIT_ITERS; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 31u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) break;
    }
  }
  *abort = 1;
  atomicOr(&g_device_error, 1u);
  return false;
}

// Spin for roughly `ns` nanoseconds (bounded by an iteration cap as well).
__device__ __forceinline__ void settle_ns(uint64_t ns) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 0; i < (1u << 22); ++i)
    if (globaltimer_ns() - t0 > ns) break;
}

// Abort path: wait for a phase that completes on its own -- an issued TMA or bulk copy
// landing, issued MMAs finishing -- so nothing asynchronous still writes this CTA's
// shared or tensor memory when it releases them and exits.  Ignores the abort flag
// and always uses the full FP8LIN_WAIT_NS; should even this run out, the thread
// settles for a further 200 us instead.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 0; i < FP8LIN_WAIT_ITERS; ++i) {
    if (mbar_try_wait(bar, parity)) return;
    if ((i & 31u) == 31u && globaltimer_ns() - t0 > FP8LIN_WAIT_NS) break;
  }
  settle_ns(200000);
}

// ----------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// L2 prefetch of one 2-D tile through a tensor map (no shared memory, no completion).
// The L2 is the point of coherence for device memory, so a prefetch issued before the
// grid-dependency wait can never hand stale data to a later load.
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap* m, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(reinterpret_cast<uint64_t>(m)),
               "r"(x), "r"(y)
               : "memory");
}

// Programmatic dependent launch.  Every kernel of the library is launched so that it
// may start while the previous kernel on the stream is finishing; pdl_wait() blocks
// the calling thread until that kernel has completed and its writes are visible, so
// each kernel calls it before its first global read or write of operand data.
// pdl_trigger() lets the next kernel be scheduled once every CTA of this grid has
// called it (or exited); a CTA that has not started cannot have called it, so the
// next grid never takes SMs this grid still needs.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// 2-D tiled bulk tensor load global -> shared, completion counted on `bar`.
// c0 is the innermost (contiguous) coordinate in elements; it must be a multiple
// of 16 for 1-byte elements (callers only pass multiples of 128).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* m, uint32_t bar,
                                            int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

// ------------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
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

// D[tmem] (+)= A[smem] * B[smem]^T, FP8 operands (kind::f8f6f4), fp32 accumulators.
__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives lane
// (quadrant*32 + i), columns [col, col+32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Call right after tmem_ld_wait() on every register array it completed.  The
// registers pass through an empty volatile asm that the compiler keeps after the
// (volatile) wait, so every later use of them -- including non-volatile
// arithmetic asm such as ffma2 -- depends on the wait and cannot be hoisted above
// it.  Emits no instruction.
template <int N>
__device__ __forceinline__ void tmem_regs_ready(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

// Shared-memory matrix descriptor for a K-major operand tile written by TMA with
// the 128-byte swizzle: rows of 128 bytes, 8-row atoms of 1024 bytes stacked
// contiguously (stride 1024 B between atoms).  Fields: start address >> 4 in
// bits [0,14), leading offset (unused for swizzled K-major, set to 1) in
// [16,30), stride offset 1024 >> 4 in [32,46), descriptor version 1 in [46,48),
// base offset 0 (atoms are 1024-byte aligned), layout SWIZZLE_128B = 2 in [61,64).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
  return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor for kind::f8f6f4: fp32 accumulator (bits [4,6) = 1),
// A and B E4M3 (format 0 in [7,10) and [10,13)), both K-major (bits 15, 16 = 0),
// N >> 3 in [17,23), M >> 4 in [24,29).
__host__ __device__ constexpr uint32_t idesc_f8_e4m3_f32(uint32_t m, uint32_t n) {
  return (1u << 4) | ((n >> 3) << 17) | ((m >> 4) << 24);
}

// ------------------------------------------------------- packed fp32 pairs
// Two fp32 values in one 64-bit register pair (low half = first value).
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 unpack2(uint64_t v) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
  return make_float2(lo, hi);
}
// acc += (p_lo, p_hi) * s2 as two independent, correctly rounded fp32 FMAs in one
// packed instruction (fma.rn.f32x2); identical results to two fmaf calls.
__device__ __forceinline__ void ffma2(uint64_t& acc, uint32_t p_lo, uint32_t p_hi, uint64_t s2) {
  asm("{\n\t.reg .b64 t;\n\tmov.b64 t, {%1, %2};\n\tfma.rn.f32x2 %0, t, %3, %0;\n\t}"
      : "+l"(acc)
      : "r"(p_lo), "r"(p_hi), "l"(s2));
}

// *p += v in global memory without waiting for (or returning) the old value.
__device__ __forceinline__ void red_add_f32(float* p, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

// ------------------------------------------------- small asynchronous copies
// 4-byte global -> shared copy that does not block the issuing thread.
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
// Wait until every cp.async this thread issued has landed in shared memory.
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// ------------------------------------------------------- register reallocation

template <uint32_t RegCount>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(RegCount));
}
template <uint32_t RegCount>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(RegCount));
}

}  // namespace fp8lin
