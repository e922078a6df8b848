// lf_ptx.cuh -- inline-PTX helpers shared by the tensor-core kernels:
// mbarriers with bounded waits, TMA tile loads, tcgen05 MMA / TMEM access,
// shared-memory and instruction descriptors, packed conversions.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "lf_common.cuh"

#define LF_WAIT_NS 1500000000ull

// ------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t lf_smem(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint64_t lf_globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void lf_mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void lf_mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void lf_mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool lf_mbar_try(uint32_t bar, uint32_t parity) {
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

// Bounded wait on an mbarrier phase.  Returns false when the CTA aborted
// (this thread's own timeout, or another role's).  abort_flag[0] is the
// CTA's abort flag; abort_flag[1] the wait limit in microseconds (0: the
// default LF_WAIT_NS), both in shared memory, set by the kernel at start.
static __device__ __noinline__ bool lf_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                     int32_t *status, int site) {
  uint64_t t0 = 0;
  const uint64_t limit = abort_flag[1] > 0 ? (uint64_t)abort_flag[1] * 1000ull : LF_WAIT_NS;
  for (uint32_t it = 0;; it++) {
    if (lf_mbar_try(bar, parity)) return true;
    if ((it & 255) == 255) {
      if (*abort_flag) return false;
      uint64_t now = lf_globaltimer();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > limit) {
        *abort_flag = 1;
        lf_set_status(status, LF_ERR_DEVICE_TIMEOUT, site);
        return false;
      }
    }
  }
}

// Wait for asynchronous work this CTA has already issued (TMA copies, MMAs)
// to complete, also after an abort: the abort flag is not consulted, the
// wait is bounded by time alone (LF_WAIT_NS); on expiry the status records
// a timeout at `site`.
static __device__ __noinline__ bool lf_wait_drain(uint32_t bar, uint32_t parity, int32_t *status,
                                                  int site) {
  uint64_t t0 = 0;
  for (uint32_t it = 0;; it++) {
    if (lf_mbar_try(bar, parity)) return true;
    if ((it & 255) == 255) {
      uint64_t now = lf_globaltimer();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > LF_WAIT_NS) {
        lf_set_status(status, LF_ERR_DEVICE_TIMEOUT, site);
        return false;
      }
    }
  }
}

// Bounded wait with an inlined first probe (the common, already-complete case).
__device__ __forceinline__ bool lf_wait_fast(uint32_t bar, uint32_t parity,
                                             volatile int *abort_flag, int32_t *status, int site) {
  if (lf_mbar_try(bar, parity)) return true;
  return lf_wait(bar, parity, abort_flag, status, site);
}

// Warp-uniform bounded wait: the converged warp polls together (every lane
// acquires the phase itself), and the outcome is made uniform before the
// warp-collective tcgen05 instructions that follow.
__device__ __forceinline__ bool lf_wait_warp(uint32_t bar, uint32_t parity,
                                             volatile int *abort_flag, int32_t *status, int site) {
  const bool ok = lf_wait_fast(bar, parity, abort_flag, status, site);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void lf_tma_load4(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                             int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void lf_tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void lf_tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---- MMA phases issued by a converged warp.  One elected lane (the same
// lane every time the full warp is converged) issues a whole phase from a
// single asm statement.  Issue cost measured on B200: one tcgen05.mma per
// asm statement from a diverged lane ~180 cycles each; a four-MMA S phase
// (128x128x64) as one statement ~380 cycles, an eight-MMA P.V phase
// (128x64x128) ~490 -- against 256 + 256 cycles of tensor-core work.  Every
// tcgen05 operation of the warp comes from that lane, so each commit tracks
// all of them.

// commit of all prior MMAs of the warp to `bar`
__device__ __forceinline__ void lf_commit_w(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          bar)
      : "memory");
}

// D = A * B^T over a 64-wide reduction: four K = 16 MMAs with K-major
// 128-byte-swizzled operands (each descriptor advances 32 bytes per step,
// i.e. +2 in its 16-byte units), then a commit to `bar`.
__device__ __forceinline__ void lf_mma_s_phase(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                               uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t.reg .b64 a1, a2, a3, b1, b2, b3;\n\t"
      "add.s64 a1, %1, 2;\n\tadd.s64 a2, %1, 4;\n\tadd.s64 a3, %1, 6;\n\t"
      "add.s64 b1, %2, 2;\n\tadd.s64 b2, %2, 4;\n\tadd.s64 b3, %2, 6;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %3, 1;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a2, b2, %3, 1;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a3, b3, %3, 1;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%4];\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(bar)
      : "memory");
}

// Two such products into two accumulators (D0 = A0 B0^T, D1 = A1 B1^T,
// same shape), interleaved step by step, then one commit to `bar`.
__device__ __forceinline__ void lf_mma_s2_phase(uint32_t d0, uint64_t a0, uint64_t b0, uint32_t d1,
                                                uint64_t a1, uint64_t b1, uint32_t idesc,
                                                uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t.reg .b64 x1, x2, x3, y1, y2, y3, u1, u2, u3, v1, v2, v3;\n\t"
      "add.s64 x1, %1, 2;\n\tadd.s64 x2, %1, 4;\n\tadd.s64 x3, %1, 6;\n\t"
      "add.s64 y1, %2, 2;\n\tadd.s64 y2, %2, 4;\n\tadd.s64 y3, %2, 6;\n\t"
      "add.s64 u1, %4, 2;\n\tadd.s64 u2, %4, 4;\n\tadd.s64 u3, %4, 6;\n\t"
      "add.s64 v1, %5, 2;\n\tadd.s64 v2, %5, 4;\n\tadd.s64 v3, %5, 6;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %6, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%3], %4, %5, %6, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], x1, y1, %6, 1;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%3], u1, v1, %6, 1;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], x2, y2, %6, 1;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%3], u2, v2, %6, 1;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], x3, y3, %6, 1;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%3], u3, v3, %6, 1;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%7];\n\t}" ::"r"(d0),
      "l"(a0), "l"(b0), "r"(d1), "l"(a1), "l"(b1), "r"(idesc), "r"(bar)
      : "memory");
}

// D (+)= A * B with A in TMEM: up to eight K = 16 MMAs, step k reading A
// columns a + 8k and the B descriptor advanced by bstep * k (16-byte units);
// step k is issued when bit k of kmask is set (kmask = 2^steps - 1, steps
// >= 1).  Step 0 accumulates iff acc0 != 0, later steps always do.  Then
// commits to bar1, bar2 and bar3, each skipped when its address is 0.
__device__ __forceinline__ void lf_mma_ts_phase(uint32_t d, uint32_t a, uint64_t b, uint32_t bstep,
                                                uint32_t idesc, uint32_t kmask, uint32_t acc0,
                                                uint32_t bar1, uint32_t bar2, uint32_t bar3) {
  asm volatile(
      "{\n\t.reg .pred e, pa, p1, p2, p3, p4, p5, p6, p7, c1, c2, c3;\n\t"
      ".reg .b32 t1, t2, t3, t4, t5, t6, t7, m;\n\t.reg .b64 s, b1, b2, b3, b4, b5, b6, b7;\n\t"
      "add.u32 t1, %1, 8;\n\tadd.u32 t2, %1, 16;\n\tadd.u32 t3, %1, 24;\n\tadd.u32 t4, %1, 32;\n\t"
      "add.u32 t5, %1, 40;\n\tadd.u32 t6, %1, 48;\n\tadd.u32 t7, %1, 56;\n\t"
      "cvt.u64.u32 s, %4;\n\t"
      "add.s64 b1, %2, s;\n\tadd.s64 b2, b1, s;\n\tadd.s64 b3, b2, s;\n\tadd.s64 b4, b3, s;\n\t"
      "add.s64 b5, b4, s;\n\tadd.s64 b6, b5, s;\n\tadd.s64 b7, b6, s;\n\t"
      "setp.ne.b32 pa, %6, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "and.b32 m, %5, 2;\n\tsetp.ne.and.b32 p1, m, 0, e;\n\t"
      "and.b32 m, %5, 4;\n\tsetp.ne.and.b32 p2, m, 0, e;\n\t"
      "and.b32 m, %5, 8;\n\tsetp.ne.and.b32 p3, m, 0, e;\n\t"
      "and.b32 m, %5, 16;\n\tsetp.ne.and.b32 p4, m, 0, e;\n\t"
      "and.b32 m, %5, 32;\n\tsetp.ne.and.b32 p5, m, 0, e;\n\t"
      "and.b32 m, %5, 64;\n\tsetp.ne.and.b32 p6, m, 0, e;\n\t"
      "and.b32 m, %5, 128;\n\tsetp.ne.and.b32 p7, m, 0, e;\n\t"
      "setp.ne.and.b32 c1, %7, 0, e;\n\t"
      "setp.ne.and.b32 c2, %8, 0, e;\n\t"
      "setp.ne.and.b32 c3, %9, 0, e;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, pa;\n\t"
      "@p1 tcgen05.mma.cta_group::1.kind::f16 [%0], [t1], b1, %3, 1;\n\t"
      "@p2 tcgen05.mma.cta_group::1.kind::f16 [%0], [t2], b2, %3, 1;\n\t"
      "@p3 tcgen05.mma.cta_group::1.kind::f16 [%0], [t3], b3, %3, 1;\n\t"
      "@p4 tcgen05.mma.cta_group::1.kind::f16 [%0], [t4], b4, %3, 1;\n\t"
      "@p5 tcgen05.mma.cta_group::1.kind::f16 [%0], [t5], b5, %3, 1;\n\t"
      "@p6 tcgen05.mma.cta_group::1.kind::f16 [%0], [t6], b6, %3, 1;\n\t"
      "@p7 tcgen05.mma.cta_group::1.kind::f16 [%0], [t7], b7, %3, 1;\n\t"
      "@c1 tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%7];\n\t"
      "@c2 tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%8];\n\t"
      "@c3 tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%9];\n\t}" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(bstep), "r"(kmask), "r"(acc0), "r"(bar1), "r"(bar2),
      "r"(bar3)
      : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane
__device__ __forceinline__ void lf_tmem_ld32(uint32_t taddr, float (&x)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int k = 0; k < 32; k++) x[k] = __uint_as_float(r[k]);
}

__device__ __forceinline__ void lf_tmem_st32(uint32_t taddr, const float (&x)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(x[0])), "r"(__float_as_uint(x[1])), "r"(__float_as_uint(x[2])),
      "r"(__float_as_uint(x[3])), "r"(__float_as_uint(x[4])), "r"(__float_as_uint(x[5])),
      "r"(__float_as_uint(x[6])), "r"(__float_as_uint(x[7])), "r"(__float_as_uint(x[8])),
      "r"(__float_as_uint(x[9])), "r"(__float_as_uint(x[10])), "r"(__float_as_uint(x[11])),
      "r"(__float_as_uint(x[12])), "r"(__float_as_uint(x[13])), "r"(__float_as_uint(x[14])),
      "r"(__float_as_uint(x[15])), "r"(__float_as_uint(x[16])), "r"(__float_as_uint(x[17])),
      "r"(__float_as_uint(x[18])), "r"(__float_as_uint(x[19])), "r"(__float_as_uint(x[20])),
      "r"(__float_as_uint(x[21])), "r"(__float_as_uint(x[22])), "r"(__float_as_uint(x[23])),
      "r"(__float_as_uint(x[24])), "r"(__float_as_uint(x[25])), "r"(__float_as_uint(x[26])),
      "r"(__float_as_uint(x[27])), "r"(__float_as_uint(x[28])), "r"(__float_as_uint(x[29])),
      "r"(__float_as_uint(x[30])), "r"(__float_as_uint(x[31]))
      : "memory");
}

// 8 consecutive fp32 columns of this thread's TMEM lane: load (waits) and store
__device__ __forceinline__ void lf_tmem_ld8(uint32_t taddr, float (&x)[8]) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
               "tcgen05.wait::ld.sync.aligned;"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
#pragma unroll
  for (int k = 0; k < 8; k++) x[k] = __uint_as_float(r[k]);
}
__device__ __forceinline__ void lf_tmem_st8(uint32_t taddr, const float (&x)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(
                   taddr),
               "r"(__float_as_uint(x[0])), "r"(__float_as_uint(x[1])), "r"(__float_as_uint(x[2])),
               "r"(__float_as_uint(x[3])), "r"(__float_as_uint(x[4])), "r"(__float_as_uint(x[5])),
               "r"(__float_as_uint(x[6])), "r"(__float_as_uint(x[7]))
               : "memory");
}

// 4 consecutive 32-bit columns of this thread's TMEM lane
__device__ __forceinline__ void lf_tmem_st4(uint32_t taddr, uint32_t a, uint32_t b, uint32_t c,
                                            uint32_t d) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(a),
               "r"(b), "r"(c), "r"(d)
               : "memory");
}

__device__ __forceinline__ void lf_tmem_st16(uint32_t taddr, const uint32_t (&w)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]),
      "r"(w[8]), "r"(w[9]), "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]),
      "r"(w[15])
      : "memory");
}

// 16 consecutive 32-bit columns of this thread's TMEM lane; the load and
// its wait are one statement, so no use of r can move above the wait
__device__ __forceinline__ void lf_tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void lf_tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float lf_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// two fp32 -> packed bf16x2 / f16x2 (lo = first element), round to nearest even
template <int kF16>
__device__ __forceinline__ uint32_t lf_pack2(float lo, float hi) {
  uint32_t r;
  if (kF16)
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  else
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Shared-memory matrix descriptor, 128-byte swizzle (tcgen05 "version 1").
// start address, leading / stride byte offsets are in 16-byte units.
__device__ __forceinline__ uint64_t lf_sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFF) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor of kind::f16: fp32 accumulate, A/B bf16 (or f16),
// M = 128, N = n, A K-major, B K-major (b_mn = 0) or MN-major (b_mn = 1).
__device__ __forceinline__ uint32_t lf_idesc(int f16, int n, int b_mn) {
  uint32_t fmt = f16 ? 0u : 1u;
  return (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// Bits k (0..31) of the 32-column chunk starting at column `base` whose
// column lies in [lo, hi].
__device__ __forceinline__ uint32_t lf_range_bits(int lo, int hi, int base) {
  const int a = lo - base, z = hi - base;  // selects, no branches
  const uint32_t ge = a <= 0 ? 0xffffffffu : (a > 31 ? 0u : (0xffffffffu << a));
  const uint32_t le = z >= 31 ? 0xffffffffu : (z < 0 ? 0u : (0xffffffffu >> (31 - z)));
  return ge & le;
}

// A value the compiler must keep in a register (it may not re-read it from
// the kernel parameter bank at each use).
__device__ __forceinline__ int lf_reg(int x) {
  int y;
  asm volatile("mov.b32 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// TMEM load of 32 columns without waiting; the caller waits with
// lf_tmem_wait_ld_regs, which also pins the registers behind the wait.
__device__ __forceinline__ void lf_tmem_ld32_nowait(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}

// Orders the use of r after an earlier tcgen05.wait::ld (no instruction).
__device__ __forceinline__ void lf_tmem_pin_regs(uint32_t (&r)[32]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                 "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                 "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                 "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

__device__ __forceinline__ void lf_tmem_wait_ld_regs(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                 "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                 "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                 "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

// Gate before the first write of P (or O) of a tile: the previous P.V of
// the same softmax group must have finished reading P.  `pending` is the
// pv_done phase still to be observed, or -1.
struct LfPvGate {
  uint32_t bar;
  int pending;
  volatile int *abort_flag;
  int32_t *status;
  __device__ __forceinline__ bool pass() {
    if (pending < 0) return true;
    const bool ok = lf_wait_warp(bar, (uint32_t)pending, abort_flag, status, 10);
    pending = -1;
    return ok;
  }
};
