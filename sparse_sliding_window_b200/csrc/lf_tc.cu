// lf_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) forward of Longformer
// attention for sm_100a, bf16 or f16 inputs, fp32 accumulation.
//
// One kernel runs two kinds of work items, one item per CTA:
//
//  * BAND items: 128 query rows t0..t0+127 of one (b, h, residue rho).  A
//    head with dilation d is split into its d residue sub-sequences
//    rho, rho+d, ... ("gaps of size d": segmentfault page, section
//    扩张滑动窗口); in sub-sequence coordinates the window is a plain band of
//    radius r (causal: [t-r, t]), so the CTA walks only the key tiles that
//    intersect the band (page section 实现: only a fixed number of diagonals
//    of QK^T are computed).  The residue view is a TMA tensor map whose row
//    stride is d rows, so dilated heads need no gather.  After the band tiles
//    come the global-column tiles: the K_s/V_s rows of the sequence's global
//    tokens (compacted by lf_gather_kernel), minus the keys already inside
//    the row's window (the union of the glossary example), merged into the
//    same online softmax.  Global query rows are skipped (their output comes
//    from the global-row items); mask-0 rows get o = 0, lse = -inf.
//  * GLOBAL items: up to 128 global query rows (Q_g, compacted) against a
//    chunk of LF_TC_CHUNK_TILES key tiles of K_g / V_g (every valid key:
//    global attention sees the whole sequence, segmentfault page section
//    全局注意力).  Each writes an unnormalised partial (acc, max, sum) that
//    lf_combine_kernel merges (split-KV).
//
// Per CTA (192 threads, two CTAs per SM): warp 0 issues TMA loads (Q once,
// then K/V tiles into a 2-stage ring), warp 1 owns TMEM and issues the
// tcgen05.mma instructions, warps 2..5 (one TMEM lane = one query row per
// thread) run the softmax.  TMEM columns: S = QK^T tile [0,128), the O
// accumulator [128,192), P (bf16/f16, packed two per column) [192,256).
// Per tile:   MMA  S_t = Q K_t^T      -> commit s_full
//             SMX  read S_t, row max, rescale O if the max grew by more than
//                  2^8, P_t = exp2(S_t*scale*log2e - m), row sum, write P_t
//                                     -> arrive p_full
//             MMA  O += P_t V_t (A operand from TMEM) -> commit kv_empty
//             MMA  S_{t+1} = Q K_{t+1}^T -> commit s_full
// so the n x w score band never leaves the SM.  The two CTAs of an SM
// interleave their MMA and softmax phases.
//
// Every wait is bounded: after LF_WAIT_NS without progress the waiting
// thread records LF_ERR_DEVICE_TIMEOUT in the status word, raises the CTA's
// abort flag and leaves its loop; all roles meet at the final barrier and
// the TMEM columns are freed before the CTA exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <stdio.h>
#include <string.h>

#include <map>
#include <utility>
#include <vector>

#include "lf_tc.cuh"

#define LF_TC_THREADS 192
#define LF_TC_NS 3
#define LF_TC_MAX_MAPS 28
#define LF_TC_MAX_SEG 32
#define LF_WAIT_NS 1500000000ull

// TMEM column map
#define LF_TM_S 0
#define LF_TM_O 128
#define LF_TM_P 192
#define LF_TM_COLS 256

// shared memory map (bytes from the 1024-aligned base)
#define LF_SM_Q 0
#define LF_SM_K(s) (16384 + (s)*16384)
#define LF_SM_V(s) (16384 + LF_TC_NS * 16384 + (s)*16384)
#define LF_SM_BAR (16384 + 2 * LF_TC_NS * 16384)
#define LF_SMEM_BYTES (LF_SM_BAR + 256)

struct LfTcSeg {
  int h0, h1, d, rho, cnt, nqb, start, map;
};

struct LfTcParams {
  CUtensorMap maps[LF_TC_MAX_MAPS];
  LfDev dev;
  LfTcSeg seg[LF_TC_MAX_SEG];
  int nseg, per_batch, n_gitems, ngq, gbox;
  int map_kg, map_vg, map_qgc, map_ksc, map_vsc;
  int f16;
  void *o;
  float *lse;
  float *part_acc;
  float2 *part_ml;
};

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
// (this thread's own timeout, or another role's).
__device__ __noinline__ bool lf_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                     int32_t *status, int site) {
  uint64_t t0 = 0;
  for (uint32_t it = 0;; it++) {
    if (lf_mbar_try(bar, parity)) return true;
    if ((it & 255) == 255) {
      if (*abort_flag) return false;
      uint64_t now = lf_globaltimer();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > LF_WAIT_NS) {
        *abort_flag = 1;
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
// acquires the phase itself), and the verdict is made uniform before the
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

__device__ __forceinline__ void lf_tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]
__device__ __forceinline__ void lf_mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]
__device__ __forceinline__ void lf_mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc,
                                          uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane
__device__ __forceinline__ void lf_tmem_ld32(uint32_t taddr, float (&x)[32]) {
  uint32_t r[32];
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
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
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

__device__ __forceinline__ void lf_tmem_st16(uint32_t taddr, const uint32_t (&w)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]),
      "r"(w[8]), "r"(w[9]), "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]),
      "r"(w[15])
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
  int a = lo - base, z = hi - base;
  if (z < 0 || a > 31 || a > z) return 0u;
  a = max(a, 0);
  z = min(z, 31);
  const uint32_t upto = z == 31 ? 0xffffffffu : ((1u << (z + 1)) - 1u);
  return upto & ~((1u << a) - 1u);
}

// One pass over the 4 column chunks of a row's S tile (TMEM lane of this
// thread).  Columns whose bit in w is clear are treated as -inf.  Tracks the
// row max of the attended raw scores in mx; when write_p, also computes
// p = 2^(s * sl2 - m) into P (TMEM, packed bf16 / f16) and their sum lt.
// Chunks no lane of the warp attends are skipped (P written as zeros).
template <int kF16>
__device__ __forceinline__ void lf_p_chunk(uint32_t tl, int cc, float (&x)[32], float sl2,
                                           float mneg, float &lt) {
  uint32_t pw[16];
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int k = 0; k < 32; k += 2) {
    const float p0 = lf_ex2(fmaf(x[k], sl2, mneg));
    const float p1 = lf_ex2(fmaf(x[k + 1], sl2, mneg));
    s0 += p0;
    s1 += p1;
    pw[k / 2] = lf_pack2<kF16>(p0, p1);
  }
  lt += s0 + s1;
  lf_tmem_st16(tl + LF_TM_P + 16 * cc, pw);
}

__device__ __forceinline__ void lf_mask_chunk(float (&x)[32], uint32_t wc) {
  if (!__all_sync(0xffffffffu, wc == 0xffffffffu)) {
#pragma unroll
    for (int k = 0; k < 32; k++) x[k] = ((wc >> k) & 1u) ? x[k] : -INFINITY;
  }
}

__device__ __forceinline__ float lf_max32(const float (&x)[32]) {
  float a = fmaxf(x[0], x[1]), b = fmaxf(x[2], x[3]), c = fmaxf(x[4], x[5]), d = fmaxf(x[6], x[7]);
#pragma unroll
  for (int k = 8; k < 32; k += 4) {
    a = fmaxf(a, x[k]);
    b = fmaxf(b, x[k + 1]);
    c = fmaxf(c, x[k + 2]);
    d = fmaxf(d, x[k + 3]);
  }
  return fmaxf(fmaxf(a, b), fmaxf(c, d));
}

// 64 consecutive fp32 columns of this thread's TMEM lane (one wait)
__device__ __forceinline__ void lf_tmem_ld32x2(uint32_t taddr, float (&x)[32], float (&y)[32]) {
  uint32_t r[32], u[32];
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
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]),
        "=r"(u[7]), "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]),
        "=r"(u[13]), "=r"(u[14]), "=r"(u[15]), "=r"(u[16]), "=r"(u[17]), "=r"(u[18]),
        "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]), "=r"(u[24]),
        "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]),
        "=r"(u[31])
      : "r"(taddr + 32));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int k = 0; k < 32; k++) {
    x[k] = __uint_as_float(r[k]);
    y[k] = __uint_as_float(u[k]);
  }
}

// One pass over the 4 column chunks of a row's S tile (TMEM lane of this
// thread).  Columns whose bit in w is clear are treated as -inf.  Tracks the
// row max of the attended raw scores in mx; when write_p, also computes
// p = 2^(s * sl2 - m) into P (TMEM, packed bf16 / f16) and their sum lt.
// Chunks no lane of the warp attends are skipped (P written as zeros); two
// attended chunks are fetched with one TMEM wait.
// Gate before the first write of P (or O) of a tile: the previous tile's
// P.V must have finished reading P.  `pending` is the pv_done phase still
// to be observed, or -1.
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

template <int kF16>
__device__ __forceinline__ void lf_softmax_tile(uint32_t tl, const uint32_t (&w)[4], float sl2,
                                                float m, float &mx, float &lt, bool write_p,
                                                LfPvGate &gate) {
  const float mneg = m == -INFINITY ? 0.f : -m;
#pragma unroll
  for (int pp = 0; pp < 2; pp++) {
    const int c0 = 2 * pp, c1 = 2 * pp + 1;
    const bool a0 = __any_sync(0xffffffffu, w[c0] != 0u);
    const bool a1 = __any_sync(0xffffffffu, w[c1] != 0u);
    if (write_p && !(a0 && a1)) {
      gate.pass();
      uint32_t z[16];
#pragma unroll
      for (int k = 0; k < 16; k++) z[k] = 0u;
      if (!a0) lf_tmem_st16(tl + LF_TM_P + 16 * c0, z);
      if (!a1) lf_tmem_st16(tl + LF_TM_P + 16 * c1, z);
    }
    if (a0 && a1) {
      float x[32], y[32];
      lf_tmem_ld32x2(tl + LF_TM_S + 32 * c0, x, y);
      lf_mask_chunk(x, w[c0]);
      lf_mask_chunk(y, w[c1]);
      mx = fmaxf(mx, fmaxf(lf_max32(x), lf_max32(y)));
      if (write_p) {
        gate.pass();
        lf_p_chunk<kF16>(tl, c0, x, sl2, mneg, lt);
        lf_p_chunk<kF16>(tl, c1, y, sl2, mneg, lt);
      }
    } else if (a0 || a1) {
      const int c = a0 ? c0 : c1;
      float x[32];
      lf_tmem_ld32(tl + LF_TM_S + 32 * c, x);
      lf_mask_chunk(x, w[c]);
      mx = fmaxf(mx, lf_max32(x));
      if (write_p) {
        gate.pass();
        lf_p_chunk<kF16>(tl, c, x, sl2, mneg, lt);
      }
    }
  }
}

// ------------------------------------------------------------ the kernel

template <int kF16>
__global__ void __launch_bounds__(LF_TC_THREADS, 2)
    lf_tc_fwd_kernel(const __grid_constant__ LfTcParams P) {
  extern __shared__ __align__(1024) uint8_t lf_smem_raw[];
  // the dynamic shared window starts 1024-byte aligned (128-byte swizzled
  // TMA tiles need it); checked rather than padded, to fit two CTAs per SM
  const uint32_t sbase = lf_smem(lf_smem_raw);
  uint8_t *gbase = lf_smem_raw;
  if (sbase & 1023u) {
    if (threadIdx.x == 0) lf_set_status(P.dev.status, LF_ERR_UNSUPPORTED, 9000);
    return;
  }

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const LfDev &D = P.dev;
  const int n = D.n;

  // ---------------------------------------------------- decode work item
  bool gitem = (int)blockIdx.x < P.n_gitems;
  int b, h, d = 1, rho = 0, cnt = n, t0 = 0, mq, mk, mv, nband = 0, nglob = 0, kt0 = 0;
  int ng, qrow0;
  if (gitem) {
    int idx = blockIdx.x;
    const int c = idx % D.nch;
    idx /= D.nch;
    const int qt = idx % P.ngq;
    idx /= P.ngq;
    h = idx % D.H;
    b = idx / D.H;
    ng = D.binfo[(size_t)b * LF_BI_WORDS + LF_BI_NG];
    if (qt * LF_BQ >= ng) return;  // uniform: no global row in this tile
    qrow0 = qt * LF_BQ;
    kt0 = c * D.chunk_tiles;
    const int ktiles = (n + LF_BK - 1) / LF_BK;
    nband = min(D.chunk_tiles, ktiles - kt0);
    if (nband <= 0) return;
    mq = P.map_qgc;
    mk = P.map_kg;
    mv = P.map_vg;
  } else {
    int idx = blockIdx.x - P.n_gitems;
    b = idx / P.per_batch;
    int rem = idx - b * P.per_batch;
    int s = 0;
    while (s + 1 < P.nseg && rem >= P.seg[s + 1].start) s++;
    const LfTcSeg &sg = P.seg[s];
    rem -= sg.start;
    h = sg.h0 + rem / sg.nqb;
    t0 = (rem % sg.nqb) * LF_BQ;
    d = sg.d;
    rho = sg.rho;
    cnt = sg.cnt;
    mq = mk = mv = sg.map;  // q, k, v maps at map, map+1, map+2
    mk += 1;
    mv += 2;
    qrow0 = t0;
    nband = lf_band_tiles(D.r, D.causal);
    const int32_t *bi = D.binfo + (size_t)b * LF_BI_WORDS;
    ng = bi[LF_BI_NG];
    bool need = ng > 0;
    if (need && d == 1 && !D.causal) {
      // every global key inside every row's window: the band covers them
      const int tlast = min(t0 + LF_BQ - 1, cnt - 1);
      if (bi[LF_BI_GMIN] >= tlast - D.r && bi[LF_BI_GMAX] <= t0 + D.r) need = false;
    }
    nglob = need ? (ng + LF_BK - 1) / LF_BK : 0;
  }
  const int T = nband + nglob;
  const int tk0 = t0 - D.r;  // first key row of band tile 0 (sub-sequence coords)

  // ---------------------------------------------------- shared state
  const uint32_t bar = sbase + LF_SM_BAR;
  const uint32_t q_full = bar, s_full = bar + 8, p_full = bar + 16, o_full = bar + 24,
                 end_bar = bar + 32, pv_done = bar + 40;
  const uint32_t kv_full0 = bar + 48, kv_empty0 = bar + 48 + 8 * LF_TC_NS;
  uint32_t *tmem_slot = (uint32_t *)(gbase + LF_SM_BAR + 128);
  volatile int *abort_flag = (volatile int *)(gbase + LF_SM_BAR + 132);

  if (threadIdx.x == 0) {
    lf_mbar_init(q_full, 1);
    lf_mbar_init(s_full, 1);
    lf_mbar_init(p_full, 4);
    lf_mbar_init(o_full, 1);
    lf_mbar_init(end_bar, 1);
    lf_mbar_init(pv_done, 1);
    for (int s = 0; s < LF_TC_NS; s++) {
      lf_mbar_init(kv_full0 + 8 * s, 1);
      lf_mbar_init(kv_empty0 + 8 * s, 1);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     lf_smem(tmem_slot)),
                 "r"(LF_TM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  lf_tc_fence_before();
  __syncthreads();
  lf_tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ================================================== TMA producer
    if (lane == 0) {
      lf_mbar_expect_tx(q_full, 16384);
      lf_tma_load4(sbase + LF_SM_Q, &P.maps[mq], q_full, 0, qrow0, h, b);
      int issued = 0;
      for (int it = 0; it < T; it++) {
        const int s = it % LF_TC_NS;
        if (it >= LF_TC_NS &&
            !lf_wait(kv_empty0 + 8 * s, ((it / LF_TC_NS) & 1) ^ 1, abort_flag, D.status, 1))
          break;
        int row;
        const CUtensorMap *km, *vm;
        uint32_t bytes;
        if (it < nband) {
          row = gitem ? (kt0 + it) * LF_BK : tk0 + it * LF_BK;
          km = &P.maps[mk];
          vm = &P.maps[mv];
          bytes = 2 * 16384;
        } else {
          row = (it - nband) * LF_BK;
          km = &P.maps[P.map_ksc];
          vm = &P.maps[P.map_vsc];
          bytes = 2 * P.gbox * 128;
        }
        lf_mbar_expect_tx(kv_full0 + 8 * s, bytes);
        lf_tma_load4(sbase + LF_SM_K(s), km, kv_full0 + 8 * s, 0, row, h, b);
        lf_tma_load4(sbase + LF_SM_V(s), vm, kv_full0 + 8 * s, 0, row, h, b);
        issued = it + 1;
      }
      if (*abort_flag) {
        // let the copies already issued land before the CTA exits
        for (int it = max(0, issued - LF_TC_NS); it < issued; it++)
          lf_wait(kv_full0 + 8 * (it % LF_TC_NS), (it / LF_TC_NS) & 1, abort_flag, D.status, 2);
      }
    }
  } else if (warp == 1) {
    // ================================================== MMA issuer
    if (lane == 0) {
      // descriptors: start-address field (16-byte units) advanced per k-step
      const uint64_t dq = lf_sdesc(sbase + LF_SM_Q, 16, 1024);
      const uint64_t dk0 = lf_sdesc(sbase + LF_SM_K(0), 16, 1024);
      const uint64_t dv0 = lf_sdesc(sbase + LF_SM_V(0), 0, 1024);
      const uint32_t id_pv = lf_idesc(kF16, 64, 1), id_s = lf_idesc(kF16, LF_BK, 0);
      const int ngk = (ng + 15) / 16 * 16;  // global key tile width, multiple of 16
      auto issue_s = [&](int it) {
        const int s = it % LF_TC_NS;
        const uint64_t dk = dk0 + (uint64_t)(s * (16384 >> 4));
        const uint32_t id = it < nband ? id_s : lf_idesc(kF16, min(LF_BK, ngk - (it - nband) * LF_BK), 0);
#pragma unroll
        for (int k = 0; k < 4; k++) lf_mma_ss(tmem + LF_TM_S, dq + 2 * k, dk + 2 * k, id, k > 0);
      };
      auto issue_pv = [&](int it) {
        const int s = it % LF_TC_NS;
        const uint64_t dv = dv0 + (uint64_t)(s * (16384 >> 4));
        const int ksteps = it < nband ? 8 : min(LF_BK, ngk - (it - nband) * LF_BK) / 16;
#pragma unroll
        for (int k = 0; k < 8; k++)
          if (k < ksteps)
            lf_mma_ts(tmem + LF_TM_O, tmem + LF_TM_P + 8 * k, dv + 128 * k, id_pv, (it > 0 || k > 0));
      };
      bool ok = lf_wait_fast(q_full, 0, abort_flag, D.status, 3) &&
                lf_wait_fast(kv_full0, 0, abort_flag, D.status, 4);
      if (ok) {
        lf_tc_fence_after();
        issue_s(0);
        lf_tc_commit(s_full);
        for (int it = 0; it < T; it++) {
          // P(it) written and S(it) consumed by the softmax warps
          if (!lf_wait_fast(p_full, it & 1, abort_flag, D.status, 5)) break;
          lf_tc_fence_after();
          if (it + 1 < T) {
            // the next scores first: they only need the S columns, now free
            const int s2 = (it + 1) % LF_TC_NS;
            if (!lf_wait_fast(kv_full0 + 8 * s2, ((it + 1) / LF_TC_NS) & 1, abort_flag, D.status, 6))
              break;
            lf_tc_fence_after();
            issue_s(it + 1);
            lf_tc_commit(s_full);
          }
          issue_pv(it);
          lf_tc_commit(kv_empty0 + 8 * (it % LF_TC_NS));
          lf_tc_commit(pv_done);  // P columns free again, O up to date
          if (it + 1 == T) lf_tc_commit(o_full);
        }
      }
      // every MMA this thread issued has completed once end_bar flips
      lf_tc_commit(end_bar);
      lf_wait(end_bar, 0, abort_flag, D.status, 7);
    }
  } else {
    // ================================================== softmax warps
    const int quarter = warp & 3;
    const int q = quarter * 32 + lane;  // query row of the tile == TMEM lane
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const int32_t *mrow = D.mask + (size_t)b * n;
    int code = 0, pos = 0;
    bool active;
    if (gitem) {
      active = qrow0 + q < ng;
    } else {
      const int t = t0 + q;
      if (t < cnt) {
        pos = rho + t * d;
        code = mrow[pos];
      }
      active = (code == 1);
    }
    const int32_t *gl = D.gidx + (size_t)b * D.G;
    const float sl2 = D.scale_log2;
    const bool padded = D.binfo[(size_t)b * LF_BI_WORDS + LF_BI_NVALID] < n;
    // Global keys already in this row's window: positions [pos - r d, pos + r d]
    // (causal: up to pos) of the row's residue.  gidx is sorted, so they form
    // the index range [e_lo, e_hi) = [rank(pos - r d), rank(pos + r d + 1)),
    // filtered by residue.
    int e_lo = 0, e_hi = 0;
    if (!gitem && nglob > 0 && active) {
      const int32_t *gr = D.grank + (size_t)b * (n + 1);
      const int lo_pos = max(pos - D.r * d, 0);
      const int hi_pos = min((D.causal ? pos : pos + D.r * d) + 1, n);
      e_lo = gr[lo_pos];
      e_hi = gr[hi_pos];
    }
    float m_ref = -INFINITY, l = 0.f;
    bool alive = true;
    for (int it = 0; it < T && alive; it++) {
      if (!lf_wait_warp(s_full, it & 1, abort_flag, D.status, 8)) {
        alive = false;
        break;
      }
      lf_tc_fence_after();
      // ---- attend mask of row q over the tile's 128 columns (4 words)
      uint32_t w[4];
      if (it < nband) {
        const int kb = gitem ? (kt0 + it) * LF_BK : tk0 + it * LF_BK;
        int lo = 0, hi = LF_BK - 1;
        if (!gitem) lf_band_cols(q, it, D.r, D.causal, lo, hi);
        lo = max(lo, -kb);            // keys exist on [0, cnt)
        hi = min(hi, cnt - 1 - kb);
        if (!active) hi = -1;
#pragma unroll
        for (int cc = 0; cc < 4; cc++) w[cc] = lf_range_bits(lo, hi, 32 * cc);
        if (padded) {
#pragma unroll
          for (int cc = 0; cc < 4; cc++) {
            const int tk = kb + 32 * cc + lane;
            const bool ok = tk >= 0 && tk < cnt && mrow[rho + tk * d] != 0;
            w[cc] &= __ballot_sync(0xffffffffu, ok);
          }
        }
      } else {
        const int gb = (it - nband) * LF_BK;
        const int hi = active ? min(LF_BK - 1, ng - 1 - gb) : -1;
#pragma unroll
        for (int cc = 0; cc < 4; cc++) {
          uint32_t inwin = lf_range_bits(e_lo - gb, e_hi - 1 - gb, 32 * cc);
          if (d > 1) {
            const int e = gb + 32 * cc + lane;
            const bool res = e < ng && (gl[e] - rho) % d == 0;
            inwin &= __ballot_sync(0xffffffffu, res);
          }
          w[cc] = lf_range_bits(0, hi, 32 * cc) & ~inwin;
        }
      }
      // ---- probabilities of the tile -> P (TMEM).  Optimistic single pass
      // against the running reference m_ref; redone (rarely) with the tile's
      // own max when some row's max grew by more than 2^8.
      LfPvGate gate{pv_done, it > 0 ? ((it - 1) & 1) : -1, abort_flag, D.status};
      const bool any_bits = (w[0] | w[1] | w[2] | w[3]) != 0u;
      const bool single = __all_sync(0xffffffffu, m_ref != -INFINITY || !any_bits);
      float mx = -INFINITY, lt = 0.f;
      if (single) lf_softmax_tile<kF16>(tl, w, sl2, m_ref, mx, lt, true, gate);
      const bool grow = any_bits && (!single || mx * sl2 > m_ref + 8.f);
      if (__any_sync(0xffffffffu, grow)) {
        if (!single) {
          float dummy = 0.f;
          lf_softmax_tile<kF16>(tl, w, sl2, m_ref, mx, dummy, false, gate);  // max only
        }
        const float ms = mx * sl2;
        const bool need = any_bits && ms > m_ref + 8.f;
        const float m_new = need ? ms : m_ref;
        const float alpha = need ? lf_ex2(m_ref - m_new) : 1.f;
        l *= alpha;
        if (it > 0 && __any_sync(0xffffffffu, need)) {
          gate.pass();
#pragma unroll
          for (int half = 0; half < 2; half++) {
            float ov[32];
            lf_tmem_ld32(tl + LF_TM_O + 32 * half, ov);
#pragma unroll
            for (int k = 0; k < 32; k++) ov[k] *= alpha;
            lf_tmem_st32(tl + LF_TM_O + 32 * half, ov);
          }
        }
        m_ref = m_new;
        lt = 0.f;
        float mx2 = -INFINITY;
        lf_softmax_tile<kF16>(tl, w, sl2, m_ref, mx2, lt, true, gate);
      }
      l += lt;
      gate.pass();  // (no-op unless every chunk of the tile was skipped)
      lf_tmem_wait_st();
      lf_tc_fence_before();
      __syncwarp();
      if (lane == 0) lf_mbar_arrive(p_full);
    }
    // ---- epilogue
    if (alive && lf_wait_warp(o_full, 0, abort_flag, D.status, 9)) {
      lf_tc_fence_after();
      float ov[64];
      {
        float a[32], c2[32];
        lf_tmem_ld32(tl + LF_TM_O, a);
        lf_tmem_ld32(tl + LF_TM_O + 32, c2);
#pragma unroll
        for (int k = 0; k < 32; k++) {
          ov[k] = a[k];
          ov[32 + k] = c2[k];
        }
      }
      const size_t bh = (size_t)b * D.H + h;
      if (gitem) {
        if (active) {
          const int e = qrow0 + q;
          const size_t pi = (bh * D.G + e) * D.nch + (kt0 / D.chunk_tiles);
          float4 *dst = reinterpret_cast<float4 *>(P.part_acc + pi * LF_HD);
#pragma unroll
          for (int k = 0; k < 16; k++)
            dst[k] = make_float4(ov[4 * k], ov[4 * k + 1], ov[4 * k + 2], ov[4 * k + 3]);
          P.part_ml[pi] = make_float2(m_ref, l);
        }
      } else if (t0 + q < cnt && code != 2) {
        const size_t orow = bh * n + pos;
        uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(P.o) + orow * LF_HD);
        const float inv = code == 1 ? 1.f / l : 0.f;
#pragma unroll
        for (int k = 0; k < 8; k++) {
          uint4 v;
          v.x = lf_pack2<kF16>(ov[8 * k + 0] * inv, ov[8 * k + 1] * inv);
          v.y = lf_pack2<kF16>(ov[8 * k + 2] * inv, ov[8 * k + 3] * inv);
          v.z = lf_pack2<kF16>(ov[8 * k + 4] * inv, ov[8 * k + 5] * inv);
          v.w = lf_pack2<kF16>(ov[8 * k + 6] * inv, ov[8 * k + 7] * inv);
          dst[k] = v;
        }
        if (P.lse) P.lse[orow] = code == 1 ? (m_ref + __log2f(l)) * LF_LN2 : -INFINITY;
      }
    }
  }

  // ---------------------------------------------------- teardown
  lf_tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    lf_tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(LF_TM_COLS)
                 : "memory");
  }
}

// ------------------------------------------------------------ gather / combine

// Compact, per (b, h), the Q_g rows (global queries) and the K_s / V_s rows
// (global keys for the band's global columns) of the global tokens; rows
// past the sequence's global count are zero.
template <typename T>
__global__ void __launch_bounds__(256)
    lf_gather_kernel(LfDev D, const T *qg, const T *ks, const T *vs, T *qg_c, T *ks_c, T *vs_c,
                     int Ga, int Gka) {
  const int lane = threadIdx.x & 31;
  const long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const long long total = (long long)D.B * D.H * Gka;
  if (w >= total) return;
  const int e = (int)(w % Gka);
  const long long bh = w / Gka;
  const int b = (int)(bh / D.H);
  const int ng = D.binfo[(size_t)b * LF_BI_WORDS + LF_BI_NG];
  uint32_t q = 0, k = 0, v = 0;
  if (e < ng) {
    const int g = D.gidx[(size_t)b * D.G + e];
    const size_t src = ((size_t)bh * D.n + g) * LF_HD + 2 * lane;
    q = *reinterpret_cast<const uint32_t *>(qg + src);
    k = *reinterpret_cast<const uint32_t *>(ks + src);
    v = *reinterpret_cast<const uint32_t *>(vs + src);
  }
  if (e < Ga) *reinterpret_cast<uint32_t *>(qg_c + ((size_t)bh * Ga + e) * LF_HD + 2 * lane) = q;
  *reinterpret_cast<uint32_t *>(ks_c + ((size_t)bh * Gka + e) * LF_HD + 2 * lane) = k;
  *reinterpret_cast<uint32_t *>(vs_c + ((size_t)bh * Gka + e) * LF_HD + 2 * lane) = v;
}

// Merge the split-KV partials of every global row: o = sum_c acc_c 2^(m_c-m)
// / sum_c l_c 2^(m_c-m), lse = (m + log2 sum) ln 2.
template <typename T>
__global__ void __launch_bounds__(256)
    lf_combine_kernel(LfDev D, const float *part_acc, const float2 *part_ml, T *o, float *lse) {
  const int lane = threadIdx.x & 31;
  const long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (w >= (long long)D.B * D.H * D.G) return;
  const int e = (int)(w % D.G);
  const long long bh = w / D.G;
  const int b = (int)(bh / D.H);
  const int ng = D.binfo[(size_t)b * LF_BI_WORDS + LF_BI_NG];
  if (e >= ng) return;
  const size_t base = ((size_t)bh * D.G + e) * D.nch;
  float m = -INFINITY;
  for (int c = 0; c < D.nch; c++) m = fmaxf(m, part_ml[base + c].x);
  float L = 0.f, a0 = 0.f, a1 = 0.f;
  for (int c = 0; c < D.nch; c++) {
    const float2 ml = part_ml[base + c];
    if (ml.y == 0.f) continue;
    const float f = exp2f(ml.x - m);
    L += ml.y * f;
    const float2 acc = *reinterpret_cast<const float2 *>(part_acc + (base + c) * LF_HD + 2 * lane);
    a0 += acc.x * f;
    a1 += acc.y * f;
  }
  const int g = D.gidx[(size_t)b * D.G + e];
  const size_t orow = (size_t)bh * D.n + g;
  LfIo<T>::st2(o + orow * LF_HD + 2 * lane, a0 / L, a1 / L);
  if (lse && lane == 0) lse[orow] = (m + log2f(L)) * LF_LN2;
}

// ------------------------------------------------------------ host side

static PFN_cuTensorMapEncodeTiled lf_encode_fn() {
  static PFN_cuTensorMapEncodeTiled fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled)p;
  }
  return fn;
}

// 4-D tiled map over rows of 64 elements: dims {64, rows, H, B}; strides in
// bytes {row_stride, head_stride, batch_stride}; box {64, box_rows, 1, 1}.
static bool lf_make_map(CUtensorMap *m, int f16, const void *base, uint64_t rows, uint64_t H,
                        uint64_t B, uint64_t row_stride, uint64_t head_stride,
                        uint64_t batch_stride, uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled enc = lf_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {64, rows, H, B};
  cuuint64_t strides[3] = {row_stride, head_stride, batch_stride};
  cuuint32_t box[4] = {64, box_rows, 1, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = enc(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                   const_cast<void *>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static bool lf_tc_attr_done[2] = {false, false};

int lf_tc_fwd(const LfLaunch &L, const LfTcArgs &a, char *err, size_t errlen) {
  const LfDev &D = L.dev;
  const int f16 = L.dtype == LF_F16 ? 1 : 0;
  LfTcParams P;  // host staging; the launch copies the parameter block
  memset(&P, 0, sizeof(P));
  P.dev = D;
  P.f16 = f16;
  const uint64_t n = D.n, H = D.H, B = D.B, rowb = 128;
  int nmaps = 0;
  // segments: runs of heads with equal dilation x residues
  std::map<std::pair<int, int>, int> rmap;
  int nseg = 0, start = 0;
  for (int h0 = 0; h0 < D.H;) {
    int h1 = h0 + 1;
    while (h1 < D.H && D.dil[h1] == D.dil[h0]) h1++;
    const int d = D.dil[h0];
    for (int rho = 0; rho < d; rho++) {
      const int cnt = lf_sub_len(D.n, d, rho);
      const int nqb = (cnt + LF_BQ - 1) / LF_BQ;
      if (nqb == 0) continue;
      auto key = std::make_pair(d, rho);
      if (!rmap.count(key)) {
        if (nmaps + 3 > LF_TC_MAX_MAPS - 5) goto too_big;
        const char *srcs[3] = {(const char *)a.qs, (const char *)a.ks, (const char *)a.vs};
        for (int k = 0; k < 3; k++)
          if (!lf_make_map(&P.maps[nmaps + k], f16, srcs[k] + rho * rowb, cnt, H, B, d * rowb,
                           n * rowb, H * n * rowb, LF_BQ)) {
            snprintf(err, errlen, "tensor map encode failed (d=%d, rho=%d)", d, rho);
            return LF_ERR_CUDA;
          }
        rmap[key] = nmaps;
        nmaps += 3;
      }
      if (nseg >= LF_TC_MAX_SEG) goto too_big;
      P.seg[nseg] = LfTcSeg{h0, h1, d, rho, cnt, nqb, start, rmap[key]};
      start += (h1 - h0) * nqb;
      nseg++;
    }
    h0 = h1;
  }
  P.nseg = nseg;
  P.per_batch = start;
  {
    // global-row (split-KV) maps and the compacted global-token rows
    const int G = D.G;
    const size_t eb = 2;
    const int Ga = L.ws.G, Gka = L.ws.Gk;
    char *qg_c = L.ws_base + L.ws.qg_c, *ks_c = L.ws_base + L.ws.ks_c, *vs_c = L.ws_base + L.ws.vs_c;
    P.map_kg = nmaps;
    P.map_vg = nmaps + 1;
    P.map_qgc = nmaps + 2;
    P.map_ksc = nmaps + 3;
    P.map_vsc = nmaps + 4;
    P.gbox = std::min(Gka, LF_BK);
    bool ok = lf_make_map(&P.maps[nmaps], f16, a.kg, n, H, B, rowb, n * rowb, H * n * rowb, LF_BK) &&
              lf_make_map(&P.maps[nmaps + 1], f16, a.vg, n, H, B, rowb, n * rowb, H * n * rowb, LF_BK) &&
              lf_make_map(&P.maps[nmaps + 2], f16, qg_c, Ga, H, B, rowb, Ga * rowb, H * Ga * rowb, LF_BQ) &&
              lf_make_map(&P.maps[nmaps + 3], f16, ks_c, Gka, H, B, rowb, Gka * rowb, H * Gka * rowb, P.gbox) &&
              lf_make_map(&P.maps[nmaps + 4], f16, vs_c, Gka, H, B, rowb, Gka * rowb, H * Gka * rowb, P.gbox);
    if (!ok) {
      snprintf(err, errlen, "tensor map encode failed (global maps)");
      return LF_ERR_CUDA;
    }
    nmaps += 5;
    P.ngq = (G + LF_BQ - 1) / LF_BQ;
    P.n_gitems = G > 0 ? D.B * D.H * P.ngq * D.nch : 0;
    P.o = a.o;
    P.lse = a.lse;
    P.part_acc = (float *)(L.ws_base + L.ws.part_acc);
    P.part_ml = (float2 *)(L.ws_base + L.ws.part_ml);
    (void)eb;
    if (G > 0) {
      const long long rows = (long long)D.B * D.H * Gka;
      const unsigned grid = (unsigned)((rows + 7) / 8);
      if (f16)
        lf_gather_kernel<__half><<<grid, 256, 0, L.stream>>>(
            D, (const __half *)a.qg, (const __half *)a.ks, (const __half *)a.vs, (__half *)qg_c,
            (__half *)ks_c, (__half *)vs_c, Ga, Gka);
      else
        lf_gather_kernel<__nv_bfloat16><<<grid, 256, 0, L.stream>>>(
            D, (const __nv_bfloat16 *)a.qg, (const __nv_bfloat16 *)a.ks,
            (const __nv_bfloat16 *)a.vs, (__nv_bfloat16 *)qg_c, (__nv_bfloat16 *)ks_c,
            (__nv_bfloat16 *)vs_c, Ga, Gka);
      lf_launches_add(1);
    }
  }
  {
    void (*kern)(const LfTcParams) = f16 ? lf_tc_fwd_kernel<1> : lf_tc_fwd_kernel<0>;
    if (!lf_tc_attr_done[f16]) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           LF_SMEM_BYTES);
      if (e != cudaSuccess) {
        snprintf(err, errlen, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        return LF_ERR_CUDA;
      }
      lf_tc_attr_done[f16] = true;
    }
    const long long items = (long long)P.n_gitems + (long long)D.B * P.per_batch;
    if (a.ev_start && a.ev_stop) cudaEventRecord(a.ev_start, L.stream);
    kern<<<(unsigned)items, LF_TC_THREADS, LF_SMEM_BYTES, L.stream>>>(P);
    lf_launches_add(1);
    if (a.ev_start && a.ev_stop) cudaEventRecord(a.ev_stop, L.stream);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
      snprintf(err, errlen, "tensor-core forward launch: %s", cudaGetErrorString(e));
      return LF_ERR_CUDA;
    }
  }
  if (D.G > 0) {
    const long long rows = (long long)D.B * D.H * D.G;
    const unsigned grid = (unsigned)((rows + 7) / 8);
    if (f16)
      lf_combine_kernel<__half><<<grid, 256, 0, L.stream>>>(
          D, (const float *)P.part_acc, (const float2 *)P.part_ml, (__half *)a.o, a.lse);
    else
      lf_combine_kernel<__nv_bfloat16><<<grid, 256, 0, L.stream>>>(
          D, (const float *)P.part_acc, (const float2 *)P.part_ml, (__nv_bfloat16 *)a.o, a.lse);
    lf_launches_add(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
      snprintf(err, errlen, "combine launch: %s", cudaGetErrorString(e));
      return LF_ERR_CUDA;
    }
  }
  return LF_OK;

too_big:
  // more (dilation, residue) views than one parameter block holds
  snprintf(err, errlen, "tensor-core path: too many distinct dilation residues (sum of distinct "
                        "dilations must stay <= %d)", (LF_TC_MAX_MAPS - 5) / 3);
  return LF_ERR_UNSUPPORTED;
}
