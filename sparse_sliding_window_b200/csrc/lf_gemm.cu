// lf_gemm.cu -- the projections around the attention (include/lf_proj.h) as
// one tcgen05 GEMM kernel for sm_100a: Y = A W^T + bias, bf16 / f16 in,
// fp32 accumulation in TMEM, one rounding to the dtype on the way out.
//
//   * input projections (segmentfault page, section 全局注意力的线性投影:
//     separate projection sets Q_s, K_s, V_s and Q_g, K_g, V_g): A = hidden
//     states [B, n, d_model]; the epilogue splits the output features into
//     projections and heads and writes each 64-wide head slice straight into
//     the attention layout [B, H, n, 64].  Q_g is needed only at the global
//     tokens: those rows are gathered first (lf_rows_gather_kernel) and the
//     epilogue scatters the results back to their positions.
//   * output projection: A = the attention output [B, H, n, 64] read through
//     a 4-D tensor map whose k-step is one head, so the heads are
//     concatenated by the loads themselves; plain [B, n, d_model] out.
//
// Persistent, one CTA of 192 threads per SM, output tiles of 128 rows x 256
// features (128 when 256-wide tiles would leave SMs idle), the reduction in
// k-steps of 64:
//   warp 0  TMA producer: per k-step a 128x64 tile of A and a 256x64 tile of
//           W (128-byte swizzle, K-major) into a 4-stage ring (48 KB each)
//   warp 1  MMA issuer (owns TMEM): four K = 16 tcgen05.mma (M = 128,
//           N = 256) per k-step into one of two 256-column fp32 accumulators
//   warps 2-5  epilogue: per 64-column box, TMEM -> registers -> + bias ->
//           dtype -> shared memory in the 128-byte swizzle layout -> one TMA
//           store (two staging boxes alternate); it frees the accumulator for
//           the tile after next, so the epilogue of one tile overlaps the
//           main loop of the next.  Gathered rows (Q_g) are scattered to their
//           positions with plain stores instead.
// Tiles go row-block-major, feature-block fastest, so the CTAs running at
// one time share their A tiles in L2.  No TMA multicast is used.
//
// Every mbarrier wait is bounded (lf_wait*): on expiry the kernel records
// LF_ERR_DEVICE_TIMEOUT in the status word, lets the copies and MMAs it
// issued land, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <cub/block/block_scan.cuh>

#include "lf_common.cuh"
#include "lf_proj.h"
#include "lf_ptx.cuh"
#include "lf_tc.cuh"

#define LG_BM 128
#define LG_BK 64
#define LG_NS 4
#define LG_THREADS 192
#define LG_A_BYTES (LG_BM * LG_BK * 2)
#define LG_MAX_OUT 8
// per output-tile width kBN (256, or 128 when the 256-wide tiles would leave
// SMs idle): stage = A tile + W tile; then two 128 x 64 output staging boxes
// (16 KB each) and the barriers
template <int kBN> struct LgLayout {
  static constexpr int B_BYTES = kBN * LG_BK * 2;
  static constexpr int STAGE = LG_A_BYTES + B_BYTES;
  static constexpr int STG = LG_NS * STAGE;
  static constexpr int BAR = STG + 2 * LG_BM * 64 * 2;
  static constexpr int SMEM = BAR + 1024;
  static_assert(SMEM <= 232448, "shared memory per CTA");
};

int lf_record_error(int code, const char *msg);

struct LgParams {
  CUtensorMap map_a;  // mode 0: {K, L, B} box {64, 128, 1}; mode 1: {64, L, H, B} box {64, 128, 1, 1}
  CUtensorMap map_b;  // W [N, K]: {K, N} box {64, 256}
  CUtensorMap map_out[LG_MAX_OUT];  // stores: head split {64, Lout, H, B} / plain {N, L, B}, box 64 x 128
  int mode;           // 0: A rows of K elements; 1: A = heads [B, H, L, 64], k-step = head
  int B, L, K, N;     // L: rows of A per sequence
  int ksteps, mblk, nblk, tiles;
  int out_mode;       // 0: head split into outs[p] [B, H, Lout, 64]; 1: plain [B, L, N]
  int H, Lout;
  const uint16_t *bias;     // [N] or null
  void *outs[LG_MAX_OUT];   // out_mode 0: one per projection; out_mode 1: outs[0] = y
  const int32_t *row_map;   // [B, L]: output row of A row r, or null (identity)
  const int32_t *row_count; // [B]: valid A rows per sequence, or null (all L)
  int32_t *status;
  int wait_us;
};

// Four K = 16 MMAs over a 64-wide k-step (K-major, 128-byte swizzle: each
// descriptor advances 32 bytes per step), the first accumulating iff acc,
// then a commit to `bar`.
__device__ __forceinline__ void lg_mma_k64(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                           uint32_t acc, uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e, pa;\n\t.reg .b64 a1, a2, a3, b1, b2, b3;\n\t"
      "add.s64 a1, %1, 2;\n\tadd.s64 a2, %1, 4;\n\tadd.s64 a3, %1, 6;\n\t"
      "add.s64 b1, %2, 2;\n\tadd.s64 b2, %2, 4;\n\tadd.s64 b3, %2, 6;\n\t"
      "setp.ne.b32 pa, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, pa;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %3, 1;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a2, b2, %3, 1;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a3, b3, %3, 1;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%5];\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void lg_tma2(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c0,
                                        int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

// TMA stores of one 128-row x 64-column box from shared memory (bulk group)
__device__ __forceinline__ void lg_store4(const CUtensorMap *map, uint32_t src, int c0, int c1, int c2,
                                          int c3) {
  asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%1, %2, %3, %4}], [%5];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(src)
               : "memory");
}
__device__ __forceinline__ void lg_store3(const CUtensorMap *map, uint32_t src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(c2), "r"(src)
               : "memory");
}

__device__ __forceinline__ void lg_tma3(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c0,
                                        int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

struct LgTile {
  int b, mb, nb;
};
__device__ __forceinline__ LgTile lg_tile(const LgParams &P, int tile) {
  LgTile t;
  t.nb = tile % P.nblk;
  const int rest = tile / P.nblk;
  t.mb = rest % P.mblk;
  t.b = rest / P.mblk;
  return t;
}

template <int kF16, int kBN>
__global__ void __launch_bounds__(LG_THREADS, 1) lf_gemm_kernel(const __grid_constant__ LgParams P) {
  using Lay = LgLayout<kBN>;
  extern __shared__ __align__(1024) uint8_t lg_smem_raw[];
  const uint32_t sbase = lf_smem(lg_smem_raw);
  if (sbase & 1023u) {  // 128-byte swizzled tiles need a 1024-byte aligned window
    if (threadIdx.x == 0) lf_set_status(P.status, LF_ERR_UNSUPPORTED, 9100);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar = sbase + Lay::BAR;
  const uint32_t full0 = bar, empty0 = bar + 8 * LG_NS, acc_full0 = bar + 16 * LG_NS,
                 acc_empty0 = acc_full0 + 16, end_bar = acc_full0 + 32;
  uint32_t *tmem_slot = (uint32_t *)(lg_smem_raw + Lay::BAR + 512);
  volatile int *abort_flag = (volatile int *)(lg_smem_raw + Lay::BAR + 520);  // [2]: flag, wait limit
  if (threadIdx.x == 0) {
    for (int s = 0; s < LG_NS; s++) {
      lf_mbar_init(full0 + 8 * s, 1);
      lf_mbar_init(empty0 + 8 * s, 1);
    }
    for (int i = 0; i < 2; i++) {
      lf_mbar_init(acc_full0 + 8 * i, 1);
      lf_mbar_init(acc_empty0 + 8 * i, 4);  // one arrival per epilogue warp
    }
    lf_mbar_init(end_bar, 1);
    abort_flag[0] = 0;
    abort_flag[1] = P.wait_us;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     lf_smem(tmem_slot)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  lf_tc_fence_before();
  __syncthreads();
  lf_tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // launched as a programmatic dependent of the row gather (when rows are
  // selected): its outputs are read only after it has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == 0) {
    // ================================================== TMA producer
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < P.tiles && ok; tile += gridDim.x) {
        const LgTile t = lg_tile(P, tile);
        for (int ks = 0; ks < P.ksteps; ks++, g++) {
          const int s = g % LG_NS;
          if (g >= LG_NS &&
              !lf_wait_fast(empty0 + 8 * s, ((g / LG_NS) & 1) ^ 1, abort_flag, P.status, 41)) {
            ok = false;
            break;
          }
          const uint32_t sa = sbase + s * Lay::STAGE, sb = sa + LG_A_BYTES;
          lf_mbar_expect_tx(full0 + 8 * s, Lay::STAGE);
          if (P.mode == 0)
            lg_tma3(sa, &P.map_a, full0 + 8 * s, ks * LG_BK, t.mb * LG_BM, t.b);
          else
            lf_tma_load4(sa, &P.map_a, full0 + 8 * s, 0, t.mb * LG_BM, ks, t.b);
          lg_tma2(sb, &P.map_b, full0 + 8 * s, ks * LG_BK, t.nb * kBN);
        }
      }
      if (*abort_flag) {
        // let the copies already issued land before the CTA exits
        for (int i = max(0, g - LG_NS); i < g; i++)
          lf_wait_drain(full0 + 8 * (i % LG_NS), (i / LG_NS) & 1, P.status, 42);
      }
    }
  } else if (warp == 1) {
    // ================================================== MMA issuer
    const uint32_t idesc = lf_idesc(kF16, kBN, 0);
    int g = 0, it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < P.tiles && ok; tile += gridDim.x, it++) {
      const int buf = it & 1;
      // the epilogue has read this accumulator's previous tile
      if (it >= 2 &&
          !lf_wait_warp(acc_empty0 + 8 * buf, ((it >> 1) & 1) ^ 1, abort_flag, P.status, 43)) {
        ok = false;
        break;
      }
      lf_tc_fence_after();
      for (int ks = 0; ks < P.ksteps; ks++, g++) {
        const int s = g % LG_NS;
        if (!lf_wait_warp(full0 + 8 * s, (g / LG_NS) & 1, abort_flag, P.status, 44)) {
          ok = false;
          break;
        }
        lf_tc_fence_after();
        const uint32_t sa = sbase + s * Lay::STAGE;
        lg_mma_k64(tmem + buf * kBN, lf_sdesc(sa, 16, 1024), lf_sdesc(sa + LG_A_BYTES, 16, 1024),
                   idesc, ks > 0 ? 1u : 0u, empty0 + 8 * s);
      }
      if (ok) lf_commit_w(acc_full0 + 8 * buf);
    }
    // every MMA issued has completed once end_bar flips (also after an
    // abort: TMEM is freed after this)
    lf_commit_w(end_bar);
    lf_wait_drain(end_bar, 0, P.status, 45);
    __syncwarp();
  } else {
    // ================================================== epilogue warps 2..5
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31 (warps 4, 5, 2, 3)
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int hw = P.H * LF_HD;  // features per projection (head split)
    const bool issuer = warp == 2 && lane == 0;  // issues the TMA stores
    int it = 0, nstore = 0;
    for (int tile = blockIdx.x; tile < P.tiles; tile += gridDim.x, it++) {
      const int buf = it & 1;
      if (!lf_wait_warp(acc_full0 + 8 * buf, (it >> 1) & 1, abort_flag, P.status, 46)) break;
      lf_tc_fence_after();
      const LgTile t = lg_tile(P, tile);
      const int r = t.mb * LG_BM + row;  // row of A within sequence t.b
      const int nvalid = P.row_count ? P.row_count[t.b] : P.L;
      const bool valid = r < nvalid && r < P.L;
      const int orow = valid ? (P.row_map ? P.row_map[(size_t)t.b * P.L + r] : r) : 0;
      const uint32_t tacc = tmem + lane_off + buf * kBN;
      // the tile in four 64-column boxes (one head of one projection each in
      // the head split), each in two 32-column TMEM loads
      for (int hb = 0; hb < kBN / 64; hb++) {
        const int n0 = t.nb * kBN + 64 * hb;
        uint32_t x[2][32];
        lf_tmem_ld32_nowait(tacc + 64 * hb, x[0]);
        lf_tmem_ld32_nowait(tacc + 64 * hb + 32, x[1]);
        lf_tmem_wait_ld_regs(x[0]);
        lf_tmem_pin_regs(x[1]);
        if (hb == kBN / 64 - 1) {
          // every column of the accumulator is in registers: the MMA warp
          // may start the tile after next in it
          lf_tc_fence_before();
          __syncwarp();
          if (lane == 0) lf_mbar_arrive(acc_empty0 + 8 * buf);
        }
        uint32_t pk[32];
#pragma unroll
        for (int hf = 0; hf < 2; hf++) {
          float bv[32];
          if (P.bias) {
            const uint4 *bp = reinterpret_cast<const uint4 *>(P.bias + n0 + 32 * hf);
#pragma unroll
            for (int q = 0; q < 4; q++) {
              const uint4 u = __ldg(bp + q);
              const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
              for (int e = 0; e < 4; e++) {
                if (kF16) {
                  const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w4[e]));
                  bv[8 * q + 2 * e] = f.x;
                  bv[8 * q + 2 * e + 1] = f.y;
                } else {
                  bv[8 * q + 2 * e] = __uint_as_float(w4[e] << 16);
                  bv[8 * q + 2 * e + 1] = __uint_as_float(w4[e] & 0xffff0000u);
                }
              }
            }
          } else {
#pragma unroll
            for (int k = 0; k < 32; k++) bv[k] = 0.f;
          }
#pragma unroll
          for (int k = 0; k < 16; k++)
            pk[16 * hf + k] = lf_pack2<kF16>(__uint_as_float(x[hf][2 * k]) + bv[2 * k],
                                             __uint_as_float(x[hf][2 * k + 1]) + bv[2 * k + 1]);
        }
        if (P.row_map) {
          // selected rows: scattered to their positions, 128 bytes per row
          if (valid) {
            const int p = n0 / hw, hn = n0 - p * hw, h = hn / LF_HD;
            uint4 *d4 = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(P.outs[p]) +
                                                  (((size_t)t.b * P.H + h) * P.Lout + orow) * LF_HD);
#pragma unroll
            for (int q = 0; q < 8; q++) d4[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
          continue;
        }
        // staged in shared memory in the 128-byte swizzle layout, then one
        // TMA store of the 128 x 64 box (rows past the tensor are clipped)
        const int sb = nstore & 1;
        const uint32_t stg = sbase + Lay::STG + sb * (LG_BM * 128);
        if (issuer && nstore >= 2)
          asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");  // box nstore-2 read out
        asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll
        for (int q = 0; q < 8; q++) {
          const uint32_t a = stg + row * 128 + ((q ^ (row & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(pk[4 * q]),
                       "r"(pk[4 * q + 1]), "r"(pk[4 * q + 2]), "r"(pk[4 * q + 3])
                       : "memory");
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (issuer) {
          if (P.out_mode == 0) {
            const int p = n0 / hw, hn = n0 - p * hw, h = hn / LF_HD;
            lg_store4(&P.map_out[p], stg, 0, t.mb * LG_BM, h, t.b);
          } else {
            lg_store3(&P.map_out[0], stg, n0, t.mb * LG_BM, t.b);
          }
          asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
        nstore++;
      }
    }
    // the stores must be complete (not only read out) before the kernel ends
    if (issuer) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }

  // ---------------------------------------------------- teardown
  lf_tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    lf_tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512)
                 : "memory");
  }
}

// One block per sequence b: the positions t with mask[b, t] == code in
// ascending order (the first max_rows of them) into rows[b, .], their number
// into count[b] (more than max_rows: LF_ERR_DEVICE_INPUT in the status
// word), and their hidden states x[b, t, :] into xs[b, r, :].
template <typename T>
__global__ void __launch_bounds__(1024)
    lf_rows_gather_kernel(const int32_t *mask, int n, int code, int max_rows, const T *x, int K,
                          int32_t *rows, int32_t *count, T *xs, int32_t *status) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  typedef cub::BlockScan<int, 1024> Scan;
  __shared__ typename Scan::TempStorage tmp;
  __shared__ int s_total;
  const int b = blockIdx.x, tid = threadIdx.x;
  const int32_t *m = mask + (size_t)b * n;
  const int per = (n + 1023) / 1024, s = tid * per, e = min(n, s + per);
  int c = 0;
  for (int i = s; i < e; i++) c += m[i] == code;
  int off, total;
  Scan(tmp).ExclusiveSum(c, off, total);
  if (tid == 0) s_total = total;
  for (int i = s; i < e; i++)
    if (m[i] == code) {
      if (off < max_rows) rows[(size_t)b * max_rows + off] = i;
      off++;
    }
  __syncthreads();
  const int cnt = min(s_total, max_rows);
  if (tid == 0) {
    count[b] = cnt;
    if (s_total > max_rows) lf_set_status(status, LF_ERR_DEVICE_INPUT, 4000000 + b);
  }
  __syncthreads();  // rows[] written
  // copy the selected rows, 16 bytes per thread per step
  const int per_row = K * (int)sizeof(T) / 16;
  for (int idx = tid; idx < cnt * per_row; idx += blockDim.x) {
    const int rr = idx / per_row, q = idx - rr * per_row;
    const int tpos = rows[(size_t)b * max_rows + rr];
    const uint4 *src = reinterpret_cast<const uint4 *>(x + ((size_t)b * n + tpos) * K) + q;
    uint4 *dst = reinterpret_cast<uint4 *>(xs + ((size_t)b * max_rows + rr) * K) + q;
    *dst = *src;
  }
}

// ------------------------------------------------------------ host side

static thread_local cudaEvent_t g_pev_start = nullptr, g_pev_stop = nullptr;

extern "C" int lf_proj_set_timing_events(void *ev_start, void *ev_stop) {
  g_pev_start = (cudaEvent_t)ev_start;
  g_pev_stop = (cudaEvent_t)ev_stop;
  return LF_OK;
}

static PFN_cuTensorMapEncodeTiled lg_encode_fn() {
  static PFN_cuTensorMapEncodeTiled fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled)p;
  }
  return fn;
}

// rank-r tiled map, innermost dimension first; 128-byte swizzle
static bool lg_make_map(CUtensorMap *m, int f16, const void *base, int rank, const cuuint64_t *dims,
                        const cuuint64_t *strides, const cuuint32_t *box) {
  PFN_cuTensorMapEncodeTiled enc = lg_encode_fn();
  if (!enc) return false;
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                   rank, const_cast<void *>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static size_t lg_align(size_t x) { return (x + 255) & ~(size_t)255; }

// Output tile width: 256 features, unless that leaves more than a quarter of
// the SMs without a tile (then 128: twice the tiles).  N is a multiple of 256.
static int lg_tile_width(int mtiles, int N) {
  const long long t256 = (long long)mtiles * (N / 256);
  return t256 * 4 >= 3LL * lf_sm_count() ? 256 : 128;
}

struct LgWs {
  size_t count, rows, xs, total;
};

static int lg_check(const lf_proj_params *p) {
  if (!p) return lf_record_error(LF_ERR_INVALID, "params is NULL");
  if (p->B < 1 || p->n < 1 || p->H < 1 || p->H > LF_MAX_H)
    return lf_record_error(LF_ERR_INVALID, "projection: B, n must be >= 1 and H in 1..128");
  if (p->dtype != LF_BF16 && p->dtype != LF_F16)
    return lf_record_error(LF_ERR_INVALID, "projection: dtype must be LF_BF16 or LF_F16");
  if (p->head_dim != LF_HD) return lf_record_error(LF_ERR_UNSUPPORTED, "projection: head_dim must be 64");
  if (p->H % 4) return lf_record_error(LF_ERR_UNSUPPORTED, "projection: H must be a multiple of 4");
  return LF_OK;
}

static LgWs lg_ws(const lf_proj_params *p, int max_rows) {
  LgWs w;
  const size_t K = (size_t)p->H * LF_HD;
  size_t off = lg_align(LF_ST_WORDS * 4);
  w.count = off;
  off = lg_align(off + (size_t)p->B * 4);
  w.rows = off;
  off = lg_align(off + (size_t)p->B * std::max(max_rows, 0) * 4);
  w.xs = off;
  off = lg_align(off + (size_t)p->B * std::max(max_rows, 0) * K * 2);
  w.total = max_rows > 0 ? off : lg_align(LF_ST_WORDS * 4);
  return w;
}

extern "C" size_t lf_proj_workspace_size(const lf_proj_params *p, int max_rows) {
  if (lg_check(p) || max_rows < 0) return 0;
  return lg_ws(p, max_rows).total;
}

static int lg_ptr(const void *ptr, const char *name, bool may_be_null = false) {
  char msg[96];
  if (!ptr) {
    if (may_be_null) return LF_OK;
    snprintf(msg, sizeof(msg), "%s is NULL", name);
    return lf_record_error(LF_ERR_INVALID, msg);
  }
  if (((uintptr_t)ptr) & 15) {
    snprintf(msg, sizeof(msg), "%s is not 16-byte aligned", name);
    return lf_record_error(LF_ERR_INVALID, msg);
  }
  return LF_OK;
}

static int lg_cuda(cudaError_t e, const char *what) {
  if (e == cudaSuccess) return LF_OK;
  char msg[160];
  snprintf(msg, sizeof(msg), "%s: %s", what, cudaGetErrorString(e));
  return lf_record_error(LF_ERR_CUDA, msg);
}

static int lg_launch(LgParams &P, int f16, int bn, cudaStream_t stream, bool pdl) {
  void (*kern)(const LgParams) = bn == 256 ? (f16 ? lf_gemm_kernel<1, 256> : lf_gemm_kernel<0, 256>)
                                           : (f16 ? lf_gemm_kernel<1, 128> : lf_gemm_kernel<0, 128>);
  const int smem = bn == 256 ? LgLayout<256>::SMEM : LgLayout<128>::SMEM;
  int st;
  if ((st = lg_cuda(lf_kernel_smem((const void *)kern, smem), "cudaFuncSetAttribute"))) return st;
  const unsigned grid = (unsigned)std::max(1, std::min(P.tiles, lf_sm_count()));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(LG_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  void *args[] = {(void *)&P};
  if (g_pev_start && g_pev_stop) cudaEventRecord(g_pev_start, stream);
  cudaError_t e = cudaLaunchKernelExC(&cfg, (const void *)kern, args);
  lf_launches_add(1);
  if (g_pev_start && g_pev_stop) cudaEventRecord(g_pev_stop, stream);
  if (e == cudaSuccess) e = cudaGetLastError();
  return lg_cuda(e, "projection GEMM launch");
}

static int lg_bind(const lf_proj_params *p, int max_rows, void *workspace, size_t ws_bytes,
                   cudaStream_t stream, LgWs &w) {
  int st;
  if ((st = lg_check(p))) return st;
  if ((st = lg_ptr(workspace, "workspace"))) return st;
  if (((uintptr_t)workspace) & 255)
    return lf_record_error(LF_ERR_INVALID, "workspace is not 256-byte aligned");
  w = lg_ws(p, max_rows);
  if (ws_bytes < w.total) return lf_record_error(LF_ERR_INVALID, "workspace too small");
  (void)stream;
  return LF_OK;  // the status word stays set until lf_attn_status reads and clears it
}

extern "C" int lf_proj_in(const lf_proj_params *p, int nproj, const void *x, const void *w_in,
                          const void *b_in, void *const *outs, const int32_t *rows_mask,
                          int rows_code, int max_rows, void *workspace, size_t ws_bytes,
                          void *stream_) {
  cudaStream_t stream = (cudaStream_t)stream_;
  int st;
  if (nproj < 1 || nproj > LG_MAX_OUT) return lf_record_error(LF_ERR_INVALID, "nproj must be 1..8");
  if (!outs) return lf_record_error(LF_ERR_INVALID, "outs is NULL");
  if ((st = lg_ptr(x, "x")) || (st = lg_ptr(w_in, "w_in")) || (st = lg_ptr(b_in, "b_in", true)))
    return st;
  for (int i = 0; i < nproj; i++)
    if ((st = lg_ptr(outs[i], "outs[i]"))) return st;
  if (rows_mask && (st = lg_ptr(rows_mask, "rows_mask"))) return st;
  if (rows_mask && max_rows < 1) return lf_record_error(LF_ERR_INVALID, "max_rows must be >= 1");
  if (rows_mask) max_rows = std::min(max_rows, p ? p->n : max_rows);
  LgWs w;
  if ((st = lg_bind(p, rows_mask ? max_rows : 0, workspace, ws_bytes, stream, w))) return st;
  const int f16 = p->dtype == LF_F16;
  const int K = p->H * LF_HD;
  char *ws = (char *)workspace;
  LgParams P;
  memset(&P, 0, sizeof(P));
  P.mode = 0;
  P.B = p->B;
  P.K = K;
  P.N = nproj * K;
  P.out_mode = 0;
  P.H = p->H;
  P.Lout = p->n;
  P.bias = (const uint16_t *)b_in;
  for (int i = 0; i < nproj; i++) P.outs[i] = outs[i];
  P.status = (int32_t *)ws;
  const void *abase = x;
  if (rows_mask) {
    // gather the selected rows into the workspace, then project those
    P.L = max_rows;
    P.row_map = (const int32_t *)(ws + w.rows);
    P.row_count = (const int32_t *)(ws + w.count);
    abase = ws + w.xs;
    if (f16)
      lf_rows_gather_kernel<__half><<<p->B, 1024, 0, stream>>>(
          rows_mask, p->n, rows_code, max_rows, (const __half *)x, K, (int32_t *)(ws + w.rows),
          (int32_t *)(ws + w.count), (__half *)(ws + w.xs), P.status);
    else
      lf_rows_gather_kernel<__nv_bfloat16><<<p->B, 1024, 0, stream>>>(
          rows_mask, p->n, rows_code, max_rows, (const __nv_bfloat16 *)x, K,
          (int32_t *)(ws + w.rows), (int32_t *)(ws + w.count), (__nv_bfloat16 *)(ws + w.xs),
          P.status);
    lf_launches_add(1);
    if ((st = lg_cuda(cudaGetLastError(), "row gather launch"))) return st;
  } else {
    P.L = p->n;
  }
  P.ksteps = K / LG_BK;
  P.mblk = (P.L + LG_BM - 1) / LG_BM;
  const int bn = lg_tile_width(P.B * P.mblk, P.N);
  P.nblk = P.N / bn;
  P.tiles = P.B * P.mblk * P.nblk;
  {
    const cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)P.L, (cuuint64_t)P.B};
    const cuuint64_t strides[2] = {(cuuint64_t)K * 2, (cuuint64_t)P.L * K * 2};
    const cuuint32_t box[3] = {LG_BK, LG_BM, 1};
    if (!lg_make_map(&P.map_a, f16, abase, 3, dims, strides, box))
      return lf_record_error(LF_ERR_CUDA, "projection: tensor map encode failed (x)");
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)P.N};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {LG_BK, (cuuint32_t)bn};
    if (!lg_make_map(&P.map_b, f16, w_in, 2, dims, strides, box))
      return lf_record_error(LF_ERR_CUDA, "projection: tensor map encode failed (w_in)");
  }
  if (!rows_mask) {
    for (int i = 0; i < nproj; i++)
      if (!lf_make_map(&P.map_out[i], f16, outs[i], (uint64_t)p->n, (uint64_t)p->H, (uint64_t)p->B,
                       128, (uint64_t)p->n * 128, (uint64_t)p->H * p->n * 128, LG_BM))
        return lf_record_error(LF_ERR_CUDA, "projection: tensor map encode failed (outs)");
  }
  return lg_launch(P, f16, bn, stream, rows_mask != nullptr);
}

extern "C" int lf_proj_out(const lf_proj_params *p, const void *o, const void *w_out,
                           const void *b_out, void *y, void *workspace, size_t ws_bytes,
                           void *stream_) {
  cudaStream_t stream = (cudaStream_t)stream_;
  int st;
  if ((st = lg_ptr(o, "o")) || (st = lg_ptr(w_out, "w_out")) || (st = lg_ptr(b_out, "b_out", true)) ||
      (st = lg_ptr(y, "y")))
    return st;
  LgWs w;
  if ((st = lg_bind(p, 0, workspace, ws_bytes, stream, w))) return st;
  const int f16 = p->dtype == LF_F16;
  const int K = p->H * LF_HD;
  LgParams P;
  memset(&P, 0, sizeof(P));
  P.mode = 1;
  P.B = p->B;
  P.L = p->n;
  P.K = K;
  P.N = K;
  P.out_mode = 1;
  P.H = p->H;
  P.Lout = p->n;
  P.bias = (const uint16_t *)b_out;
  P.outs[0] = y;
  P.status = (int32_t *)workspace;
  P.ksteps = p->H;  // one head per k-step
  P.mblk = (P.L + LG_BM - 1) / LG_BM;
  const int bn = lg_tile_width(P.B * P.mblk, P.N);
  P.nblk = P.N / bn;
  P.tiles = P.B * P.mblk * P.nblk;
  if (!lf_make_map(&P.map_a, f16, o, (uint64_t)p->n, (uint64_t)p->H, (uint64_t)p->B, 128,
                   (uint64_t)p->n * 128, (uint64_t)p->H * p->n * 128, LG_BM))
    return lf_record_error(LF_ERR_CUDA, "projection: tensor map encode failed (o)");
  {
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)P.N};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {LG_BK, (cuuint32_t)bn};
    if (!lg_make_map(&P.map_b, f16, w_out, 2, dims, strides, box))
      return lf_record_error(LF_ERR_CUDA, "projection: tensor map encode failed (w_out)");
  }
  {
    const cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)P.L, (cuuint64_t)P.B};
    const cuuint64_t strides[2] = {(cuuint64_t)K * 2, (cuuint64_t)P.L * K * 2};
    const cuuint32_t box[3] = {64, LG_BM, 1};
    if (!lg_make_map(&P.map_out[0], f16, y, 3, dims, strides, box))
      return lf_record_error(LF_ERR_CUDA, "projection: tensor map encode failed (y)");
  }
  return lg_launch(P, f16, bn, stream, false);
}
