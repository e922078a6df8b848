// lf_common.cuh -- shared device-side definitions of the attention library:
// kernel parameter block, workspace layout, dtype load/store helpers, the
// attention-pattern predicates (one definition used by every kernel, by the
// pair counter and by the pattern dump) and the device status word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lf_attn.h"

#define LF_HD 64          // head_dim built
#define LF_MAX_H 128      // heads per call
#define LF_BQ 128         // query rows per tensor-core block
#define LF_BK 128         // keys per band tile

// status word slots (int32 each) at the start of the workspace
#define LF_ST_CODE 0      // first error code (atomicCAS from 0)
#define LF_ST_DETAIL 1    // kernel-specific detail of the first error
#define LF_ST_SCHED 2     // work-item counter of the persistent forward (zero at each call)
#define LF_ST_WORDS 8

// per-sequence info written by the mask pass (int32 each)
#define LF_BI_NG 0        // number of global tokens (clamped to max_global)
#define LF_BI_NVALID 1    // number of mask != 0 tokens
#define LF_BI_GMIN 2      // smallest global position (n if none)
#define LF_BI_GMAX 3      // largest global position (-1 if none)
#define LF_BI_WORDS 8

// Workspace carve-up (byte offsets, each 256-byte aligned); computed on the
// host from the params, passed to every kernel.
struct LfWs {
  size_t status;    // int32[LF_ST_WORDS]
  size_t status_bytes;  // bytes of the status block, zeroed at the start of every call
  size_t binfo;     // int32[B][LF_BI_WORDS]
  size_t gidx;      // int32[B][G]           global positions, ascending
  size_t grank;     // int32[B][n+1]         globals at positions < p
  size_t qg_c;      // T[B][H][G][64]        Q_g rows of the global tokens
  size_t ks_c;      // T[B][H][Gk][64]       K_s rows of the global tokens (zero padded)
  size_t vs_c;      // T[B][H][Gk][64]       V_s rows of the global tokens (zero padded)
  size_t part_acc;  // float[B][H][G][NCH][64] split-KV partial sums of global rows
  size_t part_ml;   // float2[B][H][G][NCH]   (running max, running sum) of each split
  size_t delta;     // float[B][H][n]        backward: rowsum(dO * O)
  size_t total;
  int G;            // rows reserved per sequence for global tokens (>= 1)
  int Gk;           // G rounded up to 16 (global key tile width)
  int nch;          // key chunks of the global-row split
};

// Kernel parameter block (by value).
struct LfDev {
  int B, H, n, r, causal, G, Gk, nch, chunk_tiles;
  float scale;        // score scale
  float scale_log2;   // scale * log2(e)
  const int32_t *mask;
  int32_t *status;
  int32_t *binfo;
  int32_t *gidx;
  int32_t *grank;
  int wait_us;    // device wait limit in microseconds (0: default); a test hook
  int skip_tile;  // > 0: CTA 0 of the forward omits the K/V load of its tile
                  // skip_tile - 1, so a bounded wait expires (a test hook)
  int cross;      // 1: cross-attention (queries = G rows of their own tensor,
                  // keys = n rows; output rows are the query rows)
  int dil[LF_MAX_H];
};

// ----------------------------------------------------------- status word --

__device__ __forceinline__ void lf_set_status(int32_t *status, int code, int detail) {
  if (atomicCAS(status + LF_ST_CODE, 0, code) == 0) status[LF_ST_DETAIL] = detail;
}

// ------------------------------------------------------------ pattern ----

// Is key j in query i's dilated window?  keys j = i + k*d, |k| <= r, and
// k <= 0 when causal (segmentfault page, sections 滑动窗口 / 扩张滑动窗口; the
// glossary example |i - j| <= window/2 is the d = 1 case).
__host__ __device__ __forceinline__ bool lf_in_window(int i, int j, int r, int d, int causal) {
  int dist = j - i;
  if (dist % d) return false;
  int k = dist / d;
  return k >= -r && k <= (causal ? 0 : r);
}

// Tensor-core tile walk.  A head with dilation d is split into d residue
// sub-sequences rho, rho+d, rho+2d, ... ; in sub-sequence coordinates t the
// window is an undilated band of radius r (causal: [t-r, t]).  A query block
// covers rows t0..t0+127; its band key tiles start at t0 - r + 128*u.
__host__ __device__ __forceinline__ int lf_band_tiles(int r, int causal) {
  int span = LF_BQ + (causal ? r : 2 * r);
  return (span + LF_BK - 1) / LF_BK;
}

// Columns c of band tile u that row q (0..127) of the block attends by its
// window: q <= 128u + c <= q + (causal ? r : 2r).  Inclusive [lo, hi];
// empty when lo > hi.
__host__ __device__ __forceinline__ void lf_band_cols(int q, int u, int r, int causal, int &lo,
                                                      int &hi) {
  int base = LF_BK * u;
  lo = q - base;
  if (lo < 0) lo = 0;
  hi = q + (causal ? r : 2 * r) - base;
  if (hi > LF_BK - 1) hi = LF_BK - 1;
}

// The same for column tiles of kW columns (band tile u starts kW*u after
// the block's first window key): band tiles of a block, and the columns of
// tile u that row q attends, q <= kW*u + c <= q + (causal ? r : 2r).
template <int kW>
__host__ __device__ __forceinline__ int lf_band_tiles_w(int r, int causal) {
  return (LF_BQ + (causal ? r : 2 * r) + kW - 1) / kW;
}
template <int kW>
__host__ __device__ __forceinline__ void lf_band_cols_w(int q, int u, int r, int causal, int &lo,
                                                        int &hi) {
  const int base = kW * u;
  lo = q - base;
  if (lo < 0) lo = 0;
  hi = q + (causal ? r : 2 * r) - base;
  if (hi > kW - 1) hi = kW - 1;
}

// Length of residue sub-sequence rho of a length-n sequence with dilation d.
__host__ __device__ __forceinline__ int lf_sub_len(int n, int d, int rho) {
  return rho < n ? (n - rho + d - 1) / d : 0;
}

// ------------------------------------------------------ dtype helpers ----

template <typename T> struct LfIo;
template <> struct LfIo<float> {
  static __device__ __forceinline__ float2 ld2(const float *p) {
    return *reinterpret_cast<const float2 *>(p);
  }
  static __device__ __forceinline__ void st2(float *p, float a, float b) {
    *reinterpret_cast<float2 *>(p) = make_float2(a, b);
  }
};
template <> struct LfIo<__nv_bfloat16> {
  static __device__ __forceinline__ float2 ld2(const __nv_bfloat16 *p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
  }
  static __device__ __forceinline__ void st2(__nv_bfloat16 *p, float a, float b) {
    *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(a, b);
  }
};
template <> struct LfIo<__half> {
  static __device__ __forceinline__ float2 ld2(const __half *p) {
    return __half22float2(*reinterpret_cast<const __half2 *>(p));
  }
  static __device__ __forceinline__ void st2(__half *p, float a, float b) {
    *reinterpret_cast<__half2 *>(p) = __floats2half2_rn(a, b);
  }
};

// 16-byte slice of a 64-element row: N elements of T as floats.  A row is
// handled by 64 / N consecutive lanes (a lane group).
template <typename T> struct LfVec;
template <> struct LfVec<float> {
  static constexpr int N = 4;
  static __device__ __forceinline__ void ld(const float *p, float (&x)[4]) {
    const float4 v = *reinterpret_cast<const float4 *>(p);
    x[0] = v.x;
    x[1] = v.y;
    x[2] = v.z;
    x[3] = v.w;
  }
  static __device__ __forceinline__ void st(float *p, const float (&x)[4]) {
    *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
  }
};
template <typename H2, typename T> struct LfVec16 {
  static constexpr int N = 8;
  static __device__ __forceinline__ void ld(const T *p, float (&x)[8]) {
    const uint4 v = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; k++) {
      const float2 f = LfIo<T>::ld2(reinterpret_cast<const T *>(&w[k]));
      x[2 * k] = f.x;
      x[2 * k + 1] = f.y;
    }
  }
  static __device__ __forceinline__ void st(T *p, const float (&x)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; k++) LfIo<T>::st2(reinterpret_cast<T *>(&w[k]), x[2 * k], x[2 * k + 1]);
    *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  }
};
template <> struct LfVec<__nv_bfloat16> : LfVec16<__nv_bfloat162, __nv_bfloat16> {};
template <> struct LfVec<__half> : LfVec16<__half2, __half> {};

// sum over an aligned group of G lanes (G a power of two dividing 32)
template <int G>
__device__ __forceinline__ float lf_group_sum(float v) {
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float lf_warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float2 lf_warp_sum2(float a, float b) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  return make_float2(a, b);
}

#define LF_LOG2E 1.4426950408889634f
#define LF_LN2 0.6931471805599453f

// Raise fn's dynamic shared-memory limit to smem_bytes on the current
// device (once per device and kernel; thread-safe).
cudaError_t lf_kernel_smem(const void *fn, int smem_bytes);
// SM count of the current device (cached per device; thread-safe).
int lf_sm_count();

// process-wide count of kernel launches made by the library
void lf_launches_add(int k);
uint64_t lf_launches_get();

// host-side launchers implemented in the .cu files
struct LfLaunch {
  LfDev dev;
  LfWs ws;
  char *ws_base;
  cudaStream_t stream;
  int dtype;
};

cudaError_t lf_launch_mask_pass(const LfLaunch &L);
cudaError_t lf_launch_cross_setup(const LfLaunch &L);
cudaError_t lf_launch_mask_gather(const LfLaunch &L, const void *qg, const void *ks, const void *vs,
                                  void *qg_c, void *ks_c, void *vs_c, int Ga, int Gka);
cudaError_t lf_launch_count(const LfLaunch &L, int64_t *counts);
cudaError_t lf_launch_decode(const LfLaunch &L, const void *q, const void *kc, const void *vc,
                             const int32_t *lengths, void *o, float *lse);
cudaError_t lf_launch_dump(const LfLaunch &L, uint8_t *out);
cudaError_t lf_launch_simt_fwd(const LfLaunch &L, const void *qs, const void *ks, const void *vs,
                               const void *qg, const void *kg, const void *vg, void *o, float *lse);
cudaError_t lf_launch_simt_bwd(const LfLaunch &L, const void *qs, const void *ks, const void *vs,
                               const void *qg, const void *kg, const void *vg, const void *o,
                               const float *lse, const void *dO, void *dqs, void *dks, void *dvs,
                               void *dqg, void *dkg, void *dvg);
