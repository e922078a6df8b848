// lf_simt.cu -- CUDA-core kernels of the attention library:
//   * the mask pass (global-token list, valid count, device input checks),
//   * the pair counter and the pattern dump (tile-walk predicates of the
//     tensor-core forward),
//   * the CUDA-core forward and backward for every dtype (the float32 path,
//     and the cross-check of the tensor-core path for bf16/f16).
//
// CUDA-core kernels use one warp per query row (forward, dQ) or per key row
// (dK, dV); lane l owns head-dim elements 2l and 2l+1, so every K/V/Q row
// read is one coalesced 128/256-byte access and each score is a warp sum.
// All sums are float32; outputs are rounded once (RNE) to the call's dtype.
#include <cooperative_groups.h>
#include <cub/block/block_scan.cuh>

namespace cg = cooperative_groups;

#include "lf_common.cuh"

// =============================================================== mask pass

// The mask scan of sequence b by one block of 1024 threads: compact the
// global positions (ascending) into gl_out[0..min(ng, G)), and, when
// write_tables, write the rank array grank[b][p] = #globals before p, the
// per-sequence info, and the status flags (bad codes, too many globals,
// causal + global).  Returns the number of global tokens (all of them).
typedef cub::BlockScan<int, 1024> LfScan;
__device__ int lf_mask_scan(const LfDev &P, int b, bool write_tables, int32_t *gl_out,
                            typename LfScan::TempStorage &tmp) {
  __shared__ int s_valid, s_gmin, s_gmax, s_bad, s_total;
  const int tid = threadIdx.x, n = P.n;
  const int32_t *m = P.mask + (size_t)b * n;
  if (tid == 0) {
    s_valid = 0;
    s_gmin = n;
    s_gmax = -1;
    s_bad = 0;
  }
  __syncthreads();
  const int per = (n + 1023) / 1024;
  const int s = tid * per, e = min(n, s + per);
  int c = 0, v = 0, bad = 0, gmin = n, gmax = -1;
  // unrolled so that several of the thread's loads are in flight at once
#pragma unroll 8
  for (int i = s; i < e; i++) {
    int x = m[i];
    if (x == 2) {
      c++;
      gmin = min(gmin, i);
      gmax = max(gmax, i);
    }
    if (x != 0) v++;
    if (x < 0 || x > 2) bad = 1;
  }
  int off, total;
  LfScan(tmp).ExclusiveSum(c, off, total);
  atomicAdd(&s_valid, v);
  atomicMin(&s_gmin, gmin);
  atomicMax(&s_gmax, gmax);
  if (bad) atomicOr(&s_bad, 1);
  if (tid == 0) s_total = total;
  int32_t *gr = P.grank + (size_t)b * (n + 1);
#pragma unroll 8
  for (int i = s; i < e; i++) {
    if (write_tables) gr[i] = off;  // globals before position i
    if (m[i] == 2) {
      if (off < P.G) gl_out[off] = i;
      off++;
    }
  }
  if (write_tables && tid == 1023) gr[n] = total;
  __syncthreads();
  if (write_tables && tid == 0) {
    int32_t *bi = P.binfo + (size_t)b * LF_BI_WORDS;
    bi[LF_BI_NG] = min(s_total, P.G);
    bi[LF_BI_NVALID] = s_valid;
    bi[LF_BI_GMIN] = s_gmin;
    bi[LF_BI_GMAX] = s_gmax;
    if (s_bad) lf_set_status(P.status, LF_ERR_DEVICE_INPUT, 1000000 + b);
    if (s_total > P.G) lf_set_status(P.status, LF_ERR_DEVICE_INPUT, 2000000 + b);
    if (P.causal && s_total > 0) lf_set_status(P.status, LF_ERR_UNSUPPORTED, 3000000 + b);
  }
  return s_total;
}

// One block per sequence b: the mask scan and its tables.
__global__ void __launch_bounds__(1024) lf_mask_pass_kernel(LfDev P) {
  __shared__ typename LfScan::TempStorage tmp;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int b = blockIdx.x;
  // the first kernel of a call: the work-item counter of the forward starts
  // at zero (read by the kernels after this one completes)
  if (b == 0 && threadIdx.x == 0) P.status[LF_ST_SCHED] = 0;
  lf_mask_scan(P, b, true, P.gidx + (size_t)b * P.G, tmp);
}

cudaError_t lf_launch_mask_pass(const LfLaunch &L) {
  lf_mask_pass_kernel<<<L.dev.B, 1024, 0, L.stream>>>(L.dev);
  lf_launches_add(1);
  return cudaGetLastError();
}

// One block per (b, h): the mask scan of sequence b (block h = 0 also writes
// its tables and the global list) followed by the compaction of head h's Q_g / K_s / V_s rows of
// the global tokens (rows past the sequence's global count are zero) -- the
// mask pass and the gather of the tensor-core forward in one launch.  The
// global list is kept in shared memory (G entries).
template <typename T>
__global__ void __launch_bounds__(1024)
    lf_mask_gather_kernel(LfDev P, const T *qg, const T *ks, const T *vs, T *qg_c, T *ks_c, T *vs_c,
                          int Ga, int Gka) {
  __shared__ typename LfScan::TempStorage tmp;
  extern __shared__ int32_t s_gl[];
  // the forward kernel launched after this one may start its set-up now
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (blockIdx.x == 0 && threadIdx.x == 0) P.status[LF_ST_SCHED] = 0;  // (as lf_mask_pass_kernel)
  const int bh = blockIdx.x, b = bh / P.H;
  const bool tables = bh % P.H == 0;
  const int ng = min(lf_mask_scan(P, b, tables, s_gl, tmp), P.G);
  __syncthreads();
  if (tables)  // the global list itself, as the mask pass writes it
    for (int e = threadIdx.x; e < ng; e += blockDim.x) P.gidx[(size_t)b * P.G + e] = s_gl[e];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // four rows per warp per round, every load of a round issued before its stores
  for (int e0 = warp; e0 < Gka; e0 += 4 * 32) {
    uint32_t q[4], k[4], v[4];
#pragma unroll
    for (int u = 0; u < 4; u++) {
      const int e = e0 + 32 * u;
      q[u] = k[u] = v[u] = 0;
      if (e < ng) {
        const size_t src = ((size_t)bh * P.n + s_gl[e]) * LF_HD + 2 * lane;
        q[u] = *reinterpret_cast<const uint32_t *>(qg + src);
        k[u] = *reinterpret_cast<const uint32_t *>(ks + src);
        v[u] = *reinterpret_cast<const uint32_t *>(vs + src);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; u++) {
      const int e = e0 + 32 * u;
      if (e >= Gka) break;
      if (e < Ga) *reinterpret_cast<uint32_t *>(qg_c + ((size_t)bh * Ga + e) * LF_HD + 2 * lane) = q[u];
      *reinterpret_cast<uint32_t *>(ks_c + ((size_t)bh * Gka + e) * LF_HD + 2 * lane) = k[u];
      *reinterpret_cast<uint32_t *>(vs_c + ((size_t)bh * Gka + e) * LF_HD + 2 * lane) = v[u];
    }
  }
}

cudaError_t lf_launch_mask_gather(const LfLaunch &L, const void *qg, const void *ks, const void *vs,
                                  void *qg_c, void *ks_c, void *vs_c, int Ga, int Gka) {
  const unsigned grid = (unsigned)(L.dev.B * L.dev.H);
  const size_t sm = (size_t)L.dev.G * sizeof(int32_t);
  if (L.dtype == LF_F16)
    lf_mask_gather_kernel<__half><<<grid, 1024, sm, L.stream>>>(
        L.dev, (const __half *)qg, (const __half *)ks, (const __half *)vs, (__half *)qg_c,
        (__half *)ks_c, (__half *)vs_c, Ga, Gka);
  else
    lf_mask_gather_kernel<__nv_bfloat16><<<grid, 1024, sm, L.stream>>>(
        L.dev, (const __nv_bfloat16 *)qg, (const __nv_bfloat16 *)ks, (const __nv_bfloat16 *)vs,
        (__nv_bfloat16 *)qg_c, (__nv_bfloat16 *)ks_c, (__nv_bfloat16 *)vs_c, Ga, Gka);
  lf_launches_add(1);
  return cudaGetLastError();
}

// ===================================================== counter and dump

// Attended keys of row t (sub-sequence coordinates, residue rho, dilation d)
// enumerated by the tensor-core tile walk: band tiles u = 0.. of the row's
// 128-row query block, then the global tile minus keys already in the window.
__device__ int64_t lf_row_pairs_tilewalk(const LfDev &P, int b, int d, int rho, int t) {
  const int n = P.n, cnt = lf_sub_len(n, d, rho);
  const int32_t *m = P.mask + (size_t)b * n;
  const int p = rho + t * d;
  const int code = m[p];
  if (code == 0) return 0;
  const int32_t *bi = P.binfo + (size_t)b * LF_BI_WORDS;
  if (code == 2) return bi[LF_BI_NVALID];
  const int t0 = (t / LF_BQ) * LF_BQ, q = t - t0;
  int64_t c = 0;
  const int nt = lf_band_tiles(P.r, P.causal);
  for (int u = 0; u < nt; u++) {
    int lo, hi;
    lf_band_cols(q, u, P.r, P.causal, lo, hi);
    for (int col = lo; col <= hi; col++) {
      int tk = t0 - P.r + LF_BK * u + col;
      if (tk >= 0 && tk < cnt && m[rho + tk * d] != 0) c++;
    }
  }
  const int ng = bi[LF_BI_NG];
  const int32_t *gl = P.gidx + (size_t)b * P.G;
  for (int g = 0; g < ng; g++)
    if (!lf_in_window(p, gl[g], P.r, d, P.causal)) c++;
  return c;
}

__global__ void __launch_bounds__(256) lf_count_kernel(LfDev P, int64_t *counts) {
  const int bh = blockIdx.x, h = bh % P.H, b = bh / P.H, d = P.dil[h];
  int64_t c = 0;
  for (int p = threadIdx.x; p < P.n; p += blockDim.x) c += lf_row_pairs_tilewalk(P, b, d, p % d, p / d);
  __shared__ unsigned long long s;
  if (threadIdx.x == 0) s = 0;
  __syncthreads();
  atomicAdd(&s, (unsigned long long)c);
  __syncthreads();
  if (threadIdx.x == 0) counts[bh] = (int64_t)s;
}

cudaError_t lf_launch_count(const LfLaunch &L, int64_t *counts) {
  lf_count_kernel<<<L.dev.B * L.dev.H, 256, 0, L.stream>>>(L.dev, counts);
  lf_launches_add(1);
  return cudaGetLastError();
}

// One block per (b, h, query position p): row p of the pattern.
__global__ void __launch_bounds__(256) lf_dump_kernel(LfDev P, uint8_t *out) {
  const int n = P.n;
  const int p = blockIdx.x, bh = blockIdx.y, h = bh % P.H, b = bh / P.H, d = P.dil[h];
  const int32_t *m = P.mask + (size_t)b * n;
  uint8_t *row = out + ((size_t)bh * n + p) * n;
  const int code = m[p];
  const int rho = p % d, t = p / d, t0 = (t / LF_BQ) * LF_BQ, q = t - t0;
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    int a = 0;
    if (code == 2) {
      a = m[j] != 0;
    } else if (code == 1 && m[j] != 0) {
      int band = 0;
      if (j % d == rho) {  // same residue: locate key j in the tile walk
        int tk = j / d;
        int rel = tk - (t0 - P.r);
        if (rel >= 0) {
          int u = rel / LF_BK, col = rel % LF_BK, lo, hi;
          if (u < lf_band_tiles(P.r, P.causal)) {
            lf_band_cols(q, u, P.r, P.causal, lo, hi);
            band = (col >= lo && col <= hi);
          }
        }
      }
      int glob = (m[j] == 2) && !lf_in_window(p, j, P.r, d, P.causal);
      a = band | glob;
    }
    row[j] = (uint8_t)a;
  }
}

cudaError_t lf_launch_dump(const LfLaunch &L, uint8_t *out) {
  dim3 grid(L.dev.n, L.dev.B * L.dev.H);
  lf_dump_kernel<<<grid, 256, 0, L.stream>>>(L.dev, out);
  lf_launches_add(1);
  return cudaGetLastError();
}

// ========================================================= CUDA-core fwd

// 64 elements of a row as float
template <typename T>
__device__ __forceinline__ void lf_load_row64(const T *p, float (&x)[64]);
template <>
__device__ __forceinline__ void lf_load_row64<float>(const float *p, float (&x)[64]) {
  const float4 *q = reinterpret_cast<const float4 *>(p);
#pragma unroll
  for (int k = 0; k < 16; k++) {
    const float4 v = q[k];
    x[4 * k] = v.x;
    x[4 * k + 1] = v.y;
    x[4 * k + 2] = v.z;
    x[4 * k + 3] = v.w;
  }
}
template <typename H2, typename T>
__device__ __forceinline__ void lf_load_row64_h(const T *p, float (&x)[64]) {
  const uint4 *q = reinterpret_cast<const uint4 *>(p);
#pragma unroll
  for (int k = 0; k < 8; k++) {
    const uint4 v = q[k];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; j++) {
      const float2 f = LfIo<T>::ld2(reinterpret_cast<const T *>(&w[j]));
      x[8 * k + 2 * j] = f.x;
      x[8 * k + 2 * j + 1] = f.y;
    }
  }
}
template <>
__device__ __forceinline__ void lf_load_row64<__nv_bfloat16>(const __nv_bfloat16 *p, float (&x)[64]) {
  lf_load_row64_h<__nv_bfloat162>(p, x);
}
template <>
__device__ __forceinline__ void lf_load_row64<__half>(const __half *p, float (&x)[64]) {
  lf_load_row64_h<__half2>(p, x);
}

// One warp per query row, keys in batches of 32 (one key per lane): the lane
// forms its key's full score, the warp updates the running max / sum, then
// every lane accumulates its two output columns over the batch's keys.
template <typename T>
struct LfRowAcc {
  float q[64];
  float mx, l, a0, a1;
  int self;  // this warp's own row (a valid address for lanes without a key)
  // j is the lane's key when `inr` (a row of the sequence); the key counts
  // when also `cond` and its mask word is nonzero (m == nullptr: no mask).  The key row is loaded
  // together with the mask word (a row that turns out masked is loaded for
  // nothing), so a batch waits for one load latency before its scores.
  __device__ __forceinline__ void batch(const T *K, const T *V, size_t base, const int32_t *m, int j,
                                        bool inr, bool cond, int lane) {
    const int jl = inr ? j : self;
    float k[64];
    lf_load_row64<T>(K + base + (size_t)jl * LF_HD, k);
    const bool ok = inr && cond && (!m || m[jl] != 0);
    j = jl;
    float s = -INFINITY;
    if (ok) {
      float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
#pragma unroll
      for (int c = 0; c < 64; c += 4) {
        d0 = fmaf(q[c], k[c], d0);
        d1 = fmaf(q[c + 1], k[c + 1], d1);
        d2 = fmaf(q[c + 2], k[c + 2], d2);
        d3 = fmaf(q[c + 3], k[c + 3], d3);
      }
      s = (d0 + d1) + (d2 + d3);  // q is pre-scaled by scale * log2(e)
    }
    float bm = s;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
    if (bm == -INFINITY) return;  // no key in this batch (warp-uniform)
    const float mn = fmaxf(mx, bm);
    const float al = exp2f(mx - mn);
    const float p = ok ? exp2f(s - mn) : 0.f;
    l = l * al + lf_warp_sum(p);
    a0 *= al;
    a1 *= al;
    // all 32 value rows of the batch are loaded before the sums (one
    // latency per batch); a lane without a key points at row `self` with p = 0
    const int js = ok ? j : self;
    float2 v[32];
#pragma unroll
    for (int src = 0; src < 32; src++) {
      const int jj = __shfl_sync(0xffffffffu, js, src);
      v[src] = LfIo<T>::ld2(V + base + (size_t)jj * LF_HD + 2 * lane);
    }
#pragma unroll
    for (int src = 0; src < 32; src++) {
      const float pj = __shfl_sync(0xffffffffu, p, src);
      a0 = fmaf(pj, v[src].x, a0);
      a1 = fmaf(pj, v[src].y, a1);
    }
    mx = mn;
  }
};

template <typename T>
__global__ void __launch_bounds__(256, 1)
    lf_simt_fwd_kernel(LfDev P, const T *qs, const T *ks, const T *vs, const T *qg, const T *kg,
                       const T *vg, T *o, float *lse) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int n = P.n;
  if (row >= (long long)P.B * P.H * n) return;
  const int i = (int)(row % n);
  const int bh = (int)(row / n), h = bh % P.H, b = bh / P.H, d = P.dil[h];
  const int32_t *m = P.mask + (size_t)b * n;
  const size_t base = (size_t)bh * n * LF_HD;
  const size_t ooff = base + (size_t)i * LF_HD + 2 * lane;
  const int code = m[i];
  if (code == 0) {
    LfIo<T>::st2(o + ooff, 0.f, 0.f);
    if (lse && lane == 0) lse[(size_t)bh * n + i] = -INFINITY;
    return;
  }
  const bool glob = code == 2;
  const T *Q = glob ? qg : qs, *K = glob ? kg : ks, *V = glob ? vg : vs;
  LfRowAcc<T> st;
  lf_load_row64<T>(Q + base + (size_t)i * LF_HD, st.q);
#pragma unroll
  for (int c = 0; c < 64; c++) st.q[c] *= P.scale_log2;
  st.mx = -INFINITY;
  st.l = st.a0 = st.a1 = 0.f;
  st.self = i;
  if (glob) {
    for (int j0 = 0; j0 < n; j0 += 32) {
      const int j = j0 + lane;
      st.batch(K, V, base, m, j, j < n, true, lane);
    }
  } else {
    // window keys j = i + k*d, k in [-r, khi], then the global keys outside it
    const int khi = P.causal ? 0 : P.r;
    for (int k0 = -P.r; k0 <= khi; k0 += 32) {
      const int k = k0 + lane, j = i + k * d;
      st.batch(K, V, base, m, j, k <= khi && j >= 0 && j < n, true, lane);
    }
    const int ng = P.binfo[(size_t)b * LF_BI_WORDS + LF_BI_NG];
    const int32_t *gl = P.gidx + (size_t)b * P.G;
    for (int t0 = 0; t0 < ng; t0 += 32) {
      const int t = t0 + lane;
      const int g = t < ng ? gl[t] : 0;
      st.batch(K, V, base, m, g, t < ng, !lf_in_window(i, g, P.r, d, P.causal), lane);
    }
  }
  const float inv = 1.f / st.l;
  LfIo<T>::st2(o + ooff, st.a0 * inv, st.a1 * inv);
  if (lse && lane == 0) lse[(size_t)bh * n + i] = (st.mx + log2f(st.l)) * LF_LN2;
}

template <typename T>
static cudaError_t lf_simt_fwd_t(const LfLaunch &L, const void *qs, const void *ks, const void *vs,
                                 const void *qg, const void *kg, const void *vg, void *o,
                                 float *lse) {
  long long rows = (long long)L.dev.B * L.dev.H * L.dev.n;
  unsigned grid = (unsigned)((rows + 7) / 8);
  lf_simt_fwd_kernel<T><<<grid, 256, 0, L.stream>>>(
      L.dev, (const T *)qs, (const T *)ks, (const T *)vs, (const T *)qg, (const T *)kg,
      (const T *)vg, (T *)o, lse);
  lf_launches_add(1);
  return cudaGetLastError();
}

cudaError_t lf_launch_simt_fwd(const LfLaunch &L, const void *qs, const void *ks, const void *vs,
                               const void *qg, const void *kg, const void *vg, void *o,
                               float *lse) {
  switch (L.dtype) {
    case LF_F32: return lf_simt_fwd_t<float>(L, qs, ks, vs, qg, kg, vg, o, lse);
    case LF_BF16: return lf_simt_fwd_t<__nv_bfloat16>(L, qs, ks, vs, qg, kg, vg, o, lse);
    default: return lf_simt_fwd_t<__half>(L, qs, ks, vs, qg, kg, vg, o, lse);
  }
}

// ========================================================= CUDA-core bwd

// delta[row] = sum_c dO[row, c] * O[row, c]   (float32; 0 for mask-0 rows).
// A lane group of 64 / N lanes per row, 16 bytes of O and of dO per lane.
template <typename T>
__global__ void __launch_bounds__(256)
    lf_bwd_delta_kernel(LfDev P, const T *o, const T *dO, float *delta) {
  constexpr int N = LfVec<T>::N, TPR = LF_HD / N;
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = t / TPR;
  const int part = (int)(t % TPR);
  const bool in = row < (long long)P.B * P.H * P.n;
  float s = 0.f;
  if (in) {
    float a[N], g[N];
    const size_t off = (size_t)row * LF_HD + part * N;
    LfVec<T>::ld(o + off, a);
    LfVec<T>::ld(dO + off, g);
#pragma unroll
    for (int k = 0; k < N; k++) s += a[k] * g[k];
  }
  s = lf_group_sum<TPR>(s);
  if (in && part == 0) delta[row] = s;
}

// dQ: one warp per query row, same key enumeration as the forward.
template <typename T>
__global__ void __launch_bounds__(256)
    lf_bwd_dq_kernel(LfDev P, const T *qs, const T *ks, const T *vs, const T *qg, const T *kg,
                     const T *vg, const float *lse, const T *dO, const float *delta, T *dqs,
                     T *dqg) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int n = P.n;
  if (row >= (long long)P.B * P.H * n) return;
  const int i = (int)(row % n);
  const int bh = (int)(row / n), h = bh % P.H, b = bh / P.H, d = P.dil[h];
  const int32_t *m = P.mask + (size_t)b * n;
  const size_t base = (size_t)bh * n * LF_HD + 2 * lane;
  const size_t ioff = base + (size_t)i * LF_HD;
  const int code = m[i];
  if (code != 1) LfIo<T>::st2(dqs + ioff, 0.f, 0.f);
  if (code != 2) LfIo<T>::st2(dqg + ioff, 0.f, 0.f);
  if (code == 0) return;
  const bool glob = code == 2;
  const T *Q = glob ? qg : qs, *K = glob ? kg : ks, *V = glob ? vg : vs;
  float2 q = LfIo<T>::ld2(Q + ioff);
  float2 g = LfIo<T>::ld2(dO + ioff);
  const float L2 = lse[row] * LF_LOG2E, Di = delta[row];
  float acc0 = 0.f, acc1 = 0.f;
  auto visit = [&](int j) {
    size_t koff = base + (size_t)j * LF_HD;
    float2 k = LfIo<T>::ld2(K + koff), v = LfIo<T>::ld2(V + koff);
    float2 sd = lf_warp_sum2(q.x * k.x + q.y * k.y, g.x * v.x + g.y * v.y);
    float pr = exp2f(sd.x * P.scale_log2 - L2);
    float ds = pr * (sd.y - Di) * P.scale;
    acc0 += ds * k.x;
    acc1 += ds * k.y;
  };
  if (glob) {
    for (int j = 0; j < n; j++)
      if (m[j] != 0) visit(j);
  } else {
    const int khi = P.causal ? 0 : P.r;
    for (int k = -P.r; k <= khi; k++) {
      int j = i + k * d;
      if (j < 0 || j >= n || m[j] == 0) continue;
      visit(j);
    }
    const int ng = P.binfo[(size_t)b * LF_BI_WORDS + LF_BI_NG];
    const int32_t *gl = P.gidx + (size_t)b * P.G;
    for (int t = 0; t < ng; t++)
      if (!lf_in_window(i, gl[t], P.r, d, P.causal)) visit(gl[t]);
  }
  LfIo<T>::st2((glob ? dqg : dqs) + ioff, acc0, acc1);
}

// dK_s, dV_s: one warp per key row j, over the LOCAL rows that attend j.
// A non-global key is attended by the rows i = j - k*d of its window; a
// global key by every local row (exactly once: window or global column).
template <typename T>
__global__ void __launch_bounds__(256)
    lf_bwd_dkv_s_kernel(LfDev P, const T *qs, const T *ks, const T *vs, const float *lse,
                        const T *dO, const float *delta, T *dks, T *dvs) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int n = P.n;
  if (row >= (long long)P.B * P.H * n) return;
  const int j = (int)(row % n);
  const int bh = (int)(row / n), h = bh % P.H, b = bh / P.H, d = P.dil[h];
  const int32_t *m = P.mask + (size_t)b * n;
  const size_t base = (size_t)bh * n * LF_HD + 2 * lane;
  const size_t joff = base + (size_t)j * LF_HD;
  const int code = m[j];
  float k0 = 0.f, k1 = 0.f, v0 = 0.f, v1 = 0.f;
  if (code != 0) {
    float2 kk = LfIo<T>::ld2(ks + joff), vv = LfIo<T>::ld2(vs + joff);
    auto visit = [&](int i) {
      size_t ioff = base + (size_t)i * LF_HD;
      size_t ir = (size_t)bh * n + i;
      float2 q = LfIo<T>::ld2(qs + ioff), g = LfIo<T>::ld2(dO + ioff);
      float2 sd = lf_warp_sum2(q.x * kk.x + q.y * kk.y, g.x * vv.x + g.y * vv.y);
      float pr = exp2f(sd.x * P.scale_log2 - lse[ir] * LF_LOG2E);
      float ds = pr * (sd.y - delta[ir]) * P.scale;
      k0 += ds * q.x;
      k1 += ds * q.y;
      v0 += pr * g.x;
      v1 += pr * g.y;
    };
    if (code == 2) {
      for (int i = 0; i < n; i++)
        if (m[i] == 1) visit(i);
    } else {
      // row i attends j when j = i + k*d with k in [-r, khi]  <=>  i = j - k*d
      const int khi = P.causal ? 0 : P.r;
      for (int k = khi; k >= -P.r; k--) {
        int i = j - k * d;
        if (i < 0 || i >= n || m[i] != 1) continue;
        visit(i);
      }
    }
  }
  LfIo<T>::st2(dks + joff, k0, k1);
  LfIo<T>::st2(dvs + joff, v0, v1);
}

// dK_g, dV_g: one lane group (64 / N lanes, 16 bytes each) per key row j,
// over the global rows (every global row attends every valid key through
// Q_g / K_g / V_g); each global row's scores are group sums.  Rows of mask-0
// keys are zero.
template <typename T>
__global__ void __launch_bounds__(256)
    lf_bwd_dkv_g_kernel(LfDev P, const T *qg, const T *kg, const T *vg, const float *lse,
                        const T *dO, const float *delta, T *dkg, T *dvg) {
  constexpr int N = LfVec<T>::N, TPR = LF_HD / N;
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long key = t / TPR;  // (b, h, j)
  const int part = (int)(t % TPR);
  const int n = P.n;
  const bool in = key < (long long)P.B * P.H * n;
  const long long kk = in ? key : 0;
  const int j = (int)(kk % n);
  const int bh = (int)(kk / n), b = bh / P.H;
  const bool on = in && P.mask[(size_t)b * n + j] != 0;
  float kx[N], vx[N], ak[N], av[N];
#pragma unroll
  for (int k = 0; k < N; k++) ak[k] = av[k] = 0.f;
  const size_t joff = (size_t)kk * LF_HD + part * N;
  LfVec<T>::ld(kg + joff, kx);
  LfVec<T>::ld(vg + joff, vx);
  // every lane of the warp runs the same global-row loop (group sums); a
  // warp's keys may belong to two (b, h): the longer count is walked
  const int ng = P.binfo[(size_t)b * LF_BI_WORDS + LF_BI_NG];
  int ngw = ng;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ngw = max(ngw, __shfl_xor_sync(0xffffffffu, ngw, o));
  const int32_t *gl = P.gidx + (size_t)b * P.G;
  for (int e = 0; e < ngw; e++) {
    const bool act = on && e < ng;
    const int i = act ? gl[e] : 0;
    float q[N], g[N];
    const size_t ioff = ((size_t)bh * n + i) * LF_HD + part * N, ir = (size_t)bh * n + i;
    LfVec<T>::ld(qg + ioff, q);
    LfVec<T>::ld(dO + ioff, g);
    float s = 0.f, dp = 0.f;
#pragma unroll
    for (int k = 0; k < N; k++) {
      s += q[k] * kx[k];
      dp += g[k] * vx[k];
    }
    s = lf_group_sum<TPR>(s);
    dp = lf_group_sum<TPR>(dp);
    if (!act) continue;
    const float pr = exp2f(s * P.scale_log2 - lse[ir] * LF_LOG2E);
    const float ds = pr * (dp - delta[ir]) * P.scale;
#pragma unroll
    for (int k = 0; k < N; k++) {
      ak[k] += ds * q[k];
      av[k] += pr * g[k];
    }
  }
  if (in) {
    LfVec<T>::st(dkg + joff, ak);
    LfVec<T>::st(dvg + joff, av);
  }
}

template <typename T>
static cudaError_t lf_simt_bwd_t(const LfLaunch &L, const void *qs, const void *ks, const void *vs,
                                 const void *qg, const void *kg, const void *vg, const void *o,
                                 const float *lse, const void *dO, void *dqs, void *dks, void *dvs,
                                 void *dqg, void *dkg, void *dvg) {
  long long rows = (long long)L.dev.B * L.dev.H * L.dev.n;
  unsigned grid = (unsigned)((rows + 7) / 8);
  float *delta = (float *)(L.ws_base + L.ws.delta);
  lf_bwd_delta_kernel<T><<<(unsigned)((rows * (LF_HD / LfVec<T>::N) + 255) / 256), 256, 0, L.stream>>>(
      L.dev, (const T *)o, (const T *)dO, delta);
  lf_bwd_dq_kernel<T><<<grid, 256, 0, L.stream>>>(
      L.dev, (const T *)qs, (const T *)ks, (const T *)vs, (const T *)qg, (const T *)kg,
      (const T *)vg, lse, (const T *)dO, delta, (T *)dqs, (T *)dqg);
  lf_bwd_dkv_s_kernel<T><<<grid, 256, 0, L.stream>>>(L.dev, (const T *)qs, (const T *)ks,
                                                     (const T *)vs, lse, (const T *)dO, delta,
                                                     (T *)dks, (T *)dvs);
  const unsigned ggrid = (unsigned)((rows * (LF_HD / LfVec<T>::N) + 255) / 256);  // a lane group per key
  lf_bwd_dkv_g_kernel<T><<<ggrid, 256, 0, L.stream>>>(L.dev, (const T *)qg, (const T *)kg,
                                                     (const T *)vg, lse, (const T *)dO, delta,
                                                     (T *)dkg, (T *)dvg);
  lf_launches_add(4);
  return cudaGetLastError();
}

cudaError_t lf_launch_simt_bwd(const LfLaunch &L, const void *qs, const void *ks, const void *vs,
                               const void *qg, const void *kg, const void *vg, const void *o,
                               const float *lse, const void *dO, void *dqs, void *dks, void *dvs,
                               void *dqg, void *dkg, void *dvg) {
  switch (L.dtype) {
    case LF_F32:
      return lf_simt_bwd_t<float>(L, qs, ks, vs, qg, kg, vg, o, lse, dO, dqs, dks, dvs, dqg, dkg,
                                  dvg);
    case LF_BF16:
      return lf_simt_bwd_t<__nv_bfloat16>(L, qs, ks, vs, qg, kg, vg, o, lse, dO, dqs, dks, dvs,
                                          dqg, dkg, dvg);
    default:
      return lf_simt_bwd_t<__half>(L, qs, ks, vs, qg, kg, vg, o, lse, dO, dqs, dks, dvs, dqg,
                                   dkg, dvg);
  }
}

// delta = rowsum(dO * O) alone (the tensor-core backward computes dK_g / dV_g
// together with dQ_g, in lf_bwd_gkey_kernel)
template <typename T>
static cudaError_t lf_bwd_delta_t(const LfLaunch &L, const void *o, const void *dO, float *delta) {
  const long long rows = (long long)L.dev.B * L.dev.H * L.dev.n;
  const unsigned grid = (unsigned)((rows * (LF_HD / LfVec<T>::N) + 255) / 256);  // a lane group per row
  lf_bwd_delta_kernel<T><<<grid, 256, 0, L.stream>>>(L.dev, (const T *)o, (const T *)dO, delta);
  lf_launches_add(1);
  return cudaGetLastError();
}

cudaError_t lf_launch_bwd_delta(const LfLaunch &L, const void *o, const void *dO, float *delta) {
  if (L.dtype == LF_F16) return lf_bwd_delta_t<__half>(L, o, dO, delta);
  if (L.dtype == LF_BF16) return lf_bwd_delta_t<__nv_bfloat16>(L, o, dO, delta);
  return lf_bwd_delta_t<float>(L, o, dO, delta);
}

// ============================================================ decode step

// A cluster of LF_DEC_CL CTAs of 4 warps per (b, h): the window offsets go
// in batches of 32 (one key per lane, as in the CUDA-core forward), warp w of
// CTA c taking batches c*4 + w, + 4*LF_DEC_CL, ...  Each CTA merges its
// warps' (max, sum, partial output) in shared memory and writes the result
// into CTA 0's shared memory (distributed shared memory); CTA 0 merges the
// cluster's partials and writes o and lse.  One window of r + 1 keys is a
// few hundred KB at most, so the step is latency-bound: spreading it over
// 32 warps on 8 SMs keeps each warp at one or two batches.
#define LF_DEC_CL 8
template <typename T>
__global__ void __cluster_dims__(LF_DEC_CL, 1, 1) __launch_bounds__(128)
    lf_decode_kernel(LfDev P, const T *q, const T *kc, const T *vc, const int32_t *lengths, T *o,
                     float *lse) {
  __shared__ float s_m[4], s_l[4], s_acc[4][LF_HD];
  __shared__ float c_m[LF_DEC_CL], c_l[LF_DEC_CL], c_acc[LF_DEC_CL][LF_HD];  // used in CTA 0
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the previous kernel's writes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  cg::cluster_group cluster = cg::this_cluster();
  const int crank = (int)cluster.block_rank();
  const int bh = blockIdx.x / LF_DEC_CL, h = bh % P.H, b = bh / P.H, d = P.dil[h], n = P.n;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = lengths[b];
  const size_t obase = (size_t)bh * LF_HD;
  const bool valid = L >= 1 && L <= n;
  cluster.sync();  // every CTA of the cluster runs before any remote access
  LfRowAcc<T> st;
  st.mx = -INFINITY;
  st.l = st.a0 = st.a1 = 0.f;
  if (valid) {
    const int t = L - 1;
    const int kmax = min(P.r, t / d);  // keys j = t - k*d >= 0
    const size_t base = (size_t)bh * n * LF_HD;
    lf_load_row64<T>(q + obase, st.q);
#pragma unroll
    for (int c = 0; c < 64; c++) st.q[c] *= P.scale_log2;
    st.self = t;
    for (int k0 = (crank * 4 + warp) * 32; k0 <= kmax; k0 += 4 * LF_DEC_CL * 32) {
      const int k = k0 + lane;
      st.batch(kc, vc, base, nullptr, t - k * d, k <= kmax, true, lane);
    }
  }
  if (lane == 0) {
    s_m[warp] = st.mx;
    s_l[warp] = st.l;
  }
  s_acc[warp][2 * lane] = st.a0;
  s_acc[warp][2 * lane + 1] = st.a1;
  __syncthreads();
  if (warp == 0) {
    // this CTA's partial, into slot crank of CTA 0
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; w++) M = fmaxf(M, s_m[w]);
    float Ls = 0.f, a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int w = 0; w < 4; w++) {
      if (s_m[w] == -INFINITY) continue;
      const float f = exp2f(s_m[w] - M);
      Ls += s_l[w] * f;
      a0 += s_acc[w][2 * lane] * f;
      a1 += s_acc[w][2 * lane + 1] * f;
    }
    float *rm = cluster.map_shared_rank(c_m, 0), *rl = cluster.map_shared_rank(c_l, 0);
    float *racc = cluster.map_shared_rank(&c_acc[0][0], 0);
    if (lane == 0) {
      rm[crank] = M;
      rl[crank] = Ls;
    }
    racc[crank * LF_HD + 2 * lane] = a0;
    racc[crank * LF_HD + 2 * lane + 1] = a1;
  }
  cluster.sync();  // partials in CTA 0
  if (crank == 0 && warp == 0) {
    if (!valid) {
      LfIo<T>::st2(o + obase + 2 * lane, 0.f, 0.f);
      if (lse && lane == 0) lse[bh] = -INFINITY;
      return;
    }
    float M = -INFINITY;
#pragma unroll
    for (int c = 0; c < LF_DEC_CL; c++) M = fmaxf(M, c_m[c]);
    float Ls = 0.f, a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int c = 0; c < LF_DEC_CL; c++) {
      if (c_m[c] == -INFINITY) continue;
      const float f = exp2f(c_m[c] - M);
      Ls += c_l[c] * f;
      a0 += c_acc[c][2 * lane] * f;
      a1 += c_acc[c][2 * lane + 1] * f;
    }
    LfIo<T>::st2(o + obase + 2 * lane, a0 / Ls, a1 / Ls);
    if (lse && lane == 0) lse[bh] = (M + log2f(Ls)) * LF_LN2;
  }
}

template <typename T>
static cudaError_t lf_launch_decode_t(const LfLaunch &L, const void *q, const void *kc,
                                      const void *vc, const int32_t *lengths, void *o, float *lse) {
  // programmatic dependent launch: a step's launch overlaps the previous
  // kernel on the stream (the kernel waits for it before reading anything)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(L.dev.B * L.dev.H * LF_DEC_CL));
  cfg.blockDim = dim3(128);
  cfg.stream = L.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, lf_decode_kernel<T>, L.dev, (const T *)q, (const T *)kc,
                            (const T *)vc, lengths, (T *)o, lse);
}

cudaError_t lf_launch_decode(const LfLaunch &L, const void *q, const void *kc, const void *vc,
                             const int32_t *lengths, void *o, float *lse) {
  cudaError_t e;
  switch (L.dtype) {
    case LF_F32: e = lf_launch_decode_t<float>(L, q, kc, vc, lengths, o, lse); break;
    case LF_BF16: e = lf_launch_decode_t<__nv_bfloat16>(L, q, kc, vc, lengths, o, lse); break;
    default: e = lf_launch_decode_t<__half>(L, q, kc, vc, lengths, o, lse);
  }
  if (e != cudaSuccess) return e;
  lf_launches_add(1);
  return cudaGetLastError();
}
