// lf_api.cu -- the C ABI (include/lf_attn.h): argument validation, the
// workspace carve-up, and the launch sequence of each call on the caller's
// stream.  No call allocates device memory; every device buffer, including
// the workspace, belongs to the caller.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <map>
#include <mutex>
#include <utility>

#include "lf_attn.h"
#include "lf_common.cuh"
#include "lf_tc.cuh"

static thread_local char g_err[512];
static std::atomic<uint64_t> g_launches{0};

void lf_launches_add(int k) { g_launches.fetch_add((uint64_t)k, std::memory_order_relaxed); }
uint64_t lf_launches_get() { return g_launches.load(std::memory_order_relaxed); }
static thread_local cudaEvent_t g_ev_start = nullptr, g_ev_stop = nullptr;
static thread_local int g_test_wait_us = 0, g_test_skip_tile = 0;

static int lf_fail(int code, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int lf_record_error(int code, const char *msg) { return lf_fail(code, "%s", msg); }

// Per-device launch state.  cudaFuncSetAttribute acts on the current
// device's context only, and the SM count differs between devices, so both
// are kept per (device ordinal, kernel), under one lock for callers on
// several host threads.
static std::mutex g_dev_mu;
static std::map<std::pair<int, const void *>, int> g_smem_set;  // kernel -> bytes set
static std::map<int, int> g_nsm;

cudaError_t lf_kernel_smem(const void *fn, int smem_bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  auto key = std::make_pair(dev, fn);
  auto it = g_smem_set.find(key);
  if (it != g_smem_set.end() && it->second >= smem_bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e == cudaSuccess) g_smem_set[key] = smem_bytes;
  return e;
}

int lf_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  auto it = g_nsm.find(dev);
  if (it != g_nsm.end()) return it->second;
  int nsm = 0;
  if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || nsm <= 0)
    nsm = 148;
  g_nsm[dev] = nsm;
  return nsm;
}

static int lf_cuda(cudaError_t e, const char *what) {
  if (e == cudaSuccess) return LF_OK;
  return lf_fail(LF_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

extern "C" int lf_attn_version(void) { return 1; }

extern "C" uint64_t lf_attn_launch_count(void) { return lf_launches_get(); }

extern "C" const char *lf_attn_last_error(void) { return g_err; }

extern "C" int lf_attn_set_test_hooks(uint32_t wait_limit_us, int skip_kv_tile) {
  g_err[0] = 0;
  if (wait_limit_us > 60000000u) return lf_fail(LF_ERR_INVALID, "wait limit above 60 s");
  if (skip_kv_tile < 0) return lf_fail(LF_ERR_INVALID, "skip_kv_tile must be >= 0");
  g_test_wait_us = (int)wait_limit_us;
  g_test_skip_tile = skip_kv_tile;
  return LF_OK;
}

extern "C" int lf_attn_set_timing_events(void *ev_start, void *ev_stop) {
  g_ev_start = (cudaEvent_t)ev_start;
  g_ev_stop = (cudaEvent_t)ev_stop;
  return LF_OK;
}

static size_t lf_align(size_t x) { return (x + 255) & ~(size_t)255; }

static size_t lf_dtype_bytes(int dt) { return dt == LF_F32 ? 4 : 2; }

// Validate params; fill the device block and the workspace layout.
static int lf_prepare(const lf_attn_params *p, int for_bwd, LfDev &dev, LfWs &ws) {
  g_err[0] = 0;
  if (!p) return lf_fail(LF_ERR_INVALID, "params is NULL");
  if (p->B < 1 || p->H < 1 || p->n < 1)
    return lf_fail(LF_ERR_INVALID, "B, H, n must be >= 1 (got %d, %d, %d)", p->B, p->H, p->n);
  if (p->H > LF_MAX_H) return lf_fail(LF_ERR_UNSUPPORTED, "H = %d > %d", p->H, LF_MAX_H);
  if (p->head_dim != LF_HD) return lf_fail(LF_ERR_UNSUPPORTED, "head_dim must be 64 (got %d)", p->head_dim);
  if (p->window < 0) return lf_fail(LF_ERR_INVALID, "window must be >= 0 (got %d)", p->window);
  if (p->causal != 0 && p->causal != 1) return lf_fail(LF_ERR_INVALID, "causal must be 0 or 1");
  if (p->dtype < LF_F32 || p->dtype > LF_F16) return lf_fail(LF_ERR_INVALID, "bad dtype %d", p->dtype);
  if (p->kernel < LF_KERNEL_AUTO || p->kernel > LF_KERNEL_TC)
    return lf_fail(LF_ERR_INVALID, "bad kernel selector %d", p->kernel);
  if (p->kernel == LF_KERNEL_TC && p->dtype == LF_F32)
    return lf_fail(LF_ERR_UNSUPPORTED, "the tensor-core path takes bf16 or f16, not f32");
  if (!(p->scale >= 0.f) || isinf(p->scale)) return lf_fail(LF_ERR_INVALID, "scale must be finite and >= 0");
  if ((long long)p->B * p->H * p->n > (1ll << 31) - 64)
    return lf_fail(LF_ERR_UNSUPPORTED, "B*H*n too large");
  memset(&dev, 0, sizeof(dev));
  const int n = p->n;
  int dmax = 1;
  for (int h = 0; h < p->H; h++) {
    int d = p->dilation ? p->dilation[h] : 1;
    if (d < 1) return lf_fail(LF_ERR_INVALID, "dilation[%d] = %d < 1", h, d);
    d = std::min(d, n);  // d >= n keeps only k = 0: same pattern as d = n
    dev.dil[h] = d;
    dmax = std::max(dmax, d);
  }
  // a window past the sequence end is the same as one that just reaches it
  const int r = std::min(p->window, n);
  if ((long long)r * dmax + n >= (1ll << 30))
    return lf_fail(LF_ERR_UNSUPPORTED, "window * dilation too large");
  const int G = p->max_global < 0 ? n : std::min(p->max_global, n);
  dev.B = p->B;
  dev.H = p->H;
  dev.n = n;
  dev.r = r;
  dev.causal = p->causal;
  dev.G = G;
  dev.Gk = (G + 15) / 16 * 16;
  dev.scale = p->scale > 0.f ? p->scale : 1.f / sqrtf((float)p->head_dim);
  dev.scale_log2 = dev.scale * LF_LOG2E;
  dev.chunk_tiles = LF_TC_CHUNK_TILES;
  dev.nch = (n + LF_BK * LF_TC_CHUNK_TILES - 1) / (LF_BK * LF_TC_CHUNK_TILES);

  const size_t B = p->B, H = p->H, eb = lf_dtype_bytes(p->dtype);
  const size_t Ga = std::max(G, 1), Gka = std::max(dev.Gk, 16);
  const bool tc = p->dtype != LF_F32 && p->kernel != LF_KERNEL_SIMT;
  size_t off = 0;
  ws.status = off;
  {
    ws.status_bytes = LF_ST_WORDS * 4;
    off = lf_align(off + ws.status_bytes);
  }
  ws.binfo = off;
  off = lf_align(off + B * LF_BI_WORDS * 4);
  ws.gidx = off;
  off = lf_align(off + B * Ga * 4);
  ws.grank = off;
  off = lf_align(off + B * ((size_t)n + 1) * 4);
  ws.qg_c = ws.ks_c = ws.vs_c = ws.part_acc = ws.part_ml = off;
  if (tc) {
    ws.qg_c = off;
    off = lf_align(off + B * H * Ga * LF_HD * eb);
    ws.ks_c = off;
    off = lf_align(off + B * H * Gka * LF_HD * eb);
    ws.vs_c = off;
    off = lf_align(off + B * H * Gka * LF_HD * eb);
    if (!for_bwd) {
      // split-KV partials of the global rows
      ws.part_acc = off;
      off = lf_align(off + B * H * Ga * dev.nch * LF_HD * 4);
      ws.part_ml = off;
      off = lf_align(off + B * H * Ga * dev.nch * 8);
    } else {
      // backward: per-chunk partials of the global columns (dK, dV) and rows (dQ_g)
      const size_t nchb = ((size_t)n + 63) / 64;  // rows per chunk of the global parts
      ws.part_acc = off;
      off = lf_align(off + B * H * Ga * nchb * 2 * LF_HD * 4);
      ws.part_ml = off;
      off = lf_align(off + B * H * Ga * nchb * LF_HD * 4);
    }
  }
  ws.delta = off;
  if (for_bwd) off = lf_align(off + B * H * (size_t)n * 4);
  ws.total = off;
  ws.G = (int)Ga;
  ws.Gk = (int)Gka;
  ws.nch = dev.nch;
  return LF_OK;
}

extern "C" size_t lf_attn_workspace_size(const lf_attn_params *p, int for_bwd) {
  LfDev dev;
  LfWs ws;
  if (lf_prepare(p, for_bwd ? 1 : 0, dev, ws) != LF_OK) return 0;
  return ws.total;
}

static int lf_check_ptr(const void *ptr, const char *name, bool may_be_null = false) {
  if (!ptr) return may_be_null ? LF_OK : lf_fail(LF_ERR_INVALID, "%s is NULL", name);
  if (((uintptr_t)ptr) & 15) return lf_fail(LF_ERR_INVALID, "%s is not 16-byte aligned", name);
  return LF_OK;
}

static int lf_bind_ws(const lf_attn_params *p, int for_bwd, void *workspace, size_t ws_bytes,
                      const int32_t *mask, void *stream, LfLaunch &L) {
  int st = lf_prepare(p, for_bwd, L.dev, L.ws);
  if (st) return st;
  if (!workspace) return lf_fail(LF_ERR_INVALID, "workspace is NULL");
  if (((uintptr_t)workspace) & 255) return lf_fail(LF_ERR_INVALID, "workspace is not 256-byte aligned");
  if (ws_bytes < L.ws.total)
    return lf_fail(LF_ERR_INVALID, "workspace too small: %zu < %zu bytes", ws_bytes, L.ws.total);
  if ((st = lf_check_ptr(mask, "mask"))) return st;
  L.ws_base = (char *)workspace;
  L.stream = (cudaStream_t)stream;
  L.dtype = p->dtype;
  L.dev.mask = mask;
  L.dev.status = (int32_t *)(L.ws_base + L.ws.status);
  L.dev.binfo = (int32_t *)(L.ws_base + L.ws.binfo);
  L.dev.gidx = (int32_t *)(L.ws_base + L.ws.gidx);
  L.dev.grank = (int32_t *)(L.ws_base + L.ws.grank);
  L.dev.wait_us = g_test_wait_us;
  L.dev.skip_tile = g_test_skip_tile;
  // No per-call reset (a memset node before every call): the first kernel
  // of each call zeroes the work-item counter, and the error word stays set
  // until lf_attn_status reads and clears it (a fresh workspace starts zeroed)
  return LF_OK;
}

extern "C" int lf_attn_fwd(const lf_attn_params *p, const void *q_s, const void *k_s,
                           const void *v_s, const void *q_g, const void *k_g, const void *v_g,
                           const int32_t *mask, void *o, float *lse, void *workspace,
                           size_t ws_bytes, void *stream) {
  int st;
  if ((st = lf_check_ptr(q_s, "q_s")) || (st = lf_check_ptr(k_s, "k_s")) ||
      (st = lf_check_ptr(v_s, "v_s")) || (st = lf_check_ptr(q_g, "q_g")) ||
      (st = lf_check_ptr(k_g, "k_g")) || (st = lf_check_ptr(v_g, "v_g")) ||
      (st = lf_check_ptr(o, "o")) || (st = lf_check_ptr(lse, "lse", true)))
    return st;
  LfLaunch L;
  if ((st = lf_bind_ws(p, 0, workspace, ws_bytes, mask, stream, L))) return st;
  const bool tc = p->dtype != LF_F32 && p->kernel != LF_KERNEL_SIMT;
  if (tc) {
    // the tensor-core path launches the mask pass itself; a shape outside its
    // parameter block is refused (LF_ERR_UNSUPPORTED), never run elsewhere
    LfTcArgs a{q_s, k_s, v_s, q_g, k_g, v_g, o, lse, g_ev_start, g_ev_stop};
    if ((st = lf_tc_fwd(L, a, g_err, sizeof(g_err)))) return st;
  } else {
    if ((st = lf_cuda(lf_launch_mask_pass(L), "mask pass"))) return st;
    if (g_ev_start && g_ev_stop) cudaEventRecord(g_ev_start, L.stream);
    if ((st = lf_cuda(lf_launch_simt_fwd(L, q_s, k_s, v_s, q_g, k_g, v_g, o, lse), "forward")))
      return st;
    if (g_ev_start && g_ev_stop) cudaEventRecord(g_ev_stop, L.stream);
  }
  return LF_OK;
}

extern "C" int lf_attn_bwd(const lf_attn_params *p, const void *q_s, const void *k_s,
                           const void *v_s, const void *q_g, const void *k_g, const void *v_g,
                           const int32_t *mask, const void *o, const float *lse, const void *d_o,
                           void *dq_s, void *dk_s, void *dv_s, void *dq_g, void *dk_g, void *dv_g,
                           void *workspace, size_t ws_bytes, void *stream) {
  int st;
  if ((st = lf_check_ptr(q_s, "q_s")) || (st = lf_check_ptr(k_s, "k_s")) ||
      (st = lf_check_ptr(v_s, "v_s")) || (st = lf_check_ptr(q_g, "q_g")) ||
      (st = lf_check_ptr(k_g, "k_g")) || (st = lf_check_ptr(v_g, "v_g")) ||
      (st = lf_check_ptr(o, "o")) || (st = lf_check_ptr(lse, "lse")) ||
      (st = lf_check_ptr(d_o, "d_o")) || (st = lf_check_ptr(dq_s, "dq_s")) ||
      (st = lf_check_ptr(dk_s, "dk_s")) || (st = lf_check_ptr(dv_s, "dv_s")) ||
      (st = lf_check_ptr(dq_g, "dq_g")) || (st = lf_check_ptr(dk_g, "dk_g")) ||
      (st = lf_check_ptr(dv_g, "dv_g")))
    return st;
  LfLaunch L;
  if ((st = lf_bind_ws(p, 1, workspace, ws_bytes, mask, stream, L))) return st;
  if ((st = lf_cuda(lf_launch_mask_pass(L), "mask pass"))) return st;
  if (p->dtype != LF_F32 && p->kernel != LF_KERNEL_SIMT) {
    LfTcBwdArgs a{q_s, k_s, v_s, q_g, k_g, v_g, o, lse, d_o, dq_s, dk_s, dv_s, dq_g, dk_g, dv_g};
    return lf_tc_bwd(L, a, g_err, sizeof(g_err));  // refused shapes stay refused
  }
  return lf_cuda(lf_launch_simt_bwd(L, q_s, k_s, v_s, q_g, k_g, v_g, o, lse, d_o, dq_s, dk_s, dv_s,
                                    dq_g, dk_g, dv_g),
                 "backward");
}

extern "C" int lf_attn_decode(const lf_attn_params *p, const void *q, const void *k_cache,
                              const void *v_cache, const int32_t *lengths, void *o, float *lse,
                              void *stream) {
  int st;
  if ((st = lf_check_ptr(q, "q")) || (st = lf_check_ptr(k_cache, "k_cache")) ||
      (st = lf_check_ptr(v_cache, "v_cache")) || (st = lf_check_ptr(lengths, "lengths")) ||
      (st = lf_check_ptr(o, "o")) || (st = lf_check_ptr(lse, "lse", true)))
    return st;
  LfLaunch L;
  LfWs ws;
  if ((st = lf_prepare(p, 0, L.dev, ws))) return st;
  if (!p->causal) return lf_fail(LF_ERR_INVALID, "the decode step is the causal window: set causal = 1");
  L.ws = ws;
  L.ws_base = nullptr;
  L.stream = (cudaStream_t)stream;
  L.dtype = p->dtype;
  return lf_cuda(lf_launch_decode(L, q, k_cache, v_cache, lengths, o, lse), "decode");
}

extern "C" int lf_attn_count_pairs(const lf_attn_params *p, const int32_t *mask, int64_t *counts,
                                   void *workspace, size_t ws_bytes, void *stream) {
  int st;
  if ((st = lf_check_ptr(counts, "counts"))) return st;
  LfLaunch L;
  if ((st = lf_bind_ws(p, 0, workspace, ws_bytes, mask, stream, L))) return st;
  if ((st = lf_cuda(lf_launch_mask_pass(L), "mask pass"))) return st;
  return lf_cuda(lf_launch_count(L, counts), "count");
}

extern "C" int lf_attn_mask_dump(const lf_attn_params *p, const int32_t *mask, uint8_t *out,
                                 void *workspace, size_t ws_bytes, void *stream) {
  int st;
  if (!out) return lf_fail(LF_ERR_INVALID, "out is NULL");
  LfLaunch L;
  if ((st = lf_bind_ws(p, 0, workspace, ws_bytes, mask, stream, L))) return st;
  if (p->n > 8192) return lf_fail(LF_ERR_UNSUPPORTED, "mask dump needs n <= 8192");
  if ((st = lf_cuda(lf_launch_mask_pass(L), "mask pass"))) return st;
  return lf_cuda(lf_launch_dump(L, out), "dump");
}

// ---------------------------------------------------------- cross-attention

// Parameters and workspace of lf_attn_cross_fwd: the forward's global-row
// work items with n = Lk keys and G = Lq query rows.  The key range of a
// 128-row query block is split so that there are about four work items per
// SM of a full B200 (148 SMs; a fixed count keeps the workspace size a
// function of the params alone): at most every 128-key tile its own chunk.
static int lf_cross_prepare(const lf_cross_params *p, LfDev &dev, LfWs &ws) {
  g_err[0] = 0;
  if (!p) return lf_fail(LF_ERR_INVALID, "params is NULL");
  if (p->B < 1 || p->H < 1 || p->Lq < 1 || p->Lk < 1)
    return lf_fail(LF_ERR_INVALID, "B, H, Lq, Lk must be >= 1");
  if (p->H > LF_MAX_H) return lf_fail(LF_ERR_UNSUPPORTED, "H = %d > %d", p->H, LF_MAX_H);
  if (p->head_dim != LF_HD) return lf_fail(LF_ERR_UNSUPPORTED, "head_dim must be 64 (got %d)", p->head_dim);
  if (p->dtype != LF_BF16 && p->dtype != LF_F16)
    return lf_fail(LF_ERR_INVALID, "cross-attention takes LF_BF16 or LF_F16");
  if (!(p->scale >= 0.f) || isinf(p->scale)) return lf_fail(LF_ERR_INVALID, "scale must be finite and >= 0");
  if ((long long)p->B * p->H * std::max(p->Lq, p->Lk) > (1ll << 31) - 64)
    return lf_fail(LF_ERR_UNSUPPORTED, "B*H*L too large");
  memset(&dev, 0, sizeof(dev));
  dev.B = p->B;
  dev.H = p->H;
  dev.n = p->Lk;
  dev.G = p->Lq;
  dev.Gk = (p->Lq + 15) / 16 * 16;
  dev.cross = 1;
  dev.scale = p->scale > 0.f ? p->scale : 1.f / sqrtf((float)p->head_dim);
  dev.scale_log2 = dev.scale * LF_LOG2E;
  const long long rowblocks = (long long)p->B * p->H * ((p->Lq + LF_BQ - 1) / LF_BQ);
  const int ktiles = (p->Lk + LF_BK - 1) / LF_BK;
  const int want = (int)std::min<long long>(ktiles, std::max<long long>(1, (4 * 148 + rowblocks - 1) / rowblocks));
  dev.chunk_tiles = (ktiles + want - 1) / want;
  dev.nch = (ktiles + dev.chunk_tiles - 1) / dev.chunk_tiles;
  const size_t B = p->B, H = p->H, Lq = p->Lq;
  size_t off = 0;
  ws = LfWs{};
  ws.status = off;
  ws.status_bytes = LF_ST_WORDS * 4;
  off = lf_align(off + ws.status_bytes);
  ws.binfo = off;
  off = lf_align(off + B * LF_BI_WORDS * 4);
  ws.gidx = ws.grank = ws.qg_c = ws.ks_c = ws.vs_c = ws.delta = off;
  ws.part_acc = off;
  off = lf_align(off + B * H * Lq * dev.nch * LF_HD * 4);
  ws.part_ml = off;
  off = lf_align(off + B * H * Lq * dev.nch * 8);
  ws.total = off;
  ws.G = p->Lq;
  ws.Gk = dev.Gk;
  ws.nch = dev.nch;
  return LF_OK;
}

extern "C" size_t lf_attn_cross_workspace_size(const lf_cross_params *p) {
  LfDev dev;
  LfWs ws;
  if (lf_cross_prepare(p, dev, ws) != LF_OK) return 0;
  return ws.total;
}

extern "C" int lf_attn_cross_fwd(const lf_cross_params *p, const void *q, const void *k,
                                 const void *v, const int32_t *key_mask, void *o, float *lse,
                                 void *workspace, size_t ws_bytes, void *stream) {
  int st;
  if ((st = lf_check_ptr(q, "q")) || (st = lf_check_ptr(k, "k")) || (st = lf_check_ptr(v, "v")) ||
      (st = lf_check_ptr(o, "o")) || (st = lf_check_ptr(lse, "lse", true)) ||
      (st = lf_check_ptr(key_mask, "key_mask", true)))
    return st;
  LfLaunch L;
  if ((st = lf_cross_prepare(p, L.dev, L.ws))) return st;
  if (!workspace) return lf_fail(LF_ERR_INVALID, "workspace is NULL");
  if (((uintptr_t)workspace) & 255) return lf_fail(LF_ERR_INVALID, "workspace is not 256-byte aligned");
  if (ws_bytes < L.ws.total)
    return lf_fail(LF_ERR_INVALID, "workspace too small (%zu < %zu)", ws_bytes, L.ws.total);
  L.ws_base = (char *)workspace;
  L.stream = (cudaStream_t)stream;
  L.dtype = p->dtype;
  L.dev.mask = key_mask;
  L.dev.status = (int32_t *)(L.ws_base + L.ws.status);
  L.dev.binfo = (int32_t *)(L.ws_base + L.ws.binfo);
  L.dev.gidx = L.dev.grank = nullptr;
  L.dev.wait_us = g_test_wait_us;
  L.dev.skip_tile = g_test_skip_tile;
  return lf_tc_cross_fwd(L, q, k, v, o, lse, g_ev_start, g_ev_stop, g_err, sizeof(g_err));
}

extern "C" int lf_attn_status(void *workspace, void *stream) {
  g_err[0] = 0;
  if (!workspace) return lf_fail(LF_ERR_INVALID, "workspace is NULL");
  int st;
  if ((st = lf_cuda(cudaStreamSynchronize((cudaStream_t)stream), "stream sync"))) return st;
  int32_t w[LF_ST_WORDS];
  if ((st = lf_cuda(cudaMemcpy(w, workspace, sizeof(w), cudaMemcpyDeviceToHost), "status read")))
    return st;
  if ((st = lf_cuda(cudaMemset(workspace, 0, sizeof(w)), "status clear"))) return st;
  if (w[LF_ST_CODE] == LF_OK) return LF_OK;
  const int code = w[LF_ST_CODE], det = w[LF_ST_DETAIL];
  switch (code) {
    case LF_ERR_DEVICE_INPUT:
      if (det >= 2000000)
        return lf_fail(code, "sequence %d has more global tokens than max_global", det - 2000000);
      return lf_fail(code, "sequence %d has a mask value outside {0,1,2}", det - 1000000);
    case LF_ERR_UNSUPPORTED:
      return lf_fail(code, "causal attention with global tokens (sequence %d)", det - 3000000);
    case LF_ERR_DEVICE_TIMEOUT:
      return lf_fail(code, "a device-side wait expired (site %d)", det);
    default: return lf_fail(code, "device status %d (detail %d)", code, det);
  }
}
