// lf_static.cu -- lf_attn_fwd_noalloc: the forward for callers that cannot
// allocate device memory.
//
// Some callers only ever receive device buffers from a host application and
// have no device allocator of their own (a plugin inside an inference engine
// that owns all device memory), or must not allocate once they are running
// (cudaMalloc can synchronise the device, and can fail under memory pressure
// in the middle of serving).  They pass inputs and outputs as usual; the
// scratch the forward needs lives in a fixed-size array that is part of this
// library's device image.  Every GPU that loads the library holds
// LF_STATIC_WORKSPACE_BYTES of device memory for it until the process exits.
//
// On the host, the array's name is only a host-side stand-in for the device
// symbol, never a device address; the device address comes from
// cudaGetSymbolAddress with the caller's device current, on every call (a
// lookup, no allocation), so nothing goes stale when a context is torn down
// and created again.
#include <stdio.h>

#include "lf_attn.h"

static __device__ __align__(256) unsigned char lf_static_ws[LF_STATIC_WORKSPACE_BYTES];

// defined in lf_api.cu: record an error for lf_attn_last_error()
int lf_record_error(int code, const char *msg);

// Device address of the static scratch on the current device.
static int lf_static_base(void **base, const char *who) {
  void *ptr = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&ptr, lf_static_ws);
  if (e != cudaSuccess || !ptr) {
    char msg[160];
    snprintf(msg, sizeof(msg), "%s: cudaGetSymbolAddress failed (%s)", who, cudaGetErrorString(e));
    return lf_record_error(LF_ERR_CUDA, msg);
  }
  *base = ptr;
  return LF_OK;
}

extern "C" int lf_attn_fwd_noalloc(const lf_attn_params *p, const void *q_s, const void *k_s,
                                   const void *v_s, const void *q_g, const void *k_g,
                                   const void *v_g, const int32_t *mask, void *o, float *lse,
                                   void *stream) {
  const size_t need = lf_attn_workspace_size(p, 0);
  if (need == 0)  // invalid params: let the regular entry point name the problem
    return lf_attn_fwd(p, q_s, k_s, v_s, q_g, k_g, v_g, mask, o, lse, nullptr, 0, stream);
  if (need > (size_t)LF_STATIC_WORKSPACE_BYTES) {
    char msg[192];
    snprintf(msg, sizeof(msg),
             "lf_attn_fwd_noalloc: this problem needs %zu bytes of scratch, the static scratch "
             "holds %zu; use lf_attn_fwd with a caller-allocated workspace",
             need, (size_t)LF_STATIC_WORKSPACE_BYTES);
    return lf_record_error(LF_ERR_UNSUPPORTED, msg);
  }
  void *base = nullptr;
  const int st = lf_static_base(&base, "lf_attn_fwd_noalloc");
  if (st != LF_OK) return st;
  // The regular forward zeroes the work-item counter in its first kernel and
  // fully writes every other scratch region before reading it; the status
  // word (zero at load, like every __device__ array) keeps the first error
  // until lf_attn_status_noalloc reads and clears it.
  return lf_attn_fwd(p, q_s, k_s, v_s, q_g, k_g, v_g, mask, o, lse, base,
                     (size_t)LF_STATIC_WORKSPACE_BYTES, stream);
}

// The device status word of the static scratch: the same read-and-clear as
// lf_attn_status, on the array of the current device.  Allocates nothing.
extern "C" int lf_attn_status_noalloc(void *stream) {
  void *base = nullptr;
  const int st = lf_static_base(&base, "lf_attn_status_noalloc");
  if (st != LF_OK) return st;
  return lf_attn_status(base, stream);
}
