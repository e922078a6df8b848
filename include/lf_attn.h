/*
 * lf_attn.h -- C ABI of the Longformer self-attention library for NVIDIA
 * B200 (sm_100a): sliding-window attention with optional per-head dilation
 * and an optional causal (one-sided) window, plus symmetric global attention
 * on the tokens the attention mask selects.
 *
 * What is computed (per batch b and head h; i = query, j = key):
 *   * attention_mask codes, int32 [B, n]: 0 = no attention (padding),
 *     1 = local attention, 2 = global attention
 *     ("Longformer", allenai README copy on gittoolsai, section 使用方法 /
 *     运行模型, the attention_mask comment).
 *   * A local query i (mask 1) attends the keys j = i + k*d, |k| <= r
 *     (causal: -r <= k <= 0), 0 <= j < n, mask[j] != 0 -- the dilated sliding
 *     window ("Longformer：处理长文档的Transformer模型", segmentfault, sections
 *     滑动窗口 and 扩张滑动窗口; the ultralytics glossary "Longformer",
 *     section "So funktioniert die Aufmerksamkeit bei Longformer": 256 tokens
 *     each side, |i - j| <= window / 2) -- plus every global token (union:
 *     a global key inside the window counts once).  Scores use Q_s, K_s,
 *     values V_s.
 *   * A global query g (mask 2) attends every key j with mask[j] != 0, with
 *     scores from Q_g, K_g and values V_g (segmentfault page, sections
 *     全局注意力 -- global attention is symmetric -- and 全局注意力的线性投影 --
 *     a second projection set Q_g, K_g, V_g for global attention).
 *   * s_ij = scale * <q_i, k_j>, scale = 1/sqrt(head_dim) unless given;
 *     o_i = sum_j softmax_j(s_ij) v_j; lse_i = log sum_j exp(s_ij).
 *   * A mask-0 query produces o_i = 0 and lse_i = -inf; its gradients are 0.
 *   * causal together with global tokens is not supported (the device sets
 *     LF_ERR_UNSUPPORTED in the status word, see lf_attn_status).
 *
 * Tensor layout: every Q/K/V/O tensor and every gradient is a contiguous
 * [B, H, n, head_dim] array of the call's dtype, 16-byte aligned; head_dim
 * must be 64.  Q_g is read only at global rows; K_g and V_g at every
 * non-masked key.  lse is float32 [B, H, n].  All pointers are DEVICE
 * pointers owned by the caller unless stated otherwise; the library keeps
 * no pointer after a call returns.  Every call is asynchronous on `stream`
 * (a cudaStream_t, NULL = legacy default stream); results are ready when
 * the stream reaches the call's end.
 *
 * Errors: each call validates its arguments on the host before any launch
 * and returns an LF_* code; the text of the last error of the calling
 * thread is lf_attn_last_error().  Problems only the device can see (a
 * mask value outside {0,1,2}, more global tokens than params.max_global,
 * causal with a global token, a bounded wait that expired) are recorded in
 * a status word inside the workspace; read it with lf_attn_status().
 */
#ifndef LF_ATTN_H
#define LF_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* return codes */
#define LF_OK 0
#define LF_ERR_INVALID 1        /* bad argument (null pointer, size, alignment, enum) */
#define LF_ERR_UNSUPPORTED 2    /* valid but not built (head_dim != 64, causal+global, ...) */
#define LF_ERR_CUDA 3           /* a CUDA runtime call or launch failed */
#define LF_ERR_DEVICE_TIMEOUT 4 /* a device-side bounded wait expired */
#define LF_ERR_DEVICE_INPUT 5   /* the device found a bad mask value or too many globals */

/* dtypes: all tensors of one call share it; lse and internal sums are fp32 */
#define LF_F32 0
#define LF_BF16 1
#define LF_F16 2

/* kernel family selection (params.kernel) */
#define LF_KERNEL_AUTO 0 /* tensor-core (tcgen05) path for bf16/f16, CUDA-core path for f32 */
#define LF_KERNEL_SIMT 1 /* CUDA-core kernels for every dtype */
#define LF_KERNEL_TC 2   /* tensor-core path; LF_ERR_UNSUPPORTED for f32 */

typedef struct lf_attn_params {
  int B;                   /* batch size, >= 1 */
  int H;                   /* heads, 1..128 */
  int n;                   /* sequence length, >= 1 */
  int head_dim;            /* must be 64 */
  int window;              /* r: one-sided window (keys i+k*d, |k| <= r), >= 0 */
  const int32_t *dilation; /* HOST array [H] of d >= 1 per head; NULL = all 1 */
  int causal;              /* 0: two-sided window; 1: k <= 0 only */
  float scale;             /* score scale; 0 => 1/sqrt(head_dim) */
  int dtype;               /* LF_F32 / LF_BF16 / LF_F16 */
  int max_global;          /* upper bound on mask==2 tokens per sequence;
                              < 0 => n.  Sizes the workspace and grids. */
  int kernel;              /* LF_KERNEL_* */
} lf_attn_params;

/* Version of this ABI (increments when a signature changes). */
int lf_attn_version(void);

/* Bytes of device workspace lf_attn_fwd (for_bwd = 0) or lf_attn_bwd
 * (for_bwd = 1) needs for these params; 0 on invalid params.  The caller
 * allocates it (256-byte aligned) and passes it to the call; the library
 * allocates nothing itself.  Its first 32 bytes are the device status
 * word: zero them once after allocating (e.g. cudaMemset); lf_attn_status
 * zeroes them again after each read, and no call needs them cleared before
 * it runs.  One workspace must not be used by two calls that may run at the
 * same time. */
size_t lf_attn_workspace_size(const lf_attn_params *p, int for_bwd);

/* Forward.  Inputs q_s..v_g [B,H,n,64], mask int32 [B,n] (device).
 * Outputs (overwritten): o [B,H,n,64]; lse float32 [B,H,n] (may be NULL
 * when no backward follows).  workspace: ws_bytes >= lf_attn_workspace_size(p,0). */
int lf_attn_fwd(const lf_attn_params *p, const void *q_s, const void *k_s,
                const void *v_s, const void *q_g, const void *k_g,
                const void *v_g, const int32_t *mask, void *o, float *lse,
                void *workspace, size_t ws_bytes, void *stream);

/* Backward of L = sum(o * d_o).  o and lse are the forward's outputs.
 * Outputs (overwritten, not accumulated): dq_s, dk_s, dv_s, dq_g, dk_g,
 * dv_g [B,H,n,64].  dq_g is zero outside global rows; every gradient row of
 * a mask-0 token is zero.  workspace: >= lf_attn_workspace_size(p,1). */
int lf_attn_bwd(const lf_attn_params *p, const void *q_s, const void *k_s,
                const void *v_s, const void *q_g, const void *k_g,
                const void *v_g, const int32_t *mask, const void *o,
                const float *lse, const void *d_o, void *dq_s, void *dk_s,
                void *dv_s, void *dq_g, void *dk_g, void *dv_g,
                void *workspace, size_t ws_bytes, void *stream);

/* Decode step of the causal (autoregressive) window: one new query per
 * sequence against a key/value cache ("Longformer：处理长文档的Transformer模型",
 * segmentfault, 实现: autoregressive language modelling with dilated
 * sliding windows).  p->causal must be 1; window r and per-head dilation d
 * as for the forward; there are no global tokens.  For sequence b with
 * lengths[b] = L >= 1 valid cache rows (the new token's own key and value
 * already appended at row L-1), the query q[b,h] attends the keys
 * j = (L-1) - k*d, k = 0..r, j >= 0.
 *   q        [B,H,64]     the new tokens' queries (device)
 *   k_cache, v_cache  [B,H,n,64]  cached keys / values, rows >= L unused
 *   lengths  int32 [B]    device
 *   o        [B,H,64]     output (overwritten); lse float32 [B,H] or NULL
 * Returns LF_ERR_INVALID for bad arguments; a length outside [1, n] gives
 * o = 0 and lse = -inf for that sequence.  Allocates nothing. */
int lf_attn_decode(const lf_attn_params *p, const void *q, const void *k_cache,
                   const void *v_cache, const int32_t *lengths, void *o,
                   float *lse, void *stream);

/* Cross-attention of the LED decoder: the decoder's queries attend the
 * whole encoder output with full (dense) attention ("Longformer：处理长文档的
 * Transformer模型", segmentfault, section Longformer-Encoder-Decoder; the LED
 * note of the allenai README copy on gittoolsai: inputs up to 16K tokens).
 * For every (b, h) and decoder position i < Lq:
 *   s_ij = scale * <q_i, k_j> over the encoder positions j < Lk with
 *   key_mask[b, j] != 0 (key_mask NULL: every j),
 *   o_i = sum_j softmax_j(s_ij) v_j,  lse_i = log sum_j exp(s_ij);
 * a query with no valid key gets o_i = 0, lse_i = -inf.
 *   q  [B,H,Lq,64], k, v [B,H,Lk,64]; o [B,H,Lq,64] (overwritten); lse
 *   float32 [B,H,Lq] or NULL; key_mask int32 [B,Lk] or NULL (device).
 * bf16 / f16 only (tensor cores); the key range of each 128-query block is
 * split over the SMs and the partial results merged (split-KV).
 * workspace: ws_bytes >= lf_attn_cross_workspace_size(p); device-side
 * problems go to its status word (lf_attn_status). */
typedef struct lf_cross_params {
  int B;        /* batch size, >= 1 */
  int H;        /* heads, 1..128 */
  int Lq;       /* decoder positions (queries) per sequence, >= 1 */
  int Lk;       /* encoder positions (keys) per sequence, >= 1 */
  int head_dim; /* must be 64 */
  float scale;  /* score scale; 0 => 1/sqrt(head_dim) */
  int dtype;    /* LF_BF16 or LF_F16 */
} lf_cross_params;

size_t lf_attn_cross_workspace_size(const lf_cross_params *p);

int lf_attn_cross_fwd(const lf_cross_params *p, const void *q, const void *k, const void *v,
                      const int32_t *key_mask, void *o, float *lse, void *workspace,
                      size_t ws_bytes, void *stream);

/* Attended (query, key) pairs per (b, h) -> counts int64 [B, H] (device),
 * enumerated with the tile walk and predicates of the forward kernels.
 * workspace: >= lf_attn_workspace_size(p, 0). */
int lf_attn_count_pairs(const lf_attn_params *p, const int32_t *mask,
                        int64_t *counts, void *workspace, size_t ws_bytes,
                        void *stream);

/* The attention pattern itself: out uint8 [B, H, n, n] (device), 1 where
 * query i attends key j, from the same predicates.  n <= 8192. */
int lf_attn_mask_dump(const lf_attn_params *p, const int32_t *mask,
                      uint8_t *out, void *workspace, size_t ws_bytes,
                      void *stream);

/* Synchronise `stream`, read and clear the device status word of
 * `workspace`; returns LF_OK or the first device-side error code recorded
 * since the previous read (LF_ERR_DEVICE_TIMEOUT, LF_ERR_DEVICE_INPUT,
 * LF_ERR_UNSUPPORTED). */
int lf_attn_status(void *workspace, void *stream);

/* Optional timing hook: when both are non-NULL cudaEvent_t handles, every
 * following lf_attn_fwd on this thread records ev_start just before and
 * ev_stop just after its main attention kernel, on the call's stream.
 * Pass NULL, NULL to turn it off. */
int lf_attn_set_timing_events(void *ev_start, void *ev_stop);

/* Test hook for the device-side failure detection, exercised without any
 * GPU fault: an expired bounded wait is made to happen on purpose.  Applies
 * to the following lf_attn_fwd /
 * lf_attn_bwd calls of the calling thread until it is called again:
 *   wait_limit_us  the limit of every bounded device wait, in microseconds
 *                  (0 = the default 1.5 s);
 *   skip_kv_tile   > 0: CTA 0 of the tensor-core forward does not load the
 *                  K/V tile of its tile stream number skip_kv_tile - 1, so the
 *                  MMA warp's wait for it expires; the CTA records
 *                  LF_ERR_DEVICE_TIMEOUT in the status word, lets its issued
 *                  copies and MMAs finish, frees its TMEM and exits (outputs of
 *                  that call are undefined).  0 = off.
 * Nothing faults, traps or hangs; the context stays usable.  Pass 0, 0 to
 * restore normal operation.  Returns LF_ERR_INVALID for a limit above 60 s
 * or a negative tile. */
int lf_attn_set_test_hooks(uint32_t wait_limit_us, int skip_kv_tile);

/* Bytes of device scratch built into the library for lf_attn_fwd_noalloc. */
#define LF_STATIC_WORKSPACE_BYTES (16u << 20)

/* Forward for callers that cannot allocate device memory -- a plugin that
 * only receives buffers from its host application, or code that must not
 * call cudaMalloc once it runs.  The pages have no counterpart of this call.
 * Same computation, arguments and results as lf_attn_fwd, without the
 * workspace: the scratch is a fixed LF_STATIC_WORKSPACE_BYTES array inside
 * the library's device image, which every GPU that loads the library holds
 * until the process exits.  Problems whose lf_attn_workspace_size exceeds it
 * are rejected with LF_ERR_UNSUPPORTED (use lf_attn_fwd).  The call allocates
 * nothing.  Every call looks up the array's device address on the current
 * device (`stream` must belong to it; a symbol lookup, no allocation, so a
 * context torn down and created again is followed); make the first call on
 * a device before any stream capture, since it may load the library's
 * device code.  All calls on a device share the one array, so calls that
 * may overlap on the GPU (other streams, other host threads) race and must
 * be serialised by the caller.  The device status word of this variant
 * lives in that array: read it with lf_attn_status_noalloc. */
int lf_attn_fwd_noalloc(const lf_attn_params *p, const void *q_s,
                        const void *k_s, const void *v_s, const void *q_g,
                        const void *k_g, const void *v_g, const int32_t *mask,
                        void *o, float *lse, void *stream);

/* Synchronise `stream`, read and clear the device status word of the
 * static scratch of lf_attn_fwd_noalloc on the current device (zero when
 * the library is loaded).  Returns LF_OK or the first device-side error of
 * the lf_attn_fwd_noalloc calls on the device since the previous read
 * (codes as for lf_attn_status).  Allocates nothing. */
int lf_attn_status_noalloc(void *stream);

/* Number of kernels this library has launched in this process so far (all
 * threads).  Lets a caller count the kernels inside a timed region. */
uint64_t lf_attn_launch_count(void);

/* Text of the calling thread's last error ("" if none). */
const char *lf_attn_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* LF_ATTN_H */
