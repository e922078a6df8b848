/*
 * lf_proj.h -- C ABI of the projections either side of the Longformer
 * attention, in the same library as lf_attn.h (liblf_attn.so).
 *
 * The hidden states of a layer are mapped by separate affine projections
 * into the local-attention set Q_s, K_s, V_s and the global-attention set
 * Q_g, K_g, V_g ("Longformer：处理长文档的Transformer模型", segmentfault,
 * section 全局注意力的线性投影: two sets of projections, one for the sliding
 * window scores and one for the global scores); after the attention the
 * heads are concatenated and projected back to the hidden size (the output
 * projection of a transformer attention layer; the pages name the layer,
 * not this step, and the standard reading is taken).
 *
 * Layouts (row-major, contiguous, 16-byte aligned DEVICE pointers owned by
 * the caller; one dtype per call, LF_BF16 or LF_F16; fp32 accumulation; each
 * result rounded once to the dtype, to nearest even):
 *   x     [B, n, d_model]                hidden states, d_model = H * 64
 *   w_in  [nproj * d_model, d_model]     projection weights, one row per
 *                                        output feature (nn.Linear layout):
 *                                        row p*d_model + h*64 + c produces
 *                                        element c of head h of output p
 *   b_in  [nproj * d_model] or NULL      biases
 *   outs  nproj device pointers (a HOST array), each [B, H, n, 64] -- the
 *         attention library's Q/K/V layout
 *   o     [B, H, n, 64]                  attention output (heads)
 *   w_out [d_model, d_model]             output projection, input feature
 *                                        h*64 + c = element c of head h
 *   b_out [d_model] or NULL
 *   y     [B, n, d_model]
 *
 * Errors: host-side checks return LF_ERR_INVALID (null pointer, bad sizes or
 * alignment, dtype) or LF_ERR_UNSUPPORTED (head_dim != 64, H not a multiple
 * of 4); device-side problems (more selected rows than max_rows, an expired
 * bounded wait) go to the status word of the workspace (its first 32 bytes:
 * zero them once after allocating), read and cleared with
 * lf_attn_status(workspace, stream).  Every call is asynchronous on
 * `stream`; the library allocates nothing.
 */
#ifndef LF_PROJ_H
#define LF_PROJ_H

#include <stddef.h>
#include <stdint.h>

#include "lf_attn.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct lf_proj_params {
  int B;        /* sequences, >= 1 */
  int n;        /* tokens per sequence, >= 1 */
  int H;        /* heads, a multiple of 4, <= 128 */
  int head_dim; /* must be 64; d_model = H * 64 */
  int dtype;    /* LF_BF16 or LF_F16 */
} lf_proj_params;

/* Bytes of device workspace lf_proj_in / lf_proj_out need: the status
 * words, plus, when rows are selected (max_rows > 0), the selected rows'
 * positions and hidden states ([B, max_rows] int32 + [B, max_rows,
 * d_model]).  0 on invalid params. */
size_t lf_proj_workspace_size(const lf_proj_params *p, int max_rows);

/* Input projections.  For p < nproj (1..8), sequence b, head h, token t:
 *   outs[p][b, h, t, c] = sum_k x[b, t, k] * w_in[p*d_model + h*64 + c, k]
 *                         + b_in[p*d_model + h*64 + c]
 * With rows_mask == NULL every token is projected.  Otherwise
 * (rows_mask int32 [B, n], device) only the tokens with rows_mask[b, t] ==
 * rows_code are, and the other rows of outs are left untouched: e.g. Q_g at
 * the global tokens (rows_code 2) of the attention mask.  max_rows bounds
 * the selected tokens per sequence (more: LF_ERR_DEVICE_INPUT in the status
 * word, the first max_rows are projected).
 * workspace: ws_bytes >= lf_proj_workspace_size(p, rows_mask ? max_rows : 0). */
int lf_proj_in(const lf_proj_params *p, int nproj, const void *x, const void *w_in,
               const void *b_in, void *const *outs, const int32_t *rows_mask, int rows_code,
               int max_rows, void *workspace, size_t ws_bytes, void *stream);

/* Output projection: y[b, t, c] = sum_{h, j} o[b, h, t, j] * w_out[c, h*64 + j]
 *                                + b_out[c].
 * workspace: ws_bytes >= lf_proj_workspace_size(p, 0). */
int lf_proj_out(const lf_proj_params *p, const void *o, const void *w_out, const void *b_out,
                void *y, void *workspace, size_t ws_bytes, void *stream);

/* Optional timing hook: when both are non-NULL cudaEvent_t handles, the
 * following lf_proj_in / lf_proj_out calls of this thread record ev_start
 * just before and ev_stop just after their GEMM kernel.  NULL, NULL: off. */
int lf_proj_set_timing_events(void *ev_start, void *ev_stop);

#ifdef __cplusplus
}
#endif

#endif /* LF_PROJ_H */
