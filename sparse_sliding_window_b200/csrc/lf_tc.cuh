// lf_tc.cuh -- host interface of the tensor-core (tcgen05) forward path.
#pragma once

#include <cuda.h>

#include "lf_common.cuh"

// key tiles (of 128 keys) per split of a global row's full-length reduction
#define LF_TC_CHUNK_TILES 8

struct LfTcArgs {
  const void *qs, *ks, *vs, *qg, *kg, *vg;
  void *o;
  float *lse;
  cudaEvent_t ev_start, ev_stop;  // optional timing of the attention kernel
};

// One run of heads with equal dilation x one residue sub-sequence: its work
// items start at `start`; `map` indexes its tensor maps (q, k, v[, dO]).
struct LfTcSeg {
  int h0, h1, d, rho, cnt, nqb, start, map;
};

// 4-D tiled TMA map over rows of 64 elements: dims {64, rows, H, B}, byte
// strides {row, head, batch}, box {64, box_rows, 1, 1}, 128-byte swizzle.
bool lf_make_map(CUtensorMap *m, int f16, const void *base, uint64_t rows, uint64_t H, uint64_t B,
                 uint64_t row_stride, uint64_t head_stride, uint64_t batch_stride,
                 uint32_t box_rows);

// Compact the Q_g / K_s / V_s rows of the global tokens (after the mask pass).
cudaError_t lf_launch_gather(const LfLaunch &L, const void *qg, const void *ks, const void *vs,
                             void *qg_c, void *ks_c, void *vs_c, int Ga, int Gka);

struct LfTcBwdArgs {
  const void *qs, *ks, *vs, *qg, *kg, *vg, *o;
  const float *lse;
  const void *dO;
  void *dqs, *dks, *dvs, *dqg, *dkg, *dvg;
};

// Enqueue the tensor-core backward (after the mask pass).
int lf_tc_bwd(const LfLaunch &L, const LfTcBwdArgs &a, char *err, size_t errlen);

// Enqueue the cross-attention forward: the global-row work items of the
// forward kernel over every query row of q against k / v (L.dev.cross = 1,
// n = keys, G = queries), then the split-KV merge.
int lf_tc_cross_fwd(const LfLaunch &L, const void *q, const void *k, const void *v, void *o,
                    float *lse, cudaEvent_t ev_start, cudaEvent_t ev_stop, char *err, size_t errlen);

// Enqueue the tensor-core forward (after the mask pass).  Returns an LF_*
// code; on failure writes a message into err.
int lf_tc_fwd(const LfLaunch &L, const LfTcArgs &a, char *err, size_t errlen);
