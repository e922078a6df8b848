// lf_tc.cuh -- host interface of the tensor-core (tcgen05) forward path.
#pragma once

#include "lf_common.cuh"

// key tiles (of 128 keys) per split of a global row's full-length reduction
#define LF_TC_CHUNK_TILES 8

struct LfTcArgs {
  const void *qs, *ks, *vs, *qg, *kg, *vg;
  void *o;
  float *lse;
  cudaEvent_t ev_start, ev_stop;  // optional timing of the attention kernel
};

// Enqueue the tensor-core forward (after the mask pass).  Returns an LF_*
// code; on failure writes a message into err.
int lf_tc_fwd(const LfLaunch &L, const LfTcArgs &a, char *err, size_t errlen);
