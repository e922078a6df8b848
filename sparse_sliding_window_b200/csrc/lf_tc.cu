// lf_tc.cu -- tensor-core forward (placeholder: routes to the CUDA-core path).
#include <stdio.h>

#include "lf_tc.cuh"

int lf_tc_fwd(const LfLaunch &L, const LfTcArgs &a, char *err, size_t errlen) {
  if (a.ev_start && a.ev_stop) cudaEventRecord(a.ev_start, L.stream);
  cudaError_t e = lf_launch_simt_fwd(L, a.qs, a.ks, a.vs, a.qg, a.kg, a.vg, a.o, a.lse);
  if (a.ev_start && a.ev_stop) cudaEventRecord(a.ev_stop, L.stream);
  if (e != cudaSuccess) {
    snprintf(err, errlen, "forward: %s", cudaGetErrorString(e));
    return LF_ERR_CUDA;
  }
  return LF_OK;
}
