// gn_gate.cuh -- host interface of the tcgen05 GEMM kernels: the GroupNorm * swish(X W_G)
// epilogue and the q / k / v / gate-logit input projection.
#pragma once
#include "common.cuh"

namespace gret {

gret_status_t launch_gn_gate(const void* o, const void* x, const void* w_g,
                             const float* gn_weight, const float* gn_bias, float eps, int64_t T,
                             int H, int d_v, int D, void* y, cudaStream_t stream);

gret_status_t launch_qkvg_projection(const void* x, const void* w, int64_t ldw, int64_t T, int H,
                                     int D, void* q, void* k, void* v, float* g,
                                     cudaStream_t stream);

}  // namespace gret
