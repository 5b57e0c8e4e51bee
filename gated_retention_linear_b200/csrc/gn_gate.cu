// gn_gate.cu -- GroupNorm * swish(X W_G) epilogue (placeholder until the tcgen05 GEMM lands).
#include "gn_gate.cuh"

namespace gret {

gret_status_t launch_gn_gate(const void*, const void*, const void*, const float*, const float*,
                             float, int64_t, int, int, int, void*, cudaStream_t) {
    return GRET_ERR_UNSUPPORTED;
}

}  // namespace gret
