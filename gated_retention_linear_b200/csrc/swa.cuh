// swa.cuh -- host interface of the sliding-window attention prefill (swa.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gret {

constexpr int SWA_DIM = 128;   // head dimension

struct SwaArgs {
    const __nv_bfloat16* q;    // [B, N, H, 128]
    const __nv_bfloat16* k;    // [B, N, H, 128]
    const __nv_bfloat16* v;    // [B, N, H, 128]
    __nv_bfloat16* o;          // [B, N, H, 128]
    float scale;               // score scale (1/sqrt(d) in the usual reading)
    int window;                // positions each query sees, itself included (>= 1)
    int B;
    int64_t N;
    int H;
};

cudaError_t launch_swa(const SwaArgs& a, cudaStream_t stream);

}  // namespace gret
