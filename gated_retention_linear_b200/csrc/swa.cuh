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

// Largest window the decode step takes: its scores live in shared memory (4 bytes each).
constexpr int SWA_DECODE_MAX_WINDOW = 32768;

struct SwaDecodeArgs {
    const __nv_bfloat16* q;    // [B, H, 128]
    const __nv_bfloat16* k;    // [B, H, 128]
    const __nv_bfloat16* v;    // [B, H, 128]
    float scale;
    int window;
    int B, H;
    const int32_t* pos;        // [B] device: index of the new token in its sequence
    __nv_bfloat16* k_cache;    // [B, H, window, 128] ring buffer, slot t % window = token t
    __nv_bfloat16* v_cache;
    __nv_bfloat16* o;          // [B, H, 128]
};

cudaError_t launch_swa_decode(const SwaDecodeArgs& a, cudaStream_t stream);

}  // namespace gret
