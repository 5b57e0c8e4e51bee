// prefill_ew.cuh -- host interface of the per-channel-gate prefill (prefill_ew.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gret {

constexpr int EW_CHUNK = 128;  // tokens per chunk (one M = 128 tensor-core tile)
constexpr int EW_DIM = 128;    // d_k = d_v

struct EwArgs {
    const __nv_bfloat16* q;    // [B, N, H, 128]
    const __nv_bfloat16* k;    // [B, N, H, 128]
    const __nv_bfloat16* v;    // [B, N, H, 128]
    const float* g;            // [B, N, H, 128] gate logits, one per key channel
    float tau, k_scale;
    int B;
    int64_t N;
    int H;
    const float* state_in;     // [B, H, 128, 128] or nullptr (zero)
    float* state_out;          // [B, H, 128, 128] or nullptr
    __nv_bfloat16* o;          // [B, N, H, 128]
    void* workspace;           // ew_workspace_bytes(B, N, H) bytes, 16-byte aligned
};

// Chunks per range (the unit of one CTA of the range kernels) for this shape on the current
// device, and the number of ranges per sequence.
int ew_range_chunks(int B, int64_t N, int H);
int64_t ew_ranges(int B, int64_t N, int H);
size_t ew_workspace_bytes(int B, int64_t N, int H);
cudaError_t launch_prefill_ew(const EwArgs& a, cudaStream_t stream);

}  // namespace gret
