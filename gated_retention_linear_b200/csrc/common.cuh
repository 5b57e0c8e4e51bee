// common.cuh -- small helpers shared by the gated-retention kernels (device side).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gret.h"

namespace gret {

// log(sigmoid(x)) without overflow: min(x, 0) - log(1 + exp(-|x|)).
// Used for the per-token log-decay log(gamma) = logsigmoid(g) / tau ("路线二" gate).
__device__ __forceinline__ float logsigmoidf_(float x) {
    return fminf(x, 0.f) - log1pf(expf(-fabsf(x)));
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Error word at the start of every prefill workspace (see gret_workspace_status).
enum : uint32_t { WS_ERR_NONE = 0, WS_ERR_TIMEOUT = 1 };

}  // namespace gret

// Host side: an NVTX range over the scope (the header-only NVTX v3 API; with no tool attached a
// push or pop is a no-op), so that profilers show each ABI call by name around its launches.
#include <nvtx3/nvToolsExt.h>

namespace gret {

struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

}  // namespace gret

// Host-side launchers (defined in the kernel files, called from api.cu).
namespace gret {

struct PrefillArgs {
    const void* q;
    const void* k;
    const void* v;
    int64_t sb, st, sh;     // q/k strides (elements)
    int64_t vsb, vst, vsh;  // v strides (elements)
    const float* g;
    float tau, k_scale;
    int B;
    int64_t N;
    int H, dk, dv;
    const int32_t* cu_seqlens;  // device, or nullptr (dense)
    int n_seqs;                 // units: B (dense) or n_seqs (varlen)
    const float* state_in;
    float* state_out;
    void* o;
    int64_t osb, ost, osh;  // o strides (elements)
    int chunk;
    void* workspace;
    size_t workspace_bytes;
    cudaStream_t stream;
    // Failure-path testing only (gret_prefill_chunkwise_testing): the limit of every bounded
    // wait of the tensor-core kernel (0 = the default), and the first span ticket handed out
    // (0 = normal; a value past span 0 of a chain leaves its look-back flag forever unset).
    uint64_t test_wait_ns = 0;
    uint32_t test_first_ticket = 0;
};

cudaError_t launch_prefill_simt(const PrefillArgs& a, bool bf16);
cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* g, float tau,
                          float k_scale, bool bf16, int B, int H, int dk, int dv, float* state,
                          void* o, cudaStream_t stream);

}  // namespace gret
