// noalloc.cu -- chunkwise prefill without a caller-supplied workspace and without allocating.
//
// gret_prefill_chunkwise needs a device workspace (the error word, the span tickets and flags,
// and two fp32 state slots per (sequence, head) for the look-back between spans).  Callers that
// cannot allocate device memory when they call -- for example a serving process that hands all
// device memory to its own pool at start-up, or a latency-critical loop in which a cudaMalloc
// would synchronize the device -- can use gret_prefill_chunkwise_noalloc instead.  Its scratch is
// the fixed static device array below; every GPU that loads this library holds it until exit.
#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t NOALLOC_SCRATCH_BYTES = size_t(8) << 20;   // 8 MiB

// The scratch.  In host code this name is only a host-side stand-in for the symbol, not a device
// address: the device address is obtained per device with cudaGetSymbolAddress.
__device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex g_mu;
void* g_ptr[MAX_DEVICES];

// Address of the scratch on the current device, looked up once per device and kept for the life
// of the process (a cudaDeviceReset after the first call is therefore not supported: the cached
// address would then be stale).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= MAX_DEVICES) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_ptr[dev]) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_ptr[dev] = ptr;
    }
    *out = g_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" gret_status_t gret_prefill_chunkwise_noalloc(
    const void* q, const void* k, int64_t stride_batch, int64_t stride_tok, int64_t stride_head,
    const void* v, int64_t v_stride_batch, int64_t v_stride_tok, int64_t v_stride_head,
    const float* g, float tau, float k_scale, gret_dtype_t dtype, int B, int64_t N, int H,
    int d_k, int d_v, const int32_t* cu_seqlens, int n_seqs, const float* state_in,
    float* state_out, void* o, int64_t o_stride_batch, int64_t o_stride_tok,
    int64_t o_stride_head, int chunk, gret_stream_t stream) {
    const gret::NvtxRange range("gret_prefill_chunkwise_noalloc");
    // size check on the host, before any CUDA call
    const int units = cu_seqlens ? n_seqs : B;
    const int64_t tokens = cu_seqlens ? N : (int64_t)B * N;
    if (units < 0 || tokens < 0) return GRET_ERR_INVALID_ARG;
    const size_t need = gret_prefill_workspace_size(dtype, tokens, units, H, d_k, d_v, chunk);
    if (need > NOALLOC_SCRATCH_BYTES) return GRET_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (need > 0 && scratch_address(&scratch) != cudaSuccess) return GRET_ERR_CUDA;
    return gret_prefill_chunkwise(q, k, stride_batch, stride_tok, stride_head, v, v_stride_batch,
                                  v_stride_tok, v_stride_head, g, tau, k_scale, dtype, B, N, H,
                                  d_k, d_v, cu_seqlens, n_seqs, state_in, state_out, o,
                                  o_stride_batch, o_stride_tok, o_stride_head, chunk, scratch,
                                  need > 0 ? NOALLOC_SCRATCH_BYTES : 0, stream);
}

extern "C" gret_status_t gret_prefill_noalloc_status(gret_stream_t stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return GRET_ERR_CUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return GRET_ERR_CUDA;
    void* ptr = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        ptr = g_ptr[dev];
    }
    if (!ptr) return GRET_OK;   // no call on this device has used the scratch yet
    // the error word sits at the start of the scratch, as at the start of every workspace
    return gret_workspace_status(ptr, stream);
}
