// decode.cu -- one recurrent gated-retention step for a batch of sequences.
//
// Page "YOCO 完全拆解：Decoder-Decoder 架构如何让 KV Cache 只存一次", section
// "单 token Decode 的实现骨架": each Self layer's decode update multiplies the old state by the
// gate and adds the outer product of the new key and value; section "路线二" then reads the
// output as o = q S with the updated state.  Per (b, h):
//     S <- gamma S + (k_scale k)^T v ,   o = q S ,   log(gamma) = logsigmoid(g) / tau.
//
// Bound: HBM.  The fp32 state (d_k x d_v x 4 bytes per head) is read once and written once;
// q, k, v, g, o are a few hundred bytes per head.  One CTA of 256 threads owns one (b, h):
// lane l of every warp owns the d_v/32 consecutive columns [l*V, l*V + V) and warp w owns the
// rows w, w+8, w+16, ...  Each warp row access is one contiguous 512-byte (d_v = 128) stretch,
// so loads and stores are fully coalesced 16-byte accesses.  All row loads of a thread are
// issued before any arithmetic to keep enough bytes in flight.  The state streams with
// evict-first hints: it is larger than L2 at batch sizes where this kernel matters.
#include "common.cuh"

namespace gret {

template <int DK, int DV, typename T>
__global__ void __launch_bounds__(256) decode_kernel(const T* __restrict__ q,
                                                     const T* __restrict__ k,
                                                     const T* __restrict__ v,
                                                     const float* __restrict__ g, float tau,
                                                     float k_scale, float* __restrict__ state,
                                                     T* __restrict__ o) {
    constexpr int V = DV / 32;            // columns per lane: 4 (d_v=128) or 2 (d_v=64)
    constexpr int R = DK / 8;             // rows per warp
    using VecF = typename std::conditional<V == 4, float4, float2>::type;
    __shared__ float sq[DK], sk[DK];
    __shared__ float partial[8][DV];

    const int64_t u = blockIdx.x;         // (b, h) flattened
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < DK; i += 256) {
        sq[i] = to_f32(q[u * DK + i]);
        sk[i] = k_scale * to_f32(k[u * DK + i]);
    }
    float vv[V];
#pragma unroll
    for (int c = 0; c < V; ++c) vv[c] = to_f32(v[u * DV + lane * V + c]);
    const float gamma = expf(logsigmoidf_(g[u]) / tau);
    __syncthreads();

    VecF* S = reinterpret_cast<VecF*>(state + u * DK * DV);
    VecF s[R];
#pragma unroll
    for (int r = 0; r < R; ++r) s[r] = __ldcs(S + (warp + 8 * r) * (DV / V) + lane);

    float acc[V];
#pragma unroll
    for (int c = 0; c < V; ++c) acc[c] = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int row = warp + 8 * r;
        const float kr = sk[row], qr = sq[row];
        float* e = reinterpret_cast<float*>(&s[r]);
#pragma unroll
        for (int c = 0; c < V; ++c) {
            e[c] = fmaf(gamma, e[c], kr * vv[c]);
            acc[c] = fmaf(qr, e[c], acc[c]);
        }
        __stcs(S + row * (DV / V) + lane, s[r]);
    }
#pragma unroll
    for (int c = 0; c < V; ++c) partial[warp][lane * V + c] = acc[c];
    __syncthreads();
    for (int j = tid; j < DV; j += 256) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) t += partial[w][j];
        o[u * DV + j] = from_f32<T>(t);
    }
}

template <typename T>
static cudaError_t launch_decode_t(const void* q, const void* k, const void* v, const float* g,
                                   float tau, float k_scale, int B, int H, int dk, int dv,
                                   float* state, void* o, cudaStream_t stream) {
    dim3 grid((unsigned)((int64_t)B * H));
    const T* Q = (const T*)q;
    const T* K = (const T*)k;
    const T* Vv = (const T*)v;
    T* O = (T*)o;
#define GRET_DECODE_CASE(DK_, DV_)                                                          \
    if (dk == DK_ && dv == DV_) {                                                           \
        decode_kernel<DK_, DV_, T><<<grid, 256, 0, stream>>>(Q, K, Vv, g, tau, k_scale,     \
                                                             state, O);                     \
        return cudaGetLastError();                                                          \
    }
    GRET_DECODE_CASE(128, 128)
    GRET_DECODE_CASE(64, 64)
    GRET_DECODE_CASE(128, 64)
    GRET_DECODE_CASE(64, 128)
#undef GRET_DECODE_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* g, float tau,
                          float k_scale, bool bf16, int B, int H, int dk, int dv, float* state,
                          void* o, cudaStream_t stream) {
    if ((int64_t)B * H == 0) return cudaSuccess;
    if (bf16)
        return launch_decode_t<__nv_bfloat16>(q, k, v, g, tau, k_scale, B, H, dk, dv, state, o,
                                              stream);
    return launch_decode_t<float>(q, k, v, g, tau, k_scale, B, H, dk, dv, state, o, stream);
}

}  // namespace gret
