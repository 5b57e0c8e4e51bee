// decode.cu -- one recurrent gated-retention step for a batch of sequences.
//
// Page "YOCO 完全拆解：Decoder-Decoder 架构如何让 KV Cache 只存一次", section
// "单 token Decode 的实现骨架": each Self layer's decode update multiplies the old state by the
// gate and adds the outer product of the new key and value; section "路线二" then reads the
// output as o = q S with the updated state.  Per (b, h):
//     S <- gamma S + (k_scale k)^T v ,   o = q S ,   log(gamma) = logsigmoid(g) / tau.
//
// Bound: HBM.  The fp32 state (d_k x d_v x 4 bytes per head) is read once and written once;
// q, k, v, g, o are a few hundred bytes per head.  One CTA of 256 threads owns one block of 64
// columns of one (b, h) state, so the output needs no reduction across CTAs and a 64 x 24 batch
// gives 3072 CTAs (finer than one per head, which left a two-thirds-empty last wave).  Lane l
// of a warp owns 4 consecutive columns and one of 32 / 16 = 2 rows per pass; each warp row
// access is one contiguous 256-byte stretch of 16-byte loads.  All row loads of a thread are
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
    constexpr int CB = 64;                // columns per CTA
    constexpr int NB = DV / CB;           // column blocks per head
    constexpr int LPR = CB / 4;           // lanes per row (one float4 each)
    constexpr int RPW = 32 / LPR;         // rows per warp per pass
    constexpr int RPP = 8 * RPW;          // rows per pass of the 8 warps
    constexpr int R = DK / RPP;           // passes
    static_assert(DV % CB == 0 && DK % RPP == 0, "decode tiling");
    __shared__ float sq[DK], sk[DK];
    __shared__ float partial[RPP][CB];

    const int64_t u = blockIdx.x / NB;    // (b, h) flattened
    const int cb = (int)(blockIdx.x % NB);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cl = lane % LPR, rs = lane / LPR;
    const int row0 = warp * RPW + rs;     // this thread's rows: row0 + RPP * r
    const int col0 = cb * CB + cl * 4;
    for (int i = tid; i < DK; i += 256) {
        sq[i] = to_f32(q[u * DK + i]);
        sk[i] = k_scale * to_f32(k[u * DK + i]);
    }
    float vv[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) vv[c] = to_f32(v[u * DV + col0 + c]);
    const float gamma = expf(logsigmoidf_(g[u]) / tau);
    __syncthreads();

    float4* S = reinterpret_cast<float4*>(state + u * DK * DV) + col0 / 4;
    float4 s[R];
#pragma unroll
    for (int r = 0; r < R; ++r) s[r] = __ldcs(S + (row0 + RPP * r) * (DV / 4));

    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int row = row0 + RPP * r;
        const float kr = sk[row], qr = sq[row];
        float* e = reinterpret_cast<float*>(&s[r]);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            e[c] = fmaf(gamma, e[c], kr * vv[c]);
            acc[c] = fmaf(qr, e[c], acc[c]);
        }
        __stcs(S + row * (DV / 4), s[r]);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) partial[warp * RPW + rs][cl * 4 + c] = acc[c];
    __syncthreads();
    for (int j = tid; j < CB; j += 256) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < RPP; ++w) t += partial[w][j];
        o[u * DV + cb * CB + j] = from_f32<T>(t);
    }
}

template <typename T>
static cudaError_t launch_decode_t(const void* q, const void* k, const void* v, const float* g,
                                   float tau, float k_scale, int B, int H, int dk, int dv,
                                   float* state, void* o, cudaStream_t stream) {
    if (dv % 64 != 0) return cudaErrorInvalidValue;
    dim3 grid((unsigned)((int64_t)B * H * (dv / 64)));
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
