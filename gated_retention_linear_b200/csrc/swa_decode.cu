// swa_decode.cu -- one decode step of sliding-window attention with a ring-buffer cache.
//
// Page "YOCO 完全拆解：Decoder-Decoder 架构如何让 KV Cache 只存一次", section
// "路线一：滑动窗口注意力": position i attends only to the most recent `window` positions, so at
// decode time only those positions' keys and values are kept.  The cache of each (b, h) is a
// ring of `window` slots: token t lives in slot t % window.  Per (b, h), with t = pos[b]:
//     cache[t % window] = (k, v)
//     o = sum_{j = max(0, t - window + 1) .. t} softmax_j(scale q . k_j) v_j .
// The slot token t overwrites held token t - window, which is just out of the window, so no
// key or value of the window is lost and nothing in the window is read from the slot being
// written (the current token's key and value are taken from the inputs).
//
// Bound: HBM.  The window's keys and values (2 x n x d x 2 bytes per (b, h)) are read once.
// One CTA of 256 threads per (b, h): 16 key groups x 16 lanes, each lane owning 8 of the 128
// dimensions (16 bytes), so every warp load covers two whole 256-byte key rows.  Pass 1 forms
// the scores (lane partial dot products reduced across the 16 lanes by shuffles) into shared
// memory; the softmax maximum and sum are block reductions; pass 2 accumulates p_j v_j per lane
// and the 16 key groups are summed through shared memory.
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "swa.cuh"

namespace gret {
namespace {

constexpr int D = SWA_DIM;
constexpr int NT = 256;
constexpr int NG = 16;          // key groups
constexpr int UNROLL = 4;       // key rows in flight per lane

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 x = __bfloat1622float2(h[e]);
        f[2 * e] = x.x;
        f[2 * e + 1] = x.y;
    }
}

__device__ __forceinline__ float block_reduce(float x, float* red, bool is_max) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float y = __shfl_xor_sync(0xffffffffu, x, o);
        x = is_max ? fmaxf(x, y) : x + y;
    }
    __syncthreads();   // red may still be read by a previous reduction
    if (lane == 0) red[warp] = x;
    __syncthreads();
    x = red[0];
#pragma unroll
    for (int w = 1; w < NT / 32; ++w) x = is_max ? fmaxf(x, red[w]) : x + red[w];
    return x;
}

__global__ void __launch_bounds__(NT) swa_decode_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, float scale, int window, int H,
    const int32_t* __restrict__ pos, __nv_bfloat16* __restrict__ kc, __nv_bfloat16* __restrict__ vc,
    __nv_bfloat16* __restrict__ o) {
    extern __shared__ float sc[];          // [window] scores, then probabilities
    __shared__ float red[NT / 32];
    __shared__ float part[NG][D];
    const int64_t bh = blockIdx.x;
    const int b = (int)(bh / H);
    const int tid = threadIdx.x, lane16 = tid & 15, grp = tid >> 4;
    const int64_t t = pos[b];
    const int n = (int)(t + 1 < window ? t + 1 : window);   // keys in the window
    const int64_t first = t - n + 1;                        // token of window index 0

    const uint4* q4 = reinterpret_cast<const uint4*>(q + bh * D);
    const uint4* knew = reinterpret_cast<const uint4*>(k + bh * D);
    const uint4* vnew = reinterpret_cast<const uint4*>(v + bh * D);
    const uint4* kcb = reinterpret_cast<const uint4*>(kc + bh * (int64_t)window * D);
    const uint4* vcb = reinterpret_cast<const uint4*>(vc + bh * (int64_t)window * D);
    float qf[8];
    bf16x8_to_f32(q4[lane16], qf);
    // the new token into its slot (read by later steps only)
    const int64_t wslot = t % window;
    if (tid < 16)
        reinterpret_cast<uint4*>(kc + (bh * window + wslot) * D)[tid] = knew[tid];
    else if (tid < 32)
        reinterpret_cast<uint4*>(vc + (bh * window + wslot) * D)[tid - 16] = vnew[tid - 16];

    // pass 1: scores.  The loop bound is uniform over each warp (its two key groups 2w, 2w + 1
    // run the same number of iterations), so the shuffles always have the full warp.
    const int warp = tid >> 5;
    for (int ib = 2 * warp; ib < n; ib += NG * UNROLL) {
        const int i0 = ib + (grp & 1);
        uint4 kr[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int i = i0 + u * NG;
            kr[u] = make_uint4(0u, 0u, 0u, 0u);
            if (i < n) {
                const int64_t tok = first + i;
                kr[u] = tok == t ? knew[lane16] : kcb[(tok % window) * (D / 8) + lane16];
            }
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            float kf[8];
            bf16x8_to_f32(kr[u], kf);
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) s = fmaf(qf[e], kf[e], s);
#pragma unroll
            for (int of = 8; of > 0; of >>= 1) s += __shfl_xor_sync(0xffffffffu, s, of);
            const int i = i0 + u * NG;
            if (lane16 == 0 && i < n) sc[i] = s * scale;
        }
    }
    __syncthreads();
    float m = __int_as_float(0xff800000);   // -inf
    for (int i = tid; i < n; i += NT) m = fmaxf(m, sc[i]);
    m = block_reduce(m, red, true);
    float l = 0.f;
    for (int i = tid; i < n; i += NT) {
        const float p = __expf(sc[i] - m);
        sc[i] = p;
        l += p;
    }
    l = block_reduce(l, red, false);   // its first barrier also publishes the probabilities

    // pass 2: o = sum p_j v_j / l
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int ib = 2 * warp; ib < n; ib += NG * UNROLL) {
        const int i0 = ib + (grp & 1);
        uint4 vr[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int i = i0 + u * NG;
            vr[u] = make_uint4(0u, 0u, 0u, 0u);
            if (i < n) {
                const int64_t tok = first + i;
                vr[u] = tok == t ? vnew[lane16] : vcb[(tok % window) * (D / 8) + lane16];
            }
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int i = i0 + u * NG;
            const float p = i < n ? sc[i] : 0.f;
            float vf[8];
            bf16x8_to_f32(vr[u], vf);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = fmaf(p, vf[e], acc[e]);
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) part[grp][lane16 * 8 + e] = acc[e];
    __syncthreads();
    if (tid < D) {
        float s = 0.f;
#pragma unroll
        for (int g2 = 0; g2 < NG; ++g2) s += part[g2][tid];
        o[bh * D + tid] = __float2bfloat16_rn(s / l);
    }
}

}  // namespace

cudaError_t launch_swa_decode(const SwaDecodeArgs& a, cudaStream_t stream) {
    const size_t smem = (size_t)a.window * sizeof(float);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(swa_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return cudaErrorInvalidValue;
    swa_decode_kernel<<<(unsigned)((int64_t)a.B * a.H), NT, smem, stream>>>(
        a.q, a.k, a.v, a.scale, a.window, a.H, a.pos, a.k_cache, a.v_cache, a.o);
    return cudaGetLastError();
}

}  // namespace gret
