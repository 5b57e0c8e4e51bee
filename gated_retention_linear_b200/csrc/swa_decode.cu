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
// Bound: HBM.  The window's keys and values (2 x n x d x 2 bytes per (b, h)) are read once, in
// one pass.  One CTA of 256 threads per (b, h): 16 key groups x 16 lanes, each lane owning 8 of
// the 128 dimensions (16 bytes), so every warp load covers two whole 256-byte rows.  Each key
// group keeps an online softmax (running maximum, sum and p-weighted sum of values) over its
// keys, with the keys' and values' loads of several keys in flight at once; the 16 groups are
// combined through shared memory at the end.
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "swa.cuh"

namespace gret {
namespace {

constexpr int D = SWA_DIM;
constexpr int NT = 256;
constexpr int NG = 16;          // key groups
constexpr int UNROLL = 2;       // keys (key row + value row) in flight per lane

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 x = __bfloat1622float2(h[e]);
        f[2 * e] = x.x;
        f[2 * e + 1] = x.y;
    }
}

__global__ void __launch_bounds__(NT, 4) swa_decode_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, float scale_log2, int window, int H,
    const int32_t* __restrict__ pos, __nv_bfloat16* __restrict__ kc, __nv_bfloat16* __restrict__ vc,
    __nv_bfloat16* __restrict__ o) {
    __shared__ float gm[NG], gl[NG];
    __shared__ float part[NG][D];
    const int64_t bh = blockIdx.x;
    const int b = (int)(bh / H);
    const int tid = threadIdx.x, lane16 = tid & 15, grp = tid >> 4, warp = tid >> 5;
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

    // One pass over the window.  Key group grp takes window indices grp, grp + 16, ...; its 16
    // lanes hold 8 dimensions each of the running sum of p_j v_j, with the group's running
    // maximum m (log2 units) and sum l of p_j = 2^(s_j - m).  The loop bound is uniform over
    // each warp (its two key groups run the same number of iterations), so the shuffles always
    // have the full warp.
    float m = -INFINITY, l = 0.f;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int ib = 2 * warp; ib < n; ib += NG * UNROLL) {
        const int i0 = ib + (grp & 1);
        uint4 kr[UNROLL], vr[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int i = i0 + u * NG;
            kr[u] = make_uint4(0u, 0u, 0u, 0u);
            vr[u] = kr[u];
            if (i < n) {
                const int64_t tok = first + i;
                const int64_t row = (tok % window) * (D / 8) + lane16;
                kr[u] = tok == t ? knew[lane16] : kcb[row];
                vr[u] = tok == t ? vnew[lane16] : vcb[row];
            }
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            float kf[8];
            bf16x8_to_f32(kr[u], kf);
            float sc = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) sc = fmaf(qf[e], kf[e], sc);
#pragma unroll
            for (int of = 8; of > 0; of >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, of);
            if (i0 + u * NG < n) {
                sc *= scale_log2;
                const float mn = fmaxf(m, sc);
                const float corr = exp2f(m - mn);   // 0 on the group's first key (m = -inf)
                const float pj = exp2f(sc - mn);
                float vf[8];
                bf16x8_to_f32(vr[u], vf);
                l = fmaf(l, corr, pj);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = fmaf(acc[e], corr, pj * vf[e]);
                m = mn;
            }
        }
    }
    // combine the 16 key groups: o = sum_g 2^(m_g - M) acc_g / sum_g 2^(m_g - M) l_g
    if (lane16 == 0) {
        gm[grp] = m;
        gl[grp] = l;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) part[grp][lane16 * 8 + e] = acc[e];
    __syncthreads();
    if (tid < D) {
        float M = -INFINITY;
#pragma unroll
        for (int g2 = 0; g2 < NG; ++g2) M = fmaxf(M, gm[g2]);
        float num = 0.f, den = 0.f;
#pragma unroll
        for (int g2 = 0; g2 < NG; ++g2) {
            const float f = gl[g2] > 0.f ? exp2f(gm[g2] - M) : 0.f;   // groups with no key add 0
            num = fmaf(part[g2][tid], f, num);
            den = fmaf(gl[g2], f, den);
        }
        o[bh * D + tid] = __float2bfloat16_rn(num / den);
    }
}

}  // namespace

cudaError_t launch_swa_decode(const SwaDecodeArgs& a, cudaStream_t stream) {
    swa_decode_kernel<<<(unsigned)((int64_t)a.B * a.H), NT, 0, stream>>>(
        a.q, a.k, a.v, a.scale * 1.4426950408889634f, a.window, a.H, a.pos, a.k_cache,
        a.v_cache, a.o);
    return cudaGetLastError();
}

}  // namespace gret
