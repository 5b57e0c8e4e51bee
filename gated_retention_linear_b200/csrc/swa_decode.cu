// swa_decode.cu -- one decode step of sliding-window attention with a ring-buffer cache.
//
// Page "YOCO 完全拆解：Decoder-Decoder 架构如何让 KV Cache 只存一次", section
// "路线一：滑动窗口注意力": position i attends only to the most recent `window` positions, so at
// decode time only those positions' keys and values are kept.  The cache of each (b, h) is a
// ring of `window` slots: token t lives in slot t % window.  Per (b, h), with t = pos[b]:
//     cache[t % window] = (k, v)
//     o = sum_{j = max(0, t - window + 1) .. t} softmax_j(scale q . k_j) v_j .
// The slot token t overwrites held token t - window, which is just out of the window, so no
// key or value of the window is lost; the current token's key and value are taken from the
// inputs, never from the slot being written.
//
// Bound: HBM.  The window's keys and values (2 x n x d x 2 bytes per (b, h)) are read once.  The
// keys of the window occupy slots 0 .. n - 1 of the ring (all of them once t >= window - 1), one
// contiguous block of the cache, and softmax attention does not depend on the order of its keys:
// a producer warp streams the block in chunks of 32 slots (8 KB of keys and 8 KB of values) by
// bulk copy into a four-stage shared-memory ring, so that three chunks are in flight per CTA
// without holding registers.  Eight consumer warps, 16 key groups x 16 lanes, each lane owning 8
// of the 128 dimensions (16 bytes), keep an online softmax per key group (running maximum, sum
// and p-weighted sum of values) over the slots they take; the 16 groups are combined through
// shared memory at the end.  Every wait is bounded; a wait that gives up makes the CTA write NaN.
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "sm100.cuh"
#include "swa.cuh"

namespace gret {

using namespace sm100;

namespace {

constexpr int D = SWA_DIM;
constexpr int NG = 16;          // key groups (two per consumer warp)
constexpr int NCW = 8;          // consumer warps
constexpr int NT = 32 * (NCW + 1);
constexpr int CH = 32;          // cache slots per chunk
constexpr int STAGES = 4;
constexpr int ROW = D * 2;      // bytes of one cached key or value
constexpr uint64_t WAIT_NS = 2000000000ull;
constexpr uint64_t DRAIN_NS = 200000000ull;

struct __align__(128) DecSmem {
    unsigned char k[STAGES][CH * ROW];
    unsigned char v[STAGES][CH * ROW];
    uint64_t full[STAGES], empty[STAGES];
    float gm[NG], gl[NG];
    float part[NG][D];
    uint32_t abort;
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 x = __bfloat1622float2(h[e]);
        f[2 * e] = x.x;
        f[2 * e + 1] = x.y;
    }
}

__global__ void __launch_bounds__(NT, 3) swa_decode_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, float scale_log2, int window, int H,
    const int32_t* __restrict__ pos, __nv_bfloat16* __restrict__ kc, __nv_bfloat16* __restrict__ vc,
    __nv_bfloat16* __restrict__ o) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    DecSmem& sm = *reinterpret_cast<DecSmem*>(smem_raw);
    const int64_t bh = blockIdx.x;
    const int b = (int)(bh / H);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t t = pos[b];
    const int n = (int)(t + 1 < window ? t + 1 : window);   // keys in the window = slots read
    const int wslot = (int)(t % window);                     // the new token's slot
    const int nch = (n + CH - 1) / CH;
    const unsigned char* kcb = reinterpret_cast<const unsigned char*>(kc + bh * (int64_t)window * D);
    const unsigned char* vcb = reinterpret_cast<const unsigned char*>(vc + bh * (int64_t)window * D);
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], NCW);
        }
        sm.abort = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == NCW) {
        // ---- producer: chunk c of the window's slots into stage c % STAGES
        if (lane == 0) {
            int c = 0;
            for (; c < nch; ++c) {
                const int s = c % STAGES;
                if (c >= STAGES &&
                    !mbar_wait(&sm.empty[s], ((c / STAGES) - 1) & 1, &sm.abort, WAIT_NS)) {
                    atomicExch(&sm.abort, 1u);
                    break;
                }
                const int rows = n - c * CH < CH ? n - c * CH : CH;
                const uint32_t bytes = (uint32_t)rows * ROW;
                mbar_arrive_expect_tx(&sm.full[s], 2 * bytes);
                bulk_load(sm.k[s], kcb + (int64_t)c * CH * ROW, bytes, &sm.full[s]);
                bulk_load(sm.v[s], vcb + (int64_t)c * CH * ROW, bytes, &sm.full[s]);
            }
            // no bulk copy into this CTA's shared memory may be in flight at exit
            for (int cc = (c >= STAGES ? c - STAGES : 0); cc < c; ++cc) {
                uint32_t never = 0;
                mbar_wait(&sm.full[cc % STAGES], (cc / STAGES) & 1, &never, DRAIN_NS);
            }
        }
    } else {
        // ---- consumers: key group grp (16 lanes, 8 dimensions each) takes slots grp and
        // grp + 16 of every chunk
        const int lane16 = lane & 15, grp = tid >> 4;
        const uint4* q4 = reinterpret_cast<const uint4*>(q + bh * D);
        const uint4* knew = reinterpret_cast<const uint4*>(k + bh * D);
        const uint4* vnew = reinterpret_cast<const uint4*>(v + bh * D);
        float qf[8];
        bf16x8_to_f32(q4[lane16], qf);
        const uint4 kn = knew[lane16], vn = vnew[lane16];
        // the new token into its slot (read by later steps only: this step takes the slot's key
        // and value from the inputs)
        if (tid < 16)
            reinterpret_cast<uint4*>(kc + (bh * window + wslot) * D)[tid] = kn;
        else if (tid < 32)
            reinterpret_cast<uint4*>(vc + (bh * window + wslot) * D)[tid - 16] = vn;
        float m = -INFINITY, l = 0.f;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int c = 0; c < nch; ++c) {
            const int s = c % STAGES;
            // lane 0 waits; the whole warp takes its outcome (the loop's shuffles and
            // __syncwarp need every lane)
            int okw = 1;
            if (lane == 0 && !mbar_wait(&sm.full[s], (c / STAGES) & 1, &sm.abort, WAIT_NS)) {
                atomicExch(&sm.abort, 1u);
                okw = 0;
            }
            if (!__shfl_sync(0xffffffffu, okw, 0)) break;
            const int rows = n - c * CH < CH ? n - c * CH : CH;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                // slot c * CH + j of the window.  Every lane computes a score (row j is always
                // inside the stage buffer), so that the 16-lane shuffles see the whole warp; only
                // slots of the window update the softmax.
                const int j = grp + NG * u;
                const bool valid = j < rows;
                const int slot = c * CH + j;
                const uint4 kr = slot == wslot ? kn
                                 : *reinterpret_cast<const uint4*>(sm.k[s] + j * ROW + lane16 * 16);
                const uint4 vr = slot == wslot ? vn
                                 : *reinterpret_cast<const uint4*>(sm.v[s] + j * ROW + lane16 * 16);
                float kf[8];
                bf16x8_to_f32(kr, kf);
                float sc = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) sc = fmaf(qf[e], kf[e], sc);
#pragma unroll
                for (int of = 8; of > 0; of >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, of, 16);
                if (!valid) continue;
                sc *= scale_log2;
                const float mn = fmaxf(m, sc);
                const float corr = exp2f(m - mn);   // 0 on the group's first key (m = -inf)
                const float pj = exp2f(sc - mn);
                float vf[8];
                bf16x8_to_f32(vr, vf);
                l = fmaf(l, corr, pj);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = fmaf(acc[e], corr, pj * vf[e]);
                m = mn;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[s]);   // this warp is done with the stage
        }
        if (lane16 == 0) {
            sm.gm[grp] = m;
            sm.gl[grp] = l;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) sm.part[grp][lane16 * 8 + e] = acc[e];
    }
    __syncthreads();
    // combine the 16 key groups: o = sum_g 2^(m_g - M) acc_g / sum_g 2^(m_g - M) l_g
    if (tid < D) {
        float M = -INFINITY;
#pragma unroll
        for (int g2 = 0; g2 < NG; ++g2) M = fmaxf(M, sm.gm[g2]);
        float num = 0.f, den = 0.f;
#pragma unroll
        for (int g2 = 0; g2 < NG; ++g2) {
            const float f = sm.gl[g2] > 0.f ? exp2f(sm.gm[g2] - M) : 0.f;   // groups with no key add 0
            num = fmaf(sm.part[g2][tid], f, num);
            den = fmaf(sm.gl[g2], f, den);
        }
        const float res = sm.abort ? __int_as_float(0x7fc00000) : num / den;
        o[bh * D + tid] = __float2bfloat16_rn(res);
    }
}

}  // namespace

cudaError_t launch_swa_decode(const SwaDecodeArgs& a, cudaStream_t stream) {
    const size_t smem = sizeof(DecSmem);
    cudaError_t e = cudaFuncSetAttribute(swa_decode_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    swa_decode_kernel<<<(unsigned)((int64_t)a.B * a.H), NT, smem, stream>>>(
        a.q, a.k, a.v, a.scale * 1.4426950408889634f, a.window, a.H, a.pos, a.k_cache,
        a.v_cache, a.o);
    return cudaGetLastError();
}

}  // namespace gret
