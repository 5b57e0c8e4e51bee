// swa.cu -- sliding-window softmax attention prefill, the other Self-Decoder mixer of YOCO
// ("路线一：滑动窗口注意力"): position i attends to the most recent W positions of its
// sequence,
//   o_i = sum_{j = i-W+1 .. i} softmax_j(scale q_i . k_j) v_j .
// FlashAttention-style, as the page suggests for it: one CTA per 64 queries of one (batch,
// head), four warps of 16 query rows.  Key/value tiles of 64 rows stream through shared memory
// (cp.async, double-buffered, XOR-swizzled 16-byte chunks) over the window only; Q K^T and P V
// run on the tensor cores as warp-level bf16 MMAs (m16n8k16, fp32 accumulate), P as a bf16
// hi + lo pair; the softmax is online, in fp32 registers, with exp2 and the scale folded into
// log2 units.
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "swa.cuh"

namespace gret {
namespace {

constexpr int BQ = 64;          // queries per CTA
constexpr int BKV = 64;         // keys per tile
constexpr int D = SWA_DIM;      // head dimension
constexpr int NTH = 128;        // four warps
constexpr int ROWB = D * 2;     // bytes per tile row
constexpr uint32_t TILE = BQ * ROWB;          // 16 KB
constexpr size_t SMEM = 5 * (size_t)TILE;     // Q, K[2], V[2]

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Byte offset of 16-byte chunk `ch` (0..15) of row `r` in a swizzled [64][128] bf16 tile: the
// chunk index is XORed with the row's low three bits, so eight rows read at one logical chunk
// hit eight different bank groups.
__device__ __forceinline__ uint32_t swz(int r, int ch) {
    return (uint32_t)(r * ROWB + ((ch ^ (r & 7)) << 4));
}

__device__ __forceinline__ void cp16(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
                 "r"(valid ? 16 : 0));
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::); }
__device__ __forceinline__ void cp_wait_1() { asm volatile("cp.async.wait_group 1;\n" ::); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// c += a (16x16, row) * b (16x8, col), bf16 in, fp32 accumulate
__device__ __forceinline__ void mma(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// (x, y) as a bf16 pair plus the bf16 pair of what that rounding left out
__device__ __forceinline__ void split_bf16(float x, float y, uint32_t& hi, uint32_t& lo) {
    __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
    const float2 hf = __bfloat1622float2(h);
    hi = *reinterpret_cast<uint32_t*>(&h);
    lo = pack_bf16(x - hf.x, y - hf.y);
}

__global__ void __launch_bounds__(NTH) swa_kernel(SwaArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t sQ = smem_addr(smem);
    const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t N = a.N;
    const int64_t q0 = (int64_t)qb * BQ;
    const int64_t qlast = min(q0 + BQ, N) - 1;
    const int64_t kstart = max((int64_t)0, q0 - a.window + 1);
    const int64_t kt0 = (kstart / BKV) * BKV;
    const int ntiles = (int)((qlast - kt0) / BKV) + 1;
    const int64_t rstride = (int64_t)a.H * D;                        // elements per token
    const int64_t base = ((int64_t)b * N * a.H + h) * D;             // token 0 of (b, h)

    // rows [r0, r0 + 64) of q, k or v into a tile; rows at or past N are zero-filled, unread
    auto load_tile = [&](uint32_t dst, const __nv_bfloat16* src, int64_t r0) {
#pragma unroll
        for (int u = 0; u < BQ * 16 / NTH; ++u) {
            const int e = tid + NTH * u, r = e >> 4, ch = e & 15;
            const int64_t n = r0 + r;
            const bool ok = n < N;
            cp16(dst + swz(r, ch), src + base + (ok ? n : 0) * rstride + ch * 8, ok);
        }
    };
    auto sK = [&](int i) { return sQ + (uint32_t)(1 + i) * TILE; };
    auto sV = [&](int i) { return sQ + (uint32_t)(3 + i) * TILE; };

    load_tile(sQ, a.q, q0);
    load_tile(sK(0), a.k, kt0);
    load_tile(sV(0), a.v, kt0);
    cp_commit();

    const float sl2 = a.scale * 1.4426950408889634f;   // scale in log2 units
    const int64_t i0 = q0 + warp * 16 + (lane >> 2);     // this thread's two query rows
    const int64_t i1 = i0 + 8;
    float o[16][4];
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
    float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
    uint32_t qf[8][4];

    for (int t = 0; t < ntiles; ++t) {
        const int buf = t & 1;
        if (t + 1 < ntiles) {
            load_tile(sK(buf ^ 1), a.k, kt0 + (int64_t)(t + 1) * BKV);
            load_tile(sV(buf ^ 1), a.v, kt0 + (int64_t)(t + 1) * BKV);
        }
        cp_commit();
        cp_wait_1();          // everything but the tile just requested has landed
        __syncthreads();
        if (t == 0) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                ldsm_x4(sQ + swz(warp * 16 + (lane & 7) + 8 * ((lane >> 3) & 1), kk * 2 + (lane >> 4)),
                        qf[kk]);
        }
        // S = Q K^T for this warp's 16 rows and the tile's 64 keys
        float s[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
        const uint32_t kb = sK(buf), vb = sV(buf);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t r[4];
                ldsm_x4(kb + swz(np * 16 + (lane & 7) + 8 * (lane >> 4), kk * 2 + ((lane >> 3) & 1)),
                        r);
                mma(s[2 * np], qf[kk], r[0], r[1]);
                mma(s[2 * np + 1], qf[kk], r[2], r[3]);
            }
        }
        // window mask (j <= i and j > i - W), scale, online softmax
        const int64_t j0 = kt0 + (int64_t)t * BKV + 2 * (lane & 3);
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int64_t i = (e < 2) ? i0 : i1;
                const int64_t j = j0 + nt * 8 + (e & 1);
                const bool ok = j <= i && j > i - a.window;
                s[nt][e] = ok ? s[nt][e] * sl2 : -INFINITY;
                mx[e >> 1] = fmaxf(mx[e >> 1], s[nt][e]);
            }
        }
        float alpha[2], mb[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
            const float mnew = fmaxf(mrow[r], mx[r]);
            mb[r] = mnew == -INFINITY ? 0.f : mnew;    // a row with nothing visible yet
            alpha[r] = exp2f(mrow[r] - mb[r]);
            mrow[r] = mnew;
            lrow[r] *= alpha[r];
        }
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                s[nt][e] = exp2f(s[nt][e] - mb[e >> 1]);
                lrow[e >> 1] += s[nt][e];
            }
        }
#pragma unroll
        for (int dt = 0; dt < 16; ++dt) {
            o[dt][0] *= alpha[0]; o[dt][1] *= alpha[0];
            o[dt][2] *= alpha[1]; o[dt][3] *= alpha[1];
        }
        // O += P V: P's accumulator layout is the A-operand layout of the next MMA.  P goes in as
        // a bf16 hi + lo pair: one bf16 rounding of P alone costs about 2e-2 of rms over a
        // 300-1024 key window.
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t ph[4], pl[4];
            split_bf16(s[2 * kk][0], s[2 * kk][1], ph[0], pl[0]);
            split_bf16(s[2 * kk][2], s[2 * kk][3], ph[1], pl[1]);
            split_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1], ph[2], pl[2]);
            split_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3], ph[3], pl[3]);
#pragma unroll
            for (int dp = 0; dp < 8; ++dp) {
                uint32_t r[4];
                ldsm_x4_t(vb + swz(kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1), dp * 2 + (lane >> 4)),
                          r);
                mma(o[2 * dp], ph, r[0], r[1]);
                mma(o[2 * dp], pl, r[0], r[1]);
                mma(o[2 * dp + 1], ph, r[2], r[3]);
                mma(o[2 * dp + 1], pl, r[2], r[3]);
            }
        }
        __syncthreads();      // the tile's buffers may be refilled next iteration
    }

    // normalise, stage the warp's 16 rows in the Q tile, write whole 16-byte chunks
    float inv[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 1);
        lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 2);
        inv[r] = lrow[r] > 0.f ? 1.f / lrow[r] : 0.f;
    }
    const int rl0 = warp * 16 + (lane >> 2);
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) {
        const int col = dt * 8 + 2 * (lane & 3);       // element column
        const int ch = col >> 3, within = (col & 7) * 2;
        const uint32_t w0 = pack_bf16(o[dt][0] * inv[0], o[dt][1] * inv[0]);
        const uint32_t w1 = pack_bf16(o[dt][2] * inv[1], o[dt][3] * inv[1]);
        asm volatile("st.shared.u32 [%0], %1;\n" ::"r"(sQ + swz(rl0, ch) + within), "r"(w0));
        asm volatile("st.shared.u32 [%0], %1;\n" ::"r"(sQ + swz(rl0 + 8, ch) + within), "r"(w1));
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < BQ * 16 / NTH; ++u) {
        const int e = tid + NTH * u, r = e >> 4, ch = e & 15;
        const int64_t n = q0 + r;
        if (n < N) {
            uint4 val;
            asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                         : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                         : "r"(sQ + swz(r, ch)));
            *reinterpret_cast<uint4*>(a.o + base + n * rstride + ch * 8) = val;
        }
    }
}

}  // namespace

cudaError_t launch_swa(const SwaArgs& a, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(swa_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((a.N + BQ - 1) / BQ), (unsigned)a.H, (unsigned)a.B);
    swa_kernel<<<grid, NTH, SMEM, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace gret
