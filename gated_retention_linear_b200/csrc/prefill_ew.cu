// prefill_ew.cu -- chunkwise prefill of gated retention with one gate per key channel: the
// element-wise gate that "路线二：Multi-Head Gated Retention" weighs against the head-wise
// scalar gate YOCO keeps.  CUDA cores, fp32 arithmetic on bf16 q, k, v.
//
// Per sequence and head, with alpha_t[i] = sigmoid(g_t[i])^(1/tau) for key channel i:
//   S_t[i][:] = alpha_t[i] S_{t-1}[i][:] + k_scale k_t[i] v_t ,   o_t = q_t S_t
// Chunks of C = 64 tokens; c_t[i] is channel i's inclusive cumulative log-decay in the chunk
// (the chunkwise re-association of "Prefill 与 Decode 为什么使用两种计算形态", per channel):
//   1. ew_chunk_state   dS_c = sum_m (k_scale k_m * e^{c_last - c_m})^T v_m ,  a_c = e^{c_last}
//   2. ew_state_scan    S_prev(0) = S_in,  S_prev(c+1) = a_c * S_prev(c) + dS_c  (row-wise
//                       scale; element-parallel over the state, serial over chunks)
//   3. ew_chunk_output  o_t = (q_t * e^{c_t}) S_prev(c) + sum_{m<=t} A[t][m] v_m ,
//                       A[t][m] = k_scale sum_i q_t[i] k_m[i] e^{c_t[i] - c_m[i]}
// Across sub-chunks A splits at p, the last token before t's sub-chunk: e^{c_t - c_p}
// e^{c_p - c_m}, both factors at most 1, so no scaled operand can overflow whatever the gates.
// Inside a 16-token sub-chunk it splits at the token before the sub-chunk when every channel's
// decay over the sub-chunk is moderate, and takes the exponentials pair by pair otherwise.
//
// With a scalar gate the decay of a (t, m) pair is one number, so the head-wise kernel folds it
// into a masked score matrix and runs every contraction on the tensor cores.  With a gate per
// channel the decay sits inside the contraction over i; this path pays for that with the
// chunk-state round trip through the workspace and with an exponential per channel for every
// scaled operand (per pair and channel when a sub-chunk's gates are extreme).
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "prefill_ew.cuh"

namespace gret {
namespace {

constexpr int C = EW_CHUNK;   // tokens per chunk
constexpr int SC = 16;        // tokens per sub-chunk
constexpr int D = EW_DIM;     // d_k = d_v
constexpr int NT = 256;       // threads per block of the chunk kernels
constexpr int CQS = D + 1;    // row stride (floats) of the log-decay / scaled-q tile
constexpr int SS = D + 4;     // row stride (floats) of the scaled q / k rows of a sub-chunk pair

constexpr size_t SMEM_STATE = (size_t)C * D * 4 + (size_t)C * D * 2 + D * 4;
constexpr size_t SMEM_OUT = (size_t)C * CQS * 4 + 2 * (size_t)C * D * 2 + (size_t)C * C * 4 +
                            (size_t)2 * SC * SS * 4;

__device__ __forceinline__ void unpack4(uint2 u, float* f) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
}

__device__ __forceinline__ uint2 pack4(float a, float b, float c, float d) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
    return make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
}

// Copy rows [0, L) of a [C][D] bf16 chunk tile into shared memory, zeros in rows [L, C).
__device__ __forceinline__ void load_tile(__nv_bfloat16* dst, const __nv_bfloat16* src,
                                          int64_t row0, int H, int L, int tid, int first,
                                          int nthreads) {
    for (int p = tid - first; p < C * D / 8; p += nthreads) {
        const int t = p / (D / 8), col = (p % (D / 8)) * 8;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (t < L) val = *reinterpret_cast<const uint4*>(src + (row0 + (int64_t)t * H) * D + col);
        *reinterpret_cast<uint4*>(dst + t * D + col) = val;
    }
}

// Log-decays logsigmoid(g) / tau of tokens [0, L) of the chunk into c[t * stride + i], by all
// threads of the block (no barrier inside).
__device__ __forceinline__ void log_decays(const EwArgs& a, int64_t row0, int L, int tid,
                                           float* c, int stride) {
    const float inv_tau = 1.f / a.tau;
    for (int e = tid; e < L * D; e += NT) {
        const int t = e / D, i = e - t * D;
        c[t * stride + i] = logsigmoidf_(a.g[(row0 + (int64_t)t * a.H) * D + i]) * inv_tau;
    }
}

// Thread `tid` < D: turn channel tid's log-decays into the inclusive cumulative sum over the
// chunk, in place.  Returns the chunk total.
__device__ __forceinline__ float channel_cumsum(int L, int tid, float* c, int stride) {
    float cum = 0.f;
#pragma unroll 16
    for (int t = 0; t < L; ++t) {
        cum += c[t * stride + tid];
        c[t * stride + tid] = cum;
    }
    return cum;
}

// 1. Chunk state and chunk decay.  Block (chunk, head, batch).
__global__ void __launch_bounds__(NT) ew_chunk_state(EwArgs a) {
    extern __shared__ float4 smem_f4[];
    float* kt = reinterpret_cast<float*>(smem_f4);                        // [C][D]
    __nv_bfloat16* vs = reinterpret_cast<__nv_bfloat16*>(kt + C * D);      // [C][D]
    float* clast = reinterpret_cast<float*>(vs + C * D);                  // [D]
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    const int64_t t0 = (int64_t)c * C;
    const int L = (int)min((int64_t)C, a.N - t0);
    const int64_t row0 = ((int64_t)b * a.N + t0) * a.H + h;
    const int64_t slot = ((int64_t)b * a.H + h) * a.nch + c;

    load_tile(vs, a.v, row0, a.H, L, tid, 0, NT);
    log_decays(a, row0, L, tid, kt, D);                      // kt holds c_t for now
    __syncthreads();
    if (tid < D) clast[tid] = channel_cumsum(L, tid, kt, D);
    __syncthreads();
    for (int e = tid; e < L * D; e += NT) {
        const int t = e / D, i = e - t * D;
        const float kv = __bfloat162float(a.k[(row0 + (int64_t)t * a.H) * D + i]);
        kt[e] = a.k_scale * kv * __expf(clast[i] - kt[e]);
    }
    if (tid < D) a.ws_a[slot * D + tid] = expf(clast[tid]);
    __syncthreads();

    // dS[i][j] = sum_m kt[m][i] v[m][j]: rows {ri..ri+3, 64+ri..}, columns {cj..cj+3, 64+cj..}
    const int ri = (tid >> 4) * 4, cj = (tid & 15) * 4;
    float acc[8][8];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int s = 0; s < 8; ++s) acc[r][s] = 0.f;
    for (int m = 0; m < L; ++m) {
        const float4 a0 = *reinterpret_cast<const float4*>(kt + m * D + ri);
        const float4 a1 = *reinterpret_cast<const float4*>(kt + m * D + 64 + ri);
        const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        float bv[8];
        unpack4(*reinterpret_cast<const uint2*>(vs + m * D + cj), bv);
        unpack4(*reinterpret_cast<const uint2*>(vs + m * D + 64 + cj), bv + 4);
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
            for (int s = 0; s < 8; ++s) acc[r][s] = fmaf(av[r], bv[s], acc[r][s]);
    }
    float* dS = a.ws_S + slot * (int64_t)(D * D);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int i = r < 4 ? ri + r : 64 + ri + (r - 4);
        *reinterpret_cast<float4*>(dS + i * D + cj) =
            make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
        *reinterpret_cast<float4*>(dS + i * D + 64 + cj) =
            make_float4(acc[r][4], acc[r][5], acc[r][6], acc[r][7]);
    }
}

// 2. Scan over chunks.  Block: one (batch, head) and 8 state rows; thread: one row, 4 columns.
// The chunk-state slot c is overwritten with the state entering chunk c.
__global__ void __launch_bounds__(256) ew_state_scan(EwArgs a) {
    constexpr int U = 8;   // chunks whose loads are issued together
    const int64_t bh = blockIdx.x / 16;
    const int i = (blockIdx.x % 16) * 8 + threadIdx.x / 32;
    const int j = (threadIdx.x % 32) * 4;
    const int64_t off = (int64_t)i * D + j;
    float4 S = make_float4(0.f, 0.f, 0.f, 0.f);
    if (a.state_in) S = *reinterpret_cast<const float4*>(a.state_in + bh * D * D + off);
    float* base = a.ws_S + bh * a.nch * (int64_t)(D * D) + off;
    const float* abase = a.ws_a + bh * a.nch * (int64_t)D + i;
    for (int c0 = 0; c0 < a.nch; c0 += U) {
        float4 d[U];
        float al[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (c0 + u < a.nch) {
                d[u] = *reinterpret_cast<const float4*>(base + (int64_t)(c0 + u) * (D * D));
                al[u] = abase[(int64_t)(c0 + u) * D];
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (c0 + u < a.nch) {
                *reinterpret_cast<float4*>(base + (int64_t)(c0 + u) * (D * D)) = S;
                S.x = fmaf(al[u], S.x, d[u].x);
                S.y = fmaf(al[u], S.y, d[u].y);
                S.z = fmaf(al[u], S.z, d[u].z);
                S.w = fmaf(al[u], S.w, d[u].w);
            }
        }
    }
    if (a.state_out) *reinterpret_cast<float4*>(a.state_out + bh * D * D + off) = S;
}

// 3. Chunk output.  Block (chunk, head, batch).
__global__ void __launch_bounds__(NT) ew_chunk_output(EwArgs a) {
    extern __shared__ float4 smem_f4[];
    float* cq = reinterpret_cast<float*>(smem_f4);                       // [C][CQS]: c, then q*e^c
    __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(cq + C * CQS);   // [C][D]
    __nv_bfloat16* kv = qs + C * D;                                      // [C][D]: k, then v
    float* At = reinterpret_cast<float*>(kv + C * D);                    // [C][C]: At[m][t] = A[t][m]
    float* scr = At + C * C;                                             // [2 SC][SS], or S rows
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int64_t t0 = (int64_t)c * C;
    const int L = (int)min((int64_t)C, a.N - t0);
    const int64_t row0 = ((int64_t)b * a.N + t0) * a.H + h;
    const int64_t slot = ((int64_t)b * a.H + h) * a.nch + c;

    load_tile(qs, a.q, row0, a.H, L, tid, 0, NT);
    load_tile(kv, a.k, row0, a.H, L, tid, 0, NT);
    for (int e = tid; e < C * C; e += NT) At[e] = 0.f;
    log_decays(a, row0, L, tid, cq, CQS);
    __syncthreads();
    if (tid < D) channel_cumsum(L, tid, cq, CQS);
    __syncthreads();

    // A inside each sub-chunk.  With r the token before the sub-chunk (c_r = 0 before the chunk),
    // e^{c_t - c_m} = e^{c_t - c_r} e^{c_r - c_m}: the block is a dot product of scaled rows, as
    // across sub-chunks.  The second factor exceeds 1, so the split is taken only while every
    // channel's decay over the sub-chunk stays within SPAN_MAX (both factors then stay normal
    // fp32 numbers); otherwise each pair takes its exponentials one by one.
    constexpr float SPAN_MAX = 80.f;
    for (int s = 0; s < C / SC && s * SC < L; ++s) {
        const int r0 = s * SC, last = min(r0 + SC, L) - 1;
        int wide = 0;
        if (tid < D) {
            const float cref = s == 0 ? 0.f : cq[(r0 - 1) * CQS + tid];
            wide = cref - cq[last * CQS + tid] > SPAN_MAX;
        }
        if (__syncthreads_or(wide)) {
            // one warp per (t, m) pair, lanes over the channels
            for (int it = warp; it < SC * SC; it += NT / 32) {
                const int tt = it / SC, mm = it % SC;
                const int t = r0 + tt, m = r0 + mm;
                if (mm > tt || t >= L) continue;
                float acc = 0.f;
#pragma unroll
                for (int u = 0; u < D / 32; ++u) {
                    const int i = lane + 32 * u;
                    acc += __bfloat162float(qs[t * D + i]) * __bfloat162float(kv[m * D + i]) *
                           __expf(cq[t * CQS + i] - cq[m * CQS + i]);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
                if (lane == 0) At[m * C + t] = a.k_scale * acc;
            }
        } else {
            for (int e = tid; e < 2 * SC * D; e += NT) {
                const int r = e / D, i = e - r * D;
                const float cref = s == 0 ? 0.f : cq[(r0 - 1) * CQS + i];
                const int t = r0 + (r < SC ? r : r - SC);
                float val = 0.f;
                if (t < L)
                    val = r < SC ? __bfloat162float(qs[t * D + i]) * __expf(cq[t * CQS + i] - cref)
                                 : __bfloat162float(kv[t * D + i]) * __expf(cref - cq[t * CQS + i]);
                scr[r * SS + i] = val;
            }
            __syncthreads();
            const int r = tid / SC, mm = tid % SC;
            const float* qr = scr + r * SS;
            const float* kr = scr + (SC + mm) * SS;
            float acc = 0.f;
#pragma unroll 8
            for (int i = 0; i < D; i += 4) {
                const float4 x = *reinterpret_cast<const float4*>(qr + i);
                const float4 y = *reinterpret_cast<const float4*>(kr + i);
                acc = fmaf(x.x, y.x, fmaf(x.y, y.y, fmaf(x.z, y.z, fmaf(x.w, y.w, acc))));
            }
            if (mm <= r && r0 + r < L) At[(r0 + mm) * C + r0 + r] = a.k_scale * acc;
        }
        __syncthreads();   // scr is reused by the next sub-chunk
    }

    // A across sub-chunks: rows of sub-chunk ts against columns of sub-chunk ms < ts, split at
    // p = ts * SC - 1:  q_t e^{c_t - c_p}  .  k_m e^{c_p - c_m}.
    for (int ts = 1; ts < C / SC && ts * SC < L; ++ts) {
        const int p = ts * SC - 1;
        for (int ms = 0; ms < ts; ++ms) {
            __syncthreads();   // previous readers of scr are done
            for (int e = tid; e < 2 * SC * D; e += NT) {
                const int r = e / D, i = e - r * D;
                float val = 0.f;
                if (r < SC) {
                    const int t = ts * SC + r;
                    if (t < L)
                        val = __bfloat162float(qs[t * D + i]) *
                              __expf(cq[t * CQS + i] - cq[p * CQS + i]);
                } else {
                    const int m = ms * SC + (r - SC);
                    val = __bfloat162float(kv[m * D + i]) *
                          __expf(cq[p * CQS + i] - cq[m * CQS + i]);
                }
                scr[r * SS + i] = val;
            }
            __syncthreads();
            const int r = tid / SC, mm = tid % SC;
            const float* qr = scr + r * SS;
            const float* kr = scr + (SC + mm) * SS;
            float acc = 0.f;
#pragma unroll 8
            for (int i = 0; i < D; i += 4) {
                const float4 x = *reinterpret_cast<const float4*>(qr + i);
                const float4 y = *reinterpret_cast<const float4*>(kr + i);
                acc = fmaf(x.x, y.x, fmaf(x.y, y.y, fmaf(x.z, y.z, fmaf(x.w, y.w, acc))));
            }
            if (ts * SC + r < L) At[(ms * SC + mm) * C + ts * SC + r] = a.k_scale * acc;
        }
    }
    __syncthreads();   // all of A written; k and the log-decays no longer needed as such

    // The entry state of the chunk is read in slices of SR rows, each fetched into registers
    // one slice ahead of its use; the first fetch overlaps the work below.
    constexpr int SR = 2 * SC, PF = SR * D / 4 / NT;
    const float4* Sp = reinterpret_cast<const float4*>(a.ws_S + slot * (int64_t)(D * D));
    float4 pf[PF];
#pragma unroll
    for (int u = 0; u < PF; ++u) pf[u] = Sp[tid + u * NT];

    // q * e^{c} in place (zero rows past L), and v into the k tile.
    for (int e = tid; e < C * D; e += NT) {
        const int t = e / D, i = e - t * D;
        float val = 0.f;
        if (t < L) val = __bfloat162float(qs[t * D + i]) * __expf(cq[t * CQS + i]);
        cq[t * CQS + i] = val;
    }
    load_tile(kv, a.v, row0, a.H, L, tid, 0, NT);
    __syncthreads();

    // o[t][j] for rows {tr..tr+3}, columns {cj..cj+3, 64+cj..}
    const int tr = (tid >> 4) * 4, cj = (tid & 15) * 4;
    float acc[4][8];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int s = 0; s < 8; ++s) acc[r][s] = 0.f;
    for (int m = 0; m < L; ++m) {
        const float4 av = *reinterpret_cast<const float4*>(At + m * C + tr);
        const float ar[4] = {av.x, av.y, av.z, av.w};
        float bv[8];
        unpack4(*reinterpret_cast<const uint2*>(kv + m * D + cj), bv);
        unpack4(*reinterpret_cast<const uint2*>(kv + m * D + 64 + cj), bv + 4);
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int s = 0; s < 8; ++s) acc[r][s] = fmaf(ar[r], bv[s], acc[r][s]);
    }
    for (int i0 = 0; i0 < D; i0 += SR) {
#pragma unroll
        for (int u = 0; u < PF; ++u) reinterpret_cast<float4*>(scr)[tid + u * NT] = pf[u];
        __syncthreads();
        if (i0 + SR < D) {
#pragma unroll
            for (int u = 0; u < PF; ++u) pf[u] = Sp[(i0 + SR) * D / 4 + tid + u * NT];
        }
#pragma unroll 4
        for (int ii = 0; ii < SR; ++ii) {
            float ar[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) ar[r] = cq[(tr + r) * CQS + i0 + ii];
            const float4 b0 = *reinterpret_cast<const float4*>(scr + ii * D + cj);
            const float4 b1 = *reinterpret_cast<const float4*>(scr + ii * D + 64 + cj);
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int s = 0; s < 8; ++s) acc[r][s] = fmaf(ar[r], bv[s], acc[r][s]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int t = tr + r;
        if (t >= L) continue;
        __nv_bfloat16* dst = a.o + (row0 + (int64_t)t * a.H) * D;
        *reinterpret_cast<uint2*>(dst + cj) = pack4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
        *reinterpret_cast<uint2*>(dst + 64 + cj) =
            pack4(acc[r][4], acc[r][5], acc[r][6], acc[r][7]);
    }
}

}  // namespace

size_t ew_workspace_bytes(int B, int64_t N, int H) {
    const int64_t nch = (N + C - 1) / C;
    return (size_t)B * H * nch * (size_t)(D * D + D) * sizeof(float);
}

cudaError_t launch_prefill_ew(const EwArgs& a, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(ew_chunk_state,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_STATE);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(ew_chunk_output, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_OUT);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)a.nch, (unsigned)a.H, (unsigned)a.B);
    ew_chunk_state<<<grid, NT, SMEM_STATE, stream>>>(a);
    ew_state_scan<<<(unsigned)((int64_t)a.B * a.H * 16), 256, 0, stream>>>(a);
    ew_chunk_output<<<grid, NT, SMEM_OUT, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace gret
