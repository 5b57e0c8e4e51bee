// prefill_simt.cu -- chunkwise gated-retention prefill on CUDA cores (fp32 arithmetic).
//
// Page "YOCO 完全拆解：Decoder-Decoder 架构如何让 KV Cache 只存一次", section
// "Prefill 与 Decode 为什么使用两种计算形态": inside a chunk [a, b] every position is computed
// in parallel from the chunk's own keys and values plus the state carried in from the previous
// chunk; only the chunk-end state is passed on.  With c_t the in-chunk inclusive cumulative
// log-decay and S the entry state:
//     o_t = sum_{m=a..t} exp(c_t - c_m) (q_t . k_m) v_m + exp(c_t) q_t S
//     S  <- exp(c_b) S + sum_{m=a..b} exp(c_b - c_m) k_m^T v_m
//
// This path serves fp32 inputs (full fp32 arithmetic; tensor-core TF32 would not hold a 1e-4
// relative error) and the shapes the tensor-core kernel does not take.  One CTA of 256 threads
// owns one (sequence, head) and walks its chunks in order; the fp32 state stays in shared
// memory for the whole sequence.  It is a correctness-first kernel, not the bf16 hot path.
#include "common.cuh"

namespace gret {

template <int DK, int DV, int C, typename T>
struct SimtSmem {
    float q[C][DK + 1];
    float k[C][DK + 1];
    float v[C][DV];
    float a[C][C + 1];
    float s[DK][DV];
    float c[C];      // in-chunk cumulative log-decay
    float w[C];      // exp(c_b - c_m): weight of token m in the chunk-end state
};

template <int DK, int DV, int C, typename T>
__global__ void __launch_bounds__(256) prefill_simt_kernel(PrefillArgs p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto& sm = *reinterpret_cast<SimtSmem<DK, DV, C, T>*>(smem_raw);
    const int tid = threadIdx.x;
    const int h = blockIdx.x;
    const int unit = blockIdx.y;

    int64_t b, t0, len;
    if (p.cu_seqlens) {
        b = 0;
        t0 = p.cu_seqlens[unit];
        len = p.cu_seqlens[unit + 1] - t0;
    } else {
        b = unit;
        t0 = 0;
        len = p.N;
    }
    const T* Q = (const T*)p.q + b * p.sb + h * p.sh;
    const T* K = (const T*)p.k + b * p.sb + h * p.sh;
    const T* V = (const T*)p.v + b * p.vsb + h * p.vsh;
    T* O = (T*)p.o + b * p.osb + h * p.osh;
    const float* G = p.g + (b * p.N) * p.H + h;
    const int64_t sidx = ((int64_t)unit * p.H + h) * DK * DV;

    for (int e = tid; e < DK * DV; e += 256)
        (&sm.s[0][0])[e] = p.state_in ? p.state_in[sidx + e] : 0.f;

    for (int64_t a0 = 0; a0 < len; a0 += C) {
        const int n = (int)((len - a0) < C ? (len - a0) : C);  // valid rows in this chunk
        __syncthreads();  // previous chunk is done with q/k/v/a/c/w
        for (int e = tid; e < C * DK; e += 256) {
            int r = e / DK, i = e % DK;
            int64_t t = t0 + a0 + r;
            float qv = 0.f, kv = 0.f;
            if (r < n) {
                qv = to_f32(Q[t * p.st + i]);
                kv = p.k_scale * to_f32(K[t * p.st + i]);
            }
            sm.q[r][i] = qv;
            sm.k[r][i] = kv;
        }
        for (int e = tid; e < C * DV; e += 256) {
            int r = e / DV, j = e % DV;
            int64_t t = t0 + a0 + r;
            sm.v[r][j] = (r < n) ? to_f32(V[t * p.vst + j]) : 0.f;
        }
        if (tid < C) sm.c[tid] = (tid < n) ? logsigmoidf_(G[(t0 + a0 + tid) * p.H]) / p.tau : 0.f;
        __syncthreads();
        if (tid == 0) {
            float run = 0.f;
            for (int r = 0; r < n; ++r) {
                run += sm.c[r];
                sm.c[r] = run;
            }
        }
        __syncthreads();
        if (tid < C) sm.w[tid] = (tid < n) ? expf(sm.c[n - 1] - sm.c[tid]) : 0.f;

        // A[t][m] = exp(c_t - c_m) (q_t . k_m) for m <= t < n, else 0
        for (int e = tid; e < C * C; e += 256) {
            int t = e / C, m = e % C;
            float acc = 0.f;
            if (m <= t && t < n) {
#pragma unroll 8
                for (int i = 0; i < DK; ++i) acc = fmaf(sm.q[t][i], sm.k[m][i], acc);
                acc *= expf(sm.c[t] - sm.c[m]);
            }
            sm.a[t][m] = acc;
        }
        __syncthreads();

        // o_t = sum_m A[t][m] v_m + exp(c_t) q_t S
        for (int e = tid; e < C * DV; e += 256) {
            int t = e / DV, j = e % DV;
            if (t >= n) continue;
            float inner = 0.f, cross = 0.f;
            for (int m = 0; m <= t; ++m) inner = fmaf(sm.a[t][m], sm.v[m][j], inner);
#pragma unroll 8
            for (int i = 0; i < DK; ++i) cross = fmaf(sm.q[t][i], sm.s[i][j], cross);
            float out = inner + expf(sm.c[t]) * cross;
            O[(t0 + a0 + t) * p.ost + j] = from_f32<T>(out);
        }
        __syncthreads();  // every read of the entry state is done

        // S <- exp(c_b) S + sum_m exp(c_b - c_m) k_m^T v_m
        const float eb = expf(sm.c[n - 1]);
        for (int e = tid; e < DK * DV; e += 256) {
            int i = e / DV, j = e % DV;
            float acc = 0.f;
            for (int m = 0; m < n; ++m) acc = fmaf(sm.w[m] * sm.k[m][i], sm.v[m][j], acc);
            sm.s[i][j] = fmaf(eb, sm.s[i][j], acc);
        }
    }
    __syncthreads();
    if (p.state_out)
        for (int e = tid; e < DK * DV; e += 256) p.state_out[sidx + e] = (&sm.s[0][0])[e];
}

template <int DK, int DV, int C, typename T>
static cudaError_t launch_simt_t(const PrefillArgs& a) {
    auto kern = prefill_simt_kernel<DK, DV, C, T>;
    const size_t smem = sizeof(SimtSmem<DK, DV, C, T>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.H, a.n_seqs);
    kern<<<grid, 256, smem, a.stream>>>(a);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_simt_dt(const PrefillArgs& a) {
    const int C = a.chunk;
#define GRET_SIMT_CASE(DK_, DV_, C_) \
    if (a.dk == DK_ && a.dv == DV_ && C == C_) return launch_simt_t<DK_, DV_, C_, T>(a);
#define GRET_SIMT_DIMS(C_)          \
    GRET_SIMT_CASE(64, 64, C_)      \
    GRET_SIMT_CASE(128, 128, C_)    \
    GRET_SIMT_CASE(64, 128, C_)     \
    GRET_SIMT_CASE(128, 64, C_)
    GRET_SIMT_DIMS(16)
    GRET_SIMT_DIMS(32)
    GRET_SIMT_DIMS(64)
#undef GRET_SIMT_DIMS
#undef GRET_SIMT_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_prefill_simt(const PrefillArgs& a, bool bf16) {
    if ((int64_t)a.H * a.n_seqs == 0) return cudaSuccess;
    return bf16 ? launch_simt_dt<__nv_bfloat16>(a) : launch_simt_dt<float>(a);
}

}  // namespace gret
