// prefill_ew.cu -- chunkwise prefill of gated retention with one gate per key channel (the
// element-wise gate that "路线二：Multi-Head Gated Retention" weighs against the head-wise scalar
// gate YOCO keeps), on the sm_100a tensor cores.
//
// Per sequence and head, with alpha_t[i] = sigmoid(g_t[i])^(1/tau) for key channel i:
//   S_t[i][:] = alpha_t[i] S_{t-1}[i][:] + k_scale k_t[i] v_t ,   o_t = q_t S_t
// Chunks of C = 128 tokens; c_t[i] is channel i's inclusive cumulative log2-decay inside the
// chunk and c_L[i] its chunk total (the chunkwise form of "Prefill 与 Decode 为什么使用两种计算
// 形态", one decay per channel).  With a scalar gate the decay of a (query, key) pair is one
// number that can scale the score matrix after Q K^T; with a gate per channel it sits inside the
// contraction over i, so here it is folded into the operands before the MMAs:
//   K~[m][i] = k_scale k_m[i] 2^(c_L[i] - c_m[i])          (<= |k_scale k|: always finite)
//   Q^[t][i] = q_t[i] 2^(c_t[i] - c_L[i])                   (>= |q|: bounded by the check below)
//   S'       = diag(2^c_L) S_prev                           (the state decayed over the chunk)
// so that, with the intra-chunk pair decay 2^(c_t - c_m) = 2^(c_t - c_L) 2^(c_L - c_m),
//   P   = mask_{m <= t}( Q^ K~^T )                          (scores, decay included)
//   o   = Q^ S' + P V                                       (cross-chunk + inner terms)
//   S   = S' + K~^T V                                       (next chunk's state)
// Every factored operand is an fp32 value split into a bf16 high half and a bf16 low half; the
// products take hi*hi + lo*hi + hi*lo (Q^ K~^T, Q^ S') or both halves against an exact bf16
// operand (P V, K~^T V), which keeps the result near 1e-5 of rms.
//
// Range of the factorisation.  Q^ grows with the chunk's decay: when some channel decays by more
// than 2^-SPAN2 over the chunk the masked (m > t) scores could overflow and Q^ loses meaning.
// Such a chunk takes the safe form: the scores come pairwise on CUDA cores,
//   P[t][m] = k_scale sum_i q_t[i] k_m[i] 2^(c_t[i] - c_m[i])   (every exponent <= 0)
// and the cross term uses Q~ = q 2^c_t (<= |q|) against the undecayed state.  Gates that decay
// that fast (below about 2^-0.5 per token per channel) are rare; the path exists for exactness.
//
// Parallelism.  A sequence's chunks are grouped into ranges of G chunks (G from a wave model on
// the host).  Three launches:
//   ew_range_state   one CTA per range: the range's aggregate sum over its keys of
//                    (decay to the range end) k^T v, one tensor-memory accumulator over the
//                    range (keys weighted by their decay to the range end: always <= 1), and
//                    the range's total decay per channel
//   ew_state_scan    per (sequence, head), serial over ranges: entry state of every range
//   ew_range_output  one CTA per range, chunks in order from the range's entry state: the
//                    outputs above, and the state carried to the next chunk of the range
// The range kernels are synchronous per CTA (one block-wide phase after another; one thread
// issues the MMAs) and take a whole SM each: 512 threads, 224 KB of shared memory.  In the
// per-channel passes a thread takes a pair of adjacent channels over 16 tokens, so that its
// shared-memory accesses and bf16 conversions come in pairs; in the state and output phases a
// thread takes a quarter (32 columns) of one TMEM lane.  Loads run ahead of the phases as far
// as the shared-memory plan allows: in the outputs kernel the next chunk's gate tile right after
// the operand build (the state operand goes into the k and y tiles once the first MMA group has
// read them) and its q, k, v after the second group; in the aggregates kernel a two-stage k / v
// ring and the gate logits read into registers one chunk ahead.
#include "prefill_ew.cuh"

#include <algorithm>

#include "common.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace gret {

using namespace sm100;

namespace {

constexpr int C = EW_CHUNK;             // tokens per chunk
constexpr int D = EW_DIM;               // d_k = d_v
constexpr int NT = 512;                 // threads of the range kernels
constexpr int TILE = C * D * 2;         // one bf16 128 x 128 tile
constexpr int SLAB = TILE / 2;          // one 64-column slab of it
constexpr int GTILE = C * D * 4;        // the chunk's fp32 gate logits
constexpr float SPAN2 = 64.f;           // largest chunk log2-decay of the factored form
constexpr uint64_t WAIT_NS = 2000000000ull;
constexpr uint64_t DRAIN_NS = 200000000ull;
constexpr uint32_t TM_A = 0, TM_O = 128, TM_S = 256;   // scores / P, output, state update
constexpr size_t WS_HEAD = 256;          // status word, then the range slots

struct EwParams {
    const float* g;        // [B][N][H][D] gate logits (read directly by the range aggregates)
    float inv_tau_log2e;   // log2(e) / tau
    float k_scale;
    int64_t N;
    int H, R, G;           // heads, ranges per sequence, chunks per range
    float* ws_S;           // [B][H][R][D][D]: range aggregates, then range entry states
    float* ws_a;           // [B][H][R][D]: range decays
    uint32_t* err;
    __nv_bfloat16* o;
};

struct __align__(1024) OutSmem {
    unsigned char q[TILE];   // q, then the high half of the query operand (in place)
    unsigned char k[TILE];   // k, then the high half of K~ (in place), then that of the state operand
    unsigned char v[TILE];
    unsigned char x[TILE];   // low half of the query operand; then the output tile
    unsigned char y[TILE];   // low half of K~, then that of the state operand  (x and y: fp32 P
                             // of a pairwise chunk)
    float g[C * D];          // gate logits -> cumulative log2-decay
    float cls[D];            // per channel: the chunk's total log2-decay c_L
    uint64_t g_full, r_full, mma_done, drain;   // gate tile; q, k, v tiles; MMA groups; exit
    uint32_t tmem_base;
};

struct __align__(1024) StateSmem {
    unsigned char k[2][TILE];   // k (two stages), then the high half of the weighted keys in place
    unsigned char v[2][TILE];
    unsigned char y[TILE];      // low half of the weighted keys
    float tot[8][D];         // per channel: log2-decay of tokens [16 s, 16 s + 16)
    float rs[D];             // per channel: log2-decay from the range's first chunk to its end
    uint64_t kv_full[2], mma_done, drain;
    uint32_t tmem_base;
};

static_assert(sizeof(OutSmem) <= 232448, "shared-memory plan exceeds 227 KB");
static_assert(sizeof(StateSmem) <= 232448, "shared-memory plan exceeds 227 KB");

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

__device__ __forceinline__ float ex2f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// log(sigmoid(x)) = min(x, 0) - log(1 + exp(-|x|)) with the fast exponential and logarithm
// (absolute error near 1e-7, which is what a cumulative sum of these sees).
__device__ __forceinline__ float logsigmoid_fast(float x) {
    return fminf(x, 0.f) - __logf(1.f + __expf(-fabsf(x)));
}

// Element (t, col) of a swizzled bf16 tile for rows t = t8 + u, t8 a multiple of 8: the
// column's slab and byte position are fixed per thread, the 16-byte chunk index is
// (col % 64) / 8 xor u.
struct ColOffset {
    uint32_t base, chunk;
    __device__ __forceinline__ explicit ColOffset(int col)
        : base((uint32_t)(col >> 6) * SLAB + (uint32_t)(col & 7) * 2u),
          chunk((uint32_t)(col & 63) >> 3) {}
    __device__ __forceinline__ uint32_t at(int t8, int u) const {
        return base + (uint32_t)(t8 + u) * 128u + ((chunk ^ (uint32_t)u) << 4);
    }
};

__device__ __forceinline__ float bf16_at(const unsigned char* tile, uint32_t off) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(tile + off));
}

__device__ __forceinline__ float2 bf16x2_at(const unsigned char* tile, uint32_t off) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(tile + off));
}

// (x0, x1) = hi + lo per element, hi = bf16(x), lo = bf16(x - hi), each pair packed
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Every thread of the block waits on the barrier itself; the block agrees on the outcome, and a
// wait that gave up records GRET_ERR_TIMEOUT in the workspace.
__device__ __forceinline__ bool block_wait(uint64_t* bar, uint32_t parity, uint32_t* err) {
    uint32_t never = 0;
    const bool ok = mbar_wait(bar, parity, &never, WAIT_NS);
    const int bad = __syncthreads_or(!ok);
    if (bad && threadIdx.x == 0) atomicExch(err, WS_ERR_TIMEOUT);
    return bad == 0;
}

// D (+)= A B over K = 128: eight K-steps of 16, bf16 operands in shared memory (64-column slabs,
// 128-byte swizzle).  a_mn / b_mn: the operand is stored MN-major (M or N contiguous).  The steps
// are unrolled with each step's descriptors formed just before its MMA (the empty asm keeps the
// compiler from computing all of them up front), so that one thread issues them back to back.
__device__ __forceinline__ void mma_128(uint32_t d, uint32_t a_base, bool a_mn, uint32_t b_base,
                                        bool b_mn, bool accumulate) {
    const uint32_t idesc = idesc_bf16(128, 128, a_mn, b_mn);
    const uint64_t ad = sdesc_sw128(a_base, a_mn ? SLAB : 16, 1024);
    const uint64_t bd = sdesc_sw128(b_base, b_mn ? SLAB : 16, 1024);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        const uint32_t aoff = a_mn ? kk * 2048u : (kk >> 2) * SLAB + (kk & 3) * 32u;
        const uint32_t boff = b_mn ? kk * 2048u : (kk >> 2) * SLAB + (kk & 3) * 32u;
        uint64_t a = ad + (aoff >> 4), bb = bd + (boff >> 4);
        asm volatile("" : "+l"(a), "+l"(bb));
        mma_ss(d, a, bb, idesc, (accumulate || kk > 0) ? 1u : 0u);
    }
}

// D += P V with P (bf16 halves, K-major) in tensor memory: per 32-token group g the columns
// [32 g, 32 g + 16) hold the high halves and [32 g + 16, 32 g + 32) the low halves, two tokens
// per column; V [token x d_v] in shared memory.
__device__ __forceinline__ void mma_pv(uint32_t d, uint32_t p_base, int half, uint32_t v_base,
                                       bool accumulate) {
    const uint32_t idesc = idesc_bf16(128, 128, 0, 1);
    const uint64_t vd = sdesc_sw128(v_base, SLAB, 1024);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        uint64_t bb = vd + ((kk * 2048u) >> 4);
        asm volatile("" : "+l"(bb));
        mma_ts(d, p_base + 32 * (kk >> 1) + 8 * (kk & 1) + 16 * half, bb, idesc,
               (accumulate || kk > 0) ? 1u : 0u);
    }
}

// Loads of one chunk, coordinates (column, head, token, batch) in every map, rows past the
// sequence read as zero: the gate logits (one unswizzled fp32 box of 128 columns), and the q, k
// and v tiles (two 64-column swizzled slabs each).
__device__ __forceinline__ void load_gate_tile(float* g, const CUtensorMap* tg, uint64_t* bar,
                                               int tok, int h, int b) {
    mbar_arrive_expect_tx(bar, GTILE);
    tma_load_4d(g, tg, bar, 0, h, tok, b);
}

__device__ __forceinline__ void load_qkv_tiles(unsigned char* q, unsigned char* k, unsigned char* v,
                                               const CUtensorMap* tq, const CUtensorMap* tk,
                                               const CUtensorMap* tv, uint64_t* bar, int tok,
                                               int h, int b) {
    mbar_arrive_expect_tx(bar, 3 * TILE);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        tma_load_4d(q + half * SLAB, tq, bar, half * 64, h, tok, b);
        tma_load_4d(k + half * SLAB, tk, bar, half * 64, h, tok, b);
        tma_load_4d(v + half * SLAB, tv, bar, half * 64, h, tok, b);
    }
}

// ----------------------------------------------------------------------------------------------
// 1. Range aggregates.  Block (range, head, batch).  The range's chunks are visited last to
// first so that each key's weight, its log2-decay to the end of the range, is a running suffix
// sum; every K~^T V MMA of the range accumulates into one tensor-memory result.  k and v tiles
// come by TMA through a two-stage ring, the next chunk's issued as soon as its stage is free;
// thread (cp, seg) reads the gate logits of its channel pair for its 16 tokens straight into registers,
// one chunk ahead.

__device__ __forceinline__ void load_kv(StateSmem& sm, int st, const CUtensorMap* tk,
                                        const CUtensorMap* tv, int tok, int h, int b) {
    mbar_arrive_expect_tx(&sm.kv_full[st], 2 * TILE);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        tma_load_4d(sm.k[st] + half * SLAB, tk, &sm.kv_full[st], half * 64, h, tok, b);
        tma_load_4d(sm.v[st] + half * SLAB, tv, &sm.kv_full[st], half * 64, h, tok, b);
    }
}

// Gate logits of tokens [t0, t0 + 16) of one (batch, head) row at a pair of adjacent channels
// (0 past the end).
__device__ __forceinline__ void load_gate16x2(const float* grow, int64_t gstride, int64_t t0,
                                              int64_t N, float2 (&x)[16]) {
#pragma unroll
    for (int u = 0; u < 16; ++u)
        x[u] = t0 + u < N ? __ldg(reinterpret_cast<const float2*>(grow + (t0 + u) * gstride))
                          : make_float2(0.f, 0.f);
}

__global__ void __launch_bounds__(NT, 1)
    ew_range_state(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                   const EwParams p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    StateSmem& sm = *reinterpret_cast<StateSmem*>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int r = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    if ((smem_u32(smem_raw) & 1023u) != 0) {   // the swizzled tiles need 1 KB alignment
        if (tid == 0) atomicExch(p.err, WS_ERR_TIMEOUT);
        return;
    }
    const int64_t nch = (p.N + C - 1) / C;
    const int c0 = r * p.G;
    const int c1 = (int)min64(nch, (int64_t)c0 + p.G);
    const int n_ch = c1 - c0;
    if (tid == 0) {
        mbar_init(&sm.kv_full[0], 1);
        mbar_init(&sm.kv_full[1], 1);
        mbar_init(&sm.mma_done, 1);
        mbar_init(&sm.drain, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // per-channel passes: thread (cp, seg) takes channels 2 cp, 2 cp + 1 over tokens
    // [16 seg, 16 seg + 16); the aggregate is read out by thread (i, qq): TMEM lane i, columns
    // [32 qq, 32 qq + 32)
    const int cp = tid & 63, seg = tid >> 6, ch = 2 * cp;
    const int i = tid & 127, qq = tid >> 7;
    const uint32_t lane_base = ((uint32_t)(warp & 3) * 32u) << 16;
    const float* grow = p.g + ((int64_t)b * p.N * p.H + h) * D + ch;
    const int64_t gstride = (int64_t)p.H * D;
    const ColOffset co(ch);   // channels ch, ch + 1: one aligned 4-byte pair

    if (tid == 0) load_kv(sm, 0, &tk, &tv, (c1 - 1) * C, h, b);
    float2 gcur[16], gnext[16];
    load_gate16x2(grow, gstride, (int64_t)(c1 - 1) * C + 16 * seg, p.N, gcur);
    // per-token log2-decays of both channels over this thread's 16 tokens of chunk cc, in place,
    // and their sum into the chunk's segment totals
    auto decays = [&](int cc) {
        const int Lc = (int)min64(C, p.N - (int64_t)cc * C);
        float2 sum = make_float2(0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const bool in = 16 * seg + u < Lc;
            gcur[u].x = in ? logsigmoid_fast(gcur[u].x) * p.inv_tau_log2e : 0.f;
            gcur[u].y = in ? logsigmoid_fast(gcur[u].y) * p.inv_tau_log2e : 0.f;
            sum.x += gcur[u].x;
            sum.y += gcur[u].y;
        }
        *reinterpret_cast<float2*>(&sm.tot[seg][ch]) = sum;
    };
    decays(c1 - 1);
    float2 R = make_float2(0.f, 0.f);   // log2-decay after the current chunk, to the range end
    int issued = 1, consumed = 0;
    uint32_t n_mma = 0;
    bool ok = true;
#pragma unroll 1
    for (int n = 0; n < n_ch; ++n) {
        const int c = c1 - 1 - n, st = n & 1;
        // the previous chunk's MMAs are done: its stage and the low-half tile are free
        if (n > 0 && !(ok = block_wait(&sm.mma_done, (n_mma - 1) & 1, p.err))) break;
        if (n + 1 < n_ch) {
            if (tid == 0) load_kv(sm, st ^ 1, &tk, &tv, (c - 1) * C, h, b);
            ++issued;
            load_gate16x2(grow, gstride, (int64_t)(c - 1) * C + 16 * seg, p.N, gnext);
        }
        // this chunk's segment totals (written at the end of the previous iteration, or before
        // the loop) are visible to every thread
        __syncthreads();
        float2 after = make_float2(0.f, 0.f), total = make_float2(0.f, 0.f);
#pragma unroll
        for (int s8 = 0; s8 < 8; ++s8) {
            const float2 t = *reinterpret_cast<const float2*>(&sm.tot[s8][ch]);
            if (s8 > seg) {
                after.x += t.x;
                after.y += t.y;
            }
            total.x += t.x;
            total.y += t.y;
        }
        if (!(ok = block_wait(&sm.kv_full[st], (n >> 1) & 1, p.err))) break;
        ++consumed;
        // weights 2^(suffix) k_scale, suffix = log2-decay from after token t to the range end,
        // last token first, in batches of 8
        float2 s2 = make_float2(R.x + after.x, R.y + after.y);
#pragma unroll
        for (int ub = 8; ub >= 0; ub -= 8) {
            float2 kv[8], sw[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) kv[u] = bf16x2_at(sm.k[st], co.at(16 * seg + ub, u));
#pragma unroll
            for (int u = 7; u >= 0; --u) {
                sw[u] = s2;
                s2.x += gcur[ub + u].x;
                s2.y += gcur[ub + u].y;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                uint32_t hi, lo;
                split2(kv[u].x * ex2f(sw[u].x) * p.k_scale, kv[u].y * ex2f(sw[u].y) * p.k_scale,
                       hi, lo);
                *reinterpret_cast<uint32_t*>(sm.k[st] + co.at(16 * seg + ub, u)) = hi;
                *reinterpret_cast<uint32_t*>(sm.y + co.at(16 * seg + ub, u)) = lo;
            }
        }
        R.x += total.x;
        R.y += total.y;
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            // Agg (+)= K~_hi^T V + K~_lo^T V: A = K~^T (channels x tokens) stored token-major
            mma_128(tmem, smem_u32(sm.k[st]), true, smem_u32(sm.v[st]), true, n > 0);
            mma_128(tmem, smem_u32(sm.y), true, smem_u32(sm.v[st]), true, true);
            mma_commit(&sm.mma_done);
        }
        ++n_mma;
        // the next chunk's decays while this chunk's MMAs run (its gate logits have arrived
        // in gnext meanwhile; the segment totals were last read before the barrier above)
        if (n + 1 < n_ch) {
#pragma unroll
            for (int u = 0; u < 16; ++u) gcur[u] = gnext[u];
            decays(c - 1);
        }
    }
    if (seg == 0) *reinterpret_cast<float2*>(&sm.rs[ch]) = R;   // read after the next barrier
    if (ok) ok = block_wait(&sm.mma_done, (n_mma - 1) & 1, p.err);
    if (ok) {
        tc_fence_after();
        const int64_t slot = ((int64_t)b * p.H + h) * p.R + r;
        float* dst = p.ws_S + slot * (D * D) + (int64_t)i * D + 32 * qq;
        float a[32];
        tmem_ld32(tmem + lane_base + 32 * qq, a);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 8; ++e)
            reinterpret_cast<float4*>(dst)[e] =
                make_float4(a[4 * e], a[4 * e + 1], a[4 * e + 2], a[4 * e + 3]);
        if (qq == 0) p.ws_a[slot * D + i] = ex2f(sm.rs[i]);
    } else if (tid == 0) {
        // a wait gave up: let the issued MMAs and the loads in flight finish before exit
        mma_commit(&sm.drain);
        uint32_t never = 0;
        mbar_wait(&sm.drain, 0, &never, DRAIN_NS);
        for (int j = consumed; j < issued; ++j)
            mbar_wait(&sm.kv_full[j & 1], (j >> 1) & 1, &never, DRAIN_NS);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

// ----------------------------------------------------------------------------------------------
// 2. Scan over ranges.  Block: one (batch, head) and 8 state rows; thread: one row, 4 columns.
// The aggregate slot of range r is overwritten with the state entering range r.
__global__ void __launch_bounds__(256) ew_state_scan(EwParams p, const float* state_in,
                                                     float* state_out) {
    constexpr int U = 8;   // ranges whose loads are issued together
    const int64_t bh = blockIdx.x / 16;
    const int i = (blockIdx.x % 16) * 8 + threadIdx.x / 32;
    const int j = (threadIdx.x % 32) * 4;
    const int64_t off = (int64_t)i * D + j;
    float4 S = make_float4(0.f, 0.f, 0.f, 0.f);
    if (state_in) S = *reinterpret_cast<const float4*>(state_in + bh * D * D + off);
    float* base = p.ws_S + bh * p.R * (int64_t)(D * D) + off;
    const float* abase = p.ws_a + bh * p.R * (int64_t)D + i;
    for (int c0 = 0; c0 < p.R; c0 += U) {
        float4 d[U];
        float al[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (c0 + u < p.R) {
                d[u] = *reinterpret_cast<const float4*>(base + (int64_t)(c0 + u) * (D * D));
                al[u] = abase[(int64_t)(c0 + u) * D];
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (c0 + u < p.R) {
                *reinterpret_cast<float4*>(base + (int64_t)(c0 + u) * (D * D)) = S;
                S.x = fmaf(al[u], S.x, d[u].x);
                S.y = fmaf(al[u], S.y, d[u].y);
                S.z = fmaf(al[u], S.z, d[u].z);
                S.w = fmaf(al[u], S.w, d[u].w);
            }
        }
    }
    if (state_out) *reinterpret_cast<float4*>(state_out + bh * D * D + off) = S;
}

// ----------------------------------------------------------------------------------------------
// 3. Outputs.  Block (range, head, batch); chunks in order from the range's entry state.

// Scores of a chunk whose decay is too fast for the factored form, pairwise on CUDA cores (every
// exponent c_t - c_m <= 0), into P^T [m][t] fp32 over the x and y tiles; then P into tensor
// memory as bf16 halves.  Needs the chunk's raw q and k tiles and the cumulative log2-decays
// over the whole chunk in sm.g.
__device__ void pairwise_scores(OutSmem& sm, const EwParams& p, uint32_t tmem, int L) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float* Pt = reinterpret_cast<float*>(sm.x);
    for (int e = tid; e < C * C; e += NT) Pt[e] = 0.f;
    __syncthreads();
    for (int pr = warp; pr < C * C; pr += NT / 32) {
        const int t = pr >> 7, m = pr & (C - 1);
        if (m > t || t >= L) continue;   // warp-uniform
        float acc = 0.f;
#pragma unroll
        for (int u = 0; u < D / 32; ++u) {
            const int ch = lane + 32 * u;
            acc += bf16_at(sm.q, sw128_offset(t, ch, SLAB)) * bf16_at(sm.k, sw128_offset(m, ch, SLAB)) *
                   ex2f(sm.g[t * D + ch] - sm.g[m * D + ch]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) Pt[m * C + t] = acc * p.k_scale;
    }
    __syncthreads();
    const int row = (warp & 3) * 32 + lane, jc = warp >> 2;   // 32 columns per thread
    const uint32_t lane_base = ((uint32_t)(warp & 3) * 32u) << 16;
    {
        uint32_t ph[32];
#pragma unroll
        for (int i2 = 0; i2 < 16; ++i2) {
            const int m0 = jc * 32 + 2 * i2;
            split2(Pt[m0 * C + row], Pt[(m0 + 1) * C + row], ph[i2], ph[16 + i2]);
        }
        tmem_st32(tmem + lane_base + TM_A + jc * 32, ph);
    }
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();
}

__global__ void __launch_bounds__(NT, 1)
    ew_range_output(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tg,
                    const __grid_constant__ CUtensorMap to, const EwParams p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    OutSmem& sm = *reinterpret_cast<OutSmem*>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    if ((smem_u32(smem_raw) & 1023u) != 0) {
        if (tid == 0) atomicExch(p.err, WS_ERR_TIMEOUT);
        return;
    }
    const int64_t nch = (p.N + C - 1) / C;
    const int c0 = r * p.G;
    const int c1 = (int)min64(nch, (int64_t)c0 + p.G);
    if (tid == 0) {
        mbar_init(&sm.g_full, 1);
        mbar_init(&sm.r_full, 1);
        mbar_init(&sm.mma_done, 1);
        mbar_init(&sm.drain, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // thread (i, qq): channel / state row i = TMEM lane, quarter qq: tokens [32 qq, 32 qq + 32)
    // in the per-channel passes, columns [32 qq, 32 qq + 32) of the state and of the output
    const int i = tid & 127, qq = tid >> 7;
    const uint32_t lane_base = ((uint32_t)(warp & 3) * 32u) << 16;
    const uint32_t qb = smem_u32(sm.q), kb = smem_u32(sm.k), vb = smem_u32(sm.v),
                   xb = smem_u32(sm.x), yb = smem_u32(sm.y);

    if (tid == 0) {
        load_gate_tile(sm.g, &tg, &sm.g_full, c0 * C, h, b);
        load_qkv_tiles(sm.q, sm.k, sm.v, &tq, &tk, &tv, &sm.r_full, c0 * C, h, b);
    }
    // entry state of the range: row i, columns [32 qq, 32 qq + 32)
    const int64_t slot = ((int64_t)b * p.H + h) * p.R + r;
    float S[32];
    {
        const float4* src =
            reinterpret_cast<const float4*>(p.ws_S + slot * (D * D) + (int64_t)i * D + 32 * qq);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float4 x = src[e];
            S[4 * e] = x.x; S[4 * e + 1] = x.y; S[4 * e + 2] = x.z; S[4 * e + 3] = x.w;
        }
    }
    uint32_t n_g = 1, n_ld = 1, n_mma = 0;   // gate and q/k/v loads issued, MMA groups committed
    // per-channel passes: thread (cp, seg) takes channels 2 cp, 2 cp + 1 over tokens
    // [16 seg, 16 seg + 16), with paired shared-memory accesses (float2, bf16x2)
    const int cp = tid & 63, seg = tid >> 6, ch = 2 * cp;
    // cumulative log2-decay of both channels over the segment of chunk cc's gate tile, in place
    // (every load first); returns the segment's total
    auto decays = [&](int cc) {
        const int Lc = (int)min64(C, p.N - (int64_t)cc * C);
        float2 x[16], cum = make_float2(0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 16; ++u)
            x[u] = *reinterpret_cast<const float2*>(&sm.g[(16 * seg + u) * D + ch]);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const bool in = 16 * seg + u < Lc;
            x[u].x = in ? logsigmoid_fast(x[u].x) * p.inv_tau_log2e : 0.f;
            x[u].y = in ? logsigmoid_fast(x[u].y) * p.inv_tau_log2e : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            cum.x += x[u].x;
            cum.y += x[u].y;
            *reinterpret_cast<float2*>(&sm.g[(16 * seg + u) * D + ch]) = cum;
        }
        return cum;
    };
    bool ok = block_wait(&sm.g_full, 0, p.err);
    float2 cum = ok ? decays(c0) : make_float2(0.f, 0.f);
    for (int c = c0; c < c1 && ok; ++c) {
        const int L = (int)min64(C, p.N - (int64_t)c * C);
        const bool last = c == c1 - 1;
        if (c > c0) {   // the previous output tile has left x
            if (tid == 0) bulk_wait_group_read0();
            __syncthreads();
        }
        // this chunk's decays are in the gate tile already (computed while the previous chunk's
        // output MMAs ran, or before the loop)
        float* tot = reinterpret_cast<float*>(sm.y);   // [8][D] segment totals; y is idle here
        *reinterpret_cast<float2*>(&tot[seg * D + ch]) = cum;
        __syncthreads();
        float2 before = make_float2(0.f, 0.f), cl2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int s8 = 0; s8 < 8; ++s8) {
            const float2 t = *reinterpret_cast<const float2*>(&tot[s8 * D + ch]);
            if (s8 < seg) {
                before.x += t.x;
                before.y += t.y;
            }
            cl2.x += t.x;
            cl2.y += t.y;
        }
        if (seg == 0) *reinterpret_cast<float2*>(&sm.cls[ch]) = cl2;
        // (also the barrier after which y may be written again)
        const bool pairwise = __syncthreads_or(fminf(cl2.x, cl2.y) < -SPAN2) != 0;
        if (!(ok = block_wait(&sm.r_full, (n_ld - 1) & 1, p.err))) break;
        if (pairwise) {
            if (seg > 0) {
#pragma unroll 4
                for (int t = 16 * seg; t < 16 * seg + 16; ++t) {
                    float2* gp = reinterpret_cast<float2*>(&sm.g[t * D + ch]);
                    const float2 c2 = *gp;
                    *gp = make_float2(c2.x + before.x, c2.y + before.y);
                }
            }
            __syncthreads();
            pairwise_scores(sm, p, tmem, L);
        }
        // operands: query (factored: 2^(c_t - c_L); pairwise: 2^(c_t)) and K~ = k_scale k
        // 2^(c_L - c_t), each as bf16 high half in place and low half in x / y
        {
            const float2 off = pairwise ? make_float2(0.f, 0.f) : before;
            const float qsx = pairwise ? 0.f : -cl2.x, qsy = pairwise ? 0.f : -cl2.y;
            const ColOffset co(ch);   // channels ch, ch + 1: one aligned 4-byte pair
#pragma unroll 1
            for (int tb = 16 * seg; tb < 16 * seg + 16; tb += 8) {
                float2 ct[8], qv[8], kv[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const float2 c2 = *reinterpret_cast<const float2*>(&sm.g[(tb + u) * D + ch]);
                    ct[u] = make_float2(c2.x + off.x, c2.y + off.y);
                    qv[u] = bf16x2_at(sm.q, co.at(tb, u));
                    kv[u] = bf16x2_at(sm.k, co.at(tb, u));
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    uint32_t qh, ql, kh, kl;
                    split2(qv[u].x * ex2f(ct[u].x + qsx), qv[u].y * ex2f(ct[u].y + qsy), qh, ql);
                    split2(kv[u].x * ex2f(cl2.x - ct[u].x) * p.k_scale,
                           kv[u].y * ex2f(cl2.y - ct[u].y) * p.k_scale, kh, kl);
                    const uint32_t o = co.at(tb, u);
                    *reinterpret_cast<uint32_t*>(sm.q + o) = qh;
                    *reinterpret_cast<uint32_t*>(sm.x + o) = ql;
                    *reinterpret_cast<uint32_t*>(sm.k + o) = kh;
                    *reinterpret_cast<uint32_t*>(sm.y + o) = kl;
                }
            }
        }
        __syncthreads();   // every read of the log2-decays is done: the next gate tile may come
        if (!last) {
            if (tid == 0) load_gate_tile(sm.g, &tg, &sm.g_full, (c + 1) * C, h, b);
            ++n_g;
        }
        fence_proxy_async_smem();
        __syncthreads();
        // first MMA group: the scores (factored chunks) and the state update dS = K~^T V (all
        // chunks but the range's last); after it the k and y tiles are free
        if (!pairwise || !last) {
            if (tid == 0) {
                tc_fence_after();
                if (!pairwise) {
                    mma_128(tmem + TM_A, qb, false, kb, false, false);   // Q_hi K~_hi^T
                    mma_128(tmem + TM_A, xb, false, kb, false, true);    //  + Q_lo K~_hi^T
                    mma_128(tmem + TM_A, qb, false, yb, false, true);    //  + Q_hi K~_lo^T
                }
                if (!last) {
                    mma_128(tmem + TM_S, kb, true, vb, true, false);     // dS = K~_hi^T V
                    mma_128(tmem + TM_S, yb, true, vb, true, true);      //    + K~_lo^T V
                }
                mma_commit(&sm.mma_done);
            }
            ++n_mma;
            if (!(ok = block_wait(&sm.mma_done, (n_mma - 1) & 1, p.err))) break;
            tc_fence_after();
        }
        const float cL = sm.cls[i];   // row i's channel total (the state rows below)
        // state operand into the k (high halves) and y (low halves) tiles: 2^c_L S (factored) or
        // S (pairwise), row i, columns [32 qq, 32 qq + 32) of the MN-major tiles (slab qq / 2,
        // 16-byte chunks 4 (qq % 2) .. 4 (qq % 2) + 3 of the row)
        {
            const float sc = pairwise ? 1.f : ex2f(cL);
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    split2(sc * S[8 * cc + 2 * e], sc * S[8 * cc + 2 * e + 1], hi[e], lo[e]);
                const int chunk = 4 * (qq & 1) + cc;
                const uint32_t off = (qq >> 1) * SLAB + i * 128 + ((chunk ^ (i & 7)) << 4);
                *reinterpret_cast<uint4*>(sm.k + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4*>(sm.y + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
        }
        const int row = (warp & 3) * 32 + lane;   // == i: this thread's TMEM lane
        if (!pairwise) {
            // causal mask, P split into bf16 halves in place: row = lane, columns [32 qq, +32)
            float a[32];
            tmem_ld32(tmem + lane_base + TM_A + qq * 32, a);
            tmem_ld_wait();
            uint32_t ph[32];
#pragma unroll
            for (int i2 = 0; i2 < 16; ++i2) {
                const int m0 = qq * 32 + 2 * i2;
                split2(m0 <= row ? a[2 * i2] : 0.f, m0 + 1 <= row ? a[2 * i2 + 1] : 0.f, ph[i2],
                       ph[16 + i2]);
            }
            tmem_st32(tmem + lane_base + TM_A + qq * 32, ph);
            tmem_st_wait();
        }
        tc_fence_before();
        fence_proxy_async_smem();
        __syncthreads();
        // second group: the output O = Q S' + P V
        if (tid == 0) {
            tc_fence_after();
            mma_128(tmem + TM_O, qb, false, kb, true, false);    // O = Q_hi S_hi
            mma_128(tmem + TM_O, xb, false, kb, true, true);     //   + Q_lo S_hi
            mma_128(tmem + TM_O, qb, false, yb, true, true);     //   + Q_hi S_lo
            mma_pv(tmem + TM_O, tmem + TM_A, 0, vb, true);       //   + P_hi V
            mma_pv(tmem + TM_O, tmem + TM_A, 1, vb, true);       //   + P_lo V
            mma_commit(&sm.mma_done);
        }
        ++n_mma;
        // while they run: the next chunk's decays, in its gate tile (loaded after pass 2)
        if (!last) {
            if (!(ok = block_wait(&sm.g_full, (n_g - 1) & 1, p.err))) break;
            cum = decays(c + 1);
        }
        if (!(ok = block_wait(&sm.mma_done, (n_mma - 1) & 1, p.err))) break;
        tc_fence_after();
        if (!last) {   // q, k, v are free: the next chunk's tiles go now
            if (tid == 0)
                load_qkv_tiles(sm.q, sm.k, sm.v, &tq, &tk, &tv, &sm.r_full, (c + 1) * C, h, b);
            ++n_ld;
        }
        // output rows: a chunk inside the sequence goes out as one tile through x (rows in the
        // swizzled layout, two TMA stores); the rows of a partial chunk one by one
        const bool full = L == C;
        const int64_t tok = (int64_t)c * C + row;
        uint4* orow = reinterpret_cast<uint4*>(p.o + (((int64_t)b * p.N + tok) * p.H + h) * D);
        {
            float o[32];
            tmem_ld32(tmem + lane_base + TM_O + qq * 32, o);
            float d[32];
            if (!last) tmem_ld32(tmem + lane_base + TM_S + qq * 32, d);
            tmem_ld_wait();
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
                uint4 u;
                u.x = pack_bf16x2(o[8 * v4 + 0], o[8 * v4 + 1]);
                u.y = pack_bf16x2(o[8 * v4 + 2], o[8 * v4 + 3]);
                u.z = pack_bf16x2(o[8 * v4 + 4], o[8 * v4 + 5]);
                u.w = pack_bf16x2(o[8 * v4 + 6], o[8 * v4 + 7]);
                const int cc = 4 * qq + v4;   // 16-byte chunk of the row
                if (full)
                    *reinterpret_cast<uint4*>(sm.x + (cc >> 3) * SLAB + row * 128 +
                                              (((cc & 7) ^ (row & 7)) << 4)) = u;
                else if (row < L)
                    orow[cc] = u;
            }
            // the state carried to the next chunk: S = 2^c_L S + dS
            if (!last) {
                const float eL = ex2f(cL);
#pragma unroll
                for (int e = 0; e < 32; ++e) S[e] = fmaf(eL, S[e], d[e]);
            }
        }
        tc_fence_before();
        if (full) fence_proxy_async_smem();
        __syncthreads();
        if (full && tid == 0) {
#pragma unroll
            for (int half = 0; half < 2; ++half)
                tma_store_4d(&to, sm.x + half * SLAB, half * 64, h, c * C, b);
            bulk_commit_group();
        }
    }
    if (tid == 0) {
        if (!ok) {   // a wait gave up: the issued MMAs and any load in flight finish first
            mma_commit(&sm.drain);
            uint32_t never = 0;
            mbar_wait(&sm.drain, 0, &never, DRAIN_NS);
            mbar_wait(&sm.g_full, (n_g - 1) & 1, &never, DRAIN_NS);
            mbar_wait(&sm.r_full, (n_ld - 1) & 1, &never, DRAIN_NS);
        }
        bulk_wait_group0();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ----------------------------------------------------------------------------------------------
// host side

int sm_count_ew() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
    if (dev < 0 || dev >= 64) dev = 0;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 0;
        cached[dev] = n > 0 ? n : 148;
    }
    return cached[dev];
}

// [B, N, H, 128] contiguous, coordinates (column, head, token, batch); bf16 with 64-column
// swizzled boxes, or fp32 with one unswizzled 128-column box.
bool make_ew_map(CUtensorMap* map, const void* base, bool fp32, int B, int64_t N, int H) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return false;
    const uint64_t es = fp32 ? 4 : 2;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
    cuuint64_t strides[3] = {D * es, (cuuint64_t)H * D * es, (cuuint64_t)N * H * D * es};
    cuuint32_t box[4] = {fp32 ? (cuuint32_t)D : 64u, 1u, (cuuint32_t)C, 1u};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(map, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              fp32 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Chunks per range.  A range kernel runs ceil(B H R / SMs) waves of CTAs (R = ceil(chunks / G)
// ranges per sequence), each about G + 1 chunk-times long: its chunks plus a start (the first
// loads and the entry state, exposed since a CTA has its SM to itself).  G minimises that, and
// among equal costs the largest G wins (fewer ranges: less workspace traffic, a shorter scan).
int ew_range_chunks(int B, int64_t N, int H) {
    const int64_t nch = (N + C - 1) / C;
    if (nch <= 1 || B < 1 || H < 1) return 1;
    const int64_t grid = sm_count_ew();
    const int64_t units = (int64_t)B * H;
    int best = 1;
    int64_t best_cost = -1;
    const int64_t gmax = std::min<int64_t>(nch, 1 << 20);
    for (int64_t g = 1; g <= gmax; ++g) {
        const int64_t ranges = (nch + g - 1) / g;
        if (g > 1 && ranges == (nch + g - 2) / (g - 1)) continue;   // same R as g - 1
        const int64_t cost = ((units * ranges + grid - 1) / grid) * (g + 1);
        if (best_cost < 0 || cost <= best_cost) {
            best = (int)g;
            best_cost = cost;
        }
    }
    return best;
}

int64_t ew_ranges(int B, int64_t N, int H) {
    const int64_t nch = (N + C - 1) / C;
    const int G = ew_range_chunks(B, N, H);
    return (nch + G - 1) / G;
}

size_t ew_workspace_bytes(int B, int64_t N, int H) {
    const int64_t R = ew_ranges(B, N, H);
    return WS_HEAD + (size_t)B * H * R * (size_t)(D * D + D) * sizeof(float);
}

cudaError_t launch_prefill_ew(const EwArgs& a, cudaStream_t stream) {
    const int G = ew_range_chunks(a.B, a.N, a.H);
    const int64_t R = ew_ranges(a.B, a.N, a.H);
    unsigned char* ws = static_cast<unsigned char*>(a.workspace);
    EwParams p;
    p.g = a.g;
    p.inv_tau_log2e = 1.4426950408889634f / a.tau;
    p.k_scale = a.k_scale;
    p.N = a.N;
    p.H = a.H;
    p.R = (int)R;
    p.G = G;
    p.err = reinterpret_cast<uint32_t*>(ws);
    p.ws_S = reinterpret_cast<float*>(ws + WS_HEAD);
    p.ws_a = p.ws_S + (size_t)a.B * a.H * R * D * D;
    p.o = a.o;
    CUtensorMap tq, tk, tv, tg, to;
    if (!make_ew_map(&tq, a.q, false, a.B, a.N, a.H) || !make_ew_map(&tk, a.k, false, a.B, a.N, a.H) ||
        !make_ew_map(&tv, a.v, false, a.B, a.N, a.H) || !make_ew_map(&tg, a.g, true, a.B, a.N, a.H) ||
        !make_ew_map(&to, a.o, false, a.B, a.N, a.H))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaMemsetAsync(ws, 0, WS_HEAD, stream);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(ew_range_state, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sizeof(StateSmem));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(ew_range_output, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sizeof(OutSmem));
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)R, (unsigned)a.H, (unsigned)a.B);
    ew_range_state<<<grid, NT, sizeof(StateSmem), stream>>>(tk, tv, p);
    ew_state_scan<<<(unsigned)((int64_t)a.B * a.H * 16), 256, 0, stream>>>(p, a.state_in,
                                                                           a.state_out);
    ew_range_output<<<grid, NT, sizeof(OutSmem), stream>>>(tq, tk, tv, tg, to, p);
    return cudaGetLastError();
}

}  // namespace gret
