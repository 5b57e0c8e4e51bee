// swa_tc.cu -- sliding-window softmax attention prefill on the sm_100a tensor cores.
//
// Page "YOCO 完全拆解：Decoder-Decoder 架构如何让 KV Cache 只存一次", section
// "路线一：滑动窗口注意力": position i attends to the most recent W positions of its sequence,
//   o_i = sum_{j = i-W+1 .. i} softmax_j(scale q_i . k_j) v_j .
// FlashAttention-style, as the page suggests for this mixer, built on tcgen05:
//   * an item of work is two 128-query tiles of one (batch, head), queries q0 .. q0 + 255; the
//     key tiles of 128 that their windows touch (ten at W = 1024) stream through two TMA stages
//     and serve both query tiles;
//   * the kernel is persistent, one CTA per SM taking items round-robin; a query tile's slot is
//     loaded with the next item's queries as soon as its output has been stored, so the next
//     item starts while the last one finishes;
//   * S = Q K^T for each query tile goes to tensor memory; two softmax warpgroups per query
//     tile (one query row per thread, keys [0, 64) and [64, 128) of the key tile) mask the
//     window, share the row's running maximum through shared memory, keep their partial sums,
//     and write P = 2^(s - m) back over S as a bf16 high + low pair; the MMA warp accumulates
//     O += P_hi V + P_lo V in tensor memory as each half of the keys arrives;
//   * the two query tiles take turns: while one runs its softmax, the tensor cores run the
//     other tile's products;
//   * the running maximum is only moved (and O rescaled) when a tile's maximum exceeds it by
//     more than 2^8, so rescaling is rare after the first tiles; P then stays below 256;
//   * the output, O / l in bf16, leaves through the query tile's own shared-memory slot by TMA
//     store (rows past the sequence end are clipped by the store).
// P is carried as two bf16 halves because a single bf16 rounding of P over a 1024-key window
// leaves errors near 1e-2 of rms; the pair (split by truncation, see split2_trunc) keeps the
// result near 1e-5.
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512).
// Warp roles (640 threads): warp 0 TMA producer, warp 1 MMA issuer (one thread), warps 4-11 the
// softmax warpgroups of query tile 0 (keys [0, 64), then [64, 128)), warps 12-19 those of query
// tile 1.  Registers: launched at 96 per thread; warps 0-3 drop to 56 and the softmax groups
// rise to 104 (each SM sub-partition holds one warp of each of the five warpgroups:
// 32 x (56 + 4 x 104) <= 32 x 5 x 96).  A softmax thread reads its 64 scores in two passes (the
// maximum, then 32 at a time for P) so that it fits its 104 registers.
// Every wait is bounded; a wait that gives up makes the CTA stop and write NaN into its output
// rows that are still to be written.  The two warpgroups of a query tile wait together: one
// thread waits while the other 255 sleep at the pair's named barrier, so that neither half can
// leave while the other is at the pair's barrier.
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "sm100.cuh"
#include "swa.cuh"
#include "tma_host.cuh"

namespace gret {

using namespace sm100;

namespace {

constexpr int D = SWA_DIM;
constexpr int BM = 128;                  // queries per tile, keys per tile
constexpr int TILE = BM * D * 2;         // one bf16 128 x 128 tile
constexpr int SLAB = TILE / 2;
constexpr int NTHREADS = 640;
constexpr int LAUNCH_REGS = 96;
constexpr uint64_t WAIT_NS = 2000000000ull;
constexpr uint64_t DRAIN_NS = 200000000ull;
constexpr float RESCALE_LOG2 = 8.f;      // move the running maximum only past this margin

struct __align__(1024) SwaSmem {
    unsigned char q[2][TILE];            // the two query tiles; later their output tiles
    unsigned char k[2][TILE];
    unsigned char v[2][TILE];
    // p_ready[w][kh]: query tile w's P over keys [64 kh, 64 kh + 64) is in tensor memory
    // q_full[w]: query tile w of the item is loaded; q_free[w]: its output has been stored (the
    // slot may be loaded again); o_free[w]: its O accumulator has been read
    uint64_t q_full[2], q_free[2], o_free[2];
    uint64_t kv_full[2], kv_empty[2], s_full[2], p_ready[2][2], pv_done[2], drain;
    uint32_t dec[2][2];                  // the softmax pairs' shared wait outcomes
    // the two halves of a query row exchange their partial maxima (double-buffered by tile) and,
    // at the end, their partial sums
    float xmax[2][2][2][BM];             // [tile parity][query tile][key half][row]
    float xl[2][2][BM];                  // [query tile][key half][row]
    uint32_t tmem_base;
    uint32_t abort;
};
static_assert(sizeof(SwaSmem) <= 232448, "shared-memory plan exceeds 227 KB");

struct SwaParams {
    float scale_log2;      // scale * log2(e)
    int window;
    int64_t N;
    int H;
    int n_qpairs;          // query-tile pairs per sequence
    int64_t n_items;       // (batch, head, query-tile pair) items
};

// One item of work: two 128-query tiles of one (batch, head), queries q0 .. q0 + 255, and the
// key tiles [kt_lo, kt_lo + ntiles) their windows touch.
struct SwaItem {
    int64_t q0, kt_lo;
    int ntiles, h, b;
};

__device__ __forceinline__ SwaItem item_of(const SwaParams& p, int64_t t) {
    SwaItem it;
    const int pair = (int)(t % p.n_qpairs);
    it.h = (int)((t / p.n_qpairs) % p.H);
    it.b = (int)(t / ((int64_t)p.n_qpairs * p.H));
    it.q0 = (int64_t)pair * 2 * 128;
    const int64_t qlast = (it.q0 + 2 * 128 - 1 < p.N - 1) ? it.q0 + 2 * 128 - 1 : p.N - 1;
    const int64_t kfirst = (it.q0 - p.window + 1 > 0) ? it.q0 - p.window + 1 : 0;
    it.kt_lo = kfirst / 128;
    it.ntiles = (int)(qlast / 128 - it.kt_lo + 1);
    return it;
}

__device__ __forceinline__ float ex2f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// x = hi + lo in bf16 without the conversion unit: hi keeps the top 16 bits of x (its sign,
// exponent and 7 fraction bits: truncation), lo = x - hi is exact in fp32 and is truncated the
// same way.  |hi + lo - x| <= 2^-15 |x|, against 2^-17 with round-to-nearest halves; all of it
// runs on the integer and FMA pipes (bit masks, one subtraction, one byte permute per pair).
__device__ __forceinline__ void split2_trunc(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const uint32_t b0 = __float_as_uint(x0), b1 = __float_as_uint(x1);
    const float l0 = x0 - __uint_as_float(b0 & 0xFFFF0000u);
    const float l1 = x1 - __uint_as_float(b1 & 0xFFFF0000u);
    hi = __byte_perm(b0, b1, 0x7632);   // upper halves: x0 in the low 16 bits, x1 in the high
    lo = __byte_perm(__float_as_uint(l0), __float_as_uint(l1), 0x7632);
}

// does query tile w (queries q0 + 128 w .. + 127) see any key of key tile kt?
__device__ __forceinline__ bool takes_part(int64_t q0, int w, int64_t kt, int window, int64_t N) {
    const int64_t qa = q0 + BM * w, qb = qa + BM - 1;
    if (qa >= N) return false;                     // the tile is past the sequence end
    const int64_t ka = BM * kt, kb = ka + BM - 1;
    return ka <= qb && kb >= qa - window + 1;
}

// Exit-time wait for this CTA's own asynchronous work; bounded, and not cut short by an abort.
__device__ __forceinline__ void mbar_wait_drain_(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    uint32_t never = 0;
    mbar_wait(bar, parity, &never, limit_ns);
}

__device__ __forceinline__ bool wait_abortable(SwaSmem& sm, uint64_t* bar, uint32_t parity) {
    if (mbar_wait(bar, parity, &sm.abort, WAIT_NS)) return true;
    atomicExch(&sm.abort, 1u);
    return false;
}

// A softmax pair's wait (the two warpgroups of one query tile): one thread polls the barrier,
// the other 255 sleep at the pair's named barrier (no issue slots burned by polling threads),
// and all take the same branch, so that neither half can leave the tile loop while the other
// waits at the pair's barrier.  The outcome word is double-buffered, so that a fast thread
// cannot overwrite it for the next wait before a slow thread of the pair has read it.
__device__ __forceinline__ bool pair_wait(SwaSmem& sm, uint64_t* bar, uint32_t parity, int w,
                                          int hf, int r, int& flip) {
    if (hf == 0 && r == 0) sm.dec[w][flip] = wait_abortable(sm, bar, parity) ? 1u : 0u;
    asm volatile("bar.sync %0, 256;" ::"r"(1 + w) : "memory");
    const bool ok = *reinterpret_cast<volatile uint32_t*>(&sm.dec[w][flip]) != 0;
    flip ^= 1;
    return ok;
}

__device__ __forceinline__ void pair_sync(int w) {
    asm volatile("bar.sync %0, 256;" ::"r"(1 + w) : "memory");
}

// The MMA issue loops are fully unrolled over constant descriptor offsets: a single thread
// issues every MMA of the CTA, and per-step descriptor arithmetic in a rolled loop (a chain of
// dependent integer operations) takes longer than a 128x128x16 MMA takes to execute.  The empty
// asm statements pin each call's descriptor bases where they are made, so that the compiler
// does not hoist every unrolled descriptor of every stage out of the key-tile loop (which would
// need more registers than the issuing warp has).

// S (+)= A B over K = 128 with both operands K-major in shared memory (A = Q, B = K).
__device__ __forceinline__ void mma_qk(uint32_t d, uint32_t a_base, uint32_t b_base) {
    constexpr uint32_t idesc = idesc_bf16(128, 128, 0, 0);
    uint64_t ad = sdesc_sw128(a_base, 16, 1024), bd = sdesc_sw128(b_base, 16, 1024);
    asm volatile("" : "+l"(ad), "+l"(bd));
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = ((kk >> 2) * SLAB + (kk & 3) * 32u) >> 4;
        mma_ss(d, ad + off, bd + off, idesc, kk > 0 ? 1u : 0u);
    }
}

// O (+)= P V over keys [64 kh, 64 kh + 64) with P (bf16 halves, K-major) in TMEM: per 32-key
// group, 16 columns of high halves then 16 of low halves; V [key x d] MN-major in shared memory.
// Both halves of P go through: four K-steps of 16 keys each for the high and the low half.
__device__ __forceinline__ void mma_pv(uint32_t d, uint32_t p_base, int kh, uint32_t v_base,
                                       bool accumulate) {
    constexpr uint32_t idesc = idesc_bf16(128, 128, 0, 1);
    uint64_t vd = sdesc_sw128(v_base + kh * 4 * 2048u, SLAB, 1024);
    uint32_t pb = p_base + 64 * kh;
    asm volatile("" : "+l"(vd), "+r"(pb));
#pragma unroll
    for (int half = 0; half < 2; ++half)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            mma_ts(d, pb + 32 * (kk >> 1) + 8 * (kk & 1) + 16 * half, vd + ((kk * 2048u) >> 4),
                   idesc, (accumulate || half > 0 || kk > 0) ? 1u : 0u);
}

__global__ void __launch_bounds__(NTHREADS, 1)
    swa_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to,
                  const SwaParams p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    SwaSmem& sm = *reinterpret_cast<SwaSmem*>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if ((smem_u32(smem_raw) & 1023u) != 0) return;   // never: dynamic shared memory starts aligned
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sm.q_full[s], 1);
            mbar_init(&sm.q_free[s], 1);
            mbar_init(&sm.o_free[s], 256);
            mbar_init(&sm.kv_full[s], 1);
            mbar_init(&sm.kv_empty[s], 1);
            mbar_init(&sm.s_full[s], 1);
            mbar_init(&sm.p_ready[s][0], 128);
            mbar_init(&sm.p_ready[s][1], 128);
            mbar_init(&sm.pv_done[s], 1);
        }
        mbar_init(&sm.drain, 1);
        sm.abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // The CTA is persistent: it takes items t = blockIdx.x, blockIdx.x + gridDim.x, ...; every
    // role walks the same list, and every barrier's phase count runs on across items.

    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
        if (warp == 0 && lane == 0) {
            // ---- producer: per item, query tile 0, the first key / value tile, query tile 1,
            // the other key / value tiles (two stages).  A query slot is loaded again once the
            // previous item's output tile has left it.
            tma_prefetch_desc(&tq);
            tma_prefetch_desc(&tk);
            tma_prefetch_desc(&tv);
            tma_prefetch_desc(&to);
            int g = 0, n = 0;      // key / value tiles and items issued
            bool ok = true;
            auto load_q = [&](const SwaItem& it, int w) {
                if (n > 0 && !(ok = wait_abortable(sm, &sm.q_free[w], (n - 1) & 1))) return;
                mbar_arrive_expect_tx(&sm.q_full[w], TILE);
                for (int half = 0; half < 2; ++half)
                    tma_load_4d(sm.q[w] + half * SLAB, &tq, &sm.q_full[w], half * 64, it.h,
                                (int)(it.q0 + BM * w), it.b);
            };
            auto load_kv = [&](const SwaItem& it, int i) {
                const int st = g & 1;
                if (g >= 2 && !(ok = wait_abortable(sm, &sm.kv_empty[st], ((g >> 1) - 1) & 1)))
                    return;
                const int tok = (int)((it.kt_lo + i) * BM);
                mbar_arrive_expect_tx(&sm.kv_full[st], 2 * TILE);
                for (int half = 0; half < 2; ++half) {
                    tma_load_4d(sm.k[st] + half * SLAB, &tk, &sm.kv_full[st], half * 64, it.h,
                                tok, it.b);
                    tma_load_4d(sm.v[st] + half * SLAB, &tv, &sm.kv_full[st], half * 64, it.h,
                                tok, it.b);
                }
                ++g;
            };
            for (int64_t t = blockIdx.x; t < p.n_items && ok; t += gridDim.x) {
                const SwaItem it = item_of(p, t);
                load_q(it, 0);
                for (int i = 0; i < it.ntiles && ok; ++i) {
                    load_kv(it, i);
                    if (i == 0 && ok) load_q(it, 1);
                }
                if (ok) ++n;
            }
            // no TMA write into this CTA's shared memory may be in flight at exit
            for (int gg = (g >= 2 ? g - 2 : 0); gg < g; ++gg)
                mbar_wait_drain_(&sm.kv_full[gg & 1], (gg >> 1) & 1, DRAIN_NS);
            if (n > 0)
                for (int w = 0; w < 2; ++w) mbar_wait_drain_(&sm.q_full[w], (n - 1) & 1, DRAIN_NS);
        } else if (warp == 1 && lane == 0) {
            // ---- MMA issuer.  Query tile 0 runs one step ahead of tile 1: Q_0 K_{i+1}^T is
            // issued right after P_0 V_i, before P_1 V_i, so that tile 0's next softmax overlaps
            // tile 1's products instead of both tiles' softmaxes running at the same time.
            // Every item waits each tile's q_full phase once and (after the first item) each
            // tile's o_free phase once, before the first use or at the item's end.
            bool ok = true;
            int cnt[2] = {0, 0};   // P V products issued per query tile (all items)
            int g = 0, n = 0;      // key / value tiles and items consumed
            for (int64_t t = blockIdx.x; t < p.n_items && ok; t += gridDim.x) {
                const SwaItem it = item_of(p, t);
                bool need_q[2] = {true, true}, need_o[2] = {n > 0, n > 0}, first[2] = {true, true};
                auto part = [&](int w, int i) {
                    return takes_part(it.q0, w, it.kt_lo + i, p.window, p.N);
                };
                auto qk = [&](int w, int i) {   // S_w = Q_w K_i^T, once P V has read the last P
                    if (need_q[w]) {
                        if (!(ok = wait_abortable(sm, &sm.q_full[w], n & 1))) return;
                        need_q[w] = false;
                    }
                    if (cnt[w] > 0 && !(ok = wait_abortable(sm, &sm.pv_done[w], (cnt[w] - 1) & 1)))
                        return;
                    tc_fence_after();
                    mma_qk(tmem + BM * w, smem_u32(sm.q[w]), smem_u32(sm.k[(g + i) & 1]));
                    mma_commit(&sm.s_full[w]);
                };
                auto pv = [&](int w, int i) {   // O_w += P_w V_i, one half of the keys at a time
                    if (need_o[w]) {   // the previous item's O_w has been read
                        if (!(ok = wait_abortable(sm, &sm.o_free[w], (n - 1) & 1))) return;
                        need_o[w] = false;
                    }
                    const uint32_t vb = smem_u32(sm.v[(g + i) & 1]);
                    for (int kh = 0; kh < 2 && ok; ++kh) {
                        if (!(ok = wait_abortable(sm, &sm.p_ready[w][kh], cnt[w] & 1))) return;
                        tc_fence_after();
                        mma_pv(tmem + 256 + BM * w, tmem + BM * w, kh, vb, !first[w] || kh > 0);
                    }
                    first[w] = false;
                    mma_commit(&sm.pv_done[w]);
                    ++cnt[w];
                };
                auto kv_wait = [&](int i) {
                    const int gi = g + i;
                    if ((ok = wait_abortable(sm, &sm.kv_full[gi & 1], (gi >> 1) & 1))) tc_fence_after();
                };
                if (it.ntiles > 0) {
                    kv_wait(0);
                    if (ok && part(0, 0)) qk(0, 0);
                    if (ok && part(1, 0)) qk(1, 0);
                }
                for (int i = 0; i < it.ntiles && ok; ++i) {
                    const bool nxt = i + 1 < it.ntiles;
                    if (part(0, i)) pv(0, i);
                    if (ok && nxt) {
                        kv_wait(i + 1);
                        if (ok && part(0, i + 1)) qk(0, i + 1);
                    }
                    if (ok && part(1, i)) pv(1, i);
                    if (!ok) break;
                    // this stage: its K was read by Q K^T of both tiles and its V by both P V
                    mma_commit(&sm.kv_empty[(g + i) & 1]);
                    if (nxt && part(1, i + 1)) qk(1, i + 1);
                }
                // the phases this item did not need
                for (int w = 0; w < 2 && ok; ++w) {
                    if (need_q[w]) ok = wait_abortable(sm, &sm.q_full[w], n & 1);
                    if (ok && need_o[w]) ok = wait_abortable(sm, &sm.o_free[w], (n - 1) & 1);
                }
                g += it.ntiles;
                ++n;
            }
            mma_commit(&sm.drain);
            mbar_wait_drain_(&sm.drain, 0, DRAIN_NS);
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 104;" ::: "memory");
        // ---- softmax warpgroup (w, hf): query row r of query tile w, keys [64 hf, 64 hf + 64)
        // of each key tile.  The two halves of a row share its running maximum (exchanged through
        // shared memory each tile) and add their sums at the end.
        const int wg = (warp - 4) >> 2;
        const int w = wg >> 1, hf = wg & 1;
        const int q = warp & 3, r = q * 32 + lane;
        const uint32_t lane_base = ((uint32_t)(q * 32)) << 16;
        const uint32_t s_addr = tmem + lane_base + BM * w + 64 * hf;        // this half of S / P
        const uint32_t o_addr = tmem + lane_base + 256 + BM * w + 64 * hf;  // this half of O
        int cnt = 0, flip = 0;   // key tiles taken part in (all items): the barriers' phases
        bool ok = true;
        for (int64_t t = blockIdx.x; t < p.n_items && ok; t += gridDim.x) {
        // token positions fit in 32 bits (the host checks N)
        int q0, kt_lo, ntiles;
        {
            const SwaItem it = item_of(p, t);
            q0 = (int)it.q0;
            kt_lo = (int)it.kt_lo;
            ntiles = it.ntiles;
        }
        const int qi = q0 + BM * w + r;          // this thread's query position
        float m_ref = -INFINITY, l = 0.f;
        int cnt_item = 0;
        for (int i = 0; i < ntiles && ok; ++i) {
            const int kt = kt_lo + i;
            if (!takes_part(q0, w, kt, p.window, p.N)) continue;
            // pair-uniform outcome: no warp may split around the warp-wide TMEM accesses, and
            // neither half may leave while the other waits at the pair's barrier
            ok = pair_wait(sm, &sm.s_full[w], cnt & 1, w, hf, r, flip);
            if (!ok) break;
            tc_fence_after();
            // visible keys of this row in this half: columns [c_lo, c_hi] of the half
            const int c_lo64 = qi - p.window + 1 - BM * kt - 64 * hf, c_hi64 = qi - BM * kt - 64 * hf;
            const int c_lo = c_lo64 < 0 ? 0 : (c_lo64 > 64 ? 64 : c_lo64);
            const int c_hi = c_hi64 > 63 ? 63 : (c_hi64 < -1 ? -1 : c_hi64);
            // scores in log2 units are c s; the half's maximum of c s over its visible keys is
            // c max(s) for c >= 0 and c min(s) otherwise (eight independent partial extrema),
            // 32 columns at a time.  Halves wholly inside every row's window skip the per-key
            // mask.
            const float c = p.scale_log2;
            const bool full = __all_sync(0xffffffffu, c_lo == 0 && c_hi == 63);
            const bool up = c >= 0.f;
            float e8[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) e8[u] = up ? -INFINITY : INFINITY;
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                float sg[32];
                tmem_ld32(s_addr + 32 * g, sg);
                tmem_ld_wait();
                if (full) {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        e8[e & 7] = up ? fmaxf(e8[e & 7], sg[e]) : fminf(e8[e & 7], sg[e]);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (32 * g + e >= c_lo && 32 * g + e <= c_hi)
                            e8[e & 7] = up ? fmaxf(e8[e & 7], sg[e]) : fminf(e8[e & 7], sg[e]);
                }
            }
#pragma unroll
            for (int u = 4; u > 0; u >>= 1)
#pragma unroll
                for (int v = 0; v < u; ++v)
                    e8[v] = up ? fmaxf(e8[v], e8[v + u]) : fminf(e8[v], e8[v + u]);
            const float ext = e8[0];
            const float mx_half = (c_lo <= c_hi) ? c * ext : -INFINITY;
            // the row's maximum over both halves
            sm.xmax[cnt & 1][w][hf][r] = mx_half;
            pair_sync(w);
            const float mx = fmaxf(mx_half, sm.xmax[cnt & 1][w][hf ^ 1][r]);
            // move the reference when the tile's maximum passes it by the margin: O and l scale
            // by 2^(m_ref - mx) (both halves take the same decision from the same maximum; each
            // scales its own columns of O and its own partial sum).  The tensor-memory accesses
            // are warp-wide instructions, so the whole warp takes the branch when any of its
            // rows needs it (factor 1 for the others).
            const bool move = mx > m_ref + RESCALE_LOG2;
            const bool rescale = move && m_ref > -INFINITY;
            if (__any_sync(0xffffffffu, rescale)) {
                const float f = rescale ? ex2f(m_ref - mx) : 1.f;
                l *= f;
#pragma unroll 1
                for (int jc = 0; jc < 2; ++jc) {
                    float t32[32];
                    tmem_ld32(o_addr + jc * 32, t32);
                    tmem_ld_wait();
                    uint32_t u[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(t32[e] * f);
                    tmem_st32(o_addr + jc * 32, u);
                }
            }
            if (move) m_ref = mx;
            const float nm = -m_ref;   // finite whenever a key of the row is visible
            float l4[4] = {0.f, 0.f, 0.f, 0.f};   // independent partial sums
            // P, one 32-key group at a time, the group's scores read again from tensor memory
            // (so that the 64 scores of the maximum pass are not held through this one) and
            // replaced in place by the group's P: 16 columns of high halves, then 16 of low
            // halves, over the 32 columns the group's scores occupied.
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                float sg[32];
                tmem_ld32(s_addr + 32 * g, sg);
                tmem_ld_wait();
                // eight key pairs at a time: their high halves to columns 32 g + 8 sub, their
                // low halves to 32 g + 16 + 8 sub (the group's scores are all in sg already)
#pragma unroll
                for (int sub = 0; sub < 2; ++sub) {
                    uint32_t hi8[8], lo8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int k2 = 8 * sub + e;            // key pair within the group
                        const int c0 = g * 32 + 2 * k2;
                        float p0 = ex2f(fmaf(sg[2 * k2], c, nm));
                        float p1 = ex2f(fmaf(sg[2 * k2 + 1], c, nm));
                        if (!full) {
                            p0 = (c0 >= c_lo && c0 <= c_hi) ? p0 : 0.f;
                            p1 = (c0 + 1 >= c_lo && c0 + 1 <= c_hi) ? p1 : 0.f;
                        }
                        l4[e & 3] += p0 + p1;
                        split2_trunc(p0, p1, hi8[e], lo8[e]);
                    }
                    tmem_st8(s_addr + 32 * g + 8 * sub, hi8);
                    tmem_st8(s_addr + 32 * g + 16 + 8 * sub, lo8);
                }
            }
            l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&sm.p_ready[w][hf]);   // P V over this half's keys may run
            ++cnt;
            ++cnt_item;
        }
        // ---- epilogue: O / l in bf16 through this tile's query slot (each half its 64
        // columns), then one TMA store.  O_w is released (o_free) once read, the query slot
        // (q_free) once the store has read it; both once per item, also for a tile that took
        // no part.
        if (cnt_item > 0) {
            if (ok) ok = pair_wait(sm, &sm.pv_done[w], (cnt - 1) & 1, w, hf, r, flip);
            tc_fence_after();
            sm.xl[w][hf][r] = l;
            pair_sync(w);
            const float lt = l + sm.xl[w][hf ^ 1][r];
            const float inv = ok && lt > 0.f ? 1.f / lt : __int_as_float(0x7fc00000);
            unsigned char* row = sm.q[w] + hf * SLAB + r * 128;
#pragma unroll 1
            for (int jc = 0; jc < 2; ++jc) {
                float t32[32];
                tmem_ld32(o_addr + jc * 32, t32);
                tmem_ld_wait();
                if (jc == 1) {
                    tc_fence_before();
                    mbar_arrive(&sm.o_free[w]);
                }
#pragma unroll
                for (int v4 = 0; v4 < 4; ++v4) {
                    uint4 u;
                    u.x = pack_bf16x2(t32[8 * v4 + 0] * inv, t32[8 * v4 + 1] * inv);
                    u.y = pack_bf16x2(t32[8 * v4 + 2] * inv, t32[8 * v4 + 3] * inv);
                    u.z = pack_bf16x2(t32[8 * v4 + 4] * inv, t32[8 * v4 + 5] * inv);
                    u.w = pack_bf16x2(t32[8 * v4 + 6] * inv, t32[8 * v4 + 7] * inv);
                    const int cc = 4 * jc + v4;   // 16-byte chunk of the half-row
                    *reinterpret_cast<uint4*>(row + ((cc ^ (r & 7)) << 4)) = u;
                }
            }
            fence_proxy_async_smem();
            pair_sync(w);   // both halves of the tile are written
            if (hf == 0 && r == 0) {
                const SwaItem it = item_of(p, t);
                for (int half = 0; half < 2; ++half)
                    tma_store_4d(&to, sm.q[w] + half * SLAB, half * 64, it.h, q0 + BM * w, it.b);
                bulk_commit_group();
                bulk_wait_group_read0();
                mbar_arrive(&sm.q_free[w]);
            }
        } else {
            mbar_arrive(&sm.o_free[w]);
            if (hf == 0 && r == 0) mbar_arrive(&sm.q_free[w]);
        }
        }   // items
        if (hf == 0 && r == 0) bulk_wait_group0();   // the last stores have completed
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

cudaError_t launch_swa(const SwaArgs& a, cudaStream_t stream) {
    // [B, N, H, 128] contiguous: dims (d, head, token, batch), box (64, 1, 128, 1)
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)a.H, (uint64_t)a.N, (uint64_t)a.B};
    const uint64_t strides[3] = {(uint64_t)D * 2, (uint64_t)a.H * D * 2,
                                 (uint64_t)a.N * a.H * D * 2};
    const uint32_t box[4] = {64, 1, BM, 1};
    CUtensorMap tq, tk, tv, to;
    if (!make_bf16_map(&tq, a.q, 4, dims, strides, box) ||
        !make_bf16_map(&tk, a.k, 4, dims, strides, box) ||
        !make_bf16_map(&tv, a.v, 4, dims, strides, box) ||
        !make_bf16_map(&to, a.o, 4, dims, strides, box))
        return cudaErrorInvalidValue;
    if (a.N > (int64_t)0x7FFFFE00) return cudaErrorInvalidValue;   // 32-bit token coordinates
    SwaParams p;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.window = a.window;
    p.N = a.N;
    p.H = a.H;
    p.n_qpairs = (int)((a.N + 2 * BM - 1) / (2 * BM));
    p.n_items = (int64_t)a.B * a.H * p.n_qpairs;
    // persistent: one CTA per SM (at most one per item)
    int dev = 0, n_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        n_sm < 1)
        return cudaErrorUnknown;
    const int64_t grid = p.n_items < n_sm ? p.n_items : n_sm;
    if (grid == 0) return cudaSuccess;   // nothing to do
    const size_t smem = sizeof(SwaSmem);
    cudaError_t e = cudaFuncSetAttribute(swa_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    static int regs = -1;
    if (regs < 0) {
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, swa_tc_kernel) != cudaSuccess) return cudaErrorUnknown;
        regs = fa.numRegs;
    }
    // the in-kernel register split (setmaxnreg) assumes exactly LAUNCH_REGS per thread
    if (regs != LAUNCH_REGS) return cudaErrorInvalidValue;
    swa_tc_kernel<<<(unsigned)grid, NTHREADS, smem, stream>>>(tq, tk, tv, to, p);
    return cudaGetLastError();
}

}  // namespace gret
