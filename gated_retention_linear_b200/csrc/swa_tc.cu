// swa_tc.cu -- sliding-window softmax attention prefill on the sm_100a tensor cores.
//
// Page "YOCO 完全拆解：Decoder-Decoder 架构如何让 KV Cache 只存一次", section
// "路线一：滑动窗口注意力": position i attends to the most recent W positions of its sequence,
//   o_i = sum_{j = i-W+1 .. i} softmax_j(scale q_i . k_j) v_j .
// FlashAttention-style, as the page suggests for this mixer, built on tcgen05:
//   * an item of work is one 128-query tile of one (batch, head); the key tiles of 128 that its
//     window touches (nine at W = 1024) stream through shared memory (two K stages, three V
//     stages).  The kernel is persistent: one CTA per SM takes items round-robin, consecutive
//     items being neighbouring query tiles of one head (their key tiles meet in L2);
//   * every key tile j of the CTA (numbered across items) has its own score buffer S[j % 3] in
//     tensor memory and its own softmax warpgroup j % 3, so that Q K^T runs up to three key
//     tiles ahead of P V and three softmaxes overlap the products, instead of one tile's
//     Q K^T -> softmax -> P V chain setting the pace;
//   * a softmax thread owns one query row of its tile (all 128 keys): it masks the window,
//     takes the row's maximum, writes P = 2^(s - m) back over S as a bf16 high + low pair, and
//     the MMA warp accumulates O += P_hi V + P_lo V as each half of the keys arrives;
//   * the row's reference maximum m is handed from tile to tile (through shared memory, one
//     mbarrier per tile parity): it only moves, and O and the running sum are rescaled, when a
//     tile's maximum exceeds it by more than 2^8, so rescaling is rare after the first tiles and
//     P stays below 256.  The running sum l is handed on the same way, one tile later;
//   * the warpgroup of an item's last key tile writes O / l in bf16 straight from its
//     registers to HBM (16-byte stores, rows past the sequence end skipped).  An item's query
//     slot is freed by the completion of its last Q K^T, so no Q K^T ever waits for a P V (with
//     Q K^T three tiles ahead, a slot freed by the output would deadlock behind items of fewer
//     than three key tiles).
// P is carried as two bf16 halves because a single bf16 rounding of P over a 1024-key window
// leaves errors near 1e-2 of rms; the pair (split by truncation, see split2_trunc) keeps the
// result near 1e-5.
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), S2 [256,384), O [384,512).
// Warp roles (512 threads): warp 0 TMA producer, warp 1 MMA issuer (one elected lane), warps 4-7,
// 8-11 and 12-15 the softmax warpgroups 0, 1, 2.  Registers: launched at 128 per thread; warps
// 0-3 drop to 80 and the softmax warpgroups rise to 144: 32 x (4 x 80 + 12 x 144) = 65536.
// Every wait is bounded; a wait that gives up makes every role of the CTA stop (the item in
// progress gets NaN rows if its last warpgroup still reaches the output).  A warpgroup waits as
// one: one thread polls the barrier while the other 127 sleep at the group's named barrier, and
// all take the same branch.
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
constexpr int NTHREADS = 512;
constexpr int LAUNCH_REGS = 128;
constexpr int NBUF = 3;                  // score buffers = softmax warpgroups = V stages
constexpr uint32_t TM_O = 384;           // O's first tensor-memory column
constexpr uint64_t WAIT_NS = 2000000000ull;
constexpr uint64_t DRAIN_NS = 200000000ull;
constexpr float RESCALE_LOG2 = 8.f;      // move the reference maximum only past this margin

struct __align__(1024) SwaSmem {
    unsigned char q[2][TILE];            // query tile of item n in slot n % 2
    unsigned char k[2][TILE];            // key tile j in stage j % 2
    unsigned char v[NBUF][TILE];         // value tile j in stage j % 3
    // q_full / q_free: an item's query tile is loaded / read by the item's last Q K^T
    uint64_t q_full[2], q_free[2], k_full[2], k_empty[2], v_full[NBUF], v_empty[NBUF];
    // s_full[b]: Q K^T of the key tile in buffer b is done; p_ready[b][h]: its P over keys
    // [64 h, 64 h + 64) is in tensor memory; pv_done[b]: P V of that tile is done
    uint64_t s_full[NBUF], p_ready[NBUF][2], pv_done[NBUF];
    // dec_full[j % 2] / l_full[j % 2]: key tile j's reference maximum / running sum is posted
    uint64_t dec_full[2], l_full[2], o_free, drain;
    uint32_t dec[NBUF][2];               // the warpgroups' shared wait outcomes
    float mref[2][BM];                   // [key tile parity][row]
    float lsum[2][BM];
    uint32_t tmem_base;
    uint32_t abort;
};
static_assert(sizeof(SwaSmem) <= 232448, "shared-memory plan exceeds 227 KB");

struct SwaParams {
    __nv_bfloat16* o;      // [B, N, H, 128]
    float scale_log2;      // scale * log2(e)
    int window;
    int64_t N;
    int H;
    int n_qt;              // query tiles per sequence
    int64_t n_items;       // (batch, head, query tile) items
};

// One item of work: the 128-query tile q0 .. q0 + 127 of one (batch, head), and the key tiles
// [kt_lo, kt_lo + ntiles) its window touches.
struct SwaItem {
    int64_t q0, kt_lo;
    int ntiles, h, b;
};

__device__ __forceinline__ SwaItem item_of(const SwaParams& p, int64_t t) {
    SwaItem it;
    const int qt = (int)(t % p.n_qt);
    it.h = (int)((t / p.n_qt) % p.H);
    it.b = (int)(t / ((int64_t)p.n_qt * p.H));
    it.q0 = (int64_t)qt * BM;
    const int64_t qlast = (it.q0 + BM - 1 < p.N - 1) ? it.q0 + BM - 1 : p.N - 1;
    const int64_t kfirst = (it.q0 - p.window + 1 > 0) ? it.q0 - p.window + 1 : 0;
    it.kt_lo = kfirst / BM;
    it.ntiles = (int)(qlast / BM - it.kt_lo + 1);
    return it;
}

// Walks this CTA's items (t = blockIdx.x, blockIdx.x + gridDim.x, ...) and their key tiles,
// numbered across items: key tile j belongs to item number n, whose first tile is jbase.
struct TileWalk {
    int64_t t;
    int n, jbase;
    SwaItem it;
    __device__ explicit TileWalk(const SwaParams& p) : t(blockIdx.x), n(0), jbase(0) {
        if (t < p.n_items) it = item_of(p, t);
    }
    // moves to the item that holds key tile j (j never decreases); false past the last item
    __device__ bool seek(const SwaParams& p, int j) {
        while (t < p.n_items && j >= jbase + it.ntiles) {
            jbase += it.ntiles;
            ++n;
            t += gridDim.x;
            if (t < p.n_items) it = item_of(p, t);
        }
        return t < p.n_items;
    }
};

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

// The same split as split2_trunc with the two remainders taken by one packed subtraction.
__device__ __forceinline__ void split2_trunc_x2(float2 x, uint32_t& hi, uint32_t& lo) {
    const uint32_t b0 = __float_as_uint(x.x), b1 = __float_as_uint(x.y);
    const float2 h = make_float2(__uint_as_float(b0 & 0xFFFF0000u), __uint_as_float(b1 & 0xFFFF0000u));
    const float2 l = add2(x, make_float2(-h.x, -h.y));
    hi = __byte_perm(b0, b1, 0x7632);
    lo = __byte_perm(__float_as_uint(l.x), __float_as_uint(l.y), 0x7632);
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

__device__ __forceinline__ void group_sync(int gid) {
    asm volatile("bar.sync %0, 128;" ::"r"(1 + gid) : "memory");
}

// A softmax warpgroup's wait: thread 0 of the group polls the barrier, the other 127 sleep at
// the group's named barrier, and all take the same branch.  The outcome word is
// double-buffered, so that thread 0 cannot overwrite it for the next wait before a slow thread
// of the group has read it.
__device__ __forceinline__ bool group_wait(SwaSmem& sm, uint64_t* bar, uint32_t parity, int gid,
                                           int r, int& flip) {
    if (r == 0) sm.dec[gid][flip] = wait_abortable(sm, bar, parity) ? 1u : 0u;
    group_sync(gid);
    const bool ok = *reinterpret_cast<volatile uint32_t*>(&sm.dec[gid][flip]) != 0;
    flip ^= 1;
    return ok;
}

// true on every thread of the warpgroup when x holds on any of them
__device__ __forceinline__ bool group_any(bool x, int gid) {
    uint32_t res;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(res)
        : "r"((uint32_t)x), "r"(1 + gid)
        : "memory");
    return res != 0;
}

// The MMA issue loops are fully unrolled over constant descriptor offsets, and the whole of
// warp 1 runs them (one elected lane issues each instruction), so that the operands can stay
// in uniform registers: issued from one lane of a diverged warp, with each step's descriptor
// formed just before its MMA, the issue took longer than a 128x128x16 MMA takes to execute.  The empty asm
// statements pin each call's descriptor bases where they are made, so that the compiler does
// not hoist every unrolled descriptor of every stage out of the key-tile loop.

// S = Q K^T over K = 128 with both operands K-major in shared memory.
__device__ __forceinline__ void mma_qk(uint32_t d, uint32_t a_base, uint32_t b_base) {
    constexpr uint32_t idesc = idesc_bf16(128, 128, 0, 0);
    uint64_t ad = sdesc_sw128(a_base, 16, 1024), bd = sdesc_sw128(b_base, 16, 1024);
    asm volatile("" : "+l"(ad), "+l"(bd));
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = ((kk >> 2) * SLAB + (kk & 3) * 32u) >> 4;
        mma_ss_w(d, ad + off, bd + off, idesc, kk > 0 ? 1u : 0u);
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
            mma_ts_w(d, pb + 32 * (kk >> 1) + 8 * (kk & 1) + 16 * half, vd + ((kk * 2048u) >> 4),
                   idesc, (accumulate || half > 0 || kk > 0) ? 1u : 0u);
}

// ---- warp 0: TMA producer.  Per item its query tile (slot n % 2, once item n - 2's last
// Q K^T has read the slot) ahead of its first key tile; key tiles j in K stage j % 2 and V stage
// j % 3.  The K stream runs one tile ahead of the V stream: K stage j % 2 is freed by Q K^T of
// tile j - 2, which completes before P V of tile j - 4 frees the V stage of tile j - 1.
__device__ void producer(SwaSmem& sm, const SwaParams& p, const CUtensorMap* tq,
                         const CUtensorMap* tk, const CUtensorMap* tv) {
    tma_prefetch_desc(tq);
    tma_prefetch_desc(tk);
    tma_prefetch_desc(tv);
    TileWalk wk(p), wv(p);
    int jk = 0, jv = 0, nq = 0;   // key tiles, value tiles and query tiles issued
    bool ok = true;
    auto load = [&](const CUtensorMap* map, unsigned char* dst, uint64_t* bar, const SwaItem& it,
                    int tok) {
        mbar_arrive_expect_tx(bar, TILE);
        for (int half = 0; half < 2; ++half)
            tma_load_4d(dst + half * SLAB, map, bar, half * 64, it.h, tok, it.b);
    };
    while (ok) {
        const bool more_k = wk.seek(p, jk);
        if (more_k) {
            const int i = jk - wk.jbase;
            if (i == 0) {   // the item's query tile
                const int n = wk.n, qs = n & 1;
                if (n >= 2 && !(ok = wait_abortable(sm, &sm.q_free[qs], ((n >> 1) - 1) & 1)))
                    break;
                load(tq, sm.q[qs], &sm.q_full[qs], wk.it, (int)wk.it.q0);
                nq = n + 1;
            }
            const int ks = jk & 1;
            if (jk >= 2 && !(ok = wait_abortable(sm, &sm.k_empty[ks], ((jk >> 1) - 1) & 1))) break;
            load(tk, sm.k[ks], &sm.k_full[ks], wk.it, (int)((wk.it.kt_lo + i) * BM));
            ++jk;
        }
        if (jv < jk - (more_k ? 1 : 0)) {
            wv.seek(p, jv);
            const int vs = jv % NBUF;
            if (jv >= NBUF && !(ok = wait_abortable(sm, &sm.v_empty[vs], (jv / NBUF - 1) & 1)))
                break;
            load(tv, sm.v[vs], &sm.v_full[vs], wv.it, (int)((wv.it.kt_lo + jv - wv.jbase) * BM));
            ++jv;
        } else if (!more_k) {
            break;
        }
    }
    // no TMA write into this CTA's shared memory may be in flight at exit
    for (int jj = (jk >= 2 ? jk - 2 : 0); jj < jk; ++jj)
        mbar_wait_drain_(&sm.k_full[jj & 1], (jj >> 1) & 1, DRAIN_NS);
    for (int jj = (jv >= NBUF ? jv - NBUF : 0); jj < jv; ++jj)
        mbar_wait_drain_(&sm.v_full[jj % NBUF], (jj / NBUF) & 1, DRAIN_NS);
    for (int nn = (nq >= 2 ? nq - 2 : 0); nn < nq; ++nn)
        mbar_wait_drain_(&sm.q_full[nn & 1], (nn >> 1) & 1, DRAIN_NS);
}

// ---- warp 1: the MMA issuer (the whole warp, converged; one elected lane issues).  Q K^T of
// key tile j into S[j % 3] once P V of tile j - 3 has read that buffer; P V of tile j as its
// softmax hands P over, half the keys at a time.  Issue order: Q K^T of tiles 0, 1, 2, then per
// tile j: P V_j, Q K^T_{j+3}.
__device__ void mma_issuer(SwaSmem& sm, const SwaParams& p, uint32_t tmem) {
    TileWalk wq(p), wp(p);   // the Q K^T and the P V streams
    int jq = 0, jp = 0;
    bool ok = true;
    auto W = [&](uint64_t* bar, uint32_t parity) {   // warp-uniform outcome (lane 0's)
        if (ok) ok = __shfl_sync(0xffffffffu, wait_abortable(sm, bar, parity) ? 1 : 0, 0) != 0;
        return ok;
    };
    auto issue_qk = [&](int j) {
        const int i = j - wq.jbase, n = wq.n, b = j % NBUF;
        if (i == 0 && !W(&sm.q_full[n & 1], (n >> 1) & 1)) return;
        if (!W(&sm.k_full[j & 1], (j >> 1) & 1)) return;
        if (j >= NBUF && !W(&sm.pv_done[b], (j / NBUF - 1) & 1)) return;
        tc_fence_after();
        mma_qk(tmem + BM * b, smem_u32(sm.q[n & 1]), smem_u32(sm.k[j & 1]));
        mma_commit_w(&sm.s_full[b]);
        mma_commit_w(&sm.k_empty[j & 1]);
        if (i + 1 == wq.it.ntiles) mma_commit_w(&sm.q_free[n & 1]);   // the item's last Q K^T
    };
    auto issue_pv = [&](int j) {
        const int i = j - wp.jbase, n = wp.n, b = j % NBUF;
        const uint32_t use = (uint32_t)(j / NBUF);
        if (i == 0 && n > 0 && !W(&sm.o_free, (n - 1) & 1)) return;   // last item's O read
        if (!W(&sm.v_full[b], use & 1)) return;
        const uint32_t vb = smem_u32(sm.v[b]);
        for (int kh = 0; kh < 2; ++kh) {
            if (!W(&sm.p_ready[b][kh], use & 1)) return;
            tc_fence_after();
            mma_pv(tmem + TM_O, tmem + BM * b, kh, vb, i > 0 || kh > 0);
        }
        mma_commit_w(&sm.pv_done[b]);
        mma_commit_w(&sm.v_empty[b]);
    };
    while (ok) {
        while (ok && jq < jp + NBUF && wq.seek(p, jq)) issue_qk(jq++);
        if (!ok || !wp.seek(p, jp)) break;
        issue_pv(jp++);
    }
    // all issued MMAs complete before tensor memory is released
    mma_commit_w(&sm.drain);
    mbar_wait_drain_(&sm.drain, 0, DRAIN_NS);
}

// ---- softmax warpgroup gid: key tiles j = gid, gid + 3, ... (score buffer S[gid], V stage
// gid); thread r owns query row r of the tile's item.
__device__ void softmax_group(SwaSmem& sm, const SwaParams& p, uint32_t tmem, int gid, int warp,
                              int lane) {
    const int q = warp & 3, r = q * 32 + lane;
    const uint32_t lane_base = ((uint32_t)(q * 32)) << 16;
    const uint32_t s_addr = tmem + lane_base + BM * gid;   // this row of S / P
    const uint32_t o_addr = tmem + lane_base + TM_O;       // this row of O
    const float c = p.scale_log2;
    const bool up = c >= 0.f;
    TileWalk wk(p);
    int flip = 0;
    bool ok = true;
    for (int j = gid; ok && wk.seek(p, j); j += NBUF) {
        const int i = j - wk.jbase;
        const uint32_t use = (uint32_t)(j / NBUF);
        // token positions fit in 32 bits (the host checks N)
        const int qi = (int)wk.it.q0 + r;            // this thread's query position
        const int kt = (int)wk.it.kt_lo + i;
        if (!(ok = group_wait(sm, &sm.s_full[gid], use & 1, gid, r, flip))) break;
        tc_fence_after();
        // visible keys of this row in this key tile: columns [c_lo, c_hi]
        const int lo128 = qi - p.window + 1 - BM * kt, hi128 = qi - BM * kt;
        const int c_lo = lo128 < 0 ? 0 : (lo128 > BM ? BM : lo128);
        const int c_hi = hi128 > BM - 1 ? BM - 1 : (hi128 < -1 ? -1 : hi128);
        const bool full = __all_sync(0xffffffffu, c_lo == 0 && c_hi == BM - 1);
        // scores in log2 units are c s; the row's maximum of c s over its visible keys is
        // c max(s) for c >= 0 and c min(s) otherwise (eight independent partial extrema)
        float e8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) e8[u] = up ? -INFINITY : INFINITY;
#pragma unroll 1
        for (int g = 0; g < 4; ++g) {
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
        const float mx = (c_lo <= c_hi) ? c * e8[0] : -INFINITY;
        // the reference maximum after the previous key tile (every tile waits for it, also the
        // first of an item, whose reference starts afresh, so that the barrier's phases stay
        // in step)
        float m_prev = -INFINITY;
        if (j > 0) {
            if (!(ok = group_wait(sm, &sm.dec_full[(j - 1) & 1], ((j - 1) >> 1) & 1, gid, r, flip)))
                break;
            if (i > 0) m_prev = sm.mref[(j - 1) & 1][r];
        }
        const bool move = mx > m_prev + RESCALE_LOG2;
        const float m = move ? mx : m_prev;
        const bool rescale = move && m_prev > -INFINITY;
        sm.mref[j & 1][r] = m;
        mbar_arrive(&sm.dec_full[j & 1]);
        // O holds the rows' sums over the item's earlier key tiles relative to m_prev; rows that
        // move scale them by 2^(m_prev - m) once P V of tile j - 1 is done, and P V of this tile
        // may only start after that.  The wait comes after this tile's P is written, so that it
        // overlaps the previous tile's products.
        const bool any_rescale = group_any(rescale, gid);
        // P, one 32-key group at a time, the group's scores read again from tensor memory and
        // replaced in place by the group's P: 16 columns of high halves, then 16 of low halves.
        // P V over the first 64 keys may start once their P is written (unless O is rescaled).
        const float nm = -m;   // finite whenever a key of the row is visible
        const float2 c2 = make_float2(c, c), nm2 = make_float2(nm, nm);
        float2 l4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};   // independent partial sums, two lanes each
#pragma unroll 1
        for (int g = 0; g < 4; ++g) {
            float sg[32];
            tmem_ld32(s_addr + 32 * g, sg);
            tmem_ld_wait();
#pragma unroll
            for (int sub = 0; sub < 2; ++sub) {
                uint32_t hi8[8], lo8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int k2 = 8 * sub + e;            // key pair within the group
                    const int c0 = g * 32 + 2 * k2;
                    const float2 arg = fma2(make_float2(sg[2 * k2], sg[2 * k2 + 1]), c2, nm2);
                    float2 pp = make_float2(ex2f(arg.x), ex2f(arg.y));
                    if (!full) {
                        pp.x = (c0 >= c_lo && c0 <= c_hi) ? pp.x : 0.f;
                        pp.y = (c0 + 1 >= c_lo && c0 + 1 <= c_hi) ? pp.y : 0.f;
                    }
                    l4[e & 3] = add2(l4[e & 3], pp);
                    split2_trunc_x2(pp, hi8[e], lo8[e]);
                }
                tmem_st8(s_addr + 32 * g + 8 * sub, hi8);
                tmem_st8(s_addr + 32 * g + 16 + 8 * sub, lo8);
            }
            if (g == 1 && !any_rescale) {
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&sm.p_ready[gid][0]);
            }
        }
        if (any_rescale) {
            // a warp rescales (by 1 for its other rows) when any of its rows moves: the tensor
            // memory accesses are warp-wide instructions
            if (!(ok = group_wait(sm, &sm.pv_done[(j - 1) % NBUF], ((j - 1) / NBUF) & 1, gid, r,
                                  flip)))
                break;
            tc_fence_after();
            if (__any_sync(0xffffffffu, rescale)) {
                const float f = rescale ? ex2f(m_prev - m) : 1.f;
#pragma unroll 1
                for (int jc = 0; jc < 4; ++jc) {
                    float t32[32];
                    tmem_ld32(o_addr + jc * 32, t32);
                    tmem_ld_wait();
                    uint32_t u[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(t32[e] * f);
                    tmem_st32(o_addr + jc * 32, u);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&sm.p_ready[gid][0]);
        } else {
            tmem_st_wait();
            tc_fence_before();
        }
        mbar_arrive(&sm.p_ready[gid][1]);
        // the running sum: the previous tile's, relative to m_prev, plus this tile's
        float l_prev = 0.f;
        if (j > 0) {
            if (!(ok = group_wait(sm, &sm.l_full[(j - 1) & 1], ((j - 1) >> 1) & 1, gid, r, flip)))
                break;
            if (i > 0) l_prev = sm.lsum[(j - 1) & 1][r];
        }
        const float2 l2 = add2(add2(l4[0], l4[1]), add2(l4[2], l4[3]));
        const float l = (rescale ? l_prev * ex2f(m_prev - m) : l_prev) + (l2.x + l2.y);
        sm.lsum[j & 1][r] = l;
        mbar_arrive(&sm.l_full[j & 1]);
        if (i + 1 < wk.it.ntiles) continue;
        // ---- the item's last key tile: O / l in bf16, row r straight to HBM.  O is released
        // (o_free) once read.
        ok = group_wait(sm, &sm.pv_done[gid], use & 1, gid, r, flip);
        tc_fence_after();
        const float inv = ok && l > 0.f ? 1.f / l : __int_as_float(0x7fc00000);
        const bool in = (int64_t)qi < p.N;
        uint4* orow = reinterpret_cast<uint4*>(
            p.o + (((int64_t)wk.it.b * p.N + (in ? qi : 0)) * p.H + wk.it.h) * D);
#pragma unroll 1
        for (int jc = 0; jc < 4; ++jc) {
            float t32[32];
            tmem_ld32(o_addr + jc * 32, t32);
            tmem_ld_wait();
            if (jc == 3) {
                tc_fence_before();
                mbar_arrive(&sm.o_free);
            }
            if (in) {
#pragma unroll
                for (int v4 = 0; v4 < 4; ++v4) {
                    uint4 u;
                    u.x = pack_bf16x2(t32[8 * v4 + 0] * inv, t32[8 * v4 + 1] * inv);
                    u.y = pack_bf16x2(t32[8 * v4 + 2] * inv, t32[8 * v4 + 3] * inv);
                    u.z = pack_bf16x2(t32[8 * v4 + 4] * inv, t32[8 * v4 + 5] * inv);
                    u.w = pack_bf16x2(t32[8 * v4 + 6] * inv, t32[8 * v4 + 7] * inv);
                    orow[4 * jc + v4] = u;
                }
            }
        }
    }
}

__global__ void __launch_bounds__(NTHREADS, 1)
    swa_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, const SwaParams p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    SwaSmem& sm = *reinterpret_cast<SwaSmem*>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if ((smem_u32(smem_raw) & 1023u) != 0) return;   // never: dynamic shared memory starts aligned
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sm.q_full[s], 1);
            mbar_init(&sm.q_free[s], 1);
            mbar_init(&sm.k_full[s], 1);
            mbar_init(&sm.k_empty[s], 1);
            mbar_init(&sm.dec_full[s], 128);
            mbar_init(&sm.l_full[s], 128);
        }
        for (int s = 0; s < NBUF; ++s) {
            mbar_init(&sm.v_full[s], 1);
            mbar_init(&sm.v_empty[s], 1);
            mbar_init(&sm.s_full[s], 1);
            mbar_init(&sm.p_ready[s][0], 128);
            mbar_init(&sm.p_ready[s][1], 128);
            mbar_init(&sm.pv_done[s], 1);
        }
        mbar_init(&sm.o_free, 128);
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
    // The CTA is persistent: every role walks the same items and key tiles, and every
    // barrier's phase count runs on across items.
    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 80;" ::: "memory");
        if (warp == 0 && lane == 0) producer(sm, p, &tq, &tk, &tv);
        else if (warp == 1) mma_issuer(sm, p, tmem);
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 144;" ::: "memory");
        softmax_group(sm, p, tmem, (warp - 4) >> 2, warp, lane);
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
    CUtensorMap tq, tk, tv;
    if (!make_bf16_map(&tq, a.q, 4, dims, strides, box) ||
        !make_bf16_map(&tk, a.k, 4, dims, strides, box) ||
        !make_bf16_map(&tv, a.v, 4, dims, strides, box))
        return cudaErrorInvalidValue;
    if (a.N > (int64_t)0x7FFFFE00) return cudaErrorInvalidValue;   // 32-bit token coordinates
    SwaParams p;
    p.o = a.o;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.window = a.window;
    p.N = a.N;
    p.H = a.H;
    p.n_qt = (int)((a.N + BM - 1) / BM);
    p.n_items = (int64_t)a.B * a.H * p.n_qt;
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
    swa_tc_kernel<<<(unsigned)grid, NTHREADS, smem, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

}  // namespace gret
