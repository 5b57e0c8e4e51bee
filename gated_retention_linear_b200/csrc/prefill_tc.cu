// prefill_tc.cu -- chunkwise gated-retention prefill on the sm_100a tensor cores.
//
// Method: page "YOCO 完全拆解：Decoder-Decoder 架构如何让 KV Cache 只存一次", section
// "Prefill 与 Decode 为什么使用两种计算形态".  Each chunk of C = 128 tokens of one head is done
// with 128x128x128 tcgen05 MMAs accumulating in fp32 tensor memory:
//     A   = Q K^T                       (intra-chunk scores, exact from the bf16 inputs)
//     P   = k_scale * exp(c_t - c_m) * A for m <= t, else 0     (decay mask, CUDA cores)
//     O   = P V                         (inner term)
//     OX  = Q S_prev                    (cross-chunk term; added as exp(c_t) * OX)
//     dS  = (w K)^T V,  w_m = k_scale * exp(c_b - c_m)     (chunk contribution to the state)
//     S   = exp(c_b) S_prev + dS        (fp32 master state, in registers)
// c_t is the in-chunk inclusive cumulative log-decay (a warp scan of logsigmoid(g)/tau), always
// used as a difference inside one chunk, so no exponent can overflow.
//
// Precision.  P, the state copy and w K are fp32 values that an MMA needs as bf16.  Rounding
// each to bf16 once costs up to 2^-8 relative per element and leaves errors near 1e-2 of rms
// on large outputs.  Each is therefore split into a bf16 high half and a bf16 low half (x - hi),
// and both halves go through the MMA: P V, Q S_prev and (w K)^T V are each two MMAs, which keeps
// the result near 1e-5 of rms.  V and Q are used exactly as loaded.
//
// Where the operands live.  Shared memory holds two stages of K and V tiles, two Q tiles and
// the bf16 state copy: 7 x 32 KB.  The weighted keys never go back to shared memory: the
// converter group reads each key column straight out of the K tile, weights it, splits it into
// bf16 halves and stores (w K)^T into tensor memory, where dS reads it as its A operand (the
// same layout P V reads P in).  Tensor memory (512 columns): A / P [0,128), OX [128,256), one
// region [256,384) that holds dS and then O (dS is folded into the registers of the state group
// before P V writes O over it), and (w K)^T [384,512).  A chunk's bf16 output tile is staged in
// its own Q slot (free once Q K^T and Q S have read it) and leaves by TMA store.
//
// Parallelism across a sequence.  The chunk chain of one (sequence, head) is sequential, and
// one 3B-shaped layer has only 24 chains for 148 SMs.  Each chain is therefore cut into spans
// of G chunks (G chosen on the host from a wave model, see span_chunks).  A persistent CTA
// takes spans from an atomic ticket in chain order and runs:
//   pass A: read K, V, g of the span's chunks, last to first, each key weighted by its decay
//           to the end of the span, so that every dS MMA of the span accumulates into one
//           tensor-memory result: the span's aggregate Agg = sum over its keys of
//           (decay to the span end) k^T v;
//   look-back: wait for the inclusive state of span s-1 of the same chain (a bounded spin on a
//           flag in the workspace), entry E = that state (or state_in for s = 0), and publish
//           the inclusive state exp(L_span) E + Agg for span s+1;
//   pass B: the full chunk pipeline above from E, writing O.
// Inclusive states live in a two-slot ring per chain: span s+2 can only overwrite the slot of
// span s after span s+1 has consumed it, because it needs span s+1's own inclusive state first.
// Tickets are taken by running CTAs in increasing order and every span depends only on a smaller
// ticket, so the chain always progresses.
//
// Warp roles (512 threads = 4 warpgroups, one CTA per SM):
//   warp 0      TMA producer (lane 0): K and V tiles (two stages), Q tiles (two slots); the
//               whole warp scans the chunk's gate logits into the stage's gate slot (in-chunk
//               cumulative log2-decay, chunk total, key weights)
//   warp 1      tcgen05 MMA issuer (one thread); owns the 512-column TMEM allocation
//   warps 4-7   P group: decay mask A -> P (bf16 halves in TMEM) and the output epilogue
//               O + exp(c_t) OX -> bf16 -> the chunk's Q slot -> TMA store
//   warps 8-11  state group: fp32 state (one row per thread), the look-back, the bf16 halves
//               of the state that Q S_prev reads
//   warps 12-15 converter group: (w K)^T in TMEM for every chunk of both passes
// Per pass-B chunk the MMA issuer runs Q K^T, Q S_hi, dS, Q S_lo, P V; the only step that waits
// for the previous chunk's state is Q S (after the state group's fold and bf16 writes), and dS
// and the converter's work depend on nothing but the chunk's own K and V.
// Registers: launched at 128 per thread (512 x 128 = 65536); warps 0-3 and the converter group
// drop to 72, the P group rises to 136 and the state group (128 fp32 state values per thread)
// to 232: 128 x (72 + 136 + 232 + 72) = 65536, and each SM sub-partition (one warp
// of each group) needs 32 x 512 = 16384.  The host refuses to launch a build whose per-thread
// register count is not 128, since a request for more registers than the block holds would
// wait forever.
// Every wait is bounded (see sm100::mbar_wait); a wait that gives up records GRET_ERR_TIMEOUT in
// the workspace, and the kernel drains its copies, frees TMEM and exits.
#include "prefill_tc.cuh"

#include <stdlib.h>

#include <algorithm>
#include <cmath>

#include "sm100.cuh"
#include "tma_host.cuh"

namespace gret {

using namespace sm100;

namespace {

constexpr int C = 128;                  // tokens per chunk
constexpr int D = 128;                  // head width (d_k = d_v)
constexpr int TILE = C * D * 2;         // one bf16 128x128 tile
constexpr int SLAB = TILE / 2;          // one 64-column slab
constexpr int NTHREADS = 512;
constexpr int LAUNCH_REGS = 128;        // 65536 / NTHREADS
constexpr int ITEM_DEPTH = 4;
constexpr uint64_t WAIT_NS = 2000000000ull;   // a wait gives up after 2 s
constexpr uint64_t DRAIN_NS = 200000000ull;   // exit-time drains give up after 0.2 s

constexpr uint32_t TM_A = 0, TM_OX = 128, TM_DO = 256, TM_KT = 384;

struct Item {
    int32_t valid;
    int32_t u, h, s;
    int32_t c_begin, c_end;   // chunk range of the span, in chunks of the unit
    int32_t first, last;      // first / last span of the chain
    int32_t b;                // batch coordinate (dense) or 0
    int32_t pad;
    int64_t len;              // tokens in the unit
    int64_t tok_first;        // token coordinate of the unit's first token
    int64_t grow0;            // row of the unit's first token in g
};

struct __align__(1024) Smem {
    unsigned char q[2][TILE];  // Q tiles of pass B; after a chunk's Q S, its bf16 output tile
    unsigned char k[2][TILE];
    unsigned char v[2][TILE];
    // bf16 high half, then low half, of the state that Q S_prev reads; the look-back stages
    // the span's entry state through it
    unsigned char sb[TILE];
    uint64_t kv_full[2], kv_empty[2];
    uint64_t q_full[2], q_empty[2];
    uint64_t item_full[ITEM_DEPTH], item_empty[ITEM_DEPTH];
    uint64_t a_full, p_ready, s_ready, s_hi_done, s_lo_ready, sb_free, kt_ready, kt_free,
        ds_full, ds_free, o_full, o_free, drain;
    // per item slot: the span's pass-A gate scans are done and span_L holds its total decay
    uint64_t span_done[ITEM_DEPTH];
    Item items[ITEM_DEPTH];
    // per stage: in-chunk inclusive cumulative log2-decay of each token, and the key weights
    // k_scale * 2^(base - c_m) (0 past the end); written as float4 by the gate scan
    alignas(16) float gc[2][C];
    alignas(16) float w[2][C];
    float gtot[2];             // per stage: the chunk's total log2-decay
    float span_L[ITEM_DEPTH];  // per item slot: log2-decay over the whole span
    uint32_t dec[3][2];        // group-uniform wait decisions (double-buffered)
    uint32_t tmem_base;
    uint32_t abort;
};

// The dynamic shared memory a block can have on sm_100.
static_assert(sizeof(Smem) <= 232448, "shared-memory plan exceeds 227 KB");

struct TcParams {
    const float* g;
    float inv_tau_log2e;       // log2(e) / tau
    float k_scale;
    __nv_bfloat16* o;
    int64_t osb, ost, osh;
    const float* state_in;
    float* state_out;
    uint32_t* err;
    uint32_t* ticket;
    uint32_t* flags;           // [units][H][2]
    int32_t* prefix;           // varlen: [units + 1] span prefix; nullptr in dense mode
    float* slots;              // [units][H][2][128*128] inclusive states
    const int32_t* cu_seqlens;
    int64_t N;                 // dense: tokens per sequence
    int H, units, G;
    int spans_per_unit;        // dense
    int qk_pos_tok, qk_pos_head, qk_pos_b;   // tensor-map dimension of each coordinate
    int v_pos_tok, v_pos_head, v_pos_b;
    int o_pos_tok, o_pos_head, o_pos_b;
    uint64_t wait_ns;          // limit of every inter-role and inter-block wait
};

__device__ __forceinline__ float ex2f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// log(sigmoid(x)) = min(x, 0) - log(1 + exp(-|x|)) with the fast exponential and logarithm:
// the absolute error stays near 1e-7, which is what the cumulative decay (a sum of these) sees.
__device__ __forceinline__ float logsigmoid_(float x) {
    return fminf(x, 0.f) - __logf(1.f + __expf(-fabsf(x)));
}

__device__ __forceinline__ void named_sync(int id, int nthreads = 128) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void set_error(uint32_t* err) { atomicExch(err, WS_ERR_TIMEOUT); }

// Exit-time wait for this CTA's own asynchronous work; bounded, and not cut short by an abort.
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    uint32_t never = 0;
    mbar_wait(bar, parity, &never, limit_ns);
}

// A wait taken by one thread of a 128-thread group and shared with the whole group through a
// named barrier, so that every thread of the group takes the same branch afterwards.
struct GroupWait {
    Smem* sm;
    const TcParams* p;
    int gid;      // 0 = P group, 1 = state group, 2 = converter group
    int tid;      // thread index within the group
    int flip = 0;

    __device__ bool wait(uint64_t* bar, uint32_t parity) {
        if (tid == 0) {
            bool ok = mbar_wait(bar, parity, &sm->abort, p->wait_ns);
            if (!ok) {
                if (!sm->abort) set_error(p->err);
                atomicExch(&sm->abort, 1u);
            }
            sm->dec[gid][flip] = ok ? 0u : 1u;
        }
        named_sync(1 + gid);
        bool ok = *reinterpret_cast<volatile uint32_t*>(&sm->dec[gid][flip]) == 0;
        flip ^= 1;
        return ok;
    }

    // Spin on a flag in global memory written by another CTA.
    __device__ bool wait_flag(const uint32_t* flag, uint32_t want) {
        if (tid == 0) {
            bool ok = false;
            const uint64_t t0 = globaltimer_ns();
            while (true) {
                uint32_t v;
                asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
                if (v == want) { ok = true; break; }
                if (*reinterpret_cast<volatile uint32_t*>(&sm->abort)) break;
                if (globaltimer_ns() - t0 > p->wait_ns) break;
                __nanosleep(64);
            }
            if (!ok) {
                if (!sm->abort) set_error(p->err);
                atomicExch(&sm->abort, 1u);
            }
            sm->dec[gid][flip] = ok ? 0u : 1u;
        }
        named_sync(1 + gid);
        bool ok = *reinterpret_cast<volatile uint32_t*>(&sm->dec[gid][flip]) == 0;
        flip ^= 1;
        return ok;
    }
};

__device__ void decode_ticket(const TcParams& p, uint32_t ticket, uint32_t total, Item& it) {
    it = Item{};
    if (ticket >= total) return;
    const uint32_t i = ticket / (uint32_t)p.H;
    it.h = (int)(ticket % (uint32_t)p.H);
    int64_t nc;
    int ns;
    if (p.prefix == nullptr) {
        ns = p.spans_per_unit;
        it.u = (int)(i / (uint32_t)ns);
        it.s = (int)(i % (uint32_t)ns);
        it.len = p.N;
        it.tok_first = 0;
        it.b = it.u;
        it.grow0 = (int64_t)it.u * p.N;
    } else {
        int lo = 0, hi = p.units;   // prefix[lo] <= i < prefix[hi]
        while (hi - lo > 1) {
            int mid = (lo + hi) >> 1;
            if ((uint32_t)p.prefix[mid] <= i) lo = mid; else hi = mid;
        }
        it.u = lo;
        it.s = (int)(i - (uint32_t)p.prefix[lo]);
        ns = p.prefix[lo + 1] - p.prefix[lo];
        const int64_t a = p.cu_seqlens[lo];
        it.len = (int64_t)p.cu_seqlens[lo + 1] - a;
        it.tok_first = a;
        it.b = 0;
        it.grow0 = a;
    }
    nc = (it.len + C - 1) / C;
    it.c_begin = it.s * p.G;
    it.c_end = (int)(nc < (int64_t)it.c_begin + p.G ? nc : (int64_t)it.c_begin + p.G);
    if (it.c_end < it.c_begin) it.c_end = it.c_begin;
    it.first = it.s == 0;
    it.last = it.s == ns - 1;
    it.valid = 1;
}

__device__ __forceinline__ void set_coord(int (&c)[4], int pos_tok, int pos_head, int pos_b,
                                          int col, int tok, int h, int b) {
    c[0] = col;
    c[pos_tok] = tok;
    c[pos_head] = h;
    c[pos_b] = b;
}

// ----------------------------------------------------------------------------------------------
// warp 0: TMA producer (lane 0) and gate scan (all lanes)

// The chunk's gate logits, 4 consecutive tokens per lane (token 0's logit past the end of the
// sequence, masked by the scan).
__device__ __forceinline__ void gate_load(const TcParams& p, const Item& it, int c, int lane,
                                          float (&g4)[4]) {
    const int64_t t0 = (int64_t)c * C + 4 * lane;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int64_t t = (t0 + e < it.len) ? t0 + e : 0;
        g4[e] = __ldg(p.g + (it.grow0 + t) * p.H + it.h);
    }
}

// The whole warp computes, for the chunk's 128 tokens, the in-chunk inclusive cumulative
// log2-decay c_t = sum of logsigmoid(g)/tau * log2(e) over the chunk up to t (0 past the end of
// the sequence), the chunk total, and the key weights w_t = k_scale * 2^(after + total - c_t)
// (0 past the end), into the stage's gate slot; returns the chunk total on every lane.
__device__ __forceinline__ float gate_scan(Smem& sm, const TcParams& p, const Item& it, int c,
                                           int st, int lane, const float (&g4)[4], float after) {
    float lam[4];
    const int64_t t0 = (int64_t)c * C + 4 * lane;
#pragma unroll
    for (int e = 0; e < 4; ++e)
        lam[e] = (t0 + e < it.len) ? logsigmoid_(g4[e]) * p.inv_tau_log2e : 0.f;
    lam[1] += lam[0];
    lam[2] += lam[1];
    lam[3] += lam[2];
    float x = lam[3];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    const float excl = x - lam[3];
    const float tot = __shfl_sync(0xffffffffu, x, 31);
    const float base = after + tot;
    float4 gc4, w4;
    float* gcp = &gc4.x;
    float* wp = &w4.x;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        gcp[e] = excl + lam[e];
        wp[e] = (t0 + e < it.len) ? ex2f(base - gcp[e]) * p.k_scale : 0.f;
    }
    reinterpret_cast<float4*>(sm.gc[st])[lane] = gc4;
    reinterpret_cast<float4*>(sm.w[st])[lane] = w4;
    if (lane == 31) sm.gtot[st] = tot;
    return tot;
}

__device__ void producer(Smem& sm, const TcParams& p, const CUtensorMap* tq, const CUtensorMap* tk,
                         const CUtensorMap* tv, uint32_t total, int lane) {
    int j = 0, b = 0, it_n = 0;
    bool aborted = false;
    while (!aborted) {
        const int slot = it_n % ITEM_DEPTH;
        int ok = 1;
        if (lane == 0 && it_n >= ITEM_DEPTH)
            ok = mbar_wait(&sm.item_empty[slot], ((it_n / ITEM_DEPTH) - 1) & 1, &sm.abort, p.wait_ns);
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
            aborted = true;
            break;
        }
        uint32_t ticket = 0;
        if (lane == 0) ticket = atomicAdd(p.ticket, 1u);
        ticket = __shfl_sync(0xffffffffu, ticket, 0);
        Item it;
        decode_ticket(p, ticket, total, it);
        if (lane == 0) {
            sm.items[slot] = it;
            mbar_arrive(&sm.item_full[slot]);
        }
        ++it_n;
        if (!it.valid) break;
        const int n = it.c_end - it.c_begin;
        if (n == 0 && lane == 0) {   // nothing to scan: the span's total decay is 0
            sm.span_L[slot] = 0.f;
            mbar_arrive(&sm.span_done[slot]);
        }
        // pass A visits the span's chunks last to first (each key weighted by its decay to the
        // end of the span); pass B first to last
        float after = 0.f;   // pass A: log2-decay of the chunks after the current one
        for (int jj = 0; jj < 2 * n; ++jj) {
            const bool pass_b = jj >= n;
            const int c = pass_b ? it.c_begin + (jj - n) : it.c_end - 1 - jj;
            const int st = j & 1;
            float g4[4];
            gate_load(p, it, c, lane, g4);   // in flight while the slots are awaited
            ok = 1;
            if (lane == 0 && j >= 2)
                ok = mbar_wait(&sm.kv_empty[st], ((j >> 1) - 1) & 1, &sm.abort, p.wait_ns);
            if (pass_b && lane == 0 && ok && b >= 2)
                ok = mbar_wait(&sm.q_empty[b & 1], ((b >> 1) - 1) & 1, &sm.abort, p.wait_ns);
            if (!__shfl_sync(0xffffffffu, ok, 0)) {
                aborted = true;
                break;
            }
            if (lane == 0) {
                const int tok = (int)(it.tok_first + (int64_t)c * C);
                mbar_arrive_expect_tx(&sm.kv_full[st], 2 * TILE);
                if (pass_b) mbar_arrive_expect_tx(&sm.q_full[b & 1], TILE);
                int ck[4], cv[4];
                for (int half = 0; half < 2; ++half) {
                    set_coord(ck, p.qk_pos_tok, p.qk_pos_head, p.qk_pos_b, half * 64, tok, it.h,
                              it.b);
                    set_coord(cv, p.v_pos_tok, p.v_pos_head, p.v_pos_b, half * 64, tok, it.h, it.b);
                    tma_load_4d(sm.k[st] + half * SLAB, tk, &sm.kv_full[st], ck[0], ck[1], ck[2],
                                ck[3]);
                    tma_load_4d(sm.v[st] + half * SLAB, tv, &sm.kv_full[st], cv[0], cv[1], cv[2],
                                cv[3]);
                    if (pass_b)
                        tma_load_4d(sm.q[b & 1] + half * SLAB, tq, &sm.q_full[b & 1], ck[0],
                                    ck[1], ck[2], ck[3]);
                }
            }
            const float tot = gate_scan(sm, p, it, c, st, lane, g4, pass_b ? 0.f : after);
            if (!pass_b) after += tot;
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sm.kv_full[st]);
                if (!pass_b && jj == n - 1) {   // the span's total decay, for the look-back
                    sm.span_L[slot] = after;
                    mbar_arrive(&sm.span_done[slot]);
                }
            }
            if (pass_b) ++b;
            ++j;
        }
    }
    if (lane == 0) {
        if (aborted) {
            set_error(p.err);
            atomicExch(&sm.abort, 1u);
        }
        // make sure no TMA write into this CTA's shared memory is still in flight at exit
        for (int jj = (j >= 2 ? j - 2 : 0); jj < j; ++jj)
            mbar_wait_drain(&sm.kv_full[jj & 1], (jj >> 1) & 1, DRAIN_NS);
        for (int bb = (b >= 2 ? b - 2 : 0); bb < b; ++bb)
            mbar_wait_drain(&sm.q_full[bb & 1], (bb >> 1) & 1, DRAIN_NS);
    }
}

// ----------------------------------------------------------------------------------------------
// warp 1: MMA issuer (one thread)

// D (+)= A B over K = 128, eight K-steps of 16; bf16 operands in shared memory.
__device__ __forceinline__ void mma_128(uint32_t d, uint32_t a_base, bool a_mn, uint32_t b_base,
                                        bool b_mn, bool accumulate) {
    const uint32_t idesc = idesc_bf16(128, 128, a_mn, b_mn);
#pragma unroll 1
    for (int kk = 0; kk < 8; ++kk) {
        const uint32_t aoff = a_mn ? kk * 2048u : (kk >> 2) * SLAB + (kk & 3) * 32u;
        const uint32_t boff = b_mn ? kk * 2048u : (kk >> 2) * SLAB + (kk & 3) * 32u;
        const uint64_t ad = a_mn ? sdesc_sw128(a_base + aoff, SLAB, 1024)
                                 : sdesc_sw128(a_base + aoff, 16, 1024);
        const uint64_t bd = b_mn ? sdesc_sw128(b_base + boff, SLAB, 1024)
                                 : sdesc_sw128(b_base + boff, 16, 1024);
        mma_ss(d, ad, bd, idesc, (accumulate || kk > 0) ? 1u : 0u);
    }
}

// D (+)= X V with X (bf16, K-major) in TMEM and V [token x d_v] in shared memory.  X is stored
// per 32-token group g = 0..3 as [16 columns of high halves | 16 columns of low halves] at
// columns 32 g; the K-step of tokens [16 kk, 16 kk + 16) of one half starts at column
// 32 (kk / 2) + 8 (kk % 2) + 16 * half.  X is P (rows = query tokens) for the inner output and
// (w K)^T (rows = key channels) for the state update.
__device__ __forceinline__ void mma_tv(uint32_t d, uint32_t x_base, int half, uint32_t v_base,
                                       bool accumulate) {
    const uint32_t idesc = idesc_bf16(128, 128, 0, 1);
#pragma unroll 1
    for (int kk = 0; kk < 8; ++kk)
        mma_ts(d, x_base + 32 * (kk >> 1) + 8 * (kk & 1) + 16 * half,
               sdesc_sw128(v_base + kk * 2048u, SLAB, 1024), idesc,
               (accumulate || kk > 0) ? 1u : 0u);
}

// Tensor-memory region [256, 384) holds, in turn, each span's aggregate, then per pass-B chunk
// dS and then O.  The two kinds of content have their own barriers, so that each consumer waits
// for consecutive phases of one barrier (a parity wait cannot tell phase n from phase n + 2): an
// aggregate or a dS completes a phase of ds_full and, once folded by the state group, of
// ds_free; an O completes a phase of o_full and, once read by the P group, of o_free.
__device__ void mma_issuer(Smem& sm, const TcParams& p, uint32_t tmem) {
    int j = 0, b = 0, it_n = 0;
    uint32_t n_ds = 0, n_o = 0;   // aggregates + dS, and O, written so far
    bool ok = true;
    auto W = [&](uint64_t* bar, uint32_t par) {
        if (ok && !mbar_wait(bar, par, &sm.abort, p.wait_ns)) {
            ok = false;
            if (!sm.abort) set_error(p.err);
            atomicExch(&sm.abort, 1u);
        }
        return ok;
    };
    const uint32_t sb = smem_u32(sm.sb);
    while (ok) {
        const int slot = it_n % ITEM_DEPTH;
        if (!W(&sm.item_full[slot], (it_n / ITEM_DEPTH) & 1)) break;
        const Item it = sm.items[slot];
        mbar_arrive(&sm.item_empty[slot]);
        ++it_n;
        if (!it.valid) break;
        const int n = it.c_end - it.c_begin;
        // pass A: the span's aggregate, one result accumulated over its chunks (delivered last to
        // first, each key weighted by its decay to the span's end).  The region's previous
        // content, if any, is the O of the last chunk of an earlier span.
        for (int i = 0; i < n && ok; ++i, ++j) {
            const int st = j & 1;
            if (!W(&sm.kv_full[st], (j >> 1) & 1)) break;
            if (!W(&sm.kt_ready, j & 1)) break;
            if (i == 0 && n_o > 0 && !W(&sm.o_free, (n_o - 1) & 1)) break;
            tc_fence_after();
            const uint32_t vb = smem_u32(sm.v[st]);
            mma_tv(tmem + TM_DO, tmem + TM_KT, 0, vb, i > 0);
            mma_tv(tmem + TM_DO, tmem + TM_KT, 1, vb, true);
            mma_commit(&sm.kt_free);
            mma_commit(&sm.kv_empty[st]);
        }
        if (!ok) break;
        if (n > 0) {
            mma_commit(&sm.ds_full);   // the aggregate
            ++n_ds;
        }
        // pass B.  Per chunk: Q K^T (once P V of the previous chunk has read P out of the
        // tensor memory it overwrites), Q S_hi, dS, Q S_lo, P V.
        for (int i = 0; i < n && ok; ++i, ++j, ++b) {
            const int st = j & 1, qs = b & 1;
            const uint32_t qb = smem_u32(sm.q[qs]), kb = smem_u32(sm.k[st]),
                           vb = smem_u32(sm.v[st]);
            if (!W(&sm.kv_full[st], (j >> 1) & 1)) break;
            if (!W(&sm.q_full[qs], (b >> 1) & 1)) break;
            if (n_o > 0 && !W(&sm.o_full, (n_o - 1) & 1)) break;    // the last P V is done
            tc_fence_after();
            mma_128(tmem + TM_A, qb, false, kb, false, false);     // A = Q K^T
            mma_commit(&sm.a_full);
            if (!W(&sm.s_ready, b & 1)) break;
            if (n_o > 0 && !W(&sm.o_free, (n_o - 1) & 1)) break;    // last O and OX read
            tc_fence_after();
            mma_128(tmem + TM_OX, qb, false, sb, true, false);     // OX = Q S_hi
            mma_commit(&sm.s_hi_done);
            if (!W(&sm.kt_ready, j & 1)) break;
            // the region's previous content: the aggregate (i = 0, folded) or O of chunk i-1
            // (read, waited for above)
            if (i == 0 && !W(&sm.ds_free, (n_ds - 1) & 1)) break;
            tc_fence_after();
            mma_tv(tmem + TM_DO, tmem + TM_KT, 0, vb, false);      // dS = (w K)_hi^T V
            mma_tv(tmem + TM_DO, tmem + TM_KT, 1, vb, true);       //    + (w K)_lo^T V
            mma_commit(&sm.kt_free);
            mma_commit(&sm.ds_full);
            ++n_ds;
            if (!W(&sm.s_lo_ready, b & 1)) break;
            tc_fence_after();
            mma_128(tmem + TM_OX, qb, false, sb, true, true);      // OX += Q S_lo
            mma_commit(&sm.sb_free);
            if (!W(&sm.p_ready, b & 1)) break;
            if (!W(&sm.ds_free, (n_ds - 1) & 1)) break;            // dS folded into the state
            tc_fence_after();
            mma_tv(tmem + TM_DO, tmem + TM_A, 0, vb, false);       // O = P_hi V
            mma_tv(tmem + TM_DO, tmem + TM_A, 1, vb, true);        //   + P_lo V
            mma_commit(&sm.o_full);
            ++n_o;
            mma_commit(&sm.kv_empty[st]);
        }
    }
    // all issued MMAs complete before TMEM is released
    mma_commit(&sm.drain);
    mbar_wait_drain(&sm.drain, 0, DRAIN_NS);
}

// ----------------------------------------------------------------------------------------------
// bf16 splitting: x = hi + lo with hi = bf16(x) and lo = bf16(x - hi).  The pair carries about
// 16 significant bits, so products with bf16 operands accumulated in fp32 keep the P V, Q S and
// K^T V contractions within a few 1e-6 of fp32.

__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    const float2 hf = __bfloat1622float2(h);
    const float2 r = fma2(hf, make_float2(-1.f, -1.f), make_float2(x0, x1));   // x - hi
    const __nv_bfloat162 l = __floats2bfloat162_rn(r.x, r.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Row r of the state into the MN-major swizzled tile read by Q S: the bf16 high halves
// (lo_half = false) or the low halves (lo_half = true) of the split of S.
template <bool lo_half>
__device__ __forceinline__ void write_state_half(unsigned char* tile, int r, const float (&S)[D]) {
#pragma unroll
    for (int cc = 0; cc < 16; ++cc) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) split2(S[8 * cc + 2 * e], S[8 * cc + 2 * e + 1], hi[e], lo[e]);
        const int half = cc >> 3, c = cc & 7;
        const uint32_t* x = lo_half ? lo : hi;
        *reinterpret_cast<uint4*>(tile + half * SLAB + r * 128 + ((c ^ (r & 7)) << 4)) =
            make_uint4(x[0], x[1], x[2], x[3]);
    }
}

// S = 2^tot * S + dS, dS read from TMEM 32 columns at a time
__device__ __forceinline__ void fold_ds(uint32_t taddr, float (&S)[D], float eb) {
#pragma unroll
    for (int jc = 0; jc < 4; ++jc) {
        float d[32];
        tmem_ld32(taddr + jc * 32, d);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) S[jc * 32 + i] = fmaf(eb, S[jc * 32 + i], d[i]);
    }
}

// ----------------------------------------------------------------------------------------------
// warps 12-15: (w K)^T into tensor memory, for every chunk of both passes

// Thread r (TMEM lane r = key channel r) reads column r of the swizzled K tile (token m at row m;
// element (m, r) in slab r / 64, 16-byte chunk ((r % 64) / 8) ^ (m % 8), position r % 8), weights
// token m by w_m, splits into bf16 halves and stores them in the layout mma_tv reads: per
// 32-token group, 16 columns of high halves then 16 of low halves, two tokens per column.  For a
// fixed token the 32 lanes of a warp read 64 consecutive bytes of one row: no bank conflict.
__device__ __forceinline__ void convert_wkt(const Smem& sm, int st, int r, uint32_t taddr) {
    const unsigned char* kt = sm.k[st] + (r >> 6) * SLAB + ((r & 7) << 1);
    const int cch = (r & 63) >> 3;
    const float2* w2 = reinterpret_cast<const float2*>(sm.w[st]);
#pragma unroll 1
    for (int jc = 0; jc < 4; ++jc) {
        uint32_t ph[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int m0 = jc * 32 + 2 * i;
            const float k0 = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                kt + m0 * 128 + ((cch ^ (m0 & 7)) << 4)));
            const float k1 = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                kt + (m0 + 1) * 128 + ((cch ^ ((m0 + 1) & 7)) << 4)));
            const float2 kw = mul2(make_float2(k0, k1), w2[m0 >> 1]);
            split2(kw.x, kw.y, ph[i], ph[16 + i]);
        }
        tmem_st32(taddr + jc * 32, ph);
    }
    tmem_st_wait();
}

__device__ void converter(Smem& sm, const TcParams& p, uint32_t tmem, int warp, int lane) {
    GroupWait gw{&sm, &p, 2, (warp - 12) * 32 + lane};
    const int r = (warp & 3) * 32 + lane;
    const uint32_t taddr = tmem + (((uint32_t)((warp & 3) * 32)) << 16) + TM_KT;
    int j = 0, it_n = 0;
    bool ok = true;
    while (ok) {
        const int slot = it_n % ITEM_DEPTH;
        if (!gw.wait(&sm.item_full[slot], (it_n / ITEM_DEPTH) & 1)) break;
        const Item it = sm.items[slot];
        mbar_arrive(&sm.item_empty[slot]);
        ++it_n;
        if (!it.valid) break;
        const int n = it.c_end - it.c_begin;
        for (int jj = 0; jj < 2 * n; ++jj, ++j) {
            const int st = j & 1;
            if (!gw.wait(&sm.kv_full[st], (j >> 1) & 1)) { ok = false; break; }
            if (j > 0 && !gw.wait(&sm.kt_free, (j - 1) & 1)) { ok = false; break; }
            tc_fence_after();
            convert_wkt(sm, st, r, taddr);
            tc_fence_before();
            mbar_arrive(&sm.kt_ready);
            mbar_arrive(&sm.kv_empty[st]);   // this group is done with the stage's K and weights
        }
    }
}

// ----------------------------------------------------------------------------------------------
// warps 4-7: decay mask (P split into bf16 halves in TMEM) and output epilogue

__device__ void p_group(Smem& sm, const TcParams& p, const CUtensorMap* to, uint32_t tmem, int warp,
                        int lane) {
    GroupWait gw{&sm, &p, 0, (warp - 4) * 32 + lane};
    const int q = warp & 3, r = q * 32 + lane;
    const uint32_t lane_base = ((uint32_t)(q * 32)) << 16;
    int b = 0, j = 0, it_n = 0;
    bool ok = true;
    while (ok) {
        const int slot = it_n % ITEM_DEPTH;
        if (!gw.wait(&sm.item_full[slot], (it_n / ITEM_DEPTH) & 1)) break;
        const Item it = sm.items[slot];
        mbar_arrive(&sm.item_empty[slot]);
        ++it_n;
        if (!it.valid) break;
        const int n = it.c_end - it.c_begin;
        j += n;             // pass A
        for (int i = 0; i < n; ++i, ++j, ++b) {
            const int st = j & 1, qs = b & 1, c = it.c_begin + i;
            if (!gw.wait(&sm.a_full, b & 1)) { ok = false; break; }
            if (!gw.wait(&sm.kv_full[st], (j >> 1) & 1)) { ok = false; break; }   // gate slot
            const float cr = sm.gc[st][r];
            tc_fence_after();
            // P = k_scale * 2^(c_r - c_m) * A[r][m] for m <= r, split into bf16 halves; each
            // 32-column group of A is replaced in place by [16 high | 16 low] columns of P.
#pragma unroll 1
            for (int jc = 0; jc < 4; ++jc) {
                uint32_t ph[32];
                if (jc <= q) {
                    float a[32];
                    tmem_ld32(tmem + lane_base + TM_A + jc * 32, a);
                    tmem_ld_wait();
#pragma unroll
                    for (int i2 = 0; i2 < 16; ++i2) {
                        const int m0 = jc * 32 + 2 * i2;
                        const float2 g2 = *reinterpret_cast<const float2*>(&sm.gc[st][m0]);
                        const float2 arg = fma2(g2, make_float2(-1.f, -1.f), make_float2(cr, cr));
                        const float2 pv = mul2(mul2(make_float2(ex2f(arg.x), ex2f(arg.y)),
                                                    make_float2(p.k_scale, p.k_scale)),
                                               make_float2(a[2 * i2], a[2 * i2 + 1]));
                        split2(m0 <= r ? pv.x : 0.f, m0 + 1 <= r ? pv.y : 0.f, ph[i2], ph[16 + i2]);
                    }
                } else {
#pragma unroll
                    for (int i2 = 0; i2 < 32; ++i2) ph[i2] = 0u;
                }
                tmem_st32(tmem + lane_base + TM_A + jc * 32, ph);
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&sm.p_ready);
            // epilogue: O = O_inner + 2^(c_r) O_cross, rounded to bf16.  o_full for O also means
            // that every earlier MMA is done, Q K^T and Q S on this chunk's Q slot included.  A
            // chunk that lies wholly inside its sequence goes out as one tile through that slot:
            // rows in the swizzled layout, then two TMA stores.  The rows of a partial chunk are
            // stored one by one, so that nothing past the end of the sequence (the next packed
            // sequence) is written.
            if (!gw.wait(&sm.o_full, b & 1)) { ok = false; break; }
            tc_fence_after();
            const float ec = ex2f(cr);
            const int64_t t = (int64_t)c * C + r;
            const bool full = (int64_t)(c + 1) * C <= it.len;
            unsigned char* tile = sm.q[qs];
            uint4* orow = reinterpret_cast<uint4*>(p.o + (int64_t)it.b * p.osb +
                                                   (it.tok_first + t) * p.ost +
                                                   (int64_t)it.h * p.osh);
#pragma unroll 1
            for (int jc = 0; jc < 4; ++jc) {
                float o[32], ox[32];
                tmem_ld32(tmem + lane_base + TM_DO + jc * 32, o);
                tmem_ld32(tmem + lane_base + TM_OX + jc * 32, ox);
                tmem_ld_wait();
#pragma unroll
                for (int v4 = 0; v4 < 4; ++v4) {
                    uint4 u;
                    const float2 ec2 = make_float2(ec, ec);
                    float2 y[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        y[e] = fma2(ec2, make_float2(ox[8 * v4 + 2 * e], ox[8 * v4 + 2 * e + 1]),
                                    make_float2(o[8 * v4 + 2 * e], o[8 * v4 + 2 * e + 1]));
                    u.x = pack_bf16x2(y[0].x, y[0].y);
                    u.y = pack_bf16x2(y[1].x, y[1].y);
                    u.z = pack_bf16x2(y[2].x, y[2].y);
                    u.w = pack_bf16x2(y[3].x, y[3].y);
                    // columns 32 jc + 8 v4 .. + 7: 16-byte chunk cc = 4 jc + v4 of the row
                    const int cc = 4 * jc + v4;
                    if (full)
                        *reinterpret_cast<uint4*>(tile + (cc >> 3) * SLAB + r * 128 +
                                                  (((cc & 7) ^ (r & 7)) << 4)) = u;
                    else if (t < it.len)
                        orow[cc] = u;
                }
            }
            tc_fence_before();
            mbar_arrive(&sm.o_free);
            if (full) {
                fence_proxy_async_smem();
                named_sync(1);   // every row of the tile is written
                if (gw.tid == 0) {
                    const int tok = (int)(it.tok_first + (int64_t)c * C);
                    int co[4];
#pragma unroll 1
                    for (int half = 0; half < 2; ++half) {
                        set_coord(co, p.o_pos_tok, p.o_pos_head, p.o_pos_b, half * 64, tok, it.h,
                                  it.b);
                        tma_store_4d(to, tile + half * SLAB, co[0], co[1], co[2], co[3]);
                    }
                    bulk_commit_group();
                    bulk_wait_group_read0();
                    mbar_arrive(&sm.q_empty[qs]);   // the producer may load the next Q here
                }
            } else if (gw.tid == 0) {
                mbar_arrive(&sm.q_empty[qs]);
            }
        }
    }
    if (gw.tid == 0) bulk_wait_group0();   // the last output tiles are written before exit
}

// ----------------------------------------------------------------------------------------------
// warps 8-11: fp32 state, look-back, bf16 halves of the state for Q S

__device__ void state_group(Smem& sm, const TcParams& p, uint32_t tmem, int warp, int lane) {
    GroupWait gw{&sm, &p, 1, (warp - 8) * 32 + lane};
    const int q = warp & 3, r = q * 32 + lane;
    const uint32_t lane_base = ((uint32_t)(q * 32)) << 16;
    float S[D];
    int j = 0, b = 0, it_n = 0;
    uint32_t n_ds = 0;   // aggregates and dS results folded so far (phases of ds_full)
    bool ok = true;
    while (ok) {
        const int slot = it_n % ITEM_DEPTH;
        if (!gw.wait(&sm.item_full[slot], (it_n / ITEM_DEPTH) & 1)) break;
        const Item& it = sm.items[slot];   // read in place; released at the end of the span
        const uint32_t use = (uint32_t)(it_n / ITEM_DEPTH);
        ++it_n;
        if (!it.valid) {
            mbar_arrive(&sm.item_empty[slot]);
            break;
        }
        // ---- pass A: the span's aggregate Agg = sum over its keys of (decay to the span's end)
        // k^T v, accumulated by the MMAs over the span's chunks; the producer sums the span's
        // log2-decay L.
        const int n = it.c_end - it.c_begin;
#pragma unroll
        for (int i = 0; i < D; ++i) S[i] = 0.f;
        if (!gw.wait(&sm.span_done[slot], use & 1)) break;
        const float L = sm.span_L[slot];
        if (n > 0) {
            if (!gw.wait(&sm.ds_full, n_ds & 1)) break;
            tc_fence_after();
            fold_ds(tmem + lane_base + TM_DO, S, 0.f);   // S = Agg
            tc_fence_before();
            mbar_arrive(&sm.ds_free);
            ++n_ds;
        }
        j += n;
        // ---- look-back: entry state E of the span; publish exp(L) E + Agg
        const int64_t chain = (int64_t)it.u * p.H + it.h;
        const float* esrc = nullptr;
        bool from_slot = false;
        if (it.first) {
            if (p.state_in) esrc = p.state_in + (chain * D + r) * D;
        } else {
            if (!gw.wait_flag(p.flags + chain * 2 + ((it.s - 1) & 1), (uint32_t)it.s)) break;
            esrc = p.slots + (chain * 2 + ((it.s - 1) & 1)) * (D * D);
            from_slot = true;
        }
        const float eL = ex2f(L);
        float4* dst = it.last ? nullptr
                              : reinterpret_cast<float4*>(p.slots + (chain * 2 + (it.s & 1)) * (D * D));
        // E comes in through the state buffer, free once the previous chunk's Q S_lo is done:
        // two rounds of 16 float4 per thread, each thread copying and reading back only its own
        // elements (no barrier between the rounds), with all 16 copies of a round in flight.
        if (b > 0 && !gw.wait(&sm.sb_free, (b - 1) & 1)) break;
        float4* ebuf = reinterpret_cast<float4*>(sm.sb) + r;
        // float4 j4 of the row: slot layout [j4][row], state_in layout [row][j4]
        const float4* esrc4 =
            reinterpret_cast<const float4*>(esrc) + (from_slot ? r : 0);
        const int estep = from_slot ? D : 1;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            if (esrc) {
#pragma unroll 1
                for (int k = 0; k < 16; ++k)
                    cp_async_16(ebuf + k * D, esrc4 + (half * 16 + k) * estep);
                cp_async_wait_all();
            }
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const int j4 = half * 16 + k;
                const float4 x = esrc ? ebuf[k * D] : make_float4(0.f, 0.f, 0.f, 0.f);
                if (dst) {
                    float4 inc;
                    inc.x = fmaf(eL, x.x, S[4 * j4 + 0]);
                    inc.y = fmaf(eL, x.y, S[4 * j4 + 1]);
                    inc.z = fmaf(eL, x.z, S[4 * j4 + 2]);
                    inc.w = fmaf(eL, x.w, S[4 * j4 + 3]);
                    __stcg(dst + j4 * D + r, inc);
                }
                S[4 * j4 + 0] = x.x;
                S[4 * j4 + 1] = x.y;
                S[4 * j4 + 2] = x.z;
                S[4 * j4 + 3] = x.w;
            }
        }
        // One barrier for two orders: every thread has read its part of E out of the state
        // buffer before any thread writes its row of the state into it (the two layouts differ),
        // and every published row is stored and fenced before the flag is raised.
        if (dst) __threadfence();
        named_sync(2);
        if (dst && r == 0) {
            uint32_t* f = p.flags + chain * 2 + (it.s & 1);
            asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(f), "r"((uint32_t)it.s + 1)
                         : "memory");
        }
        // ---- pass B: running state from E.  Per chunk: the bf16 high half of the state into
        // the state buffer for Q S_hi, then (once Q S_hi has read it) the low half for Q S_lo,
        // then the fold of the chunk's dS.
#pragma unroll 1
        for (int i = 0; i < n; ++i, ++j, ++b) {
            const int st = j & 1;
            if (i > 0 && !gw.wait(&sm.sb_free, (b - 1) & 1)) { ok = false; break; }
            write_state_half<false>(sm.sb, r, S);
            fence_proxy_async_smem();
            mbar_arrive(&sm.s_ready);
            if (!gw.wait(&sm.s_hi_done, b & 1)) { ok = false; break; }
            write_state_half<true>(sm.sb, r, S);
            fence_proxy_async_smem();
            mbar_arrive(&sm.s_lo_ready);
            if (!gw.wait(&sm.kv_full[st], (j >> 1) & 1)) { ok = false; break; }   // gate slot
            const float tot = sm.gtot[st];
            if (!gw.wait(&sm.ds_full, n_ds & 1)) { ok = false; break; }           // dS
            tc_fence_after();
            fold_ds(tmem + lane_base + TM_DO, S, ex2f(tot));
            tc_fence_before();
            mbar_arrive(&sm.ds_free);
            ++n_ds;
        }
        if (!ok) break;
        if (it.last && p.state_out) {
            float4* so = reinterpret_cast<float4*>(p.state_out + (chain * D + r) * D);
#pragma unroll
            for (int j4 = 0; j4 < D / 4; ++j4)
                so[j4] = make_float4(S[4 * j4], S[4 * j4 + 1], S[4 * j4 + 2], S[4 * j4 + 3]);
        }
        mbar_arrive(&sm.item_empty[slot]);
    }
}

__global__ void __launch_bounds__(NTHREADS, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                      const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to,
                      const TcParams p, uint32_t total_dense) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if ((smem_u32(smem_raw) & 1023u) != 0) {   // the swizzled tiles need 1 KB alignment
        if (tid == 0) set_error(p.err);
        return;
    }
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sm.kv_full[s], 2);      // TMA bytes + expect_tx arrival, gate arrival
            mbar_init(&sm.kv_empty[s], 1 + 128);   // last MMA on the stage, converter group
            mbar_init(&sm.q_full[s], 1);
            mbar_init(&sm.q_empty[s], 1);
        }
        for (int s = 0; s < ITEM_DEPTH; ++s) {
            mbar_init(&sm.item_full[s], 1);
            mbar_init(&sm.item_empty[s], 1 + 3 * 128);
            mbar_init(&sm.span_done[s], 1);
        }
        mbar_init(&sm.a_full, 1);
        mbar_init(&sm.p_ready, 128);
        mbar_init(&sm.s_ready, 128);
        mbar_init(&sm.s_hi_done, 1);
        mbar_init(&sm.s_lo_ready, 128);
        mbar_init(&sm.sb_free, 1);
        mbar_init(&sm.kt_ready, 128);
        mbar_init(&sm.kt_free, 1);
        mbar_init(&sm.ds_full, 1);
        mbar_init(&sm.ds_free, 128);
        mbar_init(&sm.o_full, 1);
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
    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 72;" ::: "memory");
        if (warp == 0) {
            if (lane == 0) {
                tma_prefetch_desc(&tq);
                tma_prefetch_desc(&tk);
                tma_prefetch_desc(&tv);
                tma_prefetch_desc(&to);
            }
            const uint32_t total =
                p.prefix ? (uint32_t)p.prefix[p.units] * (uint32_t)p.H : total_dense;
            producer(sm, p, &tq, &tk, &tv, total, lane);
        } else if (warp == 1) {
            if (lane == 0) mma_issuer(sm, p, tmem);
        }
    } else if (warp < 8) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 136;" ::: "memory");
        p_group(sm, p, &to, tmem, warp, lane);
    } else if (warp < 12) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 232;" ::: "memory");
        state_group(sm, p, tmem, warp, lane);
    } else {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 72;" ::: "memory");
        converter(sm, p, tmem, warp, lane);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// One 32-bit word of the workspace (the failure-path test's first span ticket).
__global__ void set_u32_kernel(uint32_t* w, uint32_t value) { *w = value; }

// Varlen: spans per sequence and their exclusive prefix (one CTA).
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* __restrict__ cu, int units, int G,
                                                    int32_t* __restrict__ prefix) {
    __shared__ int32_t warp_tot[32];
    __shared__ int32_t carry;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < units; base += 1024) {
        const int u = base + tid;
        int ns = 0;
        if (u < units) {
            const int64_t len = (int64_t)cu[u + 1] - cu[u];
            const int64_t nc = (len + C - 1) / C;
            ns = (int)((nc + G - 1) / G > 1 ? (nc + G - 1) / G : 1);
        }
        int x = ns;
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_tot[w] = x;
        __syncthreads();
        if (w == 0) {
            int t = warp_tot[lane];
            for (int o = 1; o < 32; o <<= 1) {
                int y = __shfl_up_sync(0xffffffffu, t, o);
                if (lane >= o) t += y;
            }
            warp_tot[lane] = t;   // inclusive over warps
        }
        __syncthreads();
        const int excl = carry + (w > 0 ? warp_tot[w - 1] : 0) + x - ns;
        if (u < units) prefix[u] = excl;
        __syncthreads();
        if (tid == 1023) carry = excl + ns;
        __syncthreads();
    }
    if (tid == 0) prefix[units] = carry;
}

struct WsLayout {
    size_t flags, prefix, slots, total;
};

WsLayout ws_layout(int units, int H) {
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    WsLayout l;
    l.flags = 256;
    l.prefix = l.flags + up((size_t)units * H * 2 * sizeof(uint32_t));
    l.slots = l.prefix + up(((size_t)units + 1) * sizeof(int32_t));
    l.total = l.slots + (size_t)units * H * 2 * D * D * sizeof(float);
    return l;
}

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (!cached[dev]) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cached[dev] = n > 0 ? n : 148;
    }
    return cached[dev];
}

// Order the (token, head, batch) dims of a [.., token, head, d] tensor by stride for the TMA map;
// returns false if the driver rejects it.
bool make_map(CUtensorMap* map, const void* base, int64_t st, int64_t sh, int64_t sb, int64_t ntok,
              int H, int B, int& pos_tok, int& pos_head, int& pos_b) {
    struct Dim { int64_t stride, extent; int which; };
    Dim d[3] = {{st, ntok, 0}, {sh, H, 1}, {sb, B, 2}};
    // a size-1 batch dimension gets a stride past the end of the other two
    if (B == 1) {
        int64_t end = 1;
        for (int i = 0; i < 2; ++i) end = d[i].stride * d[i].extent > end ? d[i].stride * d[i].extent : end;
        d[2].stride = end;
    }
    for (int i = 0; i < 3; ++i)
        for (int k = i + 1; k < 3; ++k)
            if (d[k].stride < d[i].stride) { Dim t = d[i]; d[i] = d[k]; d[k] = t; }
    uint64_t dims[4] = {D, 0, 0, 0}, strides[3];
    uint32_t box[4] = {64, 1, 1, 1};
    for (int i = 0; i < 3; ++i) {
        dims[i + 1] = (uint64_t)d[i].extent;
        strides[i] = (uint64_t)d[i].stride * 2;
        if (d[i].which == 0) { pos_tok = i + 1; box[i + 1] = C; }
        if (d[i].which == 1) pos_head = i + 1;
        if (d[i].which == 2) pos_b = i + 1;
    }
    return make_bf16_map(map, base, 4, dims, strides, box);
}

// Chunks per span.  Spans run in waves of `grid` CTAs; a span costs about G chunk-times plus a
// fixed overhead of about 1.5 (its look-back and the switches between passes), and the
// look-backs of one chain run one after another at about half a chunk-time each.  G minimises
// the larger of the two over [2, 128]: at 32K x 24 heads it picks 43 (144 spans, one wave; the
// fastest span size of a measured sweep), at 512K x 24 heads 111.  With several packed
// sequences of unequal lengths (`ragged`, where the host knows only their mean,
// chunks_per_unit) each sequence's last span is on average half empty, so a chain has
// chunks / G + 1/2 spans: on the eight sequences of 1024 to 65536 tokens x 24 heads that
// picks 28 (2.71 ms) where the mean alone picked 82 (2.88 ms; a measured sweep was flat at
// 2.68-2.74 ms over G = 12..32).
// GRET_SPAN_CHUNKS overrides the choice.
int span_chunks(double chunks_per_unit, int64_t chains, int grid, bool ragged) {
    static int forced = -2;
    if (forced == -2) {
        const char* e = getenv("GRET_SPAN_CHUNKS");
        forced = e ? atoi(e) : -1;
        if (forced < 1) forced = -1;
    }
    if (forced > 0) return forced;
    int best = 2;
    double best_cost = -1.0;
    for (int g = 2; g <= 128; ++g) {
        const double whole = std::max(1.0, std::ceil(chunks_per_unit / g));
        const double spans = ragged ? chunks_per_unit / g + 0.5 : whole;
        const double waves = std::ceil(std::ceil((double)chains * spans) / grid);
        const double cost = std::max(waves * (g + 1.5), 0.5 * spans + g);
        if (best_cost < 0.0 || cost < best_cost) {
            best = g;
            best_cost = cost;
        }
        if (!ragged && whole == 1.0) break;   // larger spans change nothing
    }
    return best;
}

}  // namespace

size_t tc_workspace_size(int64_t, int n_units, int H) { return ws_layout(n_units, H).total; }

gret_status_t launch_prefill_tc(const PrefillArgs& a) {
    const bool varlen = a.cu_seqlens != nullptr;
    const int units = a.n_seqs;
    const WsLayout L = ws_layout(units, a.H);
    unsigned char* ws = (unsigned char*)a.workspace;
    // chunks per sequence (varlen: their mean)
    const double chunks_per_unit =
        units <= 0 ? 0.0
        : varlen   ? (double)a.N / units / C
                   : (double)((a.N + C - 1) / C);
    // packed sequences of unequal length: more than one (with one, the mean is its length)
    const int G = span_chunks(chunks_per_unit, (int64_t)units * a.H, sm_count(),
                              varlen && units > 1);

    TcParams p;
    p.g = a.g;
    p.inv_tau_log2e = 1.4426950408889634f / a.tau;
    p.k_scale = a.k_scale;
    p.o = (__nv_bfloat16*)a.o;
    p.osb = a.osb; p.ost = a.ost; p.osh = a.osh;
    p.state_in = a.state_in;
    p.state_out = a.state_out;
    p.err = (uint32_t*)ws;
    p.ticket = (uint32_t*)(ws + 4);
    p.flags = (uint32_t*)(ws + L.flags);
    p.prefix = varlen ? (int32_t*)(ws + L.prefix) : nullptr;
    p.slots = (float*)(ws + L.slots);
    p.cu_seqlens = a.cu_seqlens;
    p.N = a.N;
    p.H = a.H;
    p.units = units;
    p.G = G;
    const int64_t nc_dense = (a.N + C - 1) / C;
    p.spans_per_unit = (int)std::max<int64_t>(1, (nc_dense + G - 1) / G);
    p.wait_ns = a.test_wait_ns > 0 ? a.test_wait_ns : WAIT_NS;

    const int64_t ntok = a.N;   // dense: tokens per sequence; varlen: packed total
    const int B = varlen ? 1 : a.B;
    CUtensorMap tq, tk, tv, to;
    if (!make_map(&tq, a.q, a.st, a.sh, a.sb, ntok, a.H, B, p.qk_pos_tok, p.qk_pos_head, p.qk_pos_b) ||
        !make_map(&tk, a.k, a.st, a.sh, a.sb, ntok, a.H, B, p.qk_pos_tok, p.qk_pos_head, p.qk_pos_b) ||
        !make_map(&tv, a.v, a.vst, a.vsh, a.vsb, ntok, a.H, B, p.v_pos_tok, p.v_pos_head, p.v_pos_b) ||
        !make_map(&to, a.o, a.ost, a.osh, a.osb, ntok, a.H, B, p.o_pos_tok, p.o_pos_head, p.o_pos_b))
        return GRET_ERR_UNSUPPORTED;

    // TMA coordinates are 32-bit: token coordinates (and the tile past the last one) must fit
    if (a.N > (int64_t)0x7FFFFF00) return GRET_ERR_UNSUPPORTED;
    uint64_t total_dense = varlen ? 0 : (uint64_t)units * p.spans_per_unit * a.H;
    if (total_dense > 0xFFFFFFF0ull) return GRET_ERR_UNSUPPORTED;
    if (varlen) {
        // tickets are counted in 32 bits on the device: a sequence of len tokens has at most
        // len / (C G) + 1 spans, so N / (C G) + n_seqs + 1 bounds the total without reading
        // cu_seqlens
        const uint64_t span_bound = (uint64_t)(a.N / ((int64_t)C * G)) + (uint64_t)units + 1;
        if (span_bound * (uint64_t)a.H > 0xFFFFFFF0ull) return GRET_ERR_UNSUPPORTED;
    }
    if (cudaMemsetAsync(ws, 0, L.prefix, a.stream) != cudaSuccess) return GRET_ERR_CUDA;
    if (a.test_first_ticket > 0) {
        set_u32_kernel<<<1, 1, 0, a.stream>>>(p.ticket, a.test_first_ticket);
        if (cudaGetLastError() != cudaSuccess) return GRET_ERR_CUDA;
    }
    if (varlen) {
        plan_kernel<<<1, 1024, 0, a.stream>>>(a.cu_seqlens, units, G, p.prefix);
        if (cudaGetLastError() != cudaSuccess) return GRET_ERR_CUDA;
    }
    const size_t smem = sizeof(Smem);
    if (cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return GRET_ERR_CUDA;
    {
        // the in-kernel register split (setmaxnreg) assumes exactly LAUNCH_REGS per thread
        static int regs = -1;
        if (regs < 0) {
            cudaFuncAttributes fa;
            if (cudaFuncGetAttributes(&fa, prefill_tc_kernel) != cudaSuccess) return GRET_ERR_CUDA;
            regs = fa.numRegs;
        }
        if (regs != LAUNCH_REGS) return GRET_ERR_UNSUPPORTED;
    }
    int grid = sm_count();
    if (!varlen && total_dense < (uint64_t)grid) grid = (int)total_dense;
    if (grid < 1) grid = 1;
    prefill_tc_kernel<<<grid, NTHREADS, smem, a.stream>>>(tq, tk, tv, to, p, (uint32_t)total_dense);
    return cudaGetLastError() == cudaSuccess ? GRET_OK : GRET_ERR_CUDA;
}

}  // namespace gret
