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
// each to bf16 once costs up to 2^-8 relative per element and, measured against an fp64
// reference, left errors of 1-3% of rms on large outputs.  Each is therefore split into a bf16
// high half and a bf16 low half (x - hi), and both halves go through the MMA: P V and Q S_prev
// and (w K)^T V are each two MMAs, which keeps them within a few 1e-6 of fp32.  V and Q are used
// exactly as loaded.
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
// Pass B reads the span's K and V a second time: from L2 when spans are short, from DRAM when
// the CTAs' spans together outgrow L2 (longer spans still win: fewer look-backs, fuller waves).
// Inclusive states live in a two-slot ring per chain: span s+2 can only overwrite the slot of
// span s after span s+1 has consumed it, because it needs span s+1's own inclusive state first.
// Tickets are taken by running CTAs in increasing order and every span depends only on a smaller
// ticket, so the chain always progresses.
//
// Warp roles (384 threads = 3 warpgroups, one CTA per SM):
//   warp 0      TMA producer (lane 0): K, V (and Q in pass B) tiles, two pipeline stages;
//               the whole warp scans the chunk's gate logits into the stage's gate slot
//   warp 1      tcgen05 MMA issuer (one thread); owns the 512-column TMEM allocation
//   warps 2-3   their share of the w K split (3 of the 16 chunks of two rows each)
//   warps 4-7   "P group": decay mask A -> P (written back into TMEM as bf16 halves), its share
//               of the w K split (6 chunks of its row), and the output epilogue
//               O + exp(c_t) OX -> bf16 -> TMA store through the state buffer
//   warps 8-11  "state group": its share of the w K split (7 chunks of its row), the fp32
//               state (one row per thread), the look-back, and the bf16 halves of the state
//               that Q S_prev reads
// Registers: launched at 168 per thread (384 x 168 = 64512); the first warpgroup drops to 88,
// the P group to 136 and the state group (128 fp32 state values per thread) rises to 256:
// 128 x (88 + 136 + 256) = 61440 <= 64512, and each SM sub-partition (one warp of each group)
// needs 32 x 480 <= 16384.  The host refuses to launch a build whose per-thread register count
// is not 168, since a request for more registers than the block holds would wait forever.
// TMEM columns: [0,128) A, then P (bf16 halves, see mma_pv); [128,256) O; [256,384) OX;
// [384,512) dS.
// Every wait is bounded (see sm100::mbar_wait); a wait that gives up records GRET_ERR_TIMEOUT in
// the workspace, and the kernel drains its copies, frees TMEM and exits.
#include "prefill_tc.cuh"

#include <stdlib.h>

#include <algorithm>

#include "sm100.cuh"
#include "tma_host.cuh"

namespace gret {

using namespace sm100;

namespace {

constexpr int C = 128;                  // tokens per chunk
constexpr int D = 128;                  // head width (d_k = d_v)
constexpr int TILE = C * D * 2;         // one bf16 128x128 tile
constexpr int SLAB = TILE / 2;          // one 64-column slab
constexpr int NTHREADS = 384;
constexpr int ITEM_DEPTH = 4;
constexpr uint64_t WAIT_NS = 2000000000ull;   // a wait gives up after 2 s
constexpr uint64_t DRAIN_NS = 200000000ull;   // exit-time drains give up after 0.2 s

constexpr uint32_t TM_A = 0, TM_O = 128, TM_OX = 256, TM_DS = 384;

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
    unsigned char q[2][TILE];  // Q tile; in pass A, and after Q S in pass B, the low half of w K
    unsigned char k[2][TILE];  // K tile; rewritten in place as the high half of w K
    unsigned char v[2][TILE];
    // bf16 high half, then low half, of the state that Q S_prev reads; between a chunk's Q S_lo
    // and the next high half, the chunk's bf16 output tile on its way out by TMA store
    unsigned char sbf[TILE];
    uint64_t kv_full[2], stage_empty[2];
    uint64_t item_full[ITEM_DEPTH], item_empty[ITEM_DEPTH];
    // k_ready / kp_ready / kh_ready (per stage): the state group's / the P group's / the helpers'
    // share of the w K split is written.  Each has one producing group, so arrivals of different groups never mix, and
    // being per stage, a group can reach the next phase of a stage's barrier only after the MMA
    // has released that stage -- so no waiter can be left two phases behind.
    uint64_t k_ready[2], kh_ready[2], kp_ready[2];
    uint64_t a_full, s3a_done, q_free, p_ready, s_lo_ready, o_full, o_free, ds_full, ds_free,
        s_ready, sbf_free, drain;
    Item items[ITEM_DEPTH];
    float gc[2][C];            // per stage: in-chunk inclusive cumulative log2-decay of each token
    float gtot[2];             // per stage: the chunk's total log2-decay
    // per stage: exponent base of the key weights w_m = k_scale * 2^(gbase - c_m): the chunk
    // total in pass B, the chunk total plus that of the span's later chunks in pass A
    float gbase[2];
    uint32_t dec[3][2];        // group-uniform wait decisions (double-buffered)
    uint32_t tmem_base;
    uint32_t abort;
};

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
    int gid;      // 0 = P group, 1 = state group, 2 = split helpers
    int tid;      // thread index within the group
    int nthreads = 128;
    int flip = 0;

    __device__ bool wait(uint64_t* bar, uint32_t parity) {
        if (tid == 0) {
            bool ok = mbar_wait(bar, parity, &sm->abort, WAIT_NS);
            if (!ok) {
                if (!sm->abort) set_error(p->err);
                atomicExch(&sm->abort, 1u);
            }
            sm->dec[gid][flip] = ok ? 0u : 1u;
        }
        named_sync(1 + gid, nthreads);
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
                if (globaltimer_ns() - t0 > WAIT_NS) break;
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
// the sequence), the chunk total and the weight base `after` + total into the stage's gate slot;
// returns the chunk total on every lane.
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
#pragma unroll
    for (int e = 0; e < 4; ++e) sm.gc[st][4 * lane + e] = excl + lam[e];
    const float tot = __shfl_sync(0xffffffffu, x, 31);
    if (lane == 31) {
        sm.gtot[st] = tot;
        sm.gbase[st] = after + tot;
    }
    return tot;
}

__device__ void producer(Smem& sm, const TcParams& p, const CUtensorMap* tq, const CUtensorMap* tk,
                         const CUtensorMap* tv, uint32_t total, int lane) {
    int j = 0, it_n = 0;
    bool aborted = false;
    while (!aborted) {
        const int slot = it_n % ITEM_DEPTH;
        int ok = 1;
        if (lane == 0 && it_n >= ITEM_DEPTH)
            ok = mbar_wait(&sm.item_empty[slot], ((it_n / ITEM_DEPTH) - 1) & 1, &sm.abort, WAIT_NS);
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
        // pass A visits the span's chunks last to first (its aggregate is accumulated by the
        // MMAs with each key weighted by its decay to the end of the span); pass B first to last
        const int n = it.c_end - it.c_begin;
        float after = 0.f;   // pass A: log2-decay of the chunks after the current one
        for (int jj = 0; jj < 2 * n; ++jj) {
            const bool pass_b = jj >= n;
            const int c = pass_b ? it.c_begin + (jj - n) : it.c_end - 1 - jj;
            const int st = j & 1;
            float g4[4];
            gate_load(p, it, c, lane, g4);   // in flight while the stage is awaited
            ok = 1;
            if (lane == 0 && j >= 2)
                ok = mbar_wait(&sm.stage_empty[st], ((j >> 1) - 1) & 1, &sm.abort, WAIT_NS);
            if (!__shfl_sync(0xffffffffu, ok, 0)) {
                aborted = true;
                break;
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(&sm.kv_full[st], pass_b ? 3 * TILE : 2 * TILE);
                const int tok = (int)(it.tok_first + (int64_t)c * C);
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
                        tma_load_4d(sm.q[st] + half * SLAB, tq, &sm.kv_full[st], ck[0], ck[1],
                                    ck[2], ck[3]);
                }
            }
            const float tot = gate_scan(sm, p, it, c, st, lane, g4, pass_b ? 0.f : after);
            if (!pass_b) after += tot;
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.kv_full[st]);
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

// D (+)= P V with P (bf16, K-major) in TMEM.  P is stored per 32-token group g = 0..3 as
// [16 columns of high halves | 16 columns of low halves] at columns 32 g; the K-step of tokens
// [16 kk, 16 kk + 16) of one half starts at column 32 (kk / 2) + 8 (kk % 2) + 16 * half.
__device__ __forceinline__ void mma_pv(uint32_t d, uint32_t p_base, int half, uint32_t v_base,
                                       bool accumulate) {
    const uint32_t idesc = idesc_bf16(128, 128, 0, 1);
#pragma unroll 1
    for (int kk = 0; kk < 8; ++kk)
        mma_ts(d, p_base + 32 * (kk >> 1) + 8 * (kk & 1) + 16 * half,
               sdesc_sw128(v_base + kk * 2048u, SLAB, 1024), idesc,
               (accumulate || kk > 0) ? 1u : 0u);
}

// dS (+)= (w K)^T V as the sum of its bf16 high half (K slot) and low half (Q slot).
__device__ __forceinline__ void mma_ds(uint32_t tmem, Smem& sm, int st, bool accumulate) {
    mma_128(tmem + TM_DS, smem_u32(sm.k[st]), true, smem_u32(sm.v[st]), true, accumulate);
    mma_128(tmem + TM_DS, smem_u32(sm.q[st]), true, smem_u32(sm.v[st]), true, true);
}

__device__ void mma_issuer(Smem& sm, const TcParams& p, uint32_t tmem) {
    int j = 0, b = 0, it_n = 0;
    int dsn = 0;   // dS results handed to the state group so far (phases of ds_full)
    bool ok = true;
    auto W = [&](uint64_t* bar, uint32_t par) {
        if (ok && !mbar_wait(bar, par, &sm.abort, WAIT_NS)) {
            ok = false;
            if (!sm.abort) set_error(p.err);
            atomicExch(&sm.abort, 1u);
        }
        return ok;
    };
    const uint32_t sbf = smem_u32(sm.sbf);
    while (ok) {
        const int slot = it_n % ITEM_DEPTH;
        if (!W(&sm.item_full[slot], (it_n / ITEM_DEPTH) & 1)) break;
        const Item it = sm.items[slot];
        mbar_arrive(&sm.item_empty[slot]);
        ++it_n;
        if (!it.valid) break;
        // pass A: the span's aggregate, one dS result accumulated over its chunks (which the
        // producer delivers last to first, each key weighted by its decay to the span's end)
        const int n = it.c_end - it.c_begin;
        for (int i = 0; i < n && ok; ++i, ++j) {
            const int st = j & 1;
            if (!W(&sm.kv_full[st], (j >> 1) & 1)) break;
            if (!W(&sm.k_ready[st], (j >> 1) & 1)) break;
            if (!W(&sm.kp_ready[st], (j >> 1) & 1)) break;
            if (!W(&sm.kh_ready[st], (j >> 1) & 1)) break;
            if (i == 0 && dsn > 0 && !W(&sm.ds_free, (dsn - 1) & 1)) break;
            tc_fence_after();
            mma_ds(tmem, sm, st, i > 0);
            mma_commit(&sm.stage_empty[st]);
        }
        if (!ok) break;
        if (n > 0) {
            mma_commit(&sm.ds_full);
            ++dsn;
        }
        // pass B: the full chunk.  Order per chunk: Q K^T (issued one chunk ahead), Q S_hi,
        // Q S_lo (after which the Q slot is free for the low half of w K), P V (which runs while
        // w K is split), dS (on the state chain, so as soon as the split is done), then Q K^T of
        // the next chunk once P V has read P out of the tensor memory it overwrites.
        auto issue_qk = [&](int jj, int bb) {
            const int st = jj & 1;
            if (!W(&sm.kv_full[st], (jj >> 1) & 1)) return false;
            if (bb > 0 && !W(&sm.o_full, (bb - 1) & 1)) return false;   // P of chunk bb-1 used
            tc_fence_after();
            mma_128(tmem + TM_A, smem_u32(sm.q[st]), false, smem_u32(sm.k[st]), false, false);
            mma_commit(&sm.a_full);
            return true;
        };
        if (it.c_end > it.c_begin && !issue_qk(j, b)) break;
        for (int c = it.c_begin; c < it.c_end && ok; ++c, ++j, ++b) {
            const int st = j & 1;
            const uint32_t qb = smem_u32(sm.q[st]), vb = smem_u32(sm.v[st]);
            if (!W(&sm.s_ready, b & 1)) break;
            if (b > 0 && !W(&sm.o_free, (b - 1) & 1)) break;     // O, OX read out
            tc_fence_after();
            mma_128(tmem + TM_OX, qb, false, sbf, true, false);   // OX = Q S_hi
            mma_commit(&sm.s3a_done);
            if (!W(&sm.s_lo_ready, b & 1)) break;
            tc_fence_after();
            mma_128(tmem + TM_OX, qb, false, sbf, true, true);    // OX += Q S_lo
            mma_commit(&sm.q_free);
            if (!W(&sm.p_ready, b & 1)) break;
            tc_fence_after();
            mma_pv(tmem + TM_O, tmem + TM_A, 0, vb, false);        // O  = P_hi V
            mma_pv(tmem + TM_O, tmem + TM_A, 1, vb, true);         // O += P_lo V
            mma_commit(&sm.o_full);
            if (!W(&sm.k_ready[st], (j >> 1) & 1)) break;
            if (!W(&sm.kp_ready[st], (j >> 1) & 1)) break;
            if (!W(&sm.kh_ready[st], (j >> 1) & 1)) break;
            if (dsn > 0 && !W(&sm.ds_free, (dsn - 1) & 1)) break;
            tc_fence_after();
            mma_ds(tmem, sm, st, false);
            mma_commit(&sm.ds_full);
            mma_commit(&sm.stage_empty[st]);
            ++dsn;
            if (c + 1 < it.c_end && !issue_qk(j + 1, b + 1)) break;
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
    const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Chunks [I0, I0 + N) of row r of a swizzled K tile (16 chunks of 8 elements per row; chunk i
// sits in slab i / 8 at slot (i % 8) ^ (r % 8)): w * K split into a high half written back in
// place and a low half written to the same position of `lotile`.  All loads are issued before
// the first store (loads cannot move past stores to the same array).
template <int I0, int N>
__device__ __forceinline__ void split_k_chunks(unsigned char* ktile, unsigned char* lotile, int r,
                                               float w) {
    uint4 row[N];
#pragma unroll
    for (int n = 0; n < N; ++n) {
        const int i = I0 + n;
        row[n] = *reinterpret_cast<const uint4*>(ktile + (i >> 3) * SLAB + r * 128 +
                                                 (((i & 7) ^ (r & 7)) << 4));
    }
#pragma unroll
    for (int n = 0; n < N; ++n) {
        const int i = I0 + n;
        const int off = (i >> 3) * SLAB + r * 128 + (((i & 7) ^ (r & 7)) << 4);
        uint32_t* x = reinterpret_cast<uint32_t*>(&row[n]);
        uint4 lo;
        uint32_t* l = reinterpret_cast<uint32_t*>(&lo);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x[e]));
            split2(f.x * w, f.y * w, x[e], l[e]);
        }
        *reinterpret_cast<uint4*>(ktile + off) = row[n];
        *reinterpret_cast<uint4*>(lotile + off) = lo;
    }
}

// The split of w K is shared by three groups, by 16-byte chunks of each 128-element row: the state
// group takes chunks 0-6 of its own row, the P group chunks 7-12 of its own row, and warps 2-3
// chunks 13-15 of two rows each.
constexpr int SPLIT_STATE = 7, SPLIT_P = 6;
constexpr int SPLIT_HELP0 = SPLIT_STATE + SPLIT_P, SPLIT_HELP = 16 - SPLIT_HELP0;

// weight of token r of chunk c: k_scale * exp(c_b - c_r), zero past the end of the sequence
__device__ __forceinline__ float k_weight(const Smem& sm, const TcParams& p, const Item& it, int c,
                                          int st, int r) {
    const bool valid = (int64_t)c * C + r < it.len;
    return valid ? ex2f(sm.gbase[st] - sm.gc[st][r]) * p.k_scale : 0.f;
}

// Row r of the state into the MN-major swizzled tile read by Q S: the bf16 high half is
// written and the low half kept in registers for write_state_lo.
__device__ __forceinline__ void write_state_hi(unsigned char* tile, int r, const float (&S)[D],
                                               uint32_t (&lo)[D / 2]) {
#pragma unroll
    for (int cc = 0; cc < 16; ++cc) {
        uint32_t hi[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            split2(S[8 * cc + 2 * e], S[8 * cc + 2 * e + 1], hi[e], lo[4 * cc + e]);
        const int half = cc >> 3, c = cc & 7;
        *reinterpret_cast<uint4*>(tile + half * SLAB + r * 128 + ((c ^ (r & 7)) << 4)) =
            make_uint4(hi[0], hi[1], hi[2], hi[3]);
    }
}

__device__ __forceinline__ void write_state_lo(unsigned char* tile, int r,
                                               const uint32_t (&lo)[D / 2]) {
#pragma unroll
    for (int cc = 0; cc < 16; ++cc) {
        const int half = cc >> 3, c = cc & 7;
        *reinterpret_cast<uint4*>(tile + half * SLAB + r * 128 + ((c ^ (r & 7)) << 4)) =
            make_uint4(lo[4 * cc], lo[4 * cc + 1], lo[4 * cc + 2], lo[4 * cc + 3]);
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
// warps 4-7: decay mask (P split into bf16 halves in TMEM) and output epilogue

__device__ void p_group(Smem& sm, const TcParams& p, const CUtensorMap* to, uint32_t tmem, int warp,
                        int lane) {
    GroupWait gw{&sm, &p, 0, (warp - 4) * 32 + lane};
    const int q = warp & 3, r = q * 32 + lane;
    const uint32_t lane_base = ((uint32_t)(q * 32)) << 16;
    int b = 0, j = 0, it_n = 0;
    while (true) {
        const int slot = it_n % ITEM_DEPTH;
        if (!gw.wait(&sm.item_full[slot], (it_n / ITEM_DEPTH) & 1)) break;
        const Item it = sm.items[slot];
        mbar_arrive(&sm.item_empty[slot]);
        ++it_n;
        if (!it.valid) break;
        bool ok = true;
        const int n = it.c_end - it.c_begin;
        // every job of the span: pass A (its share of the w K split only), then pass B
        for (int jj = 0; jj < 2 * n; ++jj, ++j) {
            const int st = j & 1;
            const bool pass_b = jj >= n;
            const int c = pass_b ? it.c_begin + (jj - n) : it.c_end - 1 - jj;
            // the stage's gate slot is read before this group's split share is released: after
            // that the stage may be refilled
            float cr = 0.f;
            if (!pass_b) {
                if (!gw.wait(&sm.kv_full[st], (j >> 1) & 1)) { ok = false; break; }
            } else {
                if (!gw.wait(&sm.a_full, b & 1)) { ok = false; break; }
                if (!gw.wait(&sm.kv_full[st], (j >> 1) & 1)) { ok = false; break; }  // gate slot
                cr = sm.gc[st][r];
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
                        for (int i = 0; i < 16; ++i) {
                            const int m0 = jc * 32 + 2 * i;
                            const float p0 =
                                (m0 <= r) ? ex2f(cr - sm.gc[st][m0]) * p.k_scale * a[2 * i] : 0.f;
                            const float p1 = (m0 + 1 <= r)
                                                 ? ex2f(cr - sm.gc[st][m0 + 1]) * p.k_scale * a[2 * i + 1]
                                                 : 0.f;
                            split2(p0, p1, ph[i], ph[16 + i]);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) ph[i] = 0u;
                    }
                    tmem_st32(tmem + lane_base + TM_A + jc * 32, ph);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&sm.p_ready);
                // both Q S MMAs are done: the Q slot takes the low half of w K
                if (!gw.wait(&sm.q_free, b & 1)) { ok = false; break; }
            }
            split_k_chunks<SPLIT_STATE, SPLIT_P>(sm.k[st], sm.q[st], r,
                                                 k_weight(sm, p, it, c, st, r));
            fence_proxy_async_smem();
            mbar_arrive(&sm.kp_ready[st]);
            if (!pass_b) continue;
            // epilogue: O = O_inner + 2^(c_r) O_cross, rounded to bf16.  A chunk that lies wholly
            // inside its sequence goes out as one tile: rows into the state buffer (free between
            // Q S_lo and the next state write) in the swizzled layout, then two TMA stores.  The
            // rows of a partial chunk are stored one by one, so that nothing past the end of the
            // sequence (the next packed sequence) is written.
            if (!gw.wait(&sm.o_full, b & 1)) { ok = false; break; }
            tc_fence_after();
            const float ec = ex2f(cr);
            const int64_t t = (int64_t)c * C + r;
            const bool full = (int64_t)(c + 1) * C <= it.len;
            const bool valid = t < it.len;
            __nv_bfloat16* orow = p.o + (int64_t)it.b * p.osb + (it.tok_first + t) * p.ost +
                                  (int64_t)it.h * p.osh;
#pragma unroll 1
            for (int jc = 0; jc < 4; ++jc) {
                float o[32], ox[32];
                tmem_ld32(tmem + lane_base + TM_O + jc * 32, o);
                tmem_ld32(tmem + lane_base + TM_OX + jc * 32, ox);
                tmem_ld_wait();
                uint4 u[4];
#pragma unroll
                for (int v4 = 0; v4 < 4; ++v4) {
                    u[v4].x = pack_bf16x2(fmaf(ec, ox[8 * v4 + 0], o[8 * v4 + 0]),
                                          fmaf(ec, ox[8 * v4 + 1], o[8 * v4 + 1]));
                    u[v4].y = pack_bf16x2(fmaf(ec, ox[8 * v4 + 2], o[8 * v4 + 2]),
                                          fmaf(ec, ox[8 * v4 + 3], o[8 * v4 + 3]));
                    u[v4].z = pack_bf16x2(fmaf(ec, ox[8 * v4 + 4], o[8 * v4 + 4]),
                                          fmaf(ec, ox[8 * v4 + 5], o[8 * v4 + 5]));
                    u[v4].w = pack_bf16x2(fmaf(ec, ox[8 * v4 + 6], o[8 * v4 + 6]),
                                          fmaf(ec, ox[8 * v4 + 7], o[8 * v4 + 7]));
                }
                if (full) {
                    // columns 32 jc .. 32 jc + 31: 16-byte chunks 4 (jc % 2) + v4 of slab jc / 2
                    unsigned char* rowp = sm.sbf + (jc >> 1) * SLAB + r * 128;
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4)
                        *reinterpret_cast<uint4*>(rowp + (((4 * (jc & 1) + v4) ^ (r & 7)) << 4)) =
                            u[v4];
                } else if (valid) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + jc * 32);
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) dst[v4] = u[v4];
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
                        tma_store_4d(to, sm.sbf + half * SLAB, co[0], co[1], co[2], co[3]);
                    }
                    bulk_commit_group();
                    bulk_wait_group_read0();
                }
            }
            if (gw.tid == 0) mbar_arrive(&sm.sbf_free);   // the state buffer can be rewritten
            ++b;
        }
        if (!ok) break;
    }
    if (gw.tid == 0) bulk_wait_group0();   // the last output tiles are written before exit
}

// ----------------------------------------------------------------------------------------------
// warps 8-11: decayed K split, fp32 state, look-back

__device__ void state_group(Smem& sm, const TcParams& p, uint32_t tmem, int warp, int lane) {
    GroupWait gw{&sm, &p, 1, (warp - 8) * 32 + lane};
    const int q = warp & 3, r = q * 32 + lane;
    const uint32_t lane_base = ((uint32_t)(q * 32)) << 16;
    float S[D];
    int j = 0, b = 0, it_n = 0;
    int dsn = 0;   // dS results taken from the MMA so far (phases of ds_full)
    bool ok = true;
    while (ok) {
        const int slot = it_n % ITEM_DEPTH;
        if (!gw.wait(&sm.item_full[slot], (it_n / ITEM_DEPTH) & 1)) break;
        const Item& it = sm.items[slot];   // read in place; released at the end of the span
        ++it_n;
        if (!it.valid) {
            mbar_arrive(&sm.item_empty[slot]);
            break;
        }
        // ---- pass A: the span's aggregate Agg = sum over its keys of (decay to the span's end)
        // k^T v is accumulated by the dS MMAs over the span's chunks, which arrive last to
        // first; this group splits its share of w K and sums the span's log2-decay L, then
        // reads Agg once.
        const int n = it.c_end - it.c_begin;
#pragma unroll
        for (int i = 0; i < D; ++i) S[i] = 0.f;
        float L = 0.f;
#pragma unroll 1
        for (int i = 0; i < n; ++i) {
            const int st = (j + i) & 1;
            if (!gw.wait(&sm.kv_full[st], ((j + i) >> 1) & 1)) { ok = false; break; }
            L += sm.gtot[st];
            split_k_chunks<0, SPLIT_STATE>(sm.k[st], sm.q[st], r,
                                           k_weight(sm, p, it, it.c_end - 1 - i, st, r));
            fence_proxy_async_smem();
            mbar_arrive(&sm.k_ready[st]);
        }
        j += n;
        if (!ok) break;
        if (n > 0) {
            if (!gw.wait(&sm.ds_full, dsn & 1)) break;
            tc_fence_after();
            fold_ds(tmem + lane_base + TM_DS, S, 0.f);   // S = Agg
            tc_fence_before();
            mbar_arrive(&sm.ds_free);
            ++dsn;
        }
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
        // E comes in through the state buffer, free once the previous chunk's output tile has
        // left it: two rounds of 16 float4 per thread, each thread copying and reading back only
        // its own elements (no barrier between the rounds), with all 16 copies of a round in
        // flight.
        if (b > 0 && !gw.wait(&sm.sbf_free, (b - 1) & 1)) break;
        float4* ebuf = reinterpret_cast<float4*>(sm.sbf) + r;
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
        // ---- pass B: running state from E.  Per chunk: the bf16 high half of the state before
        // it goes into the state buffer (once the previous chunk's output tile has left it) for
        // Q S_hi, then its low half (kept in registers) once Q S_hi is done, then the chunk's
        // split of w K (into the Q slot, free after Q S_lo) and the fold of its dS.
#pragma unroll 1
        for (int i = 0; i < n; ++i) {
            const int st = (j + i) & 1;
            uint32_t slo[D / 2];   // bf16 low half of the state row, between its two writes
            if (b + i > 0 && !gw.wait(&sm.sbf_free, (b + i - 1) & 1)) { ok = false; break; }
            write_state_hi(sm.sbf, r, S, slo);
            fence_proxy_async_smem();
            mbar_arrive(&sm.s_ready);
            if (!gw.wait(&sm.kv_full[st], ((j + i) >> 1) & 1)) { ok = false; break; }
            if (!gw.wait(&sm.s3a_done, (b + i) & 1)) { ok = false; break; }
            write_state_lo(sm.sbf, r, slo);
            fence_proxy_async_smem();
            mbar_arrive(&sm.s_lo_ready);
            const float tot = sm.gtot[st];
            // every MMA reading Q has completed: its slot takes the low half of w K
            if (!gw.wait(&sm.q_free, (b + i) & 1)) { ok = false; break; }
            split_k_chunks<0, SPLIT_STATE>(sm.k[st], sm.q[st], r,
                                         k_weight(sm, p, it, it.c_begin + i, st, r));
            fence_proxy_async_smem();
            mbar_arrive(&sm.k_ready[st]);
            if (!gw.wait(&sm.ds_full, dsn & 1)) { ok = false; break; }
            tc_fence_after();
            fold_ds(tmem + lane_base + TM_DS, S, ex2f(tot));
            tc_fence_before();
            mbar_arrive(&sm.ds_free);
            ++dsn;
        }
        j += n;
        b += n;
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

// ----------------------------------------------------------------------------------------------
// warps 2-3: their share of the w K split (chunks 11-15 of rows 2t and 2t + 1), every chunk

__device__ void split_helper(Smem& sm, const TcParams& p, int warp, int lane) {
    GroupWait gw{&sm, &p, 2, (warp - 2) * 32 + lane, 64};
    const int t = (warp - 2) * 32 + lane;
    int j = 0, b = 0, it_n = 0;
    bool ok = true;
    while (ok) {
        const int slot = it_n % ITEM_DEPTH;
        if (!gw.wait(&sm.item_full[slot], (it_n / ITEM_DEPTH) & 1)) break;
        const Item it = sm.items[slot];
        mbar_arrive(&sm.item_empty[slot]);
        ++it_n;
        if (!it.valid) break;
        const int n_ch = it.c_end - it.c_begin;
        for (int jj = 0; jj < 2 * n_ch; ++jj, ++j) {
            const int st = j & 1;
            const int c = jj < n_ch ? it.c_end - 1 - jj : it.c_begin + (jj - n_ch);
            if (!gw.wait(&sm.kv_full[st], (j >> 1) & 1)) { ok = false; break; }
            if (jj >= n_ch) {   // pass B: the Q slot is free once both Q S MMAs are done
                if (!gw.wait(&sm.q_free, b & 1)) { ok = false; break; }
                ++b;
            }
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
                const int r = 2 * t + h;
                split_k_chunks<SPLIT_HELP0, SPLIT_HELP>(sm.k[st], sm.q[st], r,
                                                        k_weight(sm, p, it, c, st, r));
            }
            fence_proxy_async_smem();
            mbar_arrive(&sm.kh_ready[st]);
        }
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
            mbar_init(&sm.kv_full[s], 2);   // TMA bytes + expect_tx arrival, gate arrival
            mbar_init(&sm.stage_empty[s], 1);
        }
        for (int s = 0; s < ITEM_DEPTH; ++s) {
            mbar_init(&sm.item_full[s], 1);
            mbar_init(&sm.item_empty[s], 1 + 128 + 128 + 64);
        }
        mbar_init(&sm.a_full, 1);
        mbar_init(&sm.s3a_done, 1);
        mbar_init(&sm.q_free, 1);
        mbar_init(&sm.p_ready, 128);
        mbar_init(&sm.s_lo_ready, 128);
        mbar_init(&sm.o_full, 1);
        mbar_init(&sm.o_free, 128);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sm.k_ready[s], 128);
            mbar_init(&sm.kp_ready[s], 128);
            mbar_init(&sm.kh_ready[s], 64);
        }
        mbar_init(&sm.ds_full, 1);
        mbar_init(&sm.ds_free, 128);
        mbar_init(&sm.s_ready, 128);
        mbar_init(&sm.sbf_free, 1);
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
        asm volatile("setmaxnreg.dec.sync.aligned.u32 88;" ::: "memory");
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
        } else {
            split_helper(sm, p, warp, lane);
        }
    } else if (warp < 8) {
        // 168 -> 136 is a decrease: setmaxnreg.inc must never ask for fewer registers than the
        // warp holds, and .dec never for more.
        asm volatile("setmaxnreg.dec.sync.aligned.u32 136;" ::: "memory");
        p_group(sm, p, &to, tmem, warp, lane);
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 256;" ::: "memory");
        state_group(sm, p, tmem, warp, lane);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

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
// the larger of the two over [2, 128]; measured at 32K x 24 heads this picks 22 (two waves) and
// at 512K x 24 heads 96 (both within 2% of the best span size found by sweeping).
// GRET_SPAN_CHUNKS overrides the choice.
int span_chunks(int64_t chunks_per_unit, int64_t chains, int grid) {
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
        const int64_t spans = std::max<int64_t>(1, (chunks_per_unit + g - 1) / g);
        const int64_t waves = (chains * spans + grid - 1) / grid;
        const double cost = std::max((double)waves * (g + 1.5), 0.5 * (double)spans + g);
        if (best_cost < 0.0 || cost < best_cost) {
            best = g;
            best_cost = cost;
        }
        if (spans == 1) break;   // larger spans change nothing
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
    const int64_t chunks_per_unit =
        units > 0 ? ((varlen ? a.N / units : a.N) + C - 1) / C : 0;   // varlen: the mean
    const int G = span_chunks(chunks_per_unit, (int64_t)units * a.H, sm_count());

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
    if (varlen) {
        plan_kernel<<<1, 1024, 0, a.stream>>>(a.cu_seqlens, units, G, p.prefix);
        if (cudaGetLastError() != cudaSuccess) return GRET_ERR_CUDA;
    }
    const size_t smem = sizeof(Smem);
    if (cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return GRET_ERR_CUDA;
    {
        // the in-kernel register split (setmaxnreg) assumes exactly 168 registers per thread
        static int regs = -1;
        if (regs < 0) {
            cudaFuncAttributes fa;
            if (cudaFuncGetAttributes(&fa, prefill_tc_kernel) != cudaSuccess) return GRET_ERR_CUDA;
            regs = fa.numRegs;
        }
        if (regs != 168) return GRET_ERR_UNSUPPORTED;
    }
    int grid = sm_count();
    if (!varlen && total_dense < (uint64_t)grid) grid = (int)total_dense;
    if (grid < 1) grid = 1;
    prefill_tc_kernel<<<grid, NTHREADS, smem, a.stream>>>(tq, tk, tv, to, p, (uint32_t)total_dense);
    return cudaGetLastError() == cudaSuccess ? GRET_OK : GRET_ERR_CUDA;
}

}  // namespace gret
