// gn_gate.cu -- the gated-retention output epilogue: per-head GroupNorm of O times swish(X W_G).
//
// Page "YOCO 完全拆解：Decoder-Decoder 架构如何让 KV Cache 只存一次", section
// "路线二：Multi-Head Gated Retention": the retention output of each head is group-normalised (one
// group per head, so heads cannot drift in scale) and multiplied element-wise by swish(X W_G),
// which chooses the channels written back to the residual stream.  For token t and head h:
//     z   = X_t W_G                                          (GEMM, [T, D] x [D, H*d_v])
//     n_j = (o_j - mean) / sqrt(var + eps) * gn_w + gn_b     (o = O_t[h*d_v .. h*d_v + d_v))
//     y_j = n_j * z_j * sigmoid(z_j)
//
// The GEMM dominates (2 D H d_v FLOP per token): a persistent tcgen05 kernel run by pairs of
// CTAs (clusters of two, one CTA per SM).  A pair computes output tiles of 256 tokens x 256
// columns (two heads) with cta_group::2 MMAs: each CTA loads its 128 rows of X and its 128
// columns of W per K block of 64 through a 6-stage TMA ring into its own shared memory, the even
// CTA issues the MMAs for both, and each CTA's tensor memory receives its 128 rows x 256
// columns in fp32.  Against single-CTA 128 x 256 tiles this cuts the operand bytes each SM
// pulls from L2 per MMA by a third (32 KB instead of 48 KB per K block), the bound of that
// version.  Two accumulator buffers let the epilogue of one tile run under the MMAs of the
// next.  The epilogue is fused: GroupNorm statistics of the O row, swish of the accumulator,
// the product, bf16 out; z never goes to memory.
//
// The same GEMM, with a plain epilogue, is the layer's input projection: X W_qkvg with
// W_qkvg = [W_Q | W_K | W_V | W_gamma] gives q, k, v (bf16, [T, H, d] each) and the gate logits
// g (fp32, [T, H]) in one pass over X (qkvg_projection below).
//
// Warp roles (384 threads per CTA): warp 0 TMA producer (both CTAs; the odd CTA's loads count
// on the even CTA's stage barrier), warp 1 MMA issuer (even CTA; warp 1 of both CTAs allocates
// the pair's TMEM), warps 2-3 idle, warps 4-7 epilogue for the first head of the CTA's rows of a
// tile, warps 8-11 for the second; the epilogue threads of both CTAs release an accumulator
// buffer on the even CTA's barrier.  Tiles are assigned round-robin over pairs, in the grouped
// order of tile_coords, so the pairs working at one time share a few X row-blocks and column
// blocks of W through L2.  Every wait is bounded; a wait that gives up makes every role exit,
// and the two CTAs leave together (cluster barrier) once the even CTA's MMAs have drained.
#include "gn_gate.cuh"

#include "sm100.cuh"
#include "tma_host.cuh"

namespace gret {

using namespace sm100;

namespace {

constexpr int BM = 128;                         // rows per CTA; a pair's tile has 2 BM
constexpr int BN = 256, BK = 64, STAGES = 6;    // columns per tile; each CTA loads BN / 2 of W
constexpr int PM = 2 * BM;                      // rows per pair tile
constexpr int A_BYTES = BM * BK * 2;            // 16 KB
constexpr int B_BYTES = (BN / 2) * BK * 2;      // 16 KB
constexpr int NTHREADS = 384;
constexpr uint64_t WAIT_NS = 2000000000ull;
constexpr uint64_t DRAIN_NS = 200000000ull;

struct __align__(1024) GSmem {
    unsigned char a[STAGES][A_BYTES];
    unsigned char b[STAGES][B_BYTES];
    uint64_t full[STAGES], empty[STAGES];
    uint64_t acc_full[2], acc_empty[2], drain;
    uint32_t tmem_base;
    uint32_t abort;
};

struct GParams {
    const __nv_bfloat16* o;
    const float* gn_w;
    const float* gn_b;
    __nv_bfloat16* y;
    float eps;
    int64_t T;
    int F, D;          // F: output columns (GroupNorm gate: H * 128; projection: 3 H 128 + H)
    int m_blocks, n_blocks, n_tiles;   // in pair tiles (PM rows x BN columns)
    int group_m;       // tile order: runs of group_m row blocks (1 = row-major)
    // projection outputs
    __nv_bfloat16* qkv[3];   // q, k, v: [T, H, 128] bf16
    float* g;                // [T, H] fp32
    int H;
};

enum EpilogueMode { EPI_GN_GATE = 0, EPI_PROJECTION = 1 };

__device__ __forceinline__ bool wait_bar(GSmem& sm, uint64_t* bar, uint32_t parity) {
    if (mbar_wait(bar, parity, &sm.abort, WAIT_NS)) return true;
    atomicExch(&sm.abort, 1u);
    return false;
}

// Tile order: runs of group_m row blocks, and inside a run the row blocks fastest, so that one
// wave of CTAs shares few rows of X and few column blocks of W and both stay in L2 while the
// wave runs.  A wide W (the projection's 37 column blocks) is otherwise streamed once per few
// row blocks; a narrow one (the gate's 12) already fits, and there row-major order (group_m 1)
// measured faster.
__device__ __forceinline__ void tile_coords(const GParams& p, int tile, int& mb, int& nb) {
    const int per_group = p.group_m * p.n_blocks;
    const int grp = tile / per_group, rem = tile - grp * per_group;
    const int rows = min(p.group_m, p.m_blocks - grp * p.group_m);
    nb = rem / rows;
    mb = grp * p.group_m + (rem - nb * rows);
}

int group_rows(int n_blocks) { return n_blocks > 16 ? 16 : 1; }

// Both CTAs: this CTA's rows of X (rows PM mb + BM rank) and its half of the column block of W
// (columns BN nb + (BN / 2) rank), into its own stage; the bytes count on the even CTA's stage
// barrier, which expects both CTAs' loads.  A stage is reused once the pair's MMAs on it are done
// (the even CTA's commit arrives on the empty barrier of both CTAs).
__device__ void producer(GSmem& sm, const GParams& p, const CUtensorMap* tx, const CUtensorMap* tw,
                         uint32_t rank, int pair, int n_pairs) {
    const int kblocks = p.D / BK;
    int it = 0;
    bool ok = true;
    for (int tile = pair; tile < p.n_tiles && ok; tile += n_pairs) {
        int mb, nb;
        tile_coords(p, tile, mb, nb);
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
            const int s = it % STAGES;
            if (it >= STAGES && !wait_bar(sm, &sm.empty[s], ((it / STAGES) - 1) & 1)) {
                ok = false;
                break;
            }
            if (rank == 0) mbar_arrive_expect_tx(&sm.full[s], 2 * (A_BYTES + B_BYTES));
            const uint32_t fb = mapa_shared(&sm.full[s], 0);
            tma_load_2d_pair(sm.a[s], tx, fb, kb * BK, mb * PM + (int)rank * BM);
#pragma unroll
            for (int j = 0; j < BN / 128; ++j)
                tma_load_2d_pair(sm.b[s] + j * (BK * 128), tw, fb,
                                 nb * BN + (int)rank * (BN / 2) + j * 64, kb * BK);
        }
    }
    // no TMA write into this CTA may be in flight when it exits: wait until the pair's MMAs have
    // consumed the last stages (the stage's empty barrier)
    uint32_t never = 0;
    for (int jj = (it >= STAGES ? it - STAGES : 0); jj < it; ++jj)
        mbar_wait(&sm.empty[jj % STAGES], (jj / STAGES) & 1, &never, DRAIN_NS);
}

// Even CTA, one thread: the pair's MMAs, M = 256 (128 rows from each CTA), N = 256 (128 columns
// from each CTA's half of W), into accumulator buffer buf of both CTAs' tensor memory.
__device__ void mma_issuer(GSmem& sm, const GParams& p, uint32_t tmem, int pair, int n_pairs) {
    const int kblocks = p.D / BK;
    const uint32_t idesc = idesc_bf16(PM, BN, 0, 1);
    int it = 0, t_local = 0;
    bool ok = true;
    for (int tile = pair; tile < p.n_tiles && ok; tile += n_pairs, ++t_local) {
        const int buf = t_local & 1;
        if (t_local >= 2 && !wait_bar(sm, &sm.acc_empty[buf], ((t_local >> 1) - 1) & 1)) break;
        tc_fence_after();
        const uint32_t d = tmem + buf * BN;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
            const int s = it % STAGES;
            if (!wait_bar(sm, &sm.full[s], (it / STAGES) & 1)) { ok = false; break; }
            tc_fence_after();
            const uint32_t ab = smem_u32(sm.a[s]), bb = smem_u32(sm.b[s]);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
                mma_ss_pair(d, sdesc_sw128(ab + kk * 32, 16, 1024),
                            sdesc_sw128(bb + kk * 2048, BK * 128, 1024), idesc,
                            (kb > 0 || kk > 0) ? 1u : 0u);
            mma_commit_pair(&sm.empty[s], 0x3);
        }
        if (!ok) break;
        mma_commit_pair(&sm.acc_full[buf], 0x3);
    }
    uint32_t never = 0;
    mma_commit_pair(&sm.drain, 0x1);
    mbar_wait(&sm.drain, 0, &never, DRAIN_NS);
}

// Projection epilogue of one thread: token row t, the 128 accumulator columns starting at
// col0 (one head of q, k or v, or the gate logits and padding).
__device__ __forceinline__ void store_projection(const GParams& p, uint32_t taddr, int64_t t,
                                                 int col0, bool valid) {
    const int hd = p.H * 128;
    if (col0 < 3 * hd) {
        const int which = col0 / hd;
        __nv_bfloat16* base = which == 0 ? p.qkv[0] : (which == 1 ? p.qkv[1] : p.qkv[2]);
        __nv_bfloat16* dst = base + t * hd + (col0 - which * hd);
#pragma unroll 1
        for (int jc = 0; jc < 4; ++jc) {
            float z[32];
            tmem_ld32(taddr + jc * 32, z);
            tmem_ld_wait();
            if (valid) {
                uint4* d4 = reinterpret_cast<uint4*>(dst + jc * 32);
#pragma unroll
                for (int v4 = 0; v4 < 4; ++v4)
                    d4[v4] = make_uint4(pack_bf16x2(z[8 * v4 + 0], z[8 * v4 + 1]),
                                        pack_bf16x2(z[8 * v4 + 2], z[8 * v4 + 3]),
                                        pack_bf16x2(z[8 * v4 + 4], z[8 * v4 + 5]),
                                        pack_bf16x2(z[8 * v4 + 6], z[8 * v4 + 7]));
            }
        }
    } else if (col0 == 3 * hd) {   // the H gate-logit columns (H <= 128), then padding
#pragma unroll 1
        for (int jc = 0; jc * 32 < p.H; ++jc) {
            float z[32];
            tmem_ld32(taddr + jc * 32, z);
            tmem_ld_wait();
            if (valid) {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (jc * 32 + i < p.H) p.g[t * p.H + jc * 32 + i] = z[i];
            }
        }
    }
}

// One epilogue thread: token row r of the tile, one head (128 columns) of it.
template <int MODE>
__device__ void epilogue(GSmem& sm, const GParams& p, uint32_t tmem, int warp, int lane,
                         uint32_t rank, int pair, int n_pairs) {
    const int q = warp & 3, r = q * 32 + lane;
    const int half = (warp - 4) >> 2;                    // which head of the 256-column tile
    const uint32_t lane_base = ((uint32_t)(q * 32)) << 16;
    // the even CTA's release barriers
    const uint32_t acc_empty_even0 = mapa_shared(&sm.acc_empty[0], 0);
    const uint32_t acc_empty_even1 = mapa_shared(&sm.acc_empty[1], 0);
    int t_local = 0;
    for (int tile = pair; tile < p.n_tiles; tile += n_pairs, ++t_local) {
        const int buf = t_local & 1;
        int mb, nb;
        tile_coords(p, tile, mb, nb);
        const int64_t t = (int64_t)mb * PM + (int64_t)rank * BM + r;
        const int col0 = nb * BN + half * 128;
        const bool valid = t < p.T;
        if (MODE == EPI_PROJECTION) {
            if (!mbar_wait(&sm.acc_full[buf], (t_local >> 1) & 1, &sm.abort, WAIT_NS)) {
                atomicExch(&sm.abort, 1u);
                return;
            }
            tc_fence_after();
            store_projection(p, tmem + lane_base + buf * BN + half * 128, t, col0, valid);
            tc_fence_before();
            mbar_arrive_cluster(buf ? acc_empty_even1 : acc_empty_even0);
            continue;
        }
        // GroupNorm statistics of this head's slice of O, computed while the MMAs run; the row
        // (256 bytes) is read again per 32 columns below, from L1
        float mean = 0.f, inv = 0.f;
        const uint4* src = reinterpret_cast<const uint4*>(p.o + t * p.F + col0);
        if (valid) {
            float s = 0.f, s2 = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint4 u = __ldg(src + i);
                const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
                    s += f.x + f.y;
                }
            }
            mean = s * (1.f / 128.f);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint4 u = __ldg(src + i);
                const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
                    s2 += (f.x - mean) * (f.x - mean) + (f.y - mean) * (f.y - mean);
                }
            }
            inv = rsqrtf(s2 * (1.f / 128.f) + p.eps);
        }
        if (!mbar_wait(&sm.acc_full[buf], (t_local >> 1) & 1, &sm.abort, WAIT_NS)) {
            atomicExch(&sm.abort, 1u);
            return;
        }
        tc_fence_after();
        __nv_bfloat16* dst = p.y + t * p.F + col0;
#pragma unroll 1
        for (int jc = 0; jc < 4; ++jc) {
            float z[32];
            tmem_ld32(tmem + lane_base + buf * BN + half * 128 + jc * 32, z);
            tmem_ld_wait();
            if (valid) {
                uint32_t ow[16];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint4 u = __ldg(src + jc * 4 + i);
                    ow[4 * i + 0] = u.x;
                    ow[4 * i + 1] = u.y;
                    ow[4 * i + 2] = u.z;
                    ow[4 * i + 3] = u.w;
                }
                uint32_t out[16];
                // (o - mean) * inv as one packed fma per pair: o * inv + (-mean * inv)
                const float2 inv2 = make_float2(inv, inv), nmi2 = make_float2(-mean * inv, -mean * inv);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int c = jc * 32 + 2 * i;
                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ow[i]));
                    const float2 nn = fma2(f, inv2, nmi2);
                    float n0 = nn.x, n1 = nn.y;
                    if (p.gn_w) {
                        n0 *= __ldg(p.gn_w + col0 + c);
                        n1 *= __ldg(p.gn_w + col0 + c + 1);
                    }
                    if (p.gn_b) {
                        n0 += __ldg(p.gn_b + col0 + c);
                        n1 += __ldg(p.gn_b + col0 + c + 1);
                    }
                    const float z0 = z[2 * i], z1 = z[2 * i + 1];
                    // swish(z) = z sigmoid(z); the fast division (a few ulp) is far below the
                    // bf16 rounding of the output
                    const float s0 = __fdividef(z0, 1.f + __expf(-z0));
                    const float s1 = __fdividef(z1, 1.f + __expf(-z1));
                    out[i] = pack_bf16x2(n0 * s0, n1 * s1);
                }
                uint4* d4 = reinterpret_cast<uint4*>(dst + jc * 32);
#pragma unroll
                for (int v4 = 0; v4 < 4; ++v4)
                    d4[v4] = make_uint4(out[4 * v4], out[4 * v4 + 1], out[4 * v4 + 2], out[4 * v4 + 3]);
            }
        }
        tc_fence_before();
        mbar_arrive_cluster(buf ? acc_empty_even1 : acc_empty_even0);
    }
}

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
    gn_gate_kernel(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap tw,
                   const GParams p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    GSmem& sm = *reinterpret_cast<GSmem*>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();
    const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
    // the swizzled tiles need 1 KB alignment; both CTAs of a pair see the same layout, so they
    // take this exit together, before any cluster-wide step
    if ((smem_u32(smem_raw) & 1023u) != 0) return;
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.acc_full[b], 1);
            mbar_init(&sm.acc_empty[b], 2 * 256);   // the epilogue threads of both CTAs
        }
        mbar_init(&sm.drain, 1);
        sm.abort = 0;
        fence_mbar_init();
    }
    cluster_sync();   // every barrier of the pair is initialised before the other CTA uses it
    if (warp == 1) {
        tmem_alloc_pair(&sm.tmem_base, 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tx);
            tma_prefetch_desc(&tw);
            producer(sm, p, &tx, &tw, rank, pair, n_pairs);
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) mma_issuer(sm, p, tmem, pair, n_pairs);
    } else if (warp >= 4) {
        epilogue<MODE>(sm, p, tmem, warp, lane, rank, pair, n_pairs);
    }
    tc_fence_before();
    __syncthreads();
    // the even CTA's MMAs have drained (its issuer waited for them before the barrier above):
    // neither CTA leaves while the pair's MMAs could still touch its memory
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, 512);
    }
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

// Pairs resident at once on this device (clusters of two need two SMs of one GPC).
template <int MODE>
int max_pairs(size_t smem) {
    static int cached[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (!cached[dev]) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (unsigned)(sm_count() / 2), 1, 1);
        cfg.blockDim = dim3(NTHREADS, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = 2;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, gn_gate_kernel<MODE>, &cfg) != cudaSuccess || n < 1)
            n = sm_count() / 2;
        cached[dev] = n;
    }
    return cached[dev];
}

template <int MODE>
gret_status_t launch_gemm(const CUtensorMap& tx, const CUtensorMap& tw, const GParams& p,
                          cudaStream_t stream) {
    const size_t smem = sizeof(GSmem);
    if (cudaFuncSetAttribute(gn_gate_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return GRET_ERR_CUDA;
    int pairs = max_pairs<MODE>(smem);
    if (p.n_tiles < pairs) pairs = p.n_tiles;
    if (pairs < 1) pairs = 1;
    gn_gate_kernel<MODE><<<2 * pairs, NTHREADS, smem, stream>>>(tx, tw, p);
    return cudaGetLastError() == cudaSuccess ? GRET_OK : GRET_ERR_CUDA;
}

}  // namespace

gret_status_t launch_gn_gate(const void* o, const void* x, const void* w_g, const float* gn_weight,
                             const float* gn_bias, float eps, int64_t T, int H, int d_v, int D,
                             void* y, cudaStream_t stream) {
    const int F = H * d_v;
    if (d_v != 128 || F % BN != 0 || D % BK != 0) return GRET_ERR_UNSUPPORTED;
    if (T > ((int64_t)1 << 31) - PM) return GRET_ERR_UNSUPPORTED;
    CUtensorMap tx, tw;
    {
        uint64_t dims[2] = {(uint64_t)D, (uint64_t)T};
        uint64_t strides[1] = {(uint64_t)D * 2};
        uint32_t box[2] = {BK, BM};
        if (!make_bf16_map(&tx, x, 2, dims, strides, box)) return GRET_ERR_UNSUPPORTED;
    }
    {
        uint64_t dims[2] = {(uint64_t)F, (uint64_t)D};
        uint64_t strides[1] = {(uint64_t)F * 2};
        uint32_t box[2] = {64, BK};
        if (!make_bf16_map(&tw, w_g, 2, dims, strides, box)) return GRET_ERR_UNSUPPORTED;
    }
    GParams p = {};
    p.o = (const __nv_bfloat16*)o;
    p.gn_w = gn_weight;
    p.gn_b = gn_bias;
    p.y = (__nv_bfloat16*)y;
    p.eps = eps;
    p.T = T;
    p.F = F;
    p.D = D;
    p.m_blocks = (int)((T + PM - 1) / PM);
    p.n_blocks = F / BN;
    p.n_tiles = p.m_blocks * p.n_blocks;
    p.group_m = group_rows(p.n_blocks);
    return launch_gemm<EPI_GN_GATE>(tx, tw, p, stream);
}

gret_status_t launch_qkvg_projection(const void* x, const void* w, int64_t ldw, int64_t T, int H,
                                     int D, void* q, void* k, void* v, float* g,
                                     cudaStream_t stream) {
    const int F = 3 * H * 128 + H;
    if (H < 1 || H > 128 || D % BK != 0) return GRET_ERR_UNSUPPORTED;
    if (T > ((int64_t)1 << 31) - PM) return GRET_ERR_UNSUPPORTED;
    CUtensorMap tx, tw;
    {
        uint64_t dims[2] = {(uint64_t)D, (uint64_t)T};
        uint64_t strides[1] = {(uint64_t)D * 2};
        uint32_t box[2] = {BK, BM};
        if (!make_bf16_map(&tx, x, 2, dims, strides, box)) return GRET_ERR_UNSUPPORTED;
    }
    {
        // columns past F (the last tile's padding) are read as zeros
        uint64_t dims[2] = {(uint64_t)F, (uint64_t)D};
        uint64_t strides[1] = {(uint64_t)ldw * 2};
        uint32_t box[2] = {64, BK};
        if (!make_bf16_map(&tw, w, 2, dims, strides, box)) return GRET_ERR_UNSUPPORTED;
    }
    GParams p = {};
    p.T = T;
    p.F = F;
    p.D = D;
    p.H = H;
    p.qkv[0] = (__nv_bfloat16*)q;
    p.qkv[1] = (__nv_bfloat16*)k;
    p.qkv[2] = (__nv_bfloat16*)v;
    p.g = g;
    p.m_blocks = (int)((T + PM - 1) / PM);
    p.n_blocks = (F + BN - 1) / BN;
    p.n_tiles = p.m_blocks * p.n_blocks;
    p.group_m = group_rows(p.n_blocks);
    return launch_gemm<EPI_PROJECTION>(tx, tw, p, stream);
}

}  // namespace gret
