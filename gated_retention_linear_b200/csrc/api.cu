// api.cu -- the C ABI declared in include/gret.h: argument checks, path choice, launches.
//
// Every check runs on the host before anything is launched, so a rejected call has no effect
// on the device.  No entry point allocates device memory.
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "prefill_tc.cuh"
#include "gn_gate.cuh"
#include "prefill_ew.cuh"
#include "swa.cuh"

using namespace gret;

namespace {

bool dim_ok(int d) { return d == 64 || d == 128; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Which prefill kernel serves a call.
enum class Path { Simt, TensorCore };

Path choose_path(gret_dtype_t dtype, int dk, int dv, int chunk) {
    if (dtype == GRET_BF16 && dk == 128 && dv == 128 && (chunk == 0 || chunk == TC_CHUNK))
        return Path::TensorCore;
    return Path::Simt;
}

int default_simt_chunk() { return 64; }

}  // namespace

extern "C" {

const char* gret_status_string(gret_status_t s) {
    switch (s) {
        case GRET_OK: return "GRET_OK";
        case GRET_ERR_INVALID_ARG: return "GRET_ERR_INVALID_ARG: argument out of range";
        case GRET_ERR_UNSUPPORTED: return "GRET_ERR_UNSUPPORTED: no kernel for this combination";
        case GRET_ERR_ALIGNMENT: return "GRET_ERR_ALIGNMENT: pointer or stride not 16-byte aligned";
        case GRET_ERR_WORKSPACE: return "GRET_ERR_WORKSPACE: workspace missing or too small";
        case GRET_ERR_CUDA: return "GRET_ERR_CUDA: a CUDA runtime call failed";
        case GRET_ERR_TIMEOUT: return "GRET_ERR_TIMEOUT: a bounded inter-block wait gave up";
    }
    return "GRET_ERR_UNKNOWN";
}

size_t gret_prefill_workspace_size(gret_dtype_t dtype, int64_t total_tokens, int n_seqs, int H,
                                   int d_k, int d_v, int chunk) {
    if (total_tokens < 0 || n_seqs < 0 || H < 0 || !dim_ok(d_k) || !dim_ok(d_v)) return 0;
    if (choose_path(dtype, d_k, d_v, chunk) == Path::TensorCore)
        return tc_workspace_size(total_tokens, n_seqs, H);
    return 0;
}

}  // extern "C"

namespace {

gret_status_t prefill_impl(const void* q, const void* k, int64_t stride_batch,
                           int64_t stride_tok, int64_t stride_head, const void* v,
                           int64_t v_stride_batch, int64_t v_stride_tok,
                           int64_t v_stride_head, const float* g, float tau,
                           float k_scale, gret_dtype_t dtype, int B, int64_t N, int H,
                           int d_k, int d_v, const int32_t* cu_seqlens, int n_seqs,
                           const float* state_in, float* state_out, void* o,
                           int64_t o_stride_batch, int64_t o_stride_tok,
                           int64_t o_stride_head, int chunk, void* workspace,
                           size_t workspace_bytes, gret_stream_t stream, uint64_t test_wait_ns,
                           uint32_t test_first_ticket) {
    if (dtype != GRET_F32 && dtype != GRET_BF16) return GRET_ERR_INVALID_ARG;
    if (!dim_ok(d_k) || !dim_ok(d_v) || H < 1 || B < 0 || N < 0) return GRET_ERR_INVALID_ARG;
    if (!(tau > 0.f) || !isfinite(tau) || !isfinite(k_scale)) return GRET_ERR_INVALID_ARG;
    if (stride_batch < 0 || stride_tok < 0 || stride_head < 0 || v_stride_batch < 0 ||
        v_stride_tok < 0 || v_stride_head < 0 || o_stride_batch < 0 || o_stride_tok < 0 ||
        o_stride_head < 0)
        return GRET_ERR_INVALID_ARG;
    int units;
    if (cu_seqlens) {
        if (B != 1 || n_seqs < 0) return GRET_ERR_INVALID_ARG;
        units = n_seqs;
    } else {
        units = B;
    }
    if (units > 65535 && choose_path(dtype, d_k, d_v, chunk) == Path::Simt)
        return GRET_ERR_UNSUPPORTED;
    const int64_t tokens = cu_seqlens ? N : (int64_t)B * N;
    if (units == 0) return GRET_OK;
    if (tokens > 0 && (!q || !k || !v || !g || !o)) return GRET_ERR_INVALID_ARG;

    PrefillArgs a;
    a.q = q; a.k = k; a.v = v;
    a.sb = stride_batch; a.st = stride_tok; a.sh = stride_head;
    a.vsb = v_stride_batch; a.vst = v_stride_tok; a.vsh = v_stride_head;
    a.g = g; a.tau = tau; a.k_scale = k_scale;
    a.B = cu_seqlens ? 1 : B; a.N = N; a.H = H; a.dk = d_k; a.dv = d_v;
    a.cu_seqlens = cu_seqlens; a.n_seqs = units;
    a.state_in = state_in; a.state_out = state_out;
    a.o = o; a.osb = o_stride_batch; a.ost = o_stride_tok; a.osh = o_stride_head;
    a.workspace = workspace; a.workspace_bytes = workspace_bytes;
    a.stream = (cudaStream_t)stream;
    a.test_wait_ns = test_wait_ns;
    a.test_first_ticket = test_first_ticket;

    if (choose_path(dtype, d_k, d_v, chunk) == Path::TensorCore) {
        a.chunk = TC_CHUNK;
        const size_t need = tc_workspace_size(tokens, units, H);
        if (!workspace || workspace_bytes < need) return GRET_ERR_WORKSPACE;
        if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GRET_ERR_ALIGNMENT;
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
            return GRET_ERR_ALIGNMENT;
        if ((stride_batch % 8) || (stride_tok % 8) || (stride_head % 8) ||
            (v_stride_batch % 8) || (v_stride_tok % 8) || (v_stride_head % 8) ||
            (o_stride_batch % 8) || (o_stride_tok % 8) || (o_stride_head % 8))
            return GRET_ERR_ALIGNMENT;
        gret_status_t st = launch_prefill_tc(a);
        return st;
    }
    a.chunk = chunk == 0 ? default_simt_chunk() : chunk;
    if (a.chunk != 16 && a.chunk != 32 && a.chunk != 64) return GRET_ERR_UNSUPPORTED;
    if (tokens == 0 && !state_out) return GRET_OK;
    cudaError_t e = launch_prefill_simt(a, dtype == GRET_BF16);
    if (e == cudaErrorInvalidValue) return GRET_ERR_UNSUPPORTED;
    return e == cudaSuccess ? GRET_OK : GRET_ERR_CUDA;
}

}  // namespace

extern "C" {

gret_status_t gret_prefill_chunkwise(const void* q, const void* k, int64_t stride_batch,
                                     int64_t stride_tok, int64_t stride_head, const void* v,
                                     int64_t v_stride_batch, int64_t v_stride_tok,
                                     int64_t v_stride_head, const float* g, float tau,
                                     float k_scale, gret_dtype_t dtype, int B, int64_t N, int H,
                                     int d_k, int d_v, const int32_t* cu_seqlens, int n_seqs,
                                     const float* state_in, float* state_out, void* o,
                                     int64_t o_stride_batch, int64_t o_stride_tok,
                                     int64_t o_stride_head, int chunk, void* workspace,
                                     size_t workspace_bytes, gret_stream_t stream) {
    const NvtxRange range("gret_prefill_chunkwise");
    return prefill_impl(q, k, stride_batch, stride_tok, stride_head, v, v_stride_batch,
                        v_stride_tok, v_stride_head, g, tau, k_scale, dtype, B, N, H, d_k, d_v,
                        cu_seqlens, n_seqs, state_in, state_out, o, o_stride_batch,
                        o_stride_tok, o_stride_head, chunk, workspace, workspace_bytes, stream, 0,
                        0);
}

gret_status_t gret_prefill_chunkwise_testing(
    const void* q, const void* k, int64_t stride_batch, int64_t stride_tok, int64_t stride_head,
    const void* v, int64_t v_stride_batch, int64_t v_stride_tok, int64_t v_stride_head,
    const float* g, float tau, float k_scale, gret_dtype_t dtype, int B, int64_t N, int H,
    int d_k, int d_v, const int32_t* cu_seqlens, int n_seqs, const float* state_in,
    float* state_out, void* o, int64_t o_stride_batch, int64_t o_stride_tok,
    int64_t o_stride_head, int chunk, void* workspace, size_t workspace_bytes,
    gret_stream_t stream, uint64_t wait_ns, uint32_t first_ticket) {
    const NvtxRange range("gret_prefill_chunkwise_testing");
    if (wait_ns == 0 || wait_ns > 2000000000ull) return GRET_ERR_INVALID_ARG;
    return prefill_impl(q, k, stride_batch, stride_tok, stride_head, v, v_stride_batch,
                        v_stride_tok, v_stride_head, g, tau, k_scale, dtype, B, N, H, d_k, d_v,
                        cu_seqlens, n_seqs, state_in, state_out, o, o_stride_batch,
                        o_stride_tok, o_stride_head, chunk, workspace, workspace_bytes, stream,
                        wait_ns, first_ticket);
}

gret_status_t gret_workspace_status(const void* workspace, gret_stream_t stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return GRET_ERR_CUDA;
    if (!workspace) return GRET_OK;
    uint32_t word = 0;
    if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
        return GRET_ERR_CUDA;
    return word == WS_ERR_NONE ? GRET_OK : GRET_ERR_TIMEOUT;
}

gret_status_t gret_decode_step(const void* q, const void* k, const void* v, const float* g,
                               float tau, float k_scale, gret_dtype_t dtype, int B, int H,
                               int d_k, int d_v, float* state, void* o, gret_stream_t stream) {
    const NvtxRange range("gret_decode_step");
    if (dtype != GRET_F32 && dtype != GRET_BF16) return GRET_ERR_INVALID_ARG;
    if (!dim_ok(d_k) || !dim_ok(d_v) || B < 0 || H < 0) return GRET_ERR_INVALID_ARG;
    if (!(tau > 0.f) || !isfinite(tau) || !isfinite(k_scale)) return GRET_ERR_INVALID_ARG;
    if ((int64_t)B * H == 0) return GRET_OK;
    if ((int64_t)B * H > 0x3fffffffLL) return GRET_ERR_INVALID_ARG;   // 2 CTAs per (b, h)
    if (!q || !k || !v || !g || !state || !o) return GRET_ERR_INVALID_ARG;
    if (!aligned16(state)) return GRET_ERR_ALIGNMENT;
    cudaError_t e = launch_decode(q, k, v, g, tau, k_scale, dtype == GRET_BF16, B, H, d_k, d_v,
                                  state, o, (cudaStream_t)stream);
    if (e == cudaErrorInvalidValue) return GRET_ERR_UNSUPPORTED;
    return e == cudaSuccess ? GRET_OK : GRET_ERR_CUDA;
}

gret_status_t gret_groupnorm_gate(const void* o, const void* x, const void* w_g,
                                  const float* gn_weight, const float* gn_bias, float eps,
                                  int64_t T, int H, int d_v, int D, void* y,
                                  gret_stream_t stream) {
    const NvtxRange range("gret_groupnorm_gate");
    if (T < 0 || H < 1 || D < 1 || !(eps >= 0.f) || !isfinite(eps)) return GRET_ERR_INVALID_ARG;
    if (d_v != 128 || D % 64 != 0) return GRET_ERR_UNSUPPORTED;
    if (T == 0) return GRET_OK;
    if (!o || !x || !w_g || !y) return GRET_ERR_INVALID_ARG;
    if (!aligned16(o) || !aligned16(x) || !aligned16(w_g) || !aligned16(y))
        return GRET_ERR_ALIGNMENT;
    return launch_gn_gate(o, x, w_g, gn_weight, gn_bias, eps, T, H, d_v, D, y,
                          (cudaStream_t)stream);
}

gret_status_t gret_qkvg_projection(const void* x, const void* w, int64_t ldw, int64_t T, int H,
                                   int d, int D, void* q, void* k, void* v, float* g,
                                   gret_stream_t stream) {
    const NvtxRange range("gret_qkvg_projection");
    if (T < 0 || H < 1 || D < 1 || d < 1) return GRET_ERR_INVALID_ARG;
    const int64_t F = 3 * (int64_t)H * d + H;
    if (ldw < F) return GRET_ERR_INVALID_ARG;
    if (d != 128 || H > 128 || D % 64 != 0) return GRET_ERR_UNSUPPORTED;
    if (T == 0) return GRET_OK;
    if (!x || !w || !q || !k || !v || !g) return GRET_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w) || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
        (reinterpret_cast<uintptr_t>(g) & 3u) != 0 || ldw % 8 != 0)
        return GRET_ERR_ALIGNMENT;
    return launch_qkvg_projection(x, w, ldw, T, H, D, q, k, v, g, (cudaStream_t)stream);
}

// Sizes the per-channel gate prefill can take: the range kernels' grid (ranges, H, B) and the
// scan's (B * H * 16 blocks) fit their limits, and the workspace byte count fits in size_t.
bool ew_sizes_ok(int B, int64_t N, int H) {
    const int64_t nch = (N + EW_CHUNK - 1) / EW_CHUNK;
    if (B > 65535 || H > 65535 || nch > 0x7fffffff || N > (int64_t)0x7FFFFF00) return false;
    if ((int64_t)B * H * 16 > 0x7fffffff) return false;
    const double bytes = (double)B * H * (double)nch * (EW_DIM * EW_DIM + EW_DIM) * 4.0;
    return bytes < 9.0e18;
}

size_t gret_prefill_elementwise_workspace_size(int B, int64_t N, int H, int d) {
    if (B < 0 || N < 0 || H < 1 || d != EW_DIM || !ew_sizes_ok(B, N, H)) return 0;
    return ew_workspace_bytes(B, N, H);
}

gret_status_t gret_prefill_elementwise(const void* q, const void* k, const void* v,
                                       const float* g, float tau, float k_scale, int B,
                                       int64_t N, int H, int d, const float* state_in,
                                       float* state_out, void* o, void* workspace,
                                       size_t workspace_bytes, gret_stream_t stream) {
    const NvtxRange range("gret_prefill_elementwise");
    if (B < 0 || N < 0 || H < 1 || d < 1) return GRET_ERR_INVALID_ARG;
    if (!(tau > 0.f) || !isfinite(tau) || !isfinite(k_scale)) return GRET_ERR_INVALID_ARG;
    if (d != EW_DIM) return GRET_ERR_UNSUPPORTED;
    if (!ew_sizes_ok(B, N, H)) return GRET_ERR_UNSUPPORTED;
    if (B == 0) return GRET_OK;
    if ((state_in && !aligned16(state_in)) || (state_out && !aligned16(state_out)))
        return GRET_ERR_ALIGNMENT;
    const cudaStream_t s = (cudaStream_t)stream;
    const size_t state_bytes = (size_t)B * H * EW_DIM * EW_DIM * sizeof(float);
    if (N == 0) {   // no tokens: the final state is the entry state
        if (!state_out || state_out == state_in) return GRET_OK;
        const cudaError_t e = state_in ? cudaMemcpyAsync(state_out, state_in, state_bytes,
                                                         cudaMemcpyDeviceToDevice, s)
                                       : cudaMemsetAsync(state_out, 0, state_bytes, s);
        return e == cudaSuccess ? GRET_OK : GRET_ERR_CUDA;
    }
    if (!q || !k || !v || !g || !o) return GRET_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(o))
        return GRET_ERR_ALIGNMENT;
    if (!workspace || workspace_bytes < ew_workspace_bytes(B, N, H)) return GRET_ERR_WORKSPACE;
    if (!aligned16(workspace)) return GRET_ERR_ALIGNMENT;
    EwArgs a;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.k = static_cast<const __nv_bfloat16*>(k);
    a.v = static_cast<const __nv_bfloat16*>(v);
    a.g = g; a.tau = tau; a.k_scale = k_scale;
    a.B = B; a.N = N; a.H = H;
    a.state_in = state_in; a.state_out = state_out;
    a.o = static_cast<__nv_bfloat16*>(o);
    a.workspace = workspace;
    const cudaError_t e = launch_prefill_ew(a, s);
    if (e == cudaErrorInvalidValue) return GRET_ERR_UNSUPPORTED;   // a tensor map was refused
    return e == cudaSuccess ? GRET_OK : GRET_ERR_CUDA;
}

// Workspace of gret_layer_forward: the prefill's workspace first (its status word at byte 0),
// then q, k, v, o (bf16 [T, H, d]) and g (fp32 [T, H]), each 256-byte aligned.
struct LayerWs {
    size_t prefill, q, k, v, o, g, total;
};

LayerWs layer_ws(int64_t T, int n_seqs, int H, int d) {
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    LayerWs l = {};
    l.prefill = gret_prefill_workspace_size(GRET_BF16, T, n_seqs, H, d, d, 0);
    if (l.prefill == 0) return l;
    const size_t act = (size_t)T * H * d * 2;
    l.q = up(l.prefill);
    l.k = l.q + up(act);
    l.v = l.k + up(act);
    l.o = l.v + up(act);
    l.g = l.o + up(act);
    l.total = l.g + up((size_t)T * H * 4);
    return l;
}

size_t gret_layer_workspace_size(int64_t T, int n_seqs, int H, int d) {
    if (T < 0 || n_seqs < 1 || H < 1 || d != 128) return 0;
    return layer_ws(T, n_seqs, H, d).total;
}

gret_status_t gret_layer_forward(const void* x, const void* w_qkvg, int64_t ldw, const void* w_g,
                                 const float* gn_weight, const float* gn_bias, float eps,
                                 float tau, float k_scale, int64_t T, int H, int d, int D,
                                 const int32_t* cu_seqlens, int n_seqs, const float* state_in,
                                 float* state_out, void* y, void* workspace,
                                 size_t workspace_bytes, gret_stream_t stream) {
    const NvtxRange range("gret_layer_forward");
    if (T < 0 || H < 1 || d < 1 || D < 1 || n_seqs < 1) return GRET_ERR_INVALID_ARG;
    if (!cu_seqlens && n_seqs != 1) return GRET_ERR_INVALID_ARG;
    if (d != 128) return GRET_ERR_UNSUPPORTED;
    // the three steps' requirements, checked before anything is launched, so that a call that
    // one step would refuse has no effect on the device
    if (!(eps >= 0.f) || !isfinite(eps) || !(tau > 0.f) || !isfinite(tau) || !isfinite(k_scale))
        return GRET_ERR_INVALID_ARG;
    if (ldw < 3 * (int64_t)H * d + H) return GRET_ERR_INVALID_ARG;
    if (H > 128 || D % 64 != 0 || (H * d) % 256 != 0) return GRET_ERR_UNSUPPORTED;
    if (T > ((int64_t)1 << 31) - 256) return GRET_ERR_UNSUPPORTED;
    const LayerWs l = layer_ws(T, n_seqs, H, d);
    if (l.total == 0) return GRET_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < l.total) return GRET_ERR_WORKSPACE;
    if (!aligned16(workspace)) return GRET_ERR_ALIGNMENT;
    if (T > 0) {
        if (!x || !w_qkvg || !w_g || !y) return GRET_ERR_INVALID_ARG;
        if (!aligned16(x) || !aligned16(w_qkvg) || !aligned16(w_g) || !aligned16(y) ||
            ldw % 8 != 0 || (state_in && !aligned16(state_in)) ||
            (state_out && !aligned16(state_out)))
            return GRET_ERR_ALIGNMENT;
    }
    if (T == 0) {   // no tokens: the final states are the entry states, y is empty
        if (!state_out || state_out == state_in) return GRET_OK;
        const size_t bytes = (size_t)n_seqs * H * d * d * sizeof(float);
        const cudaStream_t s = (cudaStream_t)stream;
        const cudaError_t e =
            state_in ? cudaMemcpyAsync(state_out, state_in, bytes, cudaMemcpyDeviceToDevice, s)
                     : cudaMemsetAsync(state_out, 0, bytes, s);
        return e == cudaSuccess ? GRET_OK : GRET_ERR_CUDA;
    }
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    void* q = ws + l.q;
    void* k = ws + l.k;
    void* v = ws + l.v;
    void* o = ws + l.o;
    float* g = reinterpret_cast<float*>(ws + l.g);
    gret_status_t st = gret_qkvg_projection(x, w_qkvg, ldw, T, H, d, D, q, k, v, g, stream);
    if (st != GRET_OK) return st;
    const int64_t td = (int64_t)H * d;   // token stride of q, k, v, o
    st = gret_prefill_chunkwise(q, k, 0, td, d, v, 0, td, d, g, tau, k_scale, GRET_BF16, 1, T, H,
                                d, d, cu_seqlens, cu_seqlens ? n_seqs : 0, state_in, state_out, o,
                                0, td, d, 0, ws, l.prefill, stream);
    if (st != GRET_OK) return st;
    return gret_groupnorm_gate(o, x, w_g, gn_weight, gn_bias, eps, T, H, d, D, y, stream);
}

gret_status_t gret_swa_prefill(const void* q, const void* k, const void* v, float scale,
                               int window, int B, int64_t N, int H, int d, void* o,
                               gret_stream_t stream) {
    const NvtxRange range("gret_swa_prefill");
    if (B < 0 || N < 0 || H < 1 || d < 1 || window < 1 || !isfinite(scale))
        return GRET_ERR_INVALID_ARG;
    if (d != SWA_DIM) return GRET_ERR_UNSUPPORTED;
    if (B > 65535 || H > 65535 || (N + 63) / 64 > 0x7fffffff) return GRET_ERR_UNSUPPORTED;
    if (B == 0 || N == 0) return GRET_OK;
    if (!q || !k || !v || !o) return GRET_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return GRET_ERR_ALIGNMENT;
    SwaArgs a;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.k = static_cast<const __nv_bfloat16*>(k);
    a.v = static_cast<const __nv_bfloat16*>(v);
    a.o = static_cast<__nv_bfloat16*>(o);
    a.scale = scale; a.window = window;
    a.B = B; a.N = N; a.H = H;
    return launch_swa(a, (cudaStream_t)stream) == cudaSuccess ? GRET_OK : GRET_ERR_CUDA;
}

}  // extern "C"

extern "C" gret_status_t gret_swa_decode_step(const void* q, const void* k, const void* v,
                                              float scale, int window, int B, int H, int d,
                                              const int32_t* pos, void* k_cache, void* v_cache,
                                              void* o, gret_stream_t stream) {
    const NvtxRange range("gret_swa_decode_step");
    if (B < 0 || H < 1 || d < 1 || window < 1 || !isfinite(scale)) return GRET_ERR_INVALID_ARG;
    if (d != SWA_DIM || window > SWA_DECODE_MAX_WINDOW) return GRET_ERR_UNSUPPORTED;
    if ((int64_t)B * H > 0x7fffffffLL) return GRET_ERR_UNSUPPORTED;
    if (B == 0) return GRET_OK;
    if (!q || !k || !v || !pos || !k_cache || !v_cache || !o) return GRET_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(k_cache) ||
        !aligned16(v_cache) || (reinterpret_cast<uintptr_t>(pos) & 3u) != 0)
        return GRET_ERR_ALIGNMENT;
    SwaDecodeArgs a;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.k = static_cast<const __nv_bfloat16*>(k);
    a.v = static_cast<const __nv_bfloat16*>(v);
    a.scale = scale; a.window = window; a.B = B; a.H = H; a.pos = pos;
    a.k_cache = static_cast<__nv_bfloat16*>(k_cache);
    a.v_cache = static_cast<__nv_bfloat16*>(v_cache);
    a.o = static_cast<__nv_bfloat16*>(o);
    const cudaError_t e = launch_swa_decode(a, (cudaStream_t)stream);
    if (e == cudaErrorInvalidValue) return GRET_ERR_UNSUPPORTED;
    return e == cudaSuccess ? GRET_OK : GRET_ERR_CUDA;
}
