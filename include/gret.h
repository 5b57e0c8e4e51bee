/*
 * gret.h -- C ABI of the gated-retention (gRet) library for NVIDIA B200 (sm_100a).
 *
 * Gated retention is the Self-Decoder mixer of YOCO.  Definitions follow the page
 * "YOCO 完全拆解：Decoder-Decoder 架构如何让 KV Cache 只存一次" (pinghaoyang.com.cn/aigc/posts/yoco/):
 *   section "路线二：Multi-Head Gated Retention"         -- gate, recurrence, GroupNorm + swish gate
 *   section "Prefill 与 Decode 为什么使用两种计算形态"   -- chunkwise prefill form
 *   section "单 token Decode 的实现骨架"                  -- the decode state update
 *
 * Per sequence and head, with row vectors q_t, k_t [1 x d_k], v_t [1 x d_v] and state S [d_k x d_v]:
 *   log(gamma_t) = logsigmoid(g_t) / tau          (gamma = sigmoid(g)^(1/tau); g is the gate logit)
 *   S_t = gamma_t S_{t-1} + (k_scale k_t)^T v_t   (decay the old state, then add the current token)
 *   o_t = q_t S_t                                 (the output reads the updated state)
 *
 * Conventions shared by every entry point
 *   - All data pointers are DEVICE pointers owned by the caller.  The library keeps no pointer
 *     after a call returns and allocates no device memory.
 *   - Every call is asynchronous on `stream` (0 = legacy default stream).
 *   - Argument errors are detected on the host and returned before anything is launched.
 *     A launch failure returns GRET_ERR_CUDA.  Faults of earlier asynchronous work surface on a
 *     later call or on stream synchronisation, as usual in CUDA.
 *   - Strides are in ELEMENTS; the last dimension of every tensor is contiguous.
 *   - Gate logits must be finite (|g| <= 1e30 is fine; +-inf and NaN give undefined results).
 *   - State tensors are fp32, [units, H, d_k, d_v], row-major (d_v contiguous).
 */
#ifndef GRET_H
#define GRET_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* gret_stream_t; /* same handle as cudaStream_t */

typedef enum {
    GRET_OK = 0,
    GRET_ERR_INVALID_ARG = 1,  /* a size, pointer or stride is out of the documented range   */
    GRET_ERR_UNSUPPORTED = 2,  /* a valid combination this build has no kernel for          */
    GRET_ERR_ALIGNMENT = 3,    /* a pointer or stride breaks the 16-byte alignment rule      */
    GRET_ERR_WORKSPACE = 4,    /* workspace NULL or smaller than gret_prefill_workspace_size */
    GRET_ERR_CUDA = 5,         /* a CUDA runtime call failed (launch or attribute setup)     */
    GRET_ERR_TIMEOUT = 6       /* a bounded inter-block wait gave up; results are invalid    */
} gret_status_t;

typedef enum { GRET_F32 = 0, GRET_BF16 = 1 } gret_dtype_t;

/* Static string naming a status code.  Never NULL. */
const char* gret_status_string(gret_status_t status);

/*
 * Bytes of device workspace gret_prefill_chunkwise needs for these sizes (0 is a valid answer
 * only when nothing is launched).  `total_tokens` is B*N in dense mode and the packed token
 * count in varlen mode; `n_seqs` is B in dense mode.  `chunk` as passed to the prefill call.
 * Returns 0 and sets nothing on invalid sizes; callers pass the result through unchanged.
 */
size_t gret_prefill_workspace_size(gret_dtype_t dtype, int64_t total_tokens, int n_seqs, int H,
                                   int d_k, int d_v, int chunk);

/*
 * Chunkwise prefill ("Prefill 与 Decode 为什么使用两种计算形态").  Tokens are cut into chunks of
 * `chunk` positions that never straddle a sequence; within a chunk [a, b], with the in-chunk
 * cumulative log-decay c_t = sum_{k=a..t} log(gamma_k) and the entry state S_{a-1}:
 *   o_t = sum_{m=a..t} exp(c_t - c_m) (q_t . k_m) v_m  +  exp(c_t) q_t S_{a-1}
 *   S_b = exp(c_b) S_{a-1} + sum_{m=a..b} exp(c_b - c_m) k_m^T v_m
 * which equals the recurrence above up to rounding.  The last chunk of a sequence may be
 * shorter; nothing needs padding.
 *
 *   q, k     [.., token, head, d_k] in `dtype`, sharing strides; element (b, t, h, i) at
 *            b*stride_batch + t*stride_tok + h*stride_head + i.  Read only.
 *   v        [.., token, head, d_v] in `dtype` with its own strides (v_stride_batch,
 *            v_stride_tok, v_stride_head).  Read only.
 *   g        fp32 gate logits, contiguous [B, N, H] (dense) or [total_tokens, H] (varlen).
 *   tau      temperature (> 0); k_scale multiplies every key (e.g. d_k^-1/2, or 1.0).
 *   dtype    GRET_BF16 (tensor-core path when d_k == d_v == 128, else a CUDA-core path with
 *            fp32 accumulation) or GRET_F32 (CUDA-core path, full fp32 arithmetic).
 *   B, N     dense mode: B sequences of N tokens each.
 *   cu_seqlens  NULL for dense mode.  Varlen mode: device int32 [n_seqs + 1], non-decreasing,
 *            cu_seqlens[0] == 0, cu_seqlens[n_seqs] == N; requires B == 1, tokens packed.
 *            Empty sequences are allowed (their state passes through).
 *   H, d_k, d_v  heads and head widths; d_k, d_v in {64, 128}.
 *   state_in   fp32 [units, H, d_k, d_v] entry states, units = B (dense) or n_seqs (varlen);
 *              NULL means zero.  Read only.
 *   state_out  fp32, same shape; the state after each sequence's last token.  NULL skips it.
 *              May alias state_in exactly (then it is read before it is overwritten).
 *   o        output, same dtype as q, [.., token, head, d_v] with its own strides
 *            (o_stride_batch, o_stride_tok, o_stride_head).  Must not overlap the inputs.
 *   chunk    0 picks the tuned default; otherwise 16, 32 or 64 (CUDA-core path) or 128
 *            (tensor-core path).  Other values return GRET_ERR_UNSUPPORTED.
 *   workspace  device scratch of at least gret_prefill_workspace_size() bytes, 256-byte
 *            aligned, owned by the caller; its contents need no initialisation and are
 *            garbage afterwards.  Concurrent calls need separate workspaces.
 * Alignment: for the tensor-core path, q/k/v/o base pointers must be 16-byte aligned and every
 * stride (times 2 bytes) a multiple of 16 bytes; otherwise GRET_ERR_ALIGNMENT.  Its tile
 * copies take 32-bit token coordinates: N (tokens per sequence, or the packed total) above
 * 2^31 - 256 returns GRET_ERR_UNSUPPORTED.
 * A bounded wait between thread blocks that gives up sets an error word in the workspace;
 * read it with gret_workspace_status() after the stream has synchronised.
 */
gret_status_t gret_prefill_chunkwise(
    const void* q, const void* k, int64_t stride_batch, int64_t stride_tok, int64_t stride_head,
    const void* v, int64_t v_stride_batch, int64_t v_stride_tok, int64_t v_stride_head,
    const float* g, float tau, float k_scale, gret_dtype_t dtype, int B,
    int64_t N, int H, int d_k, int d_v, const int32_t* cu_seqlens, int n_seqs,
    const float* state_in, float* state_out, void* o, int64_t o_stride_batch,
    int64_t o_stride_tok, int64_t o_stride_head, int chunk, void* workspace,
    size_t workspace_bytes, gret_stream_t stream);

/*
 * gret_prefill_chunkwise with two settings that exist only to test its failure path; production
 * callers use gret_prefill_chunkwise.  The paper has no counterpart.
 *   wait_ns       limit of every bounded wait of the tensor-core kernel, in ns (the regular entry
 *                 point uses 2 s); 1 .. 2e9, else GRET_ERR_INVALID_ARG.
 *   first_ticket  the first span ticket handed out (0 as in the regular call).  A value past span
 *                 0 of a chain leaves that span's look-back flag unset, so the waits of the later
 *                 spans of the chain give up after wait_ns: the call then records
 *                 GRET_ERR_TIMEOUT for gret_workspace_status, the kernel stops, and its outputs
 *                 are invalid.  The CUDA context stays usable.
 * Other arguments, results and errors as gret_prefill_chunkwise.
 */
gret_status_t gret_prefill_chunkwise_testing(
    const void* q, const void* k, int64_t stride_batch, int64_t stride_tok, int64_t stride_head,
    const void* v, int64_t v_stride_batch, int64_t v_stride_tok, int64_t v_stride_head,
    const float* g, float tau, float k_scale, gret_dtype_t dtype, int B,
    int64_t N, int H, int d_k, int d_v, const int32_t* cu_seqlens, int n_seqs,
    const float* state_in, float* state_out, void* o, int64_t o_stride_batch,
    int64_t o_stride_tok, int64_t o_stride_head, int chunk, void* workspace,
    size_t workspace_bytes, gret_stream_t stream, uint64_t wait_ns, uint32_t first_ticket);

/*
 * gret_prefill_chunkwise without a workspace argument and without allocating.  The paper has no
 * counterpart: this entry point exists for callers that cannot allocate device memory when they
 * call, for example a serving process that gives all device memory to its own pool at start-up,
 * or a latency-critical loop in which a cudaMalloc would synchronize the device.
 *   - Arguments, results and errors are those of gret_prefill_chunkwise, minus the workspace.
 *   - Its scratch is one static device array of 8 MiB inside this library, present on every GPU
 *     that loads the library until the process exits.  A call whose workspace need
 *     (gret_prefill_workspace_size) exceeds 8 MiB returns GRET_ERR_WORKSPACE before doing
 *     anything; with d_k = d_v = 128 and bf16 that allows about 63 (sequence, head) chains.
 *   - The first call on a device looks up the scratch's device address (once per device); make
 *     that first call before any stream capture.
 *   - Every call shares the one scratch array: calls that overlap on the GPU (other streams, or
 *     other host threads using the same device) race and give wrong results.  The call clears
 *     what must start at zero itself; the array keeps the previous call's contents otherwise.
 *   - A bounded wait that gives up records GRET_ERR_TIMEOUT in the scratch, where
 *     gret_prefill_noalloc_status() reads it.  Each call clears the word first, so the status
 *     describes the latest call on the device.
 *   - The scratch's device address is kept for the life of the process: calling
 *     cudaDeviceReset after this entry point has run on a device is not supported.
 */
gret_status_t gret_prefill_chunkwise_noalloc(
    const void* q, const void* k, int64_t stride_batch, int64_t stride_tok, int64_t stride_head,
    const void* v, int64_t v_stride_batch, int64_t v_stride_tok, int64_t v_stride_head,
    const float* g, float tau, float k_scale, gret_dtype_t dtype, int B,
    int64_t N, int H, int d_k, int d_v, const int32_t* cu_seqlens, int n_seqs,
    const float* state_in, float* state_out, void* o, int64_t o_stride_batch,
    int64_t o_stride_tok, int64_t o_stride_head, int chunk, gret_stream_t stream);

/*
 * Status of the latest gret_prefill_chunkwise_noalloc call on the current device: synchronises
 * `stream` (use the stream that call ran on), then reads the error word of the library's static
 * scratch.  Returns GRET_OK (also when no call has used the scratch yet), GRET_ERR_TIMEOUT if a
 * bounded wait of that call gave up (its results are invalid), or GRET_ERR_CUDA.  Blocking; not
 * for use inside stream capture.  Allocates nothing.  The paper has no counterpart.
 */
gret_status_t gret_prefill_noalloc_status(gret_stream_t stream);

/*
 * Synchronises `stream`, then reads the error word that gret_prefill_chunkwise keeps at the
 * start of `workspace`.  Returns GRET_OK, GRET_ERR_TIMEOUT, or GRET_ERR_CUDA if the copy or the
 * synchronisation failed.  Blocking; not for use inside stream capture.
 */
gret_status_t gret_workspace_status(const void* workspace, gret_stream_t stream);

/*
 * One recurrent decode step for a batch ("单 token Decode 的实现骨架"): for every (b, h)
 *   S <- gamma S + (k_scale k)^T v ;  o = q S
 *   q, k   [B, H, d_k] contiguous, `dtype`;   v [B, H, d_v];   g fp32 [B, H] gate logits.
 *   state  fp32 [B, H, d_k, d_v], updated IN PLACE; 16-byte aligned.
 *   o      [B, H, d_v] in `dtype`; must not overlap state or inputs.
 * d_k, d_v in {64, 128}; B * H at most 2^30 - 1 (GRET_ERR_INVALID_ARG beyond).  Memory-bound:
 * the state is read and written once.
 */
gret_status_t gret_decode_step(const void* q, const void* k, const void* v, const float* g,
                               float tau, float k_scale, gret_dtype_t dtype, int B, int H,
                               int d_k, int d_v, float* state, void* o, gret_stream_t stream);

/*
 * Output epilogue ("路线二：Multi-Head Gated Retention"): per-head GroupNorm of the retention
 * output times swish(X W_G):
 *   z = X_t W_G ;  y_t[h*d_v + j] = GN_h(o_t)[j] * z[h*d_v + j] * sigmoid(z[h*d_v + j])
 *   GN_h: mean and biased variance of o_t[h*d_v .. h*d_v + d_v - 1], (x - mean)/sqrt(var + eps),
 *         then * gn_weight + gn_bias per channel (each may be NULL = identity).
 *   o    bf16 [T, H*d_v] row-major;  x bf16 [T, D] row-major;  w_g bf16 [D, H*d_v] row-major.
 *   gn_weight, gn_bias  fp32 [H*d_v] or NULL.      y  bf16 [T, H*d_v], must not overlap inputs.
 * Requires d_v == 128, D a positive multiple of 64, T >= 0; pointers 16-byte aligned.
 */
gret_status_t gret_groupnorm_gate(const void* o, const void* x, const void* w_g,
                                  const float* gn_weight, const float* gn_bias, float eps,
                                  int64_t T, int H, int d_v, int D, void* y,
                                  gret_stream_t stream);

/*
 * The layer's input projection in one GEMM ("路线二：Multi-Head Gated Retention": the per-head
 * gate comes from a learned projection of the layer input, next to the query, key and value
 * projections):
 *   [q | k | v | g]_t = X_t W_qkvg ,  W_qkvg = [W_Q | W_K | W_V | W_gamma]
 *   x    bf16 [T, D] row-major.
 *   w    bf16 [D, F] with F = 3 H d + H columns (H d each for W_Q, W_K, W_V, then H for
 *        W_gamma), row stride ldw >= F elements (a multiple of 8: rows start 16-byte aligned).
 *   q, k, v  bf16 [T, H, d] (token-major, contiguous), ready for gret_prefill_chunkwise.
 *   g    fp32 [T, H] gate logits (gamma = sigmoid(g)^(1/tau) is taken by the prefill).
 * fp32 accumulation; q, k, v rounded to bf16 once.  Requires d == 128, 1 <= H <= 128, D a
 * positive multiple of 64; x, w, q, k, v 16-byte aligned, g 4-byte aligned
 * (GRET_ERR_ALIGNMENT otherwise).  Outputs must not overlap the inputs or each other.
 */
gret_status_t gret_qkvg_projection(const void* x, const void* w, int64_t ldw, int64_t T, int H,
                                   int d, int D, void* q, void* k, void* v, float* g,
                                   gret_stream_t stream);

/*
 * One gated-retention mixer layer in one call: the input projection (gret_qkvg_projection), the
 * chunkwise prefill (gret_prefill_chunkwise, tensor-core path) and the per-head GroupNorm and
 * swish output gate (gret_groupnorm_gate), chained on one stream in the order the page
 * "路线二：Multi-Head Gated Retention" draws the mixer:
 *   [q | k | v | g] = X W_qkvg,   o = gRet(q, k_scale k, v; gamma = sigmoid(g)^(1/tau)),
 *   y = GN_h(o) * swish(X W_G)
 *   x        bf16 [T, D] row-major; one packed batch of sequences.
 *   w_qkvg   bf16 [D, ldw] as in gret_qkvg_projection (3 H d + H used columns).
 *   w_g      bf16 [D, H d];  gn_weight, gn_bias fp32 [H d] or NULL;  eps > 0.
 *   cu_seqlens  int32 [n_seqs + 1] on the device (offsets into x), or NULL for one sequence
 *               (n_seqs must then be 1).
 *   state_in / state_out  fp32 [n_seqs, H, d, d] or NULL (zero entry state / no final state).
 *   y        bf16 [T, H d].
 *   workspace  at least gret_layer_workspace_size(T, n_seqs, H, d) bytes of device memory,
 *              16-byte aligned, owned by the caller; it holds the intermediates q, k, v, g and o
 *              and, at its start, the prefill's workspace (gret_workspace_status reads it).
 * Requires d == 128 and what the three calls require (H <= 128, D a multiple of 64, H d a
 * multiple of 256, 16-byte aligned pointers and ldw a multiple of 8).  These are all checked
 * before the first launch, so a refused call has no effect on the device.  y must not overlap
 * x or the workspace.
 */
gret_status_t gret_layer_forward(const void* x, const void* w_qkvg, int64_t ldw, const void* w_g,
                                 const float* gn_weight, const float* gn_bias, float eps,
                                 float tau, float k_scale, int64_t T, int H, int d, int D,
                                 const int32_t* cu_seqlens, int n_seqs, const float* state_in,
                                 float* state_out, void* y, void* workspace,
                                 size_t workspace_bytes, gret_stream_t stream);

/* Workspace bytes gret_layer_forward needs; 0 for invalid or unsupported sizes. */
size_t gret_layer_workspace_size(int64_t T, int n_seqs, int H, int d);

/*
 * Chunkwise prefill with one gate per key channel: the element-wise alternative that
 * "路线二：Multi-Head Gated Retention" weighs against the head-wise scalar gate (YOCO keeps the
 * head-wise one because it keeps every contraction a plain matrix product).  Per sequence and
 * head, with a gate logit per key channel i:
 *   alpha_t[i] = sigmoid(g_t[i])^(1/tau)
 *   S_t[i][:] = alpha_t[i] S_{t-1}[i][:] + (k_scale k_t[i]) v_t      (each state row decays
 *                                                                     at its channel's rate)
 *   o_t = q_t S_t
 * A gate shared by all channels of a head gives gret_prefill_chunkwise's result.
 *   q, k, v, o  bf16 [B, N, H, d] contiguous (token-major);  g  fp32 [B, N, H, d] contiguous.
 *   state_in    fp32 [B, H, d, d] or NULL (zero entry state);  state_out likewise, or NULL;
 *               state_out may alias state_in.
 *   workspace   device memory of at least gret_prefill_elementwise_workspace_size(B, N, H, d)
 *               bytes, 16-byte aligned, owned by the caller; its contents on entry do not
 *               matter and are overwritten.  Its first word is the status word that
 *               gret_workspace_status reads (GRET_ERR_TIMEOUT if a bounded wait gave up).
 * Runs on the tensor cores (three launches: per range of chunks the decayed sum of k^T v, a
 * scan over ranges, the outputs range by range) with each channel's decay folded into bf16
 * high/low operand pairs; chunks whose decay is too fast for that take their in-chunk scores
 * pairwise on CUDA cores.  Requires d == 128, B <= 65535, H <= 65535, N <= 2^31 - 256,
 * B * H * 16 < 2^31 and a workspace size below 9e18 bytes (GRET_ERR_UNSUPPORTED otherwise);
 * q, k, v, g, o and the states 16-byte aligned (GRET_ERR_ALIGNMENT otherwise).  N == 0 copies
 * state_in (or zeros) to state_out.  o must not overlap the inputs.
 */
gret_status_t gret_prefill_elementwise(const void* q, const void* k, const void* v,
                                       const float* g, float tau, float k_scale, int B,
                                       int64_t N, int H, int d, const float* state_in,
                                       float* state_out, void* o, void* workspace,
                                       size_t workspace_bytes, gret_stream_t stream);

/* Workspace bytes gret_prefill_elementwise needs: 256 + B * H * R * (d*d + d) * 4, with R the
 * ranges of chunks per sequence that the launch uses on the current device (a wave model over
 * its SM count: R = 6 at N = 32768, H = 24 on 148 SMs).  Query it on the device that runs the
 * call.  Returns 0 on invalid or unsupported sizes (d != 128 among them). */
size_t gret_prefill_elementwise_workspace_size(int B, int64_t N, int H, int d);

/*
 * Sliding-window attention prefill, the other Self-Decoder mixer ("路线一：滑动窗口注意力"):
 * position i attends to the most recent `window` positions of its sequence, itself included,
 * with softmax over exactly those:
 *   o_i = sum_{j = max(0, i-window+1) .. i} softmax_j(scale * q_i . k_j) v_j
 *   q, k, v, o  bf16 [B, N, H, d] contiguous (token-major); each batch row is one sequence.
 *   scale       score scale (d^-1/2 in the usual reading); window >= 1 (the page's 1024).
 * bf16 tensor-core products with fp32 accumulation and an fp32 online softmax; o rounded to
 * bf16 once.  Requires d == 128, B <= 65535, H <= 65535; q, k, v, o 16-byte aligned
 * (GRET_ERR_ALIGNMENT otherwise).  o must not overlap the inputs.
 */
gret_status_t gret_swa_prefill(const void* q, const void* k, const void* v, float scale,
                               int window, int B, int64_t N, int H, int d, void* o,
                               gret_stream_t stream);

/*
 * One decode step of sliding-window attention ("路线一：滑动窗口注意力": at decode time only the
 * most recent `window` positions' keys and values are kept).  Each (b, h) keeps a ring of
 * `window` cache slots, token t in slot t % window.  With t = pos[b], the index of the new token
 * in sequence b (0 for its first token):
 *   k_cache[b, h, t % window] = k[b, h] ;  v_cache[b, h, t % window] = v[b, h]
 *   o[b, h] = sum_{j = max(0, t-window+1) .. t} softmax_j(scale q . k_j) v_j
 * which is gret_swa_prefill's output at position t.  The slot written held token t - window,
 * which has just left the window.
 *   q, k, v, o   bf16 [B, H, d] contiguous.
 *   pos          device int32 [B], pos[b] >= 0; read only (the caller advances it).
 *   k_cache, v_cache  bf16 [B, H, window, d] contiguous, owned by the caller and updated in
 *                place; slots of tokens not yet seen are never read.
 * Requires d == 128 and window <= 32768 (GRET_ERR_UNSUPPORTED otherwise); pointers 16-byte
 * aligned, pos 4-byte aligned (GRET_ERR_ALIGNMENT).  fp32 scores and softmax; o rounded to bf16
 * once.  Memory-bound: the window's keys and values are read once.
 */
gret_status_t gret_swa_decode_step(const void* q, const void* k, const void* v, float scale,
                                   int window, int B, int H, int d, const int32_t* pos,
                                   void* k_cache, void* v_cache, void* o, gret_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GRET_H */
