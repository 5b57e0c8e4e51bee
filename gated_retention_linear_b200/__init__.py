"""gated_retention_linear_b200 -- gated retention (the YOCO Self-Decoder mixer) on B200.

A thin Python binding over the C ABI in include/gret.h (libgret.so, built in-tree by
`python gated_retention_linear_b200/build.py`).  The functions here only marshal arguments:
they read shapes and strides off torch tensors, allocate outputs and workspaces with torch, pass
raw device pointers and the current CUDA stream, and raise on a non-OK status.  Every step of
the computation runs in the library's CUDA kernels; there is no fallback.  If libgret.so is
missing this import fails.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgret.so")

if not os.path.exists(LIB_PATH):
    raise ImportError("libgret.so not found at %s; build it with "
                      "`python gated_retention_linear_b200/build.py`" % LIB_PATH)

_lib = ctypes.CDLL(LIB_PATH)

GRET_F32, GRET_BF16 = 0, 1
STATUS = {0: "GRET_OK", 1: "GRET_ERR_INVALID_ARG", 2: "GRET_ERR_UNSUPPORTED",
          3: "GRET_ERR_ALIGNMENT", 4: "GRET_ERR_WORKSPACE", 5: "GRET_ERR_CUDA",
          6: "GRET_ERR_TIMEOUT"}

_vp, _i64, _i32, _f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float

_lib.gret_status_string.argtypes = [_i32]
_lib.gret_status_string.restype = ctypes.c_char_p
_lib.gret_prefill_workspace_size.argtypes = [_i32, _i64, _i32, _i32, _i32, _i32, _i32]
_lib.gret_prefill_workspace_size.restype = ctypes.c_size_t
_lib.gret_prefill_chunkwise.argtypes = [_vp, _vp, _i64, _i64, _i64, _vp, _i64, _i64, _i64, _vp,
                                        _f32, _f32, _i32,
                                        _i32, _i64, _i32, _i32, _i32, _vp, _i32, _vp, _vp, _vp,
                                        _i64, _i64, _i64, _i32, _vp, ctypes.c_size_t, _vp]
_lib.gret_prefill_chunkwise.restype = _i32
_lib.gret_prefill_chunkwise_noalloc.argtypes = [_vp, _vp, _i64, _i64, _i64, _vp, _i64, _i64, _i64,
                                                _vp, _f32, _f32, _i32, _i32, _i64, _i32, _i32,
                                                _i32, _vp, _i32, _vp, _vp, _vp, _i64, _i64, _i64,
                                                _i32, _vp]
_lib.gret_prefill_chunkwise_noalloc.restype = _i32
_lib.gret_prefill_chunkwise_testing.argtypes = _lib.gret_prefill_chunkwise.argtypes + [
    ctypes.c_uint64, ctypes.c_uint32]
_lib.gret_prefill_chunkwise_testing.restype = _i32
_lib.gret_prefill_noalloc_status.argtypes = [_vp]
_lib.gret_prefill_noalloc_status.restype = _i32
_lib.gret_workspace_status.argtypes = [_vp, _vp]
_lib.gret_workspace_status.restype = _i32
_lib.gret_decode_step.argtypes = [_vp, _vp, _vp, _vp, _f32, _f32, _i32, _i32, _i32, _i32, _i32,
                                  _vp, _vp, _vp]
_lib.gret_decode_step.restype = _i32
_lib.gret_groupnorm_gate.argtypes = [_vp, _vp, _vp, _vp, _vp, _f32, _i64, _i32, _i32, _i32, _vp,
                                     _vp]
_lib.gret_groupnorm_gate.restype = _i32
_lib.gret_qkvg_projection.argtypes = [_vp, _vp, _i64, _i64, _i32, _i32, _i32, _vp, _vp, _vp, _vp,
                                      _vp]
_lib.gret_qkvg_projection.restype = _i32
_lib.gret_prefill_elementwise.argtypes = [_vp, _vp, _vp, _vp, _f32, _f32, _i32, _i64, _i32, _i32,
                                          _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
_lib.gret_prefill_elementwise.restype = _i32
_lib.gret_prefill_elementwise_workspace_size.argtypes = [_i32, _i64, _i32, _i32]
_lib.gret_prefill_elementwise_workspace_size.restype = ctypes.c_size_t
_lib.gret_layer_forward.argtypes = [_vp, _vp, _i64, _vp, _vp, _vp, _f32, _f32, _f32, _i64, _i32,
                                    _i32, _i32, _vp, _i32, _vp, _vp, _vp, _vp, ctypes.c_size_t,
                                    _vp]
_lib.gret_layer_forward.restype = _i32
_lib.gret_layer_workspace_size.argtypes = [_i64, _i32, _i32, _i32]
_lib.gret_layer_workspace_size.restype = ctypes.c_size_t
_lib.gret_swa_prefill.argtypes = [_vp, _vp, _vp, _f32, _i32, _i32, _i64, _i32, _i32, _vp, _vp]
_lib.gret_swa_prefill.restype = _i32
_lib.gret_swa_decode_step.argtypes = [_vp, _vp, _vp, _f32, _i32, _i32, _i32, _i32, _vp, _vp, _vp,
                                      _vp, _vp]
_lib.gret_swa_decode_step.restype = _i32


class GretError(RuntimeError):
    def __init__(self, fn, code):
        self.code = code
        super().__init__("%s failed: %s" % (fn, _lib.gret_status_string(code).decode()))


def _check(fn, code):
    if code != 0:
        raise GretError(fn, code)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return GRET_BF16
    if t.dtype == torch.float32:
        return GRET_F32
    raise TypeError("q/k/v must be bfloat16 or float32, got %s" % t.dtype)


def gret_status_string(code):
    return _lib.gret_status_string(int(code)).decode()


def gret_prefill_workspace_size(dtype, total_tokens, n_seqs, H, d_k, d_v, chunk=0):
    code = dtype if isinstance(dtype, int) else _dtype_code(torch.empty(0, dtype=dtype))
    return int(_lib.gret_prefill_workspace_size(code, total_tokens, n_seqs, H, d_k, d_v, chunk))


def _layout(t, head_major):
    """(stride_batch, stride_tok, stride_head) of a 4-D [B,N,H,d] or [B,H,N,d] tensor, or of a
    3-D packed [T,H,d] tensor (stride_batch = 0)."""
    if t.stride(-1) != 1:
        raise ValueError("last dimension must be contiguous")
    if t.dim() == 3:
        return 0, t.stride(0), t.stride(1)
    if head_major:
        return t.stride(0), t.stride(2), t.stride(1)
    return t.stride(0), t.stride(1), t.stride(2)


def _prefill_args(q, k, v, g, cu_seqlens, state_out, o, head_major):
    """Shapes, strides and checks shared by both prefill wrappers.  Returns a dict of the C
    arguments (sizes and strides) plus the (possibly allocated) o and state_out."""
    if k.stride() != q.stride():
        raise ValueError("q and k must share strides")
    if q.dim() == 3:
        B, (N, H, dk) = 1, q.shape
    elif head_major:
        B, H, N, dk = q.shape
    else:
        B, N, H, dk = q.shape
    dv = v.shape[-1]
    sb, st, sh = _layout(q, head_major)
    vsb, vst, vsh = _layout(v, head_major)
    if o is None:
        o = torch.empty(q.shape[:-1] + (dv,), dtype=q.dtype, device=q.device)
    osb, ost, osh = _layout(o, head_major)
    if not g.is_contiguous() or g.dtype != torch.float32:
        raise ValueError("g must be contiguous fp32")
    n_seqs = 0
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1:
            raise ValueError("cu_seqlens must be 1-D int32")
        n_seqs = cu_seqlens.numel() - 1
    units = n_seqs if cu_seqlens is not None else B
    if state_out is True:
        state_out = torch.empty((units, H, dk, dv), dtype=torch.float32, device=q.device)
    return dict(B=B, N=N, H=H, dk=dk, dv=dv, sb=sb, st=st, sh=sh, vsb=vsb, vst=vst, vsh=vsh,
                osb=osb, ost=ost, osh=osh, n_seqs=n_seqs, units=units, code=_dtype_code(q),
                total=N if cu_seqlens is not None else B * N, o=o, state_out=state_out)


def gret_prefill_chunkwise(q, k, v, g, tau=16.0, k_scale=1.0, cu_seqlens=None, state_in=None,
                           state_out=None, o=None, chunk=0, head_major=False, workspace=None,
                           stream=None):
    """Chunkwise gated-retention prefill through the C ABI.

    q, k [B,N,H,dk] (head_major=False) or [B,H,N,dk] (head_major=True); v likewise with dv;
    packed varlen: q, k, v [T,H,d] with cu_seqlens int32 [n_seqs+1] on the device.
    g fp32 [B,N,H] or [T,H].  state_in / state_out fp32 [units,H,dk,dv] (state_out=True
    allocates one).  Returns (o, state_out)."""
    a = _prefill_args(q, k, v, g, cu_seqlens, state_out, o, head_major)
    o, state_out = a["o"], a["state_out"]
    need = int(_lib.gret_prefill_workspace_size(a["code"], a["total"], a["units"], a["H"],
                                                a["dk"], a["dv"], chunk))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("gret_prefill_chunkwise", _lib.gret_prefill_chunkwise(
        _ptr(q), _ptr(k), a["sb"], a["st"], a["sh"], _ptr(v), a["vsb"], a["vst"], a["vsh"],
        _ptr(g), tau, k_scale, a["code"], a["B"], a["N"], a["H"], a["dk"], a["dv"],
        _ptr(cu_seqlens), a["n_seqs"], _ptr(state_in), _ptr(state_out), _ptr(o), a["osb"],
        a["ost"], a["osh"], chunk, _ptr(workspace), wbytes, _stream(stream)))
    return o, state_out


def gret_prefill_chunkwise_testing(q, k, v, g, wait_ns, first_ticket, tau=16.0, k_scale=1.0,
                                   cu_seqlens=None, state_in=None, state_out=None, o=None,
                                   workspace=None, stream=None):
    """gret_prefill_chunkwise with the failure-path settings of the C entry point of the same
    name: every bounded wait gives up after wait_ns, and span tickets start at first_ticket.
    For tests of the timeout path only.  Returns (o, state_out, workspace)."""
    a = _prefill_args(q, k, v, g, cu_seqlens, state_out, o, False)
    o, state_out = a["o"], a["state_out"]
    need = int(_lib.gret_prefill_workspace_size(a["code"], a["total"], a["units"], a["H"],
                                                a["dk"], a["dv"], 0))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _check("gret_prefill_chunkwise_testing", _lib.gret_prefill_chunkwise_testing(
        _ptr(q), _ptr(k), a["sb"], a["st"], a["sh"], _ptr(v), a["vsb"], a["vst"], a["vsh"],
        _ptr(g), tau, k_scale, a["code"], a["B"], a["N"], a["H"], a["dk"], a["dv"],
        _ptr(cu_seqlens), a["n_seqs"], _ptr(state_in), _ptr(state_out), _ptr(o), a["osb"],
        a["ost"], a["osh"], 0, _ptr(workspace), workspace.numel(), _stream(stream),
        int(wait_ns), int(first_ticket)))
    return o, state_out, workspace


def gret_prefill_chunkwise_noalloc(q, k, v, g, tau=16.0, k_scale=1.0, cu_seqlens=None,
                                   state_in=None, state_out=None, o=None, chunk=0,
                                   head_major=False, stream=None):
    """gret_prefill_chunkwise through the entry point that needs no workspace and allocates no
    device memory (its scratch is a fixed 8 MiB array inside the library; calls that overlap
    on the GPU race).  Same arguments, checks and results as gret_prefill_chunkwise; `o` and
    `state_out=True` are allocated here by torch for convenience, so pass them in to allocate
    nothing at call time.  gret_prefill_noalloc_status() reports a timed-out wait."""
    a = _prefill_args(q, k, v, g, cu_seqlens, state_out, o, head_major)
    o, state_out = a["o"], a["state_out"]
    _check("gret_prefill_chunkwise_noalloc", _lib.gret_prefill_chunkwise_noalloc(
        _ptr(q), _ptr(k), a["sb"], a["st"], a["sh"], _ptr(v), a["vsb"], a["vst"], a["vsh"],
        _ptr(g), tau, k_scale, a["code"], a["B"], a["N"], a["H"], a["dk"], a["dv"],
        _ptr(cu_seqlens), a["n_seqs"], _ptr(state_in), _ptr(state_out), _ptr(o), a["osb"],
        a["ost"], a["osh"], chunk, _stream(stream)))
    return o, state_out


def gret_prefill_noalloc_status(stream=None):
    """Synchronise and return the status of the latest allocation-free prefill on the current
    device (0 = OK, 6 = a bounded wait gave up)."""
    return int(_lib.gret_prefill_noalloc_status(_stream(stream)))


def gret_workspace_status(workspace, stream=None):
    """Synchronise and return the status word of a prefill workspace (0 = OK)."""
    return int(_lib.gret_workspace_status(_ptr(workspace), _stream(stream)))


def gret_decode_step(q, k, v, g, state, tau=16.0, k_scale=1.0, o=None, stream=None):
    """One decode step: q, k [B,H,dk], v [B,H,dv], g fp32 [B,H], state fp32 [B,H,dk,dv]
    updated in place.  Returns o [B,H,dv]."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    for t in (q, k, v, g, state):
        if not t.is_contiguous():
            raise ValueError("decode tensors must be contiguous")
    if o is None:
        o = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    _check("gret_decode_step", _lib.gret_decode_step(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), tau, k_scale, _dtype_code(q), B, H, dk, dv,
        _ptr(state), _ptr(o), _stream(stream)))
    return o


def gret_groupnorm_gate(o, x, w_g, H, gn_weight=None, gn_bias=None, eps=1e-5, y=None,
                        stream=None):
    """y = GroupNorm_per_head(o) * swish(x @ w_g); o [T,H*dv], x [T,D], w_g [D,H*dv], bf16."""
    T, F = o.shape
    D = x.shape[1]
    for t in (o, x, w_g):
        if not t.is_contiguous() or t.dtype != torch.bfloat16:
            raise ValueError("o, x, w_g must be contiguous bf16")
    if y is None:
        y = torch.empty((T, F), dtype=torch.bfloat16, device=o.device)
    _check("gret_groupnorm_gate", _lib.gret_groupnorm_gate(
        _ptr(o), _ptr(x), _ptr(w_g), _ptr(gn_weight), _ptr(gn_bias), eps, T, H, F // H, D,
        _ptr(y), _stream(stream)))
    return y


def gret_qkvg_projection(x, w, H, d=128, out=None, stream=None):
    """[q | k | v | g] = x @ w in one GEMM: x [T, D] bf16, w [D, >= 3*H*d + H] bf16 (W_Q, W_K,
    W_V, W_gamma side by side; extra columns, if any, are padding).  Returns q, k, v bf16
    [T, H, d] and the gate logits g fp32 [T, H], written into `out` = (q, k, v, g) when given
    (contiguous tensors of those shapes and types)."""
    T, D = x.shape
    for t in (x, w):
        if t.dtype != torch.bfloat16 or t.stride(-1) != 1:
            raise ValueError("x and w must be bfloat16 with contiguous rows")
    if x.stride(0) != D:
        raise ValueError("x must be contiguous")
    if out is None:
        q = torch.empty((T, H, d), dtype=torch.bfloat16, device=x.device)
        k = torch.empty_like(q)
        v = torch.empty_like(q)
        g = torch.empty((T, H), dtype=torch.float32, device=x.device)
    else:
        q, k, v, g = out
        for t in (q, k, v):
            if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.shape != (T, H, d):
                raise ValueError("q, k, v outputs must be contiguous bfloat16 [T, H, d]")
        if g.dtype != torch.float32 or not g.is_contiguous() or g.shape != (T, H):
            raise ValueError("g output must be contiguous float32 [T, H]")
    _check("gret_qkvg_projection", _lib.gret_qkvg_projection(
        _ptr(x), _ptr(w), w.stride(0), T, H, d, D, _ptr(q), _ptr(k), _ptr(v), _ptr(g),
        _stream(stream)))
    return q, k, v, g


def gret_prefill_elementwise_workspace_size(B, N, H, d=128):
    return int(_lib.gret_prefill_elementwise_workspace_size(B, N, H, d))


def gret_prefill_elementwise(q, k, v, g, tau=16.0, k_scale=1.0, state_in=None, state_out=None,
                             o=None, workspace=None, stream=None):
    """Chunkwise prefill with one gate per key channel (state row i decays by
    sigmoid(g[..., i])^(1/tau)).  q, k, v [B, N, H, 128] bf16 and g [B, N, H, 128] fp32, all
    contiguous; state_in / state_out fp32 [B, H, 128, 128] (state_out=True allocates one).
    Returns (o, state_out)."""
    B, N, H, d = q.shape
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.shape != (B, N, H, d):
            raise ValueError("q, k, v must be contiguous bfloat16 [B, N, H, d]")
    if g.dtype != torch.float32 or not g.is_contiguous() or g.shape != (B, N, H, d):
        raise ValueError("g must be contiguous float32 [B, N, H, d]")
    if o is None:
        o = torch.empty_like(q)
    if state_out is True:
        state_out = torch.empty((B, H, d, d), dtype=torch.float32, device=q.device)
    if workspace is None:
        need = gret_prefill_elementwise_workspace_size(B, N, H, d)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check("gret_prefill_elementwise", _lib.gret_prefill_elementwise(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), tau, k_scale, B, N, H, d, _ptr(state_in),
        _ptr(state_out), _ptr(o), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))
    return o, state_out


def gret_swa_prefill(q, k, v, window=1024, scale=None, o=None, stream=None):
    """Sliding-window softmax attention: position i attends to the last `window` positions of
    its sequence.  q, k, v [B, N, H, 128] bf16 contiguous; scale defaults to d^-1/2.
    Returns o [B, N, H, 128] bf16."""
    B, N, H, d = q.shape
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.shape != (B, N, H, d):
            raise ValueError("q, k, v must be contiguous bfloat16 [B, N, H, d]")
    if o is None:
        o = torch.empty_like(q)
    _check("gret_swa_prefill", _lib.gret_swa_prefill(
        _ptr(q), _ptr(k), _ptr(v), d ** -0.5 if scale is None else scale, window, B, N, H, d,
        _ptr(o), _stream(stream)))
    return o


def gret_swa_decode_step(q, k, v, pos, k_cache, v_cache, window=None, scale=None, o=None,
                         stream=None):
    """One sliding-window attention decode step with a ring-buffer cache: token t = pos[b] of
    every sequence is written to slot t % window of k_cache / v_cache [B, H, window, 128] and
    attends to its sequence's last `window` tokens.  q, k, v [B, H, 128] bf16; pos int32 [B] on
    the device (not advanced here).  Returns o [B, H, 128] bf16."""
    B, H, d = q.shape
    W = k_cache.shape[2] if window is None else window
    for t in (q, k, v, k_cache, v_cache):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("q, k, v and the caches must be contiguous bfloat16")
    if k_cache.shape != (B, H, W, d) or v_cache.shape != (B, H, W, d):
        raise ValueError("caches must be [B, H, window, d]")
    if pos.dtype != torch.int32 or pos.shape != (B,):
        raise ValueError("pos must be int32 [B]")
    if o is None:
        o = torch.empty_like(q)
    _check("gret_swa_decode_step", _lib.gret_swa_decode_step(
        _ptr(q), _ptr(k), _ptr(v), d ** -0.5 if scale is None else scale, W, B, H, d, _ptr(pos),
        _ptr(k_cache), _ptr(v_cache), _ptr(o), _stream(stream)))
    return o


def gret_layer_workspace_size(T, n_seqs, H, d=128):
    return int(_lib.gret_layer_workspace_size(T, n_seqs, H, d))


def gret_layer_forward(x, w_qkvg, w_g, H, d=128, cu_seqlens=None, state_in=None, tau=16.0,
                       k_scale=None, gn_weight=None, gn_bias=None, eps=1e-5, y=None,
                       state_out=True, workspace=None, stream=None):
    """One gated-retention mixer layer through the C entry point gret_layer_forward: the
    q / k / v / gate-logit projection of x, the chunkwise prefill (k scaled by d^-1/2 unless
    k_scale is given), and the per-head GroupNorm * swish(x @ w_g) output gate.  x [T, D] bf16 is
    one packed batch (cu_seqlens marks its sequences; None means one sequence).  Returns y
    [T, H*d] bf16 and the final fp32 states [n_seqs, H, d, d] (state_out=True allocates them,
    None skips them).  The workspace holds the intermediates; it is allocated here unless given."""
    T, D = x.shape
    for t in (x, w_qkvg, w_g):
        if t.dtype != torch.bfloat16 or t.stride(-1) != 1:
            raise ValueError("x, w_qkvg and w_g must be bfloat16 with contiguous rows")
    if x.stride(0) != D or not w_g.is_contiguous():
        raise ValueError("x and w_g must be contiguous")
    if cu_seqlens is not None and (cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1):
        raise ValueError("cu_seqlens must be 1-D int32")
    n_seqs = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    if y is None:
        y = torch.empty((T, H * d), dtype=torch.bfloat16, device=x.device)
    if state_out is True:
        state_out = torch.empty((n_seqs, H, d, d), dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = torch.empty(max(16, gret_layer_workspace_size(T, n_seqs, H, d)),
                                dtype=torch.uint8, device=x.device)
    _check("gret_layer_forward", _lib.gret_layer_forward(
        _ptr(x), _ptr(w_qkvg), w_qkvg.stride(0), _ptr(w_g), _ptr(gn_weight), _ptr(gn_bias), eps,
        tau, d ** -0.5 if k_scale is None else k_scale, T, H, d, D, _ptr(cu_seqlens), n_seqs,
        _ptr(state_in), _ptr(state_out), _ptr(y), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return y, state_out
