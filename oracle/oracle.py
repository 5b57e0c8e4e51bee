"""Python access to the fp64 CPU oracle for gated retention (gret_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the benchmark's
CPU-baseline leg, never by the library.  The arithmetic lives in gret_oracle.c; this module only
converts arrays to contiguous fp64 and passes pointers.  See gret_oracle.c for the passages each
function follows ("YOCO 完全拆解", sections "路线二：Multi-Head Gated Retention",
"Prefill 与 Decode 为什么使用两种计算形态" and "单 token Decode 的实现骨架").

Layout: q, k [T, H, dk]; v [T, H, dv]; g [T, H]; cu_seqlens [n_seqs+1];
state [n_seqs, H, dk, dv]; returns o [T, H, dv] and the final state.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int64)
        common = [dp, dp, dp, dp, ctypes.c_double, ctypes.c_double, ctypes.c_int64,
                  ctypes.c_int, ctypes.c_int, ctypes.c_int, ip, ctypes.c_int, dp, dp, dp]
        for name in ("oracle_gret_recurrent", "oracle_gret_parallel"):
            f = getattr(L, name)
            f.argtypes = common
            f.restype = ctypes.c_int
        L.oracle_gret_recurrent_ew.argtypes = common
        L.oracle_gret_recurrent_ew.restype = ctypes.c_int
        L.oracle_gret_chunkwise.argtypes = common + [ctypes.c_int]
        L.oracle_gret_chunkwise.restype = ctypes.c_int
        L.oracle_gret_decode_step.argtypes = [dp, dp, dp, dp, ctypes.c_double, ctypes.c_double,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, dp, dp]
        L.oracle_gret_decode_step.restype = ctypes.c_int
        L.oracle_groupnorm_gate.argtypes = [dp, dp, dp, dp, dp, ctypes.c_double, ctypes.c_int64,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_int, ip,
                                            ctypes.c_int64, dp]
        L.oracle_groupnorm_gate.restype = ctypes.c_int
        L.oracle_swa.argtypes = [dp, dp, dp, ctypes.c_double, ctypes.c_int, ctypes.c_int64,
                                 ctypes.c_int, ctypes.c_int, ctypes.c_int, ip, ctypes.c_int, dp]
        L.oracle_swa.restype = ctypes.c_int
        L.oracle_log_gamma.argtypes = [ctypes.c_double, ctypes.c_double]
        L.oracle_log_gamma.restype = ctypes.c_double
        _lib = L
    return _lib


def _d(a):
    """Contiguous fp64 copy of an array-like (torch tensors are moved to the CPU first)."""
    if a is None:
        return None
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _cu(cu_seqlens, T):
    if cu_seqlens is None:
        cu_seqlens = [0, T]
    if hasattr(cu_seqlens, "detach"):
        cu_seqlens = cu_seqlens.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))


def threads():
    """OpenMP threads the oracle will use (OMP_NUM_THREADS, else the usable cores)."""
    env = os.environ.get("OMP_NUM_THREADS")
    if env:
        return int(env)
    return len(os.sched_getaffinity(0))


def _run(fname, q, k, v, g, tau, k_scale, cu_seqlens, state_in, extra=(), g_per_channel=False):
    q, k, v, g = _d(q), _d(k), _d(v), _d(g)
    T, H, dk = q.shape
    dv = v.shape[2]
    assert k.shape == (T, H, dk) and v.shape == (T, H, dv)
    assert g.shape == ((T, H, dk) if g_per_channel else (T, H))
    cu = _cu(cu_seqlens, T)
    n = len(cu) - 1
    s_in = _d(state_in)
    if s_in is not None:
        assert s_in.shape == (n, H, dk, dv)
    o = np.zeros((T, H, dv))
    s_out = np.zeros((n, H, dk, dv))
    rc = getattr(lib(), fname)(_p(q), _p(k), _p(v), _p(g), float(tau), float(k_scale), T, H,
                              dk, dv, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), n,
                              _p(s_in), _p(s_out), _p(o), *extra)
    if rc != 0:
        raise ValueError("%s rejected its arguments (rc=%d)" % (fname, rc))
    return o, s_out


def gret_recurrent(q, k, v, g, tau=16.0, k_scale=1.0, cu_seqlens=None, state_in=None):
    """Recurrent gRet (the definition).  Returns (o [T,H,dv], state [n_seqs,H,dk,dv])."""
    return _run("oracle_gret_recurrent", q, k, v, g, tau, k_scale, cu_seqlens, state_in)


def gret_recurrent_ew(q, k, v, g, tau=16.0, k_scale=1.0, cu_seqlens=None, state_in=None):
    """Recurrent gated retention with one gate per key channel: g [T, H, dk], the state row i
    decays by sigmoid(g[..., i])^(1/tau).  Returns (o [T,H,dv], state [n_seqs,H,dk,dv])."""
    return _run("oracle_gret_recurrent_ew", q, k, v, g, tau, k_scale, cu_seqlens, state_in,
                g_per_channel=True)


def swa(q, k, v, window, scale=None, cu_seqlens=None):
    """Sliding-window softmax attention ("路线一：滑动窗口注意力"): position i attends to the
    last `window` positions of its sequence, j in [i - window + 1, i].  q, k [T, H, d],
    v [T, H, dv]; scale defaults to d^-1/2.  Returns o [T, H, dv]."""
    q, k, v = _d(q), _d(k), _d(v)
    T, H, d = q.shape
    dv = v.shape[2]
    assert k.shape == (T, H, d) and v.shape == (T, H, dv)
    cu = _cu(cu_seqlens, T)
    o = np.zeros((T, H, dv))
    rc = lib().oracle_swa(_p(q), _p(k), _p(v), float(d ** -0.5 if scale is None else scale),
                          int(window), T, H, d, dv,
                          cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), len(cu) - 1, _p(o))
    if rc != 0:
        raise ValueError("oracle_swa rejected its arguments (rc=%d)" % rc)
    return o


def gret_parallel(q, k, v, g, tau=16.0, k_scale=1.0, cu_seqlens=None, state_in=None):
    """Brute-force unrolled form with explicit decay products (tiny inputs only)."""
    return _run("oracle_gret_parallel", q, k, v, g, tau, k_scale, cu_seqlens, state_in)


def gret_chunkwise(q, k, v, g, chunk, tau=16.0, k_scale=1.0, cu_seqlens=None, state_in=None):
    """Chunkwise re-association evaluated in fp64 (checks the decomposition, not the GPU)."""
    return _run("oracle_gret_chunkwise", q, k, v, g, tau, k_scale, cu_seqlens, state_in,
                extra=(int(chunk),))


def gret_decode_step(q, k, v, g, state, tau=16.0, k_scale=1.0):
    """One decode step on [B,H,d] inputs; returns (o [B,H,dv], new state [B,H,dk,dv])."""
    q, k, v, g = _d(q), _d(k), _d(v), _d(g)
    S = _d(state).copy()
    B, H, dk = q.shape
    dv = v.shape[2]
    assert S.shape == (B, H, dk, dv) and g.shape == (B, H)
    o = np.zeros((B, H, dv))
    rc = lib().oracle_gret_decode_step(_p(q), _p(k), _p(v), _p(g), float(tau), float(k_scale),
                                       B, H, dk, dv, _p(S), _p(o))
    if rc != 0:
        raise ValueError("oracle_gret_decode_step rc=%d" % rc)
    return o, S


def groupnorm_gate(o, x, w_g, H, gn_weight=None, gn_bias=None, eps=1e-5, rows=None):
    """Per-head GroupNorm(o) * swish(x @ w_g) for the listed rows (all rows if None).

    o [T, H*dv], x [T, D], w_g [D, H*dv].  Returns y [len(rows) or T, H*dv]."""
    o, x, w_g = _d(o), _d(x), _d(w_g)
    T, F = o.shape
    D = x.shape[1]
    assert F % H == 0 and x.shape[0] == T and w_g.shape == (D, F)
    dv = F // H
    gw, gb = _d(gn_weight), _d(gn_bias)
    if rows is not None:
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        rp, nr = r.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), len(r)
    else:
        r, rp, nr = None, None, T
    y = np.zeros((nr, F))
    rc = lib().oracle_groupnorm_gate(_p(o), _p(x), _p(w_g), _p(gw), _p(gb), float(eps), T, H,
                                     dv, D, rp, nr, _p(y))
    if rc != 0:
        raise ValueError("oracle_groupnorm_gate rc=%d" % rc)
    return y


def log_gamma(g, tau=16.0):
    return lib().oracle_log_gamma(float(g), float(tau))


def qkvg_projection(x, w, H, d=128):
    """The layer's input projection, [q | k | v | g] = x @ w, in fp64 ("路线二：Multi-Head Gated
    Retention": the gate is a learned projection of the layer input, beside the query, key and
    value projections).  x [T, D]; w [D, >= 3 H d + H] (W_Q, W_K, W_V, W_gamma side by side).
    A library matmul is the whole step; the blocks are then read off by column.
    Returns q, k, v [T, H, d] and g [T, H]."""
    x, w = _d(x), _d(w)
    T = x.shape[0]
    hd = H * d
    z = x @ w[:, :3 * hd + H]
    q = z[:, 0:hd].reshape(T, H, d)
    k = z[:, hd:2 * hd].reshape(T, H, d)
    v = z[:, 2 * hd:3 * hd].reshape(T, H, d)
    g = z[:, 3 * hd:3 * hd + H]
    return q, k, v, g


def _round_bf16(a):
    """Round fp64 values to bfloat16 (round to nearest even), back in fp64."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).double().numpy()


def layer_forward(x, w_qkvg, w_g, H, d=128, cu_seqlens=None, state_in=None, tau=16.0,
                  k_scale=None, gn_weight=None, gn_bias=None, eps=1e-5, rows=None, with_o=False):
    """One gated-retention mixer layer from the oracle's own steps: the projection (q, k, v
    stored in bf16, the layer's dtype; g kept as computed), the recurrence, and the GroupNorm *
    swish(x W_G) gate on the retention output rounded to bf16 (as the layer stores it).
    Returns y [T or len(rows), H d] and the final states (and the bf16-rounded retention
    output o [T, H d] when with_o is set)."""
    q, k, v, g = qkvg_projection(x, w_qkvg, H, d)
    q, k, v = _round_bf16(q), _round_bf16(k), _round_bf16(v)
    o, s = gret_recurrent(q, k, v, g, tau=tau, k_scale=d ** -0.5 if k_scale is None else k_scale,
                          cu_seqlens=cu_seqlens, state_in=state_in)
    T = o.shape[0]
    o = _round_bf16(o).reshape(T, H * d)
    y = groupnorm_gate(o, x, w_g, H, gn_weight=gn_weight, gn_bias=gn_bias, eps=eps, rows=rows)
    return (y, s, o) if with_o else (y, s)
