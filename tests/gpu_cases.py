"""Shared helpers for the GPU parity tests: run a prefill through the C ABI and through the
fp64 oracle on the same seeded inputs, in the oracle's token-major layout."""
import numpy as np
import torch

import synth_inputs as SI
from oracle import oracle
from parity import assert_parity

# The tensor-core prefill (bf16, d_k = d_v = 128, chunk 128) carries P, the state copy and the
# weighted keys as bf16 high + low pairs, which keeps its error near 1e-5 of rms against the
# fp64 oracle.  This second bar, far below the 1e-2 parity bar, catches a regression of that
# precision (one dropped low half alone costs about 1e-2).
TC_TIGHT = 1e-3


def tc_path(dtype, dk, dv, chunk):
    return dtype == torch.bfloat16 and dk == 128 and dv == 128 and chunk in (0, 128)


def lib():
    import gated_retention_linear_b200 as G
    return G


def token_major(x, head_major):
    """[B,N,H,d] or [B,H,N,d] -> [B*N, H, d] (a copy on the CPU)."""
    if head_major:
        x = x.permute(0, 2, 1, 3)
    B, N, H, d = x.shape
    return x.reshape(B * N, H, d).cpu()


def run_dense(B, N, H, dk, dv, dtype, chunk=0, g_mean=2.0, g_std=1.0, seed=0,
              head_major=False, state=False, g_fill=None, tau=16.0, k_scale=1.0, tol=None,
              g_edit=None):
    G = lib()
    inp = SI.gret_inputs(B, N, H, dk, dv, dtype=dtype, g_mean=g_mean, g_std=g_std, seed=seed,
                         device="cpu", layout="bhnd" if head_major else "bnhd", with_state=state)
    if g_fill is not None:
        inp["g"].fill_(g_fill)
    if g_edit is not None:
        g_edit(inp["g"])
    d = {k: v.cuda() for k, v in inp.items()}
    o, s = G.gret_prefill_chunkwise(d["q"], d["k"], d["v"], d["g"], tau=tau, k_scale=k_scale,
                                    state_in=d.get("s"), state_out=True, chunk=chunk,
                                    head_major=head_major)
    torch.cuda.synchronize()
    cu = np.arange(B + 1) * N
    o_ref, s_ref = oracle.gret_recurrent(
        token_major(inp["q"], head_major), token_major(inp["k"], head_major),
        token_major(inp["v"], head_major), inp["g"].reshape(B * N, H), tau=tau,
        k_scale=k_scale, cu_seqlens=cu, state_in=inp.get("s"))
    bf16 = dtype == torch.bfloat16
    tol = tol if tol is not None else (1e-2 if bf16 else 1e-4)
    tight = TC_TIGHT if tc_path(dtype, dk, dv, chunk) else None
    eo = assert_parity("o", token_major(o, head_major), o_ref, tol, stored_bf16=bf16, tight=tight)
    es = assert_parity("state", s, s_ref, tol, stored_bf16=False, tight=tight)
    return eo, es


def run_varlen(lengths, H, dk, dv, dtype, chunk=0, g_mean=0.0, g_std=2.0, seed=0, state=False,
               alias_state=False, tol=None):
    G = lib()
    cu = SI.cu_seqlens_of(lengths)
    T, n = cu[-1], len(lengths)
    inp = SI.gret_inputs(1, T, H, dk, dv, dtype=dtype, g_mean=g_mean, g_std=g_std, seed=seed,
                         device="cpu")
    q, k, v = (inp[x][0] for x in ("q", "k", "v"))     # packed [T, H, d]
    g = inp["g"][0]
    s0 = SI.gret_inputs(n, 1, H, dk, dv, seed=seed + 1, with_state=True)["s"] if state else None
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    s_in = s0.cuda() if s0 is not None else None
    s_out = s_in if alias_state else True
    o, s = G.gret_prefill_chunkwise(q.cuda(), k.cuda(), v.cuda(), g.cuda(), cu_seqlens=cu_d,
                                    state_in=s_in, state_out=s_out, chunk=chunk)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.gret_recurrent(q, k, v, g, cu_seqlens=cu, state_in=s0)
    bf16 = dtype == torch.bfloat16
    tol = tol if tol is not None else (1e-2 if bf16 else 1e-4)
    tight = TC_TIGHT if tc_path(dtype, dk, dv, chunk) else None
    eo = assert_parity("o", o, o_ref, tol, stored_bf16=bf16, tight=tight)
    es = assert_parity("state", s, s_ref, tol, stored_bf16=False, tight=tight)
    return eo, es
