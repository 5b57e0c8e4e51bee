"""Seeded synthetic inputs for gated retention, shared by the tests, the benchmark and the oracle
checks.

This module draws random numbers and nothing else: it holds none of the method's arithmetic.
Every tensor is drawn from a torch.Generator seeded from (seed, tensor tag), so one call with
the same arguments always returns the same values.  Inputs are drawn in fp32 and then rounded
to the requested dtype; the rounded values are what both the CUDA path and the oracle see.

Recipes (the 3B shapes of the YOCO pages: 24 heads of width 128, hidden 3072):
  * q, k, v ~ N(0, 1) / sqrt(d)         (the 1/sqrt(d_h) key scaling is folded into the draw,
                                          so the library is called with k_scale = 1)
  * gate logits g ~ N(mean, std), fp32  (N(2, 1) for the dense configs, N(0, 2) for varlen);
    the per-key-channel gate variant draws one such logit per channel
  * packed varlen lengths ~ U[lo, hi] (torch.randint, inclusive bounds)
  * epilogue: x ~ N(0, 1), w_g ~ N(0, 0.02), bf16
  * layer: x ~ N(0, 1) with a constant column x[:, 0] = 1; W_Q, W_K, W_V ~ N(0, 1/D);
    W_gamma ~ N(0, 0.05^2 / D) plus a per-head bias ~ N(2, 1) on the constant row, so the
    gate logits sit near N(2, 1) per head; w_g ~ N(0, 0.02); bf16
"""
import math

import torch

_TAGS = {"q": 1, "k": 2, "v": 3, "g": 4, "s": 5, "x": 6, "w": 7, "len": 8, "gnw": 9, "gnb": 10,
         "wqkvg": 11, "gbias": 12, "gch": 13}


def _gen(seed, tag, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1000003 + _TAGS[tag] * 7919)
    return g


def _randn(shape, seed, tag, device, std=1.0, mean=0.0):
    gen = _gen(seed, tag, device)
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    if mean != 0.0:
        t.add_(mean)
    return t


def gret_inputs(B, N, H, dk, dv=None, dtype=torch.bfloat16, g_mean=2.0, g_std=1.0, seed=0,
                device="cpu", layout="bnhd", with_state=False, state_std=1.0):
    """q, k [B,N,H,dk] (or [B,H,N,dk] when layout == "bhnd"), v [..,dv], g [B,N,H] fp32.

    Returns a dict with q, k, v, g and, if with_state, an fp32 entry state s [B,H,dk,dv]
    ~ N(0, state_std)."""
    dv = dk if dv is None else dv
    if layout == "bnhd":
        shq, shv = (B, N, H, dk), (B, N, H, dv)
    elif layout == "bhnd":
        shq, shv = (B, H, N, dk), (B, H, N, dv)
    else:
        raise ValueError(layout)
    out = {
        "q": _randn(shq, seed, "q", device, std=1.0 / math.sqrt(dk)).to(dtype),
        "k": _randn(shq, seed, "k", device, std=1.0 / math.sqrt(dk)).to(dtype),
        "v": _randn(shv, seed, "v", device, std=1.0 / math.sqrt(dv)).to(dtype),
        "g": _randn((B, N, H), seed, "g", device, std=g_std, mean=g_mean),
    }
    if with_state:
        out["s"] = _randn((B, H, dk, dv), seed, "s", device, std=state_std)
    return out


def varlen_lengths(n_seqs, lo, hi, seed):
    """n_seqs lengths drawn uniformly from [lo, hi] (inclusive), on the CPU."""
    gen = _gen(seed, "len", "cpu")
    return [int(x) for x in torch.randint(lo, hi + 1, (n_seqs,), generator=gen)]


def cu_seqlens_of(lengths):
    """Offsets [0, l0, l0+l1, ...] as a Python list."""
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return cu


def epilogue_inputs(T, D, F, seed=0, device="cpu", w_std=0.02, affine=False):
    """x [T,D] ~ N(0,1) and w_g [D,F] ~ N(0, w_std) in bf16; optional GroupNorm affine
    parameters (fp32, weight ~ 1 + N(0, 0.1), bias ~ N(0, 0.1))."""
    out = {
        "x": _randn((T, D), seed, "x", device).to(torch.bfloat16),
        "w_g": _randn((D, F), seed, "w", device, std=w_std).to(torch.bfloat16),
    }
    if affine:
        out["gn_weight"] = _randn((F,), seed, "gnw", device, std=0.1, mean=1.0)
        out["gn_bias"] = _randn((F,), seed, "gnb", device, std=0.1)
    return out


def channel_gates(B, N, H, dk, g_mean=2.0, g_std=1.0, seed=0, device="cpu"):
    """Gate logits with one value per key channel, g [B, N, H, dk] fp32 ~ N(g_mean, g_std)."""
    return _randn((B, N, H, dk), seed, "gch", device, std=g_std, mean=g_mean)


def layer_inputs(T, D, H, d=128, seed=0, device="cpu", pad=0, pad_value=float("nan"),
                 exact_projection=False):
    """One mixer layer's input and weights, bf16: x [T, D], w_qkvg [D, 3 H d + H + pad] (W_Q,
    W_K, W_V and W_gamma side by side; the pad columns, if any, hold pad_value) and
    w_g [D, H d].

    exact_projection: the same distributions drawn on coarse dyadic grids (x on multiples of
    1/8 within [-4, 4]; the q, k, v weight columns on multiples of 2^-10, the gate-logit columns
    on 2^-14, their bias row on 2^-5), so that every partial sum of x W is an integer multiple
    of the grid unit below 2^24 units: the projection is then exact in fp32 and fp64 alike, and
    both round the same q, k, v to bf16.  For D <= 3072 (the bounds below)."""
    F = 3 * H * d + H
    x = _randn((T, D), seed, "x", device)
    x[:, 0] = 1.0
    w = _randn((D, F + pad), seed, "wqkvg", device, std=D ** -0.5)
    w[:, 3 * H * d:F] *= 0.05
    w[0, 3 * H * d:F] = _randn((H,), seed, "gbias", device, mean=2.0)
    if exact_projection:
        # |x| <= 32 units of 1/8; |w| <= 127 units (7 bits, exact in bf16): a q, k, v sum is at
        # most D * 32 * 127 < 2^24 units of 2^-13, a gate-logit sum at most D * 32 * 127 plus the
        # bias row's 8 * 127 * 2^9 units of 2^-17
        assert D <= 3072
        x = torch.clamp(torch.round(x * 8.0), -32.0, 32.0) / 8.0
        qkv = w[:, :3 * H * d]
        w[:, :3 * H * d] = torch.clamp(torch.round(qkv * 1024.0), -127.0, 127.0) / 1024.0
        gcol = w[1:, 3 * H * d:F]
        w[1:, 3 * H * d:F] = torch.clamp(torch.round(gcol * 16384.0), -127.0, 127.0) / 16384.0
        w[0, 3 * H * d:F] = torch.clamp(torch.round(w[0, 3 * H * d:F] * 32.0), -127.0, 127.0) / 32.0
    if pad:
        w[:, F:] = pad_value
    w_g = _randn((D, H * d), seed, "w", device, std=0.02)
    return {"x": x.to(torch.bfloat16), "w_qkvg": w.to(torch.bfloat16),
            "w_g": w_g.to(torch.bfloat16)}


# The five workloads, by what they are.
TINY = dict(B=1, N=512, H=2, dk=64, dtype=torch.float32, g_mean=2.0, g_std=1.0, seed=1,
            layout="bhnd", chunk=64)
PREFILL_32K = dict(B=1, N=32768, H=24, dk=128, dtype=torch.bfloat16, g_mean=2.0, g_std=1.0,
                   seed=2)
PREFILL_512K = dict(B=1, N=524288, H=24, dk=128, dtype=torch.bfloat16, g_mean=2.0, g_std=1.0,
                    seed=3)
DECODE_BS64 = dict(B=64, prefill_N=4096, steps=256, H=24, dk=128, dtype=torch.bfloat16,
                   g_mean=2.0, g_std=1.0, seed=4)
SWA_32K = dict(B=1, N=32768, H=24, dk=128, window=1024, seed=8)
ELEMENTWISE_32K = dict(B=1, N=32768, H=24, dk=128, g_mean=2.0, g_std=1.0, seed=7)
LAYER_32K = dict(T=32768, D=3072, H=24, dk=128, seed=6)
VARLEN_EPILOGUE = dict(n_seqs=8, lo=1024, hi=65536, H=24, dk=128, dtype=torch.bfloat16,
                       g_mean=0.0, g_std=2.0, D=3072, eps=1e-5, seed=5)
