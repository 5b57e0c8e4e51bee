"""GPU parity of the sliding-window attention prefill (gret_swa_prefill) against the fp64
oracle, through the C ABI ("路线一：滑动窗口注意力": position i attends to positions
i-C+1 .. i with softmax over exactly those; the page's scaling runs use C = 1024)."""
import numpy as np
import pytest
import torch

import synth_inputs as SI
from oracle import oracle
from parity import assert_parity

pytestmark = pytest.mark.gpu


def lib():
    import gated_retention_linear_b200 as G
    return G


def inputs(B, N, H, seed):
    inp = SI.gret_inputs(B, N, H, 128, dtype=torch.bfloat16, seed=seed)
    # unit-variance queries and keys give scores ~ N(0, 1) after the 1/sqrt(d) scale
    return (inp["q"] * 128 ** 0.5).to(torch.bfloat16), (inp["k"] * 128 ** 0.5).to(torch.bfloat16), \
        inp["v"]


@pytest.mark.parametrize("B,N,H,W", [
    (1, 200, 2, 64),       # window of one tile, ragged tail
    (2, 150, 3, 40),       # window not a multiple of the tile
    (1, 1, 2, 1024),       # a single token
    (1, 130, 1, 1),        # window 1: o = v
    (1, 1000, 2, 300),     # several tiles per window
    (1, 700, 2, 1024),     # window longer than the sequence: causal attention
    (2, 2100, 2, 1024),    # the page's window, 17 tiles per query block
    (1, 2000, 48, 100),    # 768 one- and two-key-tile items: several per CTA, back to back
    (1, 1500, 40, 300),    # items of one to four key tiles, several per CTA
])
def test_swa_matches_oracle(B, N, H, W):
    G = lib()
    q, k, v = inputs(B, N, H, seed=N + W)
    o = G.gret_swa_prefill(q.cuda(), k.cuda(), v.cuda(), window=W)
    torch.cuda.synchronize()
    cu = [i * N for i in range(B + 1)]
    ref = oracle.swa(q.reshape(B * N, H, 128), k.reshape(B * N, H, 128), v.reshape(B * N, H, 128),
                     W, cu_seqlens=cu)
    assert_parity("o", o.reshape(B * N, H, 128), ref, 1e-2, stored_bf16=True)


def test_swa_full_size_sampled_rows():
    """32768 tokens x 24 heads with window 1024, as the benchmark runs it; four blocks of 64
    queries of heads 0 and 23 checked against the oracle, each on the slice of keys its
    windows cover (a query's output depends on nothing else)."""
    G = lib()
    N, H, W = 32768, 24, 1024
    q, k, v = inputs(1, N, H, seed=8)
    o = G.gret_swa_prefill(q.cuda(), k.cuda(), v.cuda(), window=W).cpu()
    for i0 in (0, 1000, 17000, N - 64):
        a = max(0, i0 - W + 1)
        sl = slice(a, i0 + 64)
        for h in (0, 23):
            ref = oracle.swa(q[0, sl, h:h + 1], k[0, sl, h:h + 1], v[0, sl, h:h + 1], W)
            assert_parity("o", o[0, i0:i0 + 64, h:h + 1], ref[i0 - a:], 1e-2, stored_bf16=True)


def test_swa_rejects_bad_arguments():
    G = lib()
    x = torch.zeros((1, 4, 1, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(G.GretError):            # d = 64: no kernel for it
        G.gret_swa_prefill(x, x, x)
    y = torch.zeros((1, 4, 1, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(G.GretError):            # window 0
        G.gret_swa_prefill(y, y, y, window=0)


def test_swa_decode_steps_match_oracle():
    """Token-by-token decode of 2 sequences x 3 heads, window 64, 200 steps through the ring
    buffer (it wraps three times): every step's output equals the sliding-window attention of
    the whole sequence at that position."""
    G = lib()
    B, T, H, W = 2, 200, 3, 64
    q, k, v = inputs(B, T, H, seed=91)
    kc = torch.zeros((B, H, W, 128), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    outs = []
    for t in range(T):
        pos = torch.full((B,), t, dtype=torch.int32, device="cuda")
        outs.append(G.gret_swa_decode_step(qd[:, t].contiguous(), kd[:, t].contiguous(),
                                           vd[:, t].contiguous(), pos, kc, vc))
    torch.cuda.synchronize()
    o = torch.stack(outs, dim=1)          # [B, T, H, 128]
    cu = [i * T for i in range(B + 1)]
    ref = oracle.swa(q.reshape(B * T, H, 128), k.reshape(B * T, H, 128), v.reshape(B * T, H, 128),
                     W, cu_seqlens=cu)
    assert_parity("o", o.reshape(B * T, H, 128), ref, 1e-2, stored_bf16=True)


def test_swa_decode_full_window_prefilled_cache():
    """Batch 4 x 24 heads, window 1024, each sequence at a different position (its first token,
    inside the first window, exactly one window, well past it); the caches are filled with the
    earlier tokens in ring order, then one step runs.  The oracle sees only the tokens of each
    window (the last position's output depends on nothing else); heads 0, 11 and 23 checked."""
    G = lib()
    H, W = 24, 1024
    tpos = [0, 700, 1024, 3001]
    B, T = len(tpos), max(tpos) + 1
    q, k, v = inputs(B, T, H, seed=92)
    kc = torch.zeros((B, H, W, 128), dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    for b, t in enumerate(tpos):
        for j in range(max(0, t - W + 1), t):          # the tokens before t still in the window
            kc[b, :, j % W] = k[b, j]
            vc[b, :, j % W] = v[b, j]
    pos = torch.tensor(tpos, dtype=torch.int32, device="cuda")
    sel = lambda x: torch.stack([x[b, t] for b, t in enumerate(tpos)]).cuda()
    kcd, vcd = kc.cuda(), vc.cuda()
    o = G.gret_swa_decode_step(sel(q), sel(k), sel(v), pos, kcd, vcd).cpu()
    for b, t in enumerate(tpos):
        a = max(0, t - W + 1)
        for h in (0, 11, 23):
            ref = oracle.swa(q[b, a:t + 1, h:h + 1], k[b, a:t + 1, h:h + 1],
                             v[b, a:t + 1, h:h + 1], W)
            assert_parity("o", o[b, h:h + 1], ref[-1], 1e-2, stored_bf16=True)
        # the new token went into its slot
        assert torch.equal(kcd[b, :, t % W].cpu(), k[b, t]) and \
            torch.equal(vcd[b, :, t % W].cpu(), v[b, t])


def test_swa_decode_rejects_bad_arguments():
    G = lib()
    x = torch.zeros((1, 1, 128), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((1, 1, 8, 128), dtype=torch.bfloat16, device="cuda")
    pos = torch.zeros((1,), dtype=torch.int32, device="cuda")
    with pytest.raises(G.GretError):            # window 0
        G._check("gret_swa_decode_step", G._lib.gret_swa_decode_step(
            G._ptr(x), G._ptr(x), G._ptr(x), 1.0, 0, 1, 1, 128, G._ptr(pos), G._ptr(kc),
            G._ptr(kc), G._ptr(x), G._stream(None)))
    with pytest.raises(G.GretError):            # window above the 32768 the step takes
        G._check("gret_swa_decode_step", G._lib.gret_swa_decode_step(
            G._ptr(x), G._ptr(x), G._ptr(x), 1.0, 40000, 1, 1, 128, G._ptr(pos), G._ptr(kc),
            G._ptr(kc), G._ptr(x), G._stream(None)))
