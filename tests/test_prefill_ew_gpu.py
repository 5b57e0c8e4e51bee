"""GPU parity of the per-key-channel-gate prefill (gret_prefill_elementwise) against the fp64
oracle, through the C ABI.  The variant is the element-wise gate that "路线二：Multi-Head Gated
Retention" weighs against the head-wise gate: state row i decays by sigmoid(g[i])^(1/tau)."""
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


def inputs(B, N, H, g_mean, g_std, seed, state):
    inp = SI.gret_inputs(B, N, H, 128, dtype=torch.bfloat16, seed=seed, with_state=state)
    g = SI.channel_gates(B, N, H, 128, g_mean=g_mean, g_std=g_std, seed=seed)
    return inp["q"], inp["k"], inp["v"], g, inp.get("s")


def run(G, q, k, v, g, **kw):
    """The prefill through an explicit workspace, whose status word must read OK afterwards."""
    B, N, H, d = q.shape
    ws = torch.empty(max(16, G.gret_prefill_elementwise_workspace_size(B, N, H, d)),
                     dtype=torch.uint8, device="cuda")
    o, s = G.gret_prefill_elementwise(q.cuda(), k.cuda(), v.cuda(), g.cuda(), workspace=ws, **kw)
    assert G.gret_workspace_status(ws) == 0
    return o, s


def reference(q, k, v, g, s0, k_scale, heads=None):
    """Oracle on [B*N, H, d] with one sequence per batch row (optionally a subset of heads)."""
    B, N, H, d = q.shape
    sel = slice(None) if heads is None else heads
    flat = lambda t: t[:, :, sel].reshape(B * N, -1, t.shape[-1])
    cu = [i * N for i in range(B + 1)]
    s_in = None if s0 is None else s0[:, sel]
    o, s = oracle.gret_recurrent_ew(flat(q), flat(k), flat(v), flat(g), k_scale=k_scale,
                                    cu_seqlens=cu, state_in=s_in)
    return o.reshape(B, N, -1, d), s


@pytest.mark.parametrize("B,N,H,g_mean,g_std,state", [
    (1, 200, 2, 2.0, 1.0, False),     # two chunks, ragged tail
    (2, 81, 3, 0.0, 2.0, True),       # two sequences, part of one chunk each, entry state
    (1, 1, 2, 0.0, 2.0, True),        # a single token
    (1, 128, 2, 2.0, 1.0, True),      # exactly one chunk
    (1, 1000, 4, 0.0, 2.0, True),     # 8 chunks, harsh gates
    (3, 300, 2, 0.0, 4.0, True),      # very harsh gates (alpha down to ~0.1)
    (1, 20000, 2, 2.0, 1.0, True),    # ranges of 3 chunks: the state carried inside a range
])
def test_elementwise_matches_oracle(B, N, H, g_mean, g_std, state):
    G = lib()
    q, k, v, g, s0 = inputs(B, N, H, g_mean, g_std, seed=N + 7 * B + H, state=state)
    o, s = run(G, q, k, v, g, k_scale=0.9, state_in=None if s0 is None else s0.cuda(),
               state_out=True)
    torch.cuda.synchronize()
    ro, rs = reference(q, k, v, g, s0, 0.9)
    # every operand is a bf16 hi/lo pair: the error stays near 1e-5 of rms
    assert_parity("o", o, ro, 1e-2, stored_bf16=True, tight=1e-3)
    assert_parity("state", s, rs, 1e-2, stored_bf16=False, tight=1e-3)


def test_elementwise_fast_and_pairwise_chunks_in_one_sequence():
    """Chunks where one channel decays by more than 2^-64 take the pairwise scores; the others
    the factored operands.  Alternate the two along a sequence that spans several ranges."""
    G = lib()
    q, k, v, g, s0 = inputs(2, 1300, 3, 1.0, 1.0, seed=21, state=True)
    for c in range(0, 11, 2):                       # chunks 0, 2, 4, ...: channel 5 and 77 of
        g[:, c * 128:(c + 1) * 128, :, 5] = -30.0   # every head decay by 2^-2.7 per token
        g[0, c * 128:(c + 1) * 128, 1, 77] = -60.0
    o, s = run(G, q, k, v, g, k_scale=0.8, state_in=s0.cuda(), state_out=True)
    torch.cuda.synchronize()
    ro, rs = reference(q, k, v, g, s0, 0.8)
    assert_parity("o", o, ro, 1e-2, stored_bf16=True, tight=1e-3)
    assert_parity("state", s, rs, 1e-2, stored_bf16=False, tight=1e-3)


@pytest.mark.parametrize("g_value", [-1e4, 200.0])
def test_elementwise_degenerate_gates(g_value):
    """alpha == 0 (only the current token survives) and alpha == 1 (causal linear attention)."""
    G = lib()
    q, k, v, _, s0 = inputs(1, 150, 2, 0.0, 1.0, seed=3, state=True)
    g = torch.full((1, 150, 2, 128), g_value)
    o, s = run(G, q, k, v, g, state_in=s0.cuda(), state_out=True)
    torch.cuda.synchronize()
    ro, rs = reference(q, k, v, g, s0, 1.0)
    assert_parity("o", o, ro, 1e-2, stored_bf16=True)
    assert_parity("state", s, rs, 1e-2, stored_bf16=False)


def test_elementwise_no_tokens_passes_the_state_through():
    G = lib()
    s0 = torch.randn(2, 3, 128, 128, device="cuda")
    e = torch.empty((2, 0, 3, 128), dtype=torch.bfloat16, device="cuda")
    ge = torch.empty((2, 0, 3, 128), dtype=torch.float32, device="cuda")
    _, s = G.gret_prefill_elementwise(e, e, e, ge, state_in=s0, state_out=True)
    _, z = G.gret_prefill_elementwise(e, e, e, ge, state_out=True)
    torch.cuda.synchronize()
    assert torch.equal(s, s0) and not torch.any(z)


def test_elementwise_full_size_sampled_heads():
    """The 32768-token, 24-head workload the benchmark times, in the same launch; heads 0 and
    23 compared element by element with the oracle (heads are independent)."""
    G = lib()
    c = SI.ELEMENTWISE_32K
    q, k, v, g, _ = inputs(c["B"], c["N"], c["H"], c["g_mean"], c["g_std"], c["seed"], False)
    o, s = run(G, q, k, v, g, state_out=True)
    torch.cuda.synchronize()
    heads = [0, 23]
    ro, rs = reference(q, k, v, g, None, 1.0, heads=heads)
    assert_parity("o", o[:, :, heads].cpu(), ro, 1e-2, stored_bf16=True, tight=1e-3)
    assert_parity("state", s[:, heads].cpu(), rs, 1e-2, stored_bf16=False, tight=1e-3)


def test_elementwise_equal_gates_match_headwise_kernel():
    """A gate shared by every channel must give the head-wise tensor-core kernel's result."""
    G = lib()
    q, k, v, g1, s0 = [t for t in SI.gret_inputs(1, 300, 2, 128, seed=9, with_state=True).values()]
    g = g1[..., None].expand(1, 300, 2, 128).contiguous()
    o_ew, s_ew = G.gret_prefill_elementwise(q.cuda(), k.cuda(), v.cuda(), g.cuda(),
                                            state_in=s0.cuda(), state_out=True)
    o_hw, s_hw = G.gret_prefill_chunkwise(q.cuda(), k.cuda(), v.cuda(), g1.cuda(),
                                          state_in=s0.cuda(), state_out=True)
    torch.cuda.synchronize()
    assert_parity("o", o_ew, o_hw.double().cpu().numpy(), 1e-2, stored_bf16=True)
    assert_parity("state", s_ew, s_hw.double().cpu().numpy(), 1e-3, stored_bf16=False)


def test_elementwise_rejects_bad_arguments():
    G = lib()
    x = torch.zeros((1, 4, 1, 64), dtype=torch.bfloat16, device="cuda")
    gx = torch.zeros((1, 4, 1, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(G.GretError):            # d = 64: no kernel for it
        G.gret_prefill_elementwise(x, x, x, gx)
    y = torch.zeros((1, 4, 1, 128), dtype=torch.bfloat16, device="cuda")
    gy = torch.zeros((1, 4, 1, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(G.GretError):            # workspace too small
        G.gret_prefill_elementwise(y, y, y, gy,
                                   workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
