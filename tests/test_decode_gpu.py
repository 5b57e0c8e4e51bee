"""GPU parity of gret_decode_step against the fp64 oracle, and decode-after-prefill equal to a
longer prefill (the recurrent decode update of "单 token Decode 的实现骨架")."""
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


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (64, 128), (128, 64)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_step_matches_oracle(dk, dv, dtype):
    G = lib()
    B, H = 5, 3
    inp = SI.gret_inputs(B, 1, H, dk, dv, dtype=dtype, seed=dk + dv, with_state=True)
    q, k, v = (inp[x][:, 0] for x in ("q", "k", "v"))
    g = inp["g"][:, 0]
    S = inp["s"]
    Sd = S.cuda()
    for step in range(3):           # three steps in a row on the same state
        o = G.gret_decode_step(q.cuda(), k.cuda(), v.cuda(), g.cuda(), Sd)
        torch.cuda.synchronize()
        o_ref, S = oracle.gret_decode_step(q, k, v, g, S)
        bf16 = dtype == torch.bfloat16
        tol = 1e-2 if bf16 else 1e-4
        assert_parity("o", o, o_ref, tol, stored_bf16=bf16)
        assert_parity("state", Sd, S, tol, stored_bf16=False)
        S = torch.from_numpy(S)


def test_decode_batch64_shape():
    G = lib()
    B, H, d = 64, 24, 128
    inp = SI.gret_inputs(B, 1, H, d, dtype=torch.bfloat16, seed=4, with_state=True)
    q, k, v = (inp[x][:, 0] for x in ("q", "k", "v"))
    g = inp["g"][:, 0]
    Sd = inp["s"].cuda()
    o = G.gret_decode_step(q.cuda(), k.cuda(), v.cuda(), g.cuda(), Sd)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.gret_decode_step(q, k, v, g, inp["s"])
    assert_parity("o", o, o_ref, 1e-2, stored_bf16=True)
    assert_parity("state", Sd, s_ref, 1e-2, stored_bf16=False)


@pytest.mark.parametrize("dtype,chunk", [(torch.float32, 64), (torch.bfloat16, 0)])
def test_decode_after_prefill_equals_longer_prefill(dtype, chunk):
    G = lib()
    B, N, H, d = 3, 200, 2, 128
    inp = SI.gret_inputs(B, N + 1, H, d, dtype=dtype, seed=21)
    qd, kd, vd, gd = (inp[x].cuda() for x in ("q", "k", "v", "g"))
    _, s = G.gret_prefill_chunkwise(qd[:, :N].contiguous(), kd[:, :N].contiguous(),
                                    vd[:, :N].contiguous(), gd[:, :N].contiguous(),
                                    state_out=True, chunk=chunk)
    o_dec = G.gret_decode_step(qd[:, N].contiguous(), kd[:, N].contiguous(),
                               vd[:, N].contiguous(), gd[:, N].contiguous(), s)
    torch.cuda.synchronize()
    T = B * (N + 1)
    o_ref, s_ref = oracle.gret_recurrent(inp["q"].reshape(T, H, d), inp["k"].reshape(T, H, d),
                                         inp["v"].reshape(T, H, d), inp["g"].reshape(T, H),
                                         cu_seqlens=np.arange(B + 1) * (N + 1))
    last = o_ref.reshape(B, N + 1, H, d)[:, N]
    bf16 = dtype == torch.bfloat16
    tol = 1e-2 if bf16 else 1e-4
    assert_parity("o_decode", o_dec, last, tol, stored_bf16=bf16)
    assert_parity("state", s, s_ref, tol, stored_bf16=False)


def test_decode_bs64_after_4096_token_prefill_256_steps():
    """The batched-decode workload as the benchmark runs it: 64 sequences x 24 heads of 128,
    each state produced by gret_prefill_chunkwise over 4096 seeded tokens, then 256 chained
    gret_decode_step calls with per-step seeded q, k, v, g (same seeds as the benchmark).  The
    oracle runs the plain recurrence over the 4352 tokens of one head of every sequence
    ((b, h) = (b, (7 b + 3) mod 24)); decode outputs at steps 1, 64 and 256 and the final states
    are compared, so error that builds up over the 256 in-place fp32 updates after a
    tensor-core prefill is checked."""
    G = lib()
    c = SI.DECODE_BS64
    B, N0, S, H, d = c["B"], c["prefill_N"], c["steps"], c["H"], c["dk"]
    pre = SI.gret_inputs(B, N0, H, d, dtype=torch.bfloat16, seed=c["seed"], device="cuda")
    _, state = G.gret_prefill_chunkwise(pre["q"], pre["k"], pre["v"], pre["g"], state_out=True)
    st = SI.gret_inputs(B, S, H, d, dtype=torch.bfloat16, seed=10 * c["seed"], device="cuda")
    qs, ks, vs = (st[x].permute(1, 0, 2, 3).contiguous() for x in ("q", "k", "v"))
    gs = st["g"].permute(1, 0, 2).contiguous()
    check = (1, 64, 256)
    outs = {}
    for s in range(S):
        o = G.gret_decode_step(qs[s], ks[s], vs[s], gs[s], state)
        if s + 1 in check:
            outs[s + 1] = o.clone()
    torch.cuda.synchronize()
    bs = torch.arange(B, device="cuda")
    hs = (7 * bs + 3) % H
    L = N0 + S

    def seq(name):   # [B, N0 + S, d] for the sampled head of each sequence, packed [B*L, 1, d]
        x = torch.cat([pre[name][bs, :, hs], st[name][bs, :, hs]], dim=1)
        return x.reshape(B * L, 1, -1).cpu()

    gseq = torch.cat([pre["g"][bs, :, hs], st["g"][bs, :, hs]], dim=1).reshape(B * L, 1).cpu()
    o_ref, s_ref = oracle.gret_recurrent(seq("q"), seq("k"), seq("v"), gseq,
                                         cu_seqlens=np.arange(B + 1) * L)
    o_ref = o_ref.reshape(B, L, d)
    for s in check:
        assert_parity("o_step%d" % s, outs[s][bs, hs], o_ref[:, N0 + s - 1], 1e-2,
                      stored_bf16=True)
    assert_parity("state", state[bs, hs], s_ref[:, 0], 1e-2, stored_bf16=False, tight=1e-3)
