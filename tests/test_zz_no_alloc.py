"""The allocation-free prefill entry point (gret_prefill_chunkwise_noalloc).

Some callers cannot allocate device memory when they call: a server that hands all device
memory to its own pool at start-up, or a latency-critical loop in which a cudaMalloc would
synchronize the device.  This entry point serves them from a fixed 8 MiB scratch array inside
the library.  Each case calls it through the C ABI twice in a row and checks both results
against the fp64 oracle with the parity tests' tolerances, against the regular entry point
(which takes a caller-allocated workspace; the same kernel, so the results are identical), and
checks that the status call reports no timed-out wait.  The cases cover dense bf16 with entry
states (the tensor-core path), packed varlen bf16 with an empty sequence (whose span prefix
lives in the scratch at an offset that depends on the number of sequences), fp32 (the CUDA-core
path, which needs no scratch) and the full 32768-token x 24-head shape (heads sampled for the
oracle).  A request larger than the scratch is refused.  This file is collected last so that a
run stopping at the first failure has already run every other test; it passes on its own in a
fresh process too, since the first call sets up the scratch address.
"""
import numpy as np
import pytest
import torch

import synth_inputs as SI
from gpu_cases import TC_TIGHT
from oracle import oracle
from parity import assert_parity

pytestmark = pytest.mark.gpu


def lib():
    import gated_retention_linear_b200 as G
    return G


CASES = {
    "dense_bf16_N1000_H4": dict(lens=None, B=1, N=1000, H=4, d=128, dtype=torch.bfloat16),
    "varlen_bf16": dict(lens=[300, 0, 1000, 129], H=3, d=128, dtype=torch.bfloat16),
    "dense_fp32_d64": dict(lens=None, B=2, N=333, H=2, d=64, dtype=torch.float32),
    "dense_bf16_N32768_H24": dict(lens=None, B=1, N=32768, H=24, d=128, dtype=torch.bfloat16,
                                  heads=[0, 13, 23]),
}


@pytest.mark.parametrize("case", list(CASES))
def test_noalloc_matches_oracle_twice(case):
    G = lib()
    c = CASES[case]
    H, d, dt = c["H"], c["d"], c["dtype"]
    if c["lens"] is None:
        B, N = c["B"], c["N"]
        inp = SI.gret_inputs(B, N, H, d, dtype=dt, seed=77, with_state=True)
        q, k, v, g = (inp[x] for x in ("q", "k", "v", "g"))
        s0 = inp["s"]
        cu, T, cu_d = list(np.arange(B + 1) * N), B * N, None
        flat = lambda x: x.reshape(T, H, -1) if x.dim() == 4 else x.reshape(T, H)
    else:
        cu = SI.cu_seqlens_of(c["lens"])
        T = cu[-1]
        inp = SI.gret_inputs(1, T, H, d, dtype=dt, seed=78, g_mean=0.0, g_std=2.0)
        q, k, v, g = (inp[x][0] for x in ("q", "k", "v", "g"))
        s0 = SI.gret_inputs(len(c["lens"]), 1, H, d, seed=79, with_state=True)["s"]
        cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
        flat = lambda x: x
    hs = c.get("heads", list(range(H)))
    o_ref, s_ref = oracle.gret_recurrent(flat(q)[:, hs], flat(k)[:, hs], flat(v)[:, hs],
                                         flat(g)[:, hs], cu_seqlens=cu, state_in=s0[:, hs])
    dq, dk_, dv_, dg, ds0 = (x.cuda() for x in (q, k, v, g, s0))
    o_ws, s_ws = G.gret_prefill_chunkwise(dq, dk_, dv_, dg, cu_seqlens=cu_d, state_in=ds0,
                                          state_out=True)
    bf16 = dt == torch.bfloat16
    tol = 1e-2 if bf16 else 1e-4
    tight = TC_TIGHT if (bf16 and d == 128) else None
    for _ in range(2):
        o = torch.full_like(o_ws, float("nan"))
        s = torch.full_like(s_ws, float("nan"))
        G.gret_prefill_chunkwise_noalloc(dq, dk_, dv_, dg, cu_seqlens=cu_d, state_in=ds0,
                                         state_out=s, o=o)
        assert G.gret_prefill_noalloc_status() == 0
        assert_parity("o", flat(o)[:, hs], o_ref, tol, stored_bf16=bf16, tight=tight)
        assert_parity("state", s[:, hs], s_ref, tol, stored_bf16=False, tight=tight)
        assert torch.equal(o, o_ws) and torch.equal(s, s_ws)


def test_noalloc_refuses_more_than_its_scratch():
    G = lib()
    # 4 sequences x 24 heads need 96 state-slot pairs (12 MiB) > 8 MiB of scratch
    inp = SI.gret_inputs(4, 300, 24, 128, dtype=torch.bfloat16, seed=78, device="cuda")
    with pytest.raises(G.GretError) as err:
        G.gret_prefill_chunkwise_noalloc(inp["q"], inp["k"], inp["v"], inp["g"])
    assert err.value.code == 4   # GRET_ERR_WORKSPACE
