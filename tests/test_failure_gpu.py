"""The bounded waits of the tensor-core prefill give up, report, and leave the GPU usable.

Every wait of the kernel (between warp roles and between thread blocks) has a time limit; a
wait that runs out records GRET_ERR_TIMEOUT in the workspace, the block's other roles stop,
drain their copies, free tensor memory and exit.  The test makes a look-back wait run out
without any fault: through gret_prefill_chunkwise_testing it hands out span tickets from past
span 0 of every chain, so the flag those spans wait for is never set, and it shortens the
limit to 20 ms.  It then checks the reported status, and that a regular call afterwards, on a
fresh workspace, matches the fp64 oracle."""
import numpy as np
import pytest
import torch

import synth_inputs as SI
from gpu_cases import TC_TIGHT, lib
from oracle import oracle
from parity import assert_parity

pytestmark = pytest.mark.gpu


def test_lookback_wait_runs_out_and_is_reported():
    G = lib()
    # 1024 tokens = 8 chunks per chain, cut into spans of 2 chunks: 4 spans per chain, tickets
    # span-major (ticket = span * H + head), so first_ticket = H skips span 0 of both chains
    B, N, H = 1, 1024, 2
    inp = SI.gret_inputs(B, N, H, 128, dtype=torch.bfloat16, seed=95, device="cuda")
    q, k, v, g = inp["q"], inp["k"], inp["v"], inp["g"]
    _, _, ws = G.gret_prefill_chunkwise_testing(q, k, v, g, wait_ns=20_000_000, first_ticket=H)
    assert G.gret_workspace_status(ws) == 6          # GRET_ERR_TIMEOUT
    # a regular call right after, on a fresh workspace, is correct
    o, s = G.gret_prefill_chunkwise(q, k, v, g, state_out=True)
    torch.cuda.synchronize()
    ref_o, ref_s = oracle.gret_recurrent(q[0].cpu(), k[0].cpu(), v[0].cpu(), g[0].cpu())
    assert_parity("o", o[0], ref_o, 1e-2, stored_bf16=True, tight=TC_TIGHT)
    assert_parity("state", s, ref_s, 1e-2, stored_bf16=False, tight=TC_TIGHT)


def test_testing_entry_point_without_poison_is_the_regular_call():
    """first_ticket 0 with a short (but sufficient) limit: same result as the regular call, and
    the status stays OK."""
    G = lib()
    inp = SI.gret_inputs(1, 1500, 3, 128, dtype=torch.bfloat16, seed=96, device="cuda")
    q, k, v, g = inp["q"], inp["k"], inp["v"], inp["g"]
    o1, s1, ws = G.gret_prefill_chunkwise_testing(q, k, v, g, wait_ns=500_000_000,
                                                  first_ticket=0, state_out=True)
    assert G.gret_workspace_status(ws) == 0
    o2, s2 = G.gret_prefill_chunkwise(q, k, v, g, state_out=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_testing_entry_point_rejects_bad_limits():
    G = lib()
    inp = SI.gret_inputs(1, 10, 1, 128, dtype=torch.bfloat16, seed=97, device="cuda")
    for w in (0, 3_000_000_000):
        with pytest.raises(G.GretError):
            G.gret_prefill_chunkwise_testing(inp["q"], inp["k"], inp["v"], inp["g"], wait_ns=w,
                                             first_ticket=0)
