"""The allocation-free prefill entry point (gret_prefill_chunkwise_noalloc).

Some callers cannot allocate device memory at call time (a server that gives all device memory
to its own pool at start-up, or a latency-critical loop where cudaMalloc would synchronize the
device); this entry point serves them from a fixed 8 MiB scratch array inside the library.  The
test calls it through the C ABI twice in a row and checks each result against the regular entry
point (which takes a caller-allocated workspace) with the tolerance the parity tests use, and
checks that a request larger than the scratch is refused.  This file is collected last so that a
run stopping at the first failure has already run every other test; it passes on its own in a
fresh process too, since the first call sets up the scratch address.
"""
import numpy as np
import pytest
import torch

import synth_inputs as SI
from parity import parity_error

pytestmark = pytest.mark.gpu


def lib():
    import gated_retention_linear_b200 as G
    return G


@pytest.mark.parametrize("N,H", [(1000, 4), (32768, 24)])
def test_noalloc_matches_workspace_entry_point_twice(N, H):
    G = lib()
    inp = SI.gret_inputs(1, N, H, 128, dtype=torch.bfloat16, seed=77, device="cuda",
                         with_state=True)
    q, k, v, g, s0 = inp["q"], inp["k"], inp["v"], inp["g"], inp["s"]
    o_ref, s_ref = G.gret_prefill_chunkwise(q, k, v, g, state_in=s0, state_out=True)
    torch.cuda.synchronize()
    for _ in range(2):
        o = torch.empty_like(o_ref)
        s = torch.empty_like(s_ref)
        G.gret_prefill_chunkwise_noalloc(q, k, v, g, state_in=s0, state_out=s, o=o)
        torch.cuda.synchronize()
        assert parity_error(o.float().cpu().numpy(), o_ref.float().cpu().numpy(), True) <= 1e-2
        assert parity_error(s.cpu().numpy(), s_ref.cpu().numpy(), False) <= 1e-2


def test_noalloc_refuses_more_than_its_scratch():
    G = lib()
    # 4 sequences x 24 heads need 96 state-slot pairs (12 MiB) > 8 MiB of scratch
    inp = SI.gret_inputs(4, 300, 24, 128, dtype=torch.bfloat16, seed=78, device="cuda")
    with pytest.raises(G.GretError) as err:
        G.gret_prefill_chunkwise_noalloc(inp["q"], inp["k"], inp["v"], inp["g"])
    assert err.value.code == 4   # GRET_ERR_WORKSPACE
