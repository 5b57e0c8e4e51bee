"""GPU parity of gret_groupnorm_gate (per-head GroupNorm of O times swish(X W_G), the output
epilogue of "路线二：Multi-Head Gated Retention") against the fp64 oracle, through the C ABI."""
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


def run(T, H, D, seed, affine=False, rows=None, eps=1e-5):
    G = lib()
    F = H * 128
    ep = SI.epilogue_inputs(T, D, F, seed=seed, affine=affine)
    o = SI.gret_inputs(1, T, H, 128, dtype=torch.bfloat16, seed=seed + 1)["v"][0].reshape(T, F)
    o = (o * 11.3).to(torch.bfloat16)            # typical retention-output scale, O(1)
    gw = ep.get("gn_weight")
    gb = ep.get("gn_bias")
    y = G.gret_groupnorm_gate(o.cuda(), ep["x"].cuda(), ep["w_g"].cuda(), H,
                              gn_weight=None if gw is None else gw.cuda(),
                              gn_bias=None if gb is None else gb.cuda(), eps=eps)
    torch.cuda.synchronize()
    y_ref = oracle.groupnorm_gate(o, ep["x"], ep["w_g"], H, gn_weight=gw, gn_bias=gb, eps=eps,
                                  rows=rows)
    yg = y.float().cpu().numpy()
    if rows is not None:
        yg = yg[np.asarray(rows)]
    return assert_parity("y", yg, y_ref, 1e-2, stored_bf16=True)


@pytest.mark.parametrize("T", [1, 127, 128, 300])
def test_ragged_tokens(T):
    run(T, 4, 256, seed=T)


def test_affine_and_wide_k():
    run(200, 2, 1024, seed=3, affine=True)


def test_many_tiles():
    run(1000, 8, 512, seed=4)


def test_3b_shape_sampled_rows():
    # config-5 shape: H = 24 heads of 128, D = 3072; rows sampled (the oracle GEMM is fp64)
    T = 20000
    rng = np.random.default_rng(0)
    rows = sorted(set(rng.integers(0, T, 256).tolist()) | {0, T - 1})
    run(T, 24, 3072, seed=5, rows=rows)
