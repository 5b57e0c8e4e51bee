"""The packed variable-length workload end to end: 8 sequences of seeded lengths in
[1024, 65536], 24 heads of 128, harsher gates g ~ N(0, 2); the varlen chunkwise prefill's bf16
output goes straight into the per-head GroupNorm * swish(X W_G) gate with X [T, 3072] and
W_G [3072, 3072] ("路线二：Multi-Head Gated Retention").  The oracle computes its own retention
output from the same inputs (the plain recurrence, all heads), rounds it to bf16 as the library
stores it, and applies its GroupNorm gate to the first and last row of every sequence and a
seeded sample of rows; nothing it uses comes from the GPU."""
import numpy as np
import pytest
import torch

import synth_inputs as SI
from gpu_cases import TC_TIGHT, lib
from oracle import oracle
from parity import assert_parity, gate_o_rounding_allowance

pytestmark = pytest.mark.gpu


def test_varlen_prefill_then_groupnorm_gate():
    G = lib()
    c = SI.VARLEN_EPILOGUE
    H, d, D = c["H"], c["dk"], c["D"]
    lens = SI.varlen_lengths(c["n_seqs"], c["lo"], c["hi"], seed=c["seed"])
    cu = SI.cu_seqlens_of(lens)
    T = cu[-1]
    inp = SI.gret_inputs(1, T, H, d, dtype=torch.bfloat16, g_mean=c["g_mean"], g_std=c["g_std"],
                         seed=c["seed"], device="cuda")
    q, k, v, g = (inp[x][0] for x in ("q", "k", "v", "g"))
    ep = SI.epilogue_inputs(T, D, H * d, seed=c["seed"], device="cuda")
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    o, s = G.gret_prefill_chunkwise(q, k, v, g, cu_seqlens=cu_d, state_out=True)
    y = G.gret_groupnorm_gate(o.view(T, H * d), ep["x"], ep["w_g"], H, eps=c["eps"])
    torch.cuda.synchronize()

    o_ref, s_ref = oracle.gret_recurrent(q.cpu(), k.cpu(), v.cpu(), g.cpu(), cu_seqlens=cu)
    rng = np.random.default_rng(c["seed"])
    ends = {cu[i] for i in range(len(lens))} | {cu[i + 1] - 1 for i in range(len(lens))}
    rows = sorted(ends | set(rng.integers(0, T, 64).tolist()))
    ro = oracle._round_bf16(o_ref[rows].reshape(len(rows), H * d))
    x_rows, w_g = ep["x"][rows].cpu(), ep["w_g"].cpu()
    y_ref = oracle.groupnorm_gate(ro, x_rows, w_g, H, eps=c["eps"])
    assert_parity("o", o[rows], o_ref[rows], 1e-2, stored_bf16=True, tight=TC_TIGHT)
    assert_parity("state", s, s_ref, 1e-2, stored_bf16=False, tight=TC_TIGHT)
    a = gate_o_rounding_allowance(ro, x_rows, w_g, H, eps=c["eps"])
    assert_parity("y", y[rows], y_ref, 1e-2, stored_bf16=True, allowance=a)
