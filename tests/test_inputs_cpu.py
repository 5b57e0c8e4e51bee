"""Properties of the seeded input generators that the parity tests rely on (no GPU)."""
import torch

import synth_inputs as SI


def test_exact_projection_inputs_make_the_projection_exact_in_fp32():
    """layer_inputs(exact_projection=True) draws x and W on dyadic grids on which every partial
    sum of x W is an exact fp32 number: the fp32 product, in two summation orders, equals the
    fp64 one, so any two implementations round the same q, k, v to bf16."""
    li = SI.layer_inputs(48, 3072, 24, 128, seed=6, exact_projection=True)
    x, w = li["x"], li["w_qkvg"]
    exact = x.double() @ w.double()
    a = (x.float() @ w.float()).double()
    b = (torch.flip(x.float(), [1]) @ torch.flip(w.float(), [0])).double()
    assert torch.equal(a, exact) and torch.equal(b, exact)
    assert 0.8 < float(exact[:, :3072].std()) < 1.2          # q columns keep unit scale
    assert 1.0 < float(exact[:, 9216:].mean()) < 3.0         # gate logits around 2
