"""Parity metric between a GPU result and the fp64 oracle.

The stated bar is max|GPU - oracle| / rms(oracle) <= 1e-4 with fp32 inputs and <= 1e-2 with
bf16 inputs, per output tensor.  Outputs stored in bf16 carry, on top of the arithmetic error,
the rounding to the stored format: up to half a bf16 ulp, 2^-8 |x| in the worst case, which on
its own exceeds 1e-2 rms for every element larger than 2.56 rms.  For bf16 outputs the
rounding allowance (half an ulp at the element's magnitude) is therefore taken off each
element's difference before the bar is applied; fp32 outputs get no allowance.
"""
import numpy as np
import torch


def _np(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def bf16_half_ulp(x):
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 8.0), 0.0)


def parity_error(gpu, ref, stored_bf16):
    g, r = _np(gpu), _np(ref)
    assert g.shape == r.shape, (g.shape, r.shape)
    if r.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(r * r)))
    if rms == 0.0:
        return float(np.max(np.abs(g)))
    d = np.abs(g - r)
    if stored_bf16:
        d = np.maximum(d - bf16_half_ulp(np.maximum(np.abs(g), np.abs(r))), 0.0)
    return float(np.max(d)) / rms


def assert_parity(name, gpu, ref, tol, stored_bf16):
    g = _np(gpu)
    assert np.all(np.isfinite(g)), "%s: non-finite values in the GPU result" % name
    err = parity_error(g, ref, stored_bf16)
    assert err <= tol, "%s: max|d|/rms = %.3e > %.1e" % (name, err, tol)
    return err
