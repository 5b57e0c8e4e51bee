"""Parity metric between a GPU result and the fp64 oracle.

The stated bar is max|GPU - oracle| / rms(oracle) <= 1e-4 with fp32 inputs and <= 1e-2 with
bf16 inputs, per output tensor.  Outputs stored in bf16 carry, on top of the arithmetic error,
the rounding to the stored format: up to half a bf16 ulp, 2^-8 |x| in the worst case, which on
its own exceeds 1e-2 rms for every element larger than 2.56 rms.  For bf16 outputs the
rounding allowance (half an ulp at the element's magnitude) is therefore taken off each
element's difference before the bar is applied; fp32 outputs get no allowance.

Every error measured through assert_parity is also recorded (test, tensor, error), and written
as JSON at the end of the session when GRET_PARITY_LOG names a file, so that the achieved
errors, not only the pass/fail against the bar, are on record.
"""
import os

import numpy as np
import torch

ERRORS = []


def _np(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def bf16_half_ulp(x):
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 8.0), 0.0)


def parity_error(gpu, ref, stored_bf16, allowance=None):
    """max over elements of (|gpu - ref| - allowances) / rms(ref).  `allowance`, if given, is an
    extra per-element bound (same shape) taken off before the maximum."""
    g, r = _np(gpu), _np(ref)
    assert g.shape == r.shape, (g.shape, r.shape)
    if r.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(r * r)))
    if rms == 0.0:
        return float(np.max(np.abs(g)))
    d = np.abs(g - r)
    if stored_bf16:
        d = d - bf16_half_ulp(np.maximum(np.abs(g), np.abs(r)))
    if allowance is not None:
        d = d - np.asarray(allowance, dtype=np.float64)
    return float(np.max(np.maximum(d, 0.0))) / rms


def record(name, err):
    test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
    ERRORS.append({"test": test, "tensor": name, "err": err})


def assert_parity(name, gpu, ref, tol, stored_bf16, tight=None, allowance=None):
    """Assert the parity bar `tol`; `tight`, when given, is a second, much lower bar near the
    error the kernel actually reaches, so that a regression well inside `tol` still fails."""
    g = _np(gpu)
    assert np.all(np.isfinite(g)), "%s: non-finite values in the GPU result" % name
    err = parity_error(g, ref, stored_bf16, allowance)
    record(name, err)
    assert err <= tol, "%s: max|d|/rms = %.3e > %.1e" % (name, err, tol)
    if tight is not None:
        assert err <= tight, "%s: max|d|/rms = %.3e within the bar %.1e but above the %.1e " \
                             "this kernel reaches" % (name, err, tol, tight)
    return err


def gate_o_rounding_allowance(o_bf16, x, w_g, H, eps=1e-5, gn_weight=None):
    """Per-element bound on how far y = GN_h(o) * swish(x W_G) moves when the retention output o
    (stored in bf16 on both sides) differs by one bf16 ulp in an element.

    Where the exact o lies within the kernel's error of a bf16 rounding midpoint, the GPU and the
    oracle round it to neighbouring values, one ulp apart.  GroupNorm and the gate carry that ulp
    into y as ulp(o_i) |gn_w_i| / sigma_head |swish(z_i)|, z = x W_G; the changes of the head's
    mean and variance that one element makes are a factor 1/d_v smaller and are not counted.
    o_bf16 [R, H d], x [R, D], w_g [D, H d]; fp64 throughout.  Returns [R, H d]."""
    o = _np(o_bf16)
    R, F = o.shape
    d = F // H
    z = _np(x) @ _np(w_g)
    sw = np.abs(z / (1.0 + np.exp(-z)))
    oh = o.reshape(R, H, d)
    sigma = np.sqrt(oh.var(axis=2) + eps)
    a = (2.0 * bf16_half_ulp(oh) / sigma[:, :, None]).reshape(R, F) * sw
    if gn_weight is not None:
        a = a * np.abs(_np(gn_weight))[None, :]
    return a
