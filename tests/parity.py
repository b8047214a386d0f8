"""Helpers shared by the GPU parity tests: moving seeded inputs to the device
and comparing GPU outputs with the oracle's."""
import numpy as np
import torch

import oracle

# fp16 output: |y_gpu - y_oracle| <= 1e-3 * max_n |y_oracle[m, n]| per row (the
# workload's stated tolerance; one fp16 ulp is at most 2^-10 |y| < 1e-3 |y|, so
# any single-rounding difference passes).  bf16 keeps 8 significant bits, so one
# bf16 ulp is up to 2^-7 |y|: its tolerance is 2^-7 * row max, derived the same way.
TOL = {oracle.F16: 1e-3, oracle.BF16: 2.0 ** -7}


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def dev_bits(bits, dt):
    """uint16 bit patterns (or an fp16 array) -> device fp16/bf16 tensor."""
    b = np.ascontiguousarray(np.asarray(bits).view(np.uint16)).view(np.int16)
    t = torch.from_numpy(b).cuda()
    return t.view(torch.float16 if dt == oracle.F16 else torch.bfloat16)


def host_bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def act(M, K, seed, dt=oracle.F16, **kw):
    from w8a8_activation_quantized_b200 import synth
    x = synth.activations(M, K, seed, dtype="f16" if dt == oracle.F16 else "bf16", **kw)
    return x.view(np.uint16)


def check_y(y_gpu, y_ref_bits, dt, rows=None):
    """Row-relative comparison of a GPU output with the oracle's bit patterns."""
    yg = oracle.as_float(host_bits(y_gpu), dt)
    yr = oracle.as_float(y_ref_bits, dt)
    if rows is not None:
        yg = yg[rows]
    assert yg.shape == yr.shape, (yg.shape, yr.shape)
    assert np.all(np.isfinite(yg)) and np.all(np.isfinite(yr))
    rowmax = np.abs(yr).max(axis=1, keepdims=True)
    err = np.abs(yg - yr)
    tol = TOL[dt] * rowmax
    zero = (rowmax[:, 0] == 0)
    assert np.all(yg[zero] == 0), "rows whose reference is all zero must be exactly zero"
    bad = err > tol
    if bad.any():
        m, n = np.argwhere(bad)[0]
        raise AssertionError(
            f"{bad.sum()} outputs out of tolerance; first at ({m},{n}): gpu={yg[m, n]!r} "
            f"oracle={yr[m, n]!r} rowmax={rowmax[m, 0]!r} max rel err={np.max(err / np.maximum(rowmax, 1e-30)):.3g}")
    return float(np.max(err / np.maximum(rowmax, 1e-30)))
