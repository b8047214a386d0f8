"""The workspace-free per-channel linear, cider_w8a8_linear_pc_noalloc.

Some callers cannot allocate device memory: an application or framework that
owns all of the GPU's memory through its own pool, or code held to a memory
budget fixed at start-up.  They cannot pass the workspace that
cider_w8a8_linear_pc needs, so this entry point keeps its scratch in a fixed
array built into the library.  These tests call it through the C ABI and
check it against the entry point that takes a workspace and against the
oracle (sampled token rows, which are independent), on calls in a row with
different inputs and shapes, so that a call reading what the previous call
left in the shared scratch would be caught.  The last of them is large
enough for the per-channel GEMM to split K, so its partial sums also live in
the scratch.

This file is named to be collected last, and it passes both on its own in a
fresh process and after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import w8a8_activation_quantized_b200 as cider
from w8a8_activation_quantized_b200 import synth
from tests.parity import TOL, check_y, dev, host_bits

pytestmark = pytest.mark.gpu


def _call_noalloc(x, w, sw, y):
    """Straight through the C ABI: no workspace argument exists to pass."""
    M, K = x.shape
    N = w.shape[0]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return cider.lib().cider_w8a8_linear_pc_noalloc(
        ctypes.c_void_p(x.data_ptr()), 0, M, K, ctypes.c_void_p(w.data_ptr()), ctypes.c_void_p(sw.data_ptr()), N,
        ctypes.c_void_p(y.data_ptr()), 0, stream)


def _close(y, y_ref):
    """Row-relative fp16 tolerance used by every parity test in this suite."""
    a = oracle.as_float(host_bits(y), oracle.F16)
    b = oracle.as_float(host_bits(y_ref), oracle.F16)
    rowmax = np.abs(b).max(axis=1, keepdims=True)
    assert np.all(np.abs(a - b) <= TOL[oracle.F16] * rowmax)


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert cider.cider_is_available()


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    old = cider.cider_get_small_m_threshold()
    try:
        cider.cider_set_small_m_threshold(0)  # every call takes the tensor-core path, which uses the scratch
        # the third shape's CTA-pair tiles leave a partial last round, cut along K
        for (M, N, K, seed) in [(300, 1032, 4096, 1), (129, 264, 2560, 2), (1024, 5120, 8192, 3)]:
            xh = synth.activations(M, K, seed)
            x = torch.from_numpy(xh).cuda()
            qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed))
            w, s = dev(qw), dev(sw)
            y_ref = cider.cider_w8a8_linear_pc(x, w, s)
            y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
            assert _call_noalloc(x, w, s, y) == 0, cider.lib().cider_last_error()
            torch.cuda.synchronize()
            _close(y, y_ref)
            rows = np.unique(np.concatenate([[r for r in (0, 127, 128, 255, 256, M - 1) if r < M],
                                             np.random.default_rng(seed).choice(M, 10, replace=False)]))
            check_y(y[torch.from_numpy(rows).cuda()], oracle.linear_pc(xh[rows], qw, sw), oracle.F16)
    finally:
        cider.cider_set_small_m_threshold(old)
    cider.cider_device_status()


def test_noalloc_small_m_and_too_large():
    M, N, K = 1, 264, 2560  # decode-shaped: the fused kernel, no scratch touched
    x = torch.from_numpy(synth.activations(M, K, 3)).cuda()
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, 3))
    w, s = dev(qw), dev(sw)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    assert _call_noalloc(x, w, s, y) == 0
    _close(y, cider.cider_w8a8_linear_pc(x, w, s))
    check_y(y, oracle.linear_pc(synth.activations(M, K, 3), qw, sw), oracle.F16)
    # beyond the built-in scratch: rejected with a message, nothing launched
    big = torch.empty((8192, 8192), dtype=torch.float16, device="cuda")
    wb = torch.empty((16, 8192), dtype=torch.int8, device="cuda")
    sb = torch.ones((16,), dtype=torch.float32, device="cuda")
    yb = torch.empty((8192, 16), dtype=torch.float16, device="cuda")
    assert _call_noalloc(big, wb, sb, yb) == 1
    assert b"scratch" in cider.lib().cider_last_error()
