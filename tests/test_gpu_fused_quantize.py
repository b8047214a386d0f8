"""Activation quantization inside the GEMM launch (the per-channel linear at
mid-size M; the juejin post "在Mac上跑大模型，MLX 不是终点", section "W8A8 对称量
化：Cider 的选择", asks the quantize step to be fast enough not to become a
new bottleneck, and the workload asks for it fused into the GEMM prologue).

The fused launch leaves the codes and scales in the workspace, so they are
checked bit for bit against the oracle's quantization; the outputs against
the oracle within the row-relative tolerance and, bit for bit, against the
unfused path (same codes, same GEMM arithmetic).  Every GEMM variant (the
single-CTA 128x80, 128x128, 128x256 tiles and the CTA pair) runs fused, with
ragged shapes, K not a multiple of the 128-wide stage, bf16 input, and more
calls in a row than there are grid-barrier slots."""
import numpy as np
import pytest
import torch

import oracle
import w8a8_activation_quantized_b200 as cider
from w8a8_activation_quantized_b200 import synth
from tests.parity import act, check_y, dev, dev_bits, host_bits

pytestmark = pytest.mark.gpu
F16, BF16 = oracle.F16, oracle.BF16


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    old = cider.cider_get_small_m_threshold()
    cider.cider_set_small_m_threshold(4)
    yield
    cider.cider_test_set_fused_quantize(0)
    cider.cider_test_set_gemm_variant(0)
    cider.cider_set_small_m_threshold(old)
    cider.cider_device_status()


def _align256(v):
    return (v + 255) // 256 * 256


def _run(x_bits, dt, qw, sw, fused, variant=0):
    M, K = x_bits.shape
    N = qw.shape[0]
    ws = torch.zeros((cider.cider_workspace_bytes_mnk(M, N, K),), dtype=torch.uint8, device="cuda")
    cider.cider_test_set_fused_quantize(2 if fused else 1)
    cider.cider_test_set_gemm_variant(variant)
    try:
        y = cider.cider_w8a8_linear_pc(dev_bits(x_bits, dt), dev(qw), dev(sw), workspace=ws)
        torch.cuda.synchronize()
    finally:
        cider.cider_test_set_fused_quantize(0)
        cider.cider_test_set_gemm_variant(0)
    q = ws[: M * K].cpu().numpy().view(np.int8).reshape(M, K)
    sx = ws[_align256(M * K): _align256(M * K) + 4 * M].cpu().numpy().view(np.float32)
    return y, q, sx


def _rows(M, seed):
    fixed = [r for r in (0, 1, 127, 128, 255, 256, M - 1) if r < M]
    rnd = np.random.default_rng(seed).choice(M, size=min(M, 16), replace=False)
    return np.unique(np.concatenate([fixed, rnd]).astype(np.int64))


SHAPES = [(128, 10240, 2560), (200, 264, 1024), (5, 1032, 4096), (129, 520, 16), (300, 1032, 12304),
          (1024, 10240, 2560), (777, 2056, 1040)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_fused_codes_and_outputs(M, N, K):
    x = act(M, K, seed=M + N + K)
    if M > 3:
        x[3] = 0  # an all-zero token: scale 0, codes 0, output row 0
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed=N + K))
    y, q, sx = _run(x, F16, qw, sw, fused=True)
    q_ref, sx_ref = oracle.quantize_act(x, F16)
    np.testing.assert_array_equal(sx.view(np.uint32), sx_ref.view(np.uint32))
    np.testing.assert_array_equal(q, q_ref)
    rows = _rows(M, seed=M)
    check_y(y[torch.from_numpy(rows).cuda()], oracle.linear_pc(x[rows], qw, sw), F16)
    y_plain, _, _ = _run(x, F16, qw, sw, fused=False)
    assert torch.equal(y.view(torch.int16), y_plain.view(torch.int16))


@pytest.mark.parametrize("variant", [1, 2, 3, 4, 5])
def test_fused_every_variant(variant):
    M, N, K = 300, 1032, 2560
    x = act(M, K, seed=variant)
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed=variant + 1))
    y, q, _ = _run(x, F16, qw, sw, fused=True, variant=variant)
    np.testing.assert_array_equal(q, oracle.quantize_act(x, F16)[0])
    check_y(y, oracle.linear_pc(x, qw, sw), F16)


def test_fused_bf16():
    M, N, K = 260, 1032, 2560
    x = act(M, K, seed=9, dt=BF16)
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed=10))
    y, q, sx = _run(x, BF16, qw, sw, fused=True)
    q_ref, sx_ref = oracle.quantize_act(x, BF16)
    np.testing.assert_array_equal(q, q_ref)
    np.testing.assert_array_equal(sx.view(np.uint32), sx_ref.view(np.uint32))
    check_y(y, oracle.linear_pc(x, qw, sw, xdt=BF16, ydt=BF16), BF16)


def test_fused_more_calls_than_barrier_slots():
    """300 fused calls in a row on one stream (the grid-barrier slots, 256,
    are handed out in turn and each is left reset): the last outputs are
    still right and no bounded wait ran out."""
    M, N, K = 136, 264, 512
    xs = [act(M, K, seed=100 + i) for i in range(3)]
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed=7))
    xd = [dev_bits(x, F16) for x in xs]
    w, s = dev(qw), dev(sw)
    ws = torch.empty((cider.cider_workspace_bytes_mnk(M, N, K),), dtype=torch.uint8, device="cuda")
    cider.cider_test_set_fused_quantize(2)
    try:
        ys = [cider.cider_w8a8_linear_pc(xd[i % 3], w, s, workspace=ws) for i in range(300)]
        torch.cuda.synchronize()
    finally:
        cider.cider_test_set_fused_quantize(0)
    cider.cider_device_status()  # raises if any barrier or wait ran out
    for i in (297, 298, 299):
        check_y(ys[i], oracle.linear_pc(xs[i % 3], qw, sw), F16)
