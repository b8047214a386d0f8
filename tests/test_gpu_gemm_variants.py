"""Every kernel variant of the per-channel GEMM against the oracle on small and
ragged shapes: single-CTA 128x80, 128x128 and 128x256 tiles, and the CTA-pair
256x256 and 256x192 tiles (tcgen05.mma.cta_group::2).  Bit-exact INT32 accumulators, and
the fused dequant within the row-relative tolerance."""
import numpy as np
import pytest
import torch

import oracle
import w8a8_activation_quantized_b200 as cider
from w8a8_activation_quantized_b200 import synth
from tests.parity import act, check_y, dev, dev_bits

pytestmark = pytest.mark.gpu

VARIANTS = {"single128": 1, "single256": 2, "pair256": 3, "single80": 4, "pair192": 5}


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    cider.cider_test_set_gemm_variant(0)
    cider.cider_device_status()


@pytest.fixture(params=sorted(VARIANTS))
def variant(request):
    cider.cider_test_set_gemm_variant(VARIANTS[request.param])
    yield request.param
    cider.cider_test_set_gemm_variant(0)


def _codes(M, N, K, seed):
    rng = np.random.default_rng(seed)
    q = rng.integers(-127, 128, size=(M, K), dtype=np.int64).astype(np.int8)
    w = rng.integers(-128, 128, size=(N, K), dtype=np.int64).astype(np.int8)
    return q, w


@pytest.mark.parametrize("M,N,K", [(256, 256, 128), (1, 8, 16), (257, 264, 272), (300, 520, 1040),
                                   (512, 1024, 2560), (130, 3080, 96), (1283, 4104, 272)])
def test_gemm_i32_variant(variant, M, N, K):
    q, w = _codes(M, N, K, seed=M * 3 + N + K)
    acc = cider.cider_test_gemm_i32(dev(q), dev(w))
    np.testing.assert_array_equal(acc.cpu().numpy(), oracle.gemm_i32(q, w))


@pytest.mark.parametrize("M,N,K", [(256, 256, 256), (300, 1032, 2560), (129, 264, 4096), (520, 2056, 1040)])
def test_linear_pc_variant(variant, M, N, K):
    cider.cider_set_small_m_threshold(4)
    x = act(M, K, seed=M + N + K)
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed=M + K))
    y = cider.cider_w8a8_linear_pc(dev_bits(x, oracle.F16), dev(qw), dev(sw))
    check_y(y, oracle.linear_pc(x, qw, sw), oracle.F16)


def test_pair_is_chosen_for_large_m():
    """The automatic choice sends the headline shape to the CTA-pair kernel; the
    result must equal the forced single-CTA result bit for bit (same arithmetic)."""
    M, N, K = 2048, 4096, 1024
    x = act(M, K, seed=5)
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed=5))
    xd, wd, sd = dev_bits(x, oracle.F16), dev(qw), dev(sw)
    cider.cider_test_set_gemm_variant(3)
    y_pair = cider.cider_w8a8_linear_pc(xd, wd, sd)
    cider.cider_test_set_gemm_variant(2)
    y_single = cider.cider_w8a8_linear_pc(xd, wd, sd)
    cider.cider_test_set_gemm_variant(0)
    y_auto = cider.cider_w8a8_linear_pc(xd, wd, sd)
    torch.cuda.synchronize()
    assert torch.equal(y_pair, y_single) and torch.equal(y_auto, y_pair)
    rows = np.arange(0, M, 97)
    check_y(y_auto, oracle.linear_pc(x[rows], qw, sw), oracle.F16, rows=rows)


@pytest.mark.parametrize("dt", [oracle.F16, oracle.BF16])
def test_pair192_is_chosen_at_m1024(dt):
    """M = 1024, N = 10240, K = 2560: 160 square pair tiles leave the 74 SM
    pairs a last round of 12 tiles, so the automatic choice takes the 256 x 192
    tile (216 tiles, three full rounds of narrower tiles).  Exact INT32 sums and
    the same dequant expression: equal to the square tile bit for bit; the
    last N tile holds 64 valid columns of 192."""
    M, N, K = 1024, 10240, 2560
    cider.cider_set_small_m_threshold(4)
    x = act(M, K, seed=1024, dt=dt)
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed=1025))
    xd, wd, sd = dev_bits(x, dt), dev(qw), dev(sw)
    outs = {}
    for name, v in (("auto", 0), ("pair192", 5), ("pair256", 3)):
        cider.cider_test_set_gemm_variant(v)
        outs[name] = cider.cider_w8a8_linear_pc(xd, wd, sd)
    cider.cider_test_set_gemm_variant(0)
    torch.cuda.synchronize()
    assert torch.equal(outs["auto"], outs["pair192"]) and torch.equal(outs["pair192"], outs["pair256"])
    rows = np.concatenate([np.arange(0, M, 61), [M - 1]])
    check_y(outs["auto"], oracle.linear_pc(x[rows], qw, sw, xdt=dt, ydt=dt), dt, rows=rows)


# ---------------------------------------------------------------- split K of the pair kernel

@pytest.mark.parametrize("splits", [2, 3, 5])
@pytest.mark.parametrize("M,N,K", [(300, 520, 2560), (513, 1032, 1280), (256, 256, 512)])
def test_linear_pc_pair_split_equals_unsplit(splits, M, N, K):
    """K pieces of the CTA-pair kernel add INT32 partial sums exactly and then
    dequantize with the fused epilogue's expression, so the split result equals
    the unsplit one bit for bit (and the oracle within tolerance)."""
    cider.cider_set_small_m_threshold(4)
    x = act(M, K, seed=M + N + K + splits)
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed=N + splits))
    xd, wd, sd = dev_bits(x, oracle.F16), dev(qw), dev(sw)
    cider.cider_test_set_gemm_variant(3)
    try:
        cider.cider_test_set_split_k(1)
        y_plain = cider.cider_w8a8_linear_pc(xd, wd, sd)
        cider.cider_test_set_split_k(splits)
        y_split = cider.cider_w8a8_linear_pc(xd, wd, sd)
    finally:
        cider.cider_test_set_split_k(0)
        cider.cider_test_set_gemm_variant(0)
    torch.cuda.synchronize()
    assert torch.equal(y_split, y_plain)
    rows = np.arange(0, M, 7)
    check_y(y_split, oracle.linear_pc(x[rows], qw, sw), oracle.F16, rows=rows)


@pytest.mark.parametrize("dt", [oracle.F16, oracle.BF16])
def test_linear_pc_tail_split_automatic(dt):
    """M=2048, N=2560, K=10240: 80 pair tiles on 74 SM pairs, so the automatic
    plan runs 74 whole tiles and cuts the 6 tiles of the last round into K
    pieces (80 k-blocks, enough to pay for the partial sums); the result
    equals the unsplit kernel's bit for bit."""
    M, N, K = 2048, 2560, 10240
    x = act(M, K, seed=31, dt=dt)
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed=32))
    xd, wd, sd = dev_bits(x, dt), dev(qw), dev(sw)
    big = torch.empty((cider.cider_workspace_bytes_mnk(M, N, K),), dtype=torch.uint8, device="cuda")
    assert big.numel() > cider.cider_workspace_bytes(M, K)
    y_auto = cider.cider_w8a8_linear_pc(xd, wd, sd, workspace=big)
    small = torch.empty((cider.cider_workspace_bytes(M, K),), dtype=torch.uint8, device="cuda")
    y_plain = cider.cider_w8a8_linear_pc(xd, wd, sd, workspace=small)
    torch.cuda.synchronize()
    assert torch.equal(y_auto, y_plain)
    rows = np.arange(0, M, 37)
    check_y(y_auto, oracle.linear_pc(x[rows], qw, sw, xdt=dt, ydt=dt), dt, rows=rows)


def test_mid_m_variants_agree_bit_for_bit():
    """M = 128, N = 10240 (the pages' table shape) takes the 128 x 80 tile by
    default (128 tiles in one round on 148 SMs); the INT32 sums are exact and
    the dequant expression is the same in every variant, so the 128 x 80,
    128 x 128 and 128 x 256 results are equal bit for bit."""
    M, N, K = 128, 10240, 2560
    cider.cider_set_small_m_threshold(4)
    x = act(M, K, seed=128)
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed=129))
    xd, wd, sd = dev_bits(x, oracle.F16), dev(qw), dev(sw)
    outs = {}
    for name, v in (("auto", 0), ("single80", 4), ("single128", 1), ("single256", 2)):
        cider.cider_test_set_gemm_variant(v)
        outs[name] = cider.cider_w8a8_linear_pc(xd, wd, sd)
    cider.cider_test_set_gemm_variant(0)
    torch.cuda.synchronize()
    for name in ("single80", "single128", "single256"):
        assert torch.equal(outs[name], outs["auto"]), name
    rows = np.arange(0, M, 9)
    check_y(outs["auto"], oracle.linear_pc(x[rows], qw, sw), oracle.F16, rows=rows)
