"""GPU parity: every kernel against the oracle, through the C ABI.

Bit-exact: activation codes and scales, weight codes/scales/packing, the INT4
unpack, INT32 accumulators and per-group INT32 partials.  Outputs: within the
row-relative tolerance of tests/parity.py.  Sizes span several tiles and
ragged tails (M, N and K not multiples of the tile), both N-tile widths of
the per-channel GEMM, both group sizes, both activation dtypes, the fused
small-M path and the tensor-core path at the same M.
"""
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
    assert cider.cider_is_available(), "current device is not sm_100-family"
    yield
    torch.cuda.synchronize()
    cider.cider_device_status()  # raises CiderError if any bounded wait ran out


@pytest.fixture
def small_m(request):
    """Set the small-M threshold for one test, restore afterwards."""
    old = cider.cider_get_small_m_threshold()
    yield cider.cider_set_small_m_threshold
    cider.cider_set_small_m_threshold(old)


# ---------------------------------------------------------------- activation quantization

@pytest.mark.parametrize("dt", [F16, BF16])
@pytest.mark.parametrize("M,K", [(1, 16), (3, 256), (17, 2560), (129, 4096), (5, 4112),
                                 (7, 10240), (2, 12288), (3, 16400), (2, 40000)])
def test_quantize_act_bitexact(M, K, dt):
    x = act(M, K, seed=M * 7 + K, dt=dt)
    if M >= 3:
        x[1] = 0  # an all-zero token
    q_ref, s_ref = oracle.quantize_act(x, dt)
    q, s = cider.cider_quantize_act(dev_bits(x, dt))
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("dt", [F16, BF16])
def test_quantize_act_row_strides(dt):
    """A strided view (a slice of a wider buffer) quantizes to the same codes and
    scales as the oracle on those rows, into a strided q; the bytes between K
    and the stride of q are left untouched."""
    M, K, LDX, LDQ = 37, 1024, 1536, 1040
    wide = act(M, LDX, seed=41, dt=dt)
    xs = wide[:, 256:256 + K]
    qbuf = torch.full((M, LDQ), 77, dtype=torch.int8, device="cuda")
    xd = dev_bits(wide, dt)[:, 256:256 + K]
    q, s = cider.cider_quantize_act(xd, q=qbuf[:, :K])
    torch.cuda.synchronize()
    qo, so = oracle.quantize_act(np.ascontiguousarray(xs), dt)
    np.testing.assert_array_equal(qbuf[:, :K].cpu().numpy(), qo)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))
    assert bool((qbuf[:, K:] == 77).all())


def test_quantize_act_ties_and_extremes():
    K = 64
    rows = np.zeros((4, K), np.float32)
    rows[0, :8] = [127, 2.5, -2.5, 0.5, -0.5, 126.5, -126.5, 1.5]         # exact .5 ties, scale 1
    rows[1, :4] = [254, 5.0, -1.0, 3.0]                                    # scale 2 -> 2.5, -0.5, 1.5
    rows[2, :3] = [65504, -65504, 1e-7]                                    # fp16 extremes
    rows[3, :3] = [6e-8, -6e-8, 0]                                         # subnormal-only token
    x = rows.astype(np.float16).view(np.uint16)
    q_ref, s_ref = oracle.quantize_act(x)
    q, s = cider.cider_quantize_act(dev_bits(x, F16))
    np.testing.assert_array_equal(s.cpu().numpy(), s_ref)
    np.testing.assert_array_equal(q.cpu().numpy(), q_ref)
    assert list(q_ref[0, :8]) == [127, 3, -3, 1, -1, 127, -127, 2]


def test_quantize_act_bf16_ties_and_extremes():
    """bf16 tokens at the ends of the fp32 range, where the fast path's
    reciprocal of the scale is huge or infinite: bit-exact codes and scales."""
    K = 64
    rows = np.zeros((5, K), np.float64)
    rows[0, :8] = [127, 2.5, -2.5, 0.5, -0.5, 126.5, -126.5, 1.5]   # exact .5 ties, scale 1
    rows[1, :4] = [1e-37, -3e-38, 5e-38, 7.1e-38]                    # amax ~1e-37: a subnormal scale, 1/scale = inf
    rows[2, :4] = [2.0 ** -130, -(2.0 ** -131), 2.0 ** -133, 0.0]    # subnormal-only token
    rows[3, :4] = [3.38e38, -3.38e38, 1.0, 2.0e38]                   # near the largest bf16
    rows[4, :4] = [4e-36, -1.3e-36, 2.2e-36, 0.9e-36]                # scale ~3e-38: 1/scale finite and huge
    x = oracle.narrow(rows, BF16)
    q_ref, s_ref = oracle.quantize_act(x, BF16)
    q, s = cider.cider_quantize_act(dev_bits(x, BF16))
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(q.cpu().numpy(), q_ref)
    assert list(q_ref[0, :8]) == [127, 3, -3, 1, -1, 127, -127, 2]
    assert s_ref[1] > 0 and s_ref[1] < np.finfo(np.float32).tiny  # the subnormal-scale case is exercised


# ---------------------------------------------------------------- offline weight quantization

@pytest.mark.parametrize("N,K", [(8, 16), (264, 2560), (33 * 8, 10240)])
def test_quantize_weight_pc_bitexact(N, K):
    W = synth.weights(N, K, seed=N + K)
    w_ref, s_ref = oracle.quantize_weight_pc(W)
    w, s = cider.cider_quantize_weight_pc(dev(W))
    np.testing.assert_array_equal(s.cpu().numpy(), s_ref)
    np.testing.assert_array_equal(w.cpu().numpy(), w_ref)


@pytest.mark.parametrize("offset", [0, 1])
@pytest.mark.parametrize("N,K", [(37, 2048), (9, 2560), (7, 1020), (5, 2564), (3, 12), (10240, 2560)])
def test_quantize_weight_pc_widths_and_offsets(N, K, offset):
    """The per-channel INT8 quantizer and INT4 packer on several row widths,
    on aligned storage and 4 bytes past a 16-byte boundary, bit for bit."""
    W = synth.weights(N, K, seed=N * 7 + K)
    W[0, : min(K, 64)] = 0.0  # a partly zero row
    flat = torch.zeros(W.size + offset, dtype=torch.float32, device="cuda")
    flat[offset:] = torch.from_numpy(W.ravel()).cuda()
    Wd = flat[offset:].view(N, K)
    w_ref, s_ref = oracle.quantize_weight_pc(W)
    w, s = cider.cider_quantize_weight_pc(Wd)
    np.testing.assert_array_equal(s.cpu().numpy(), s_ref)
    np.testing.assert_array_equal(w.cpu().numpy(), w_ref)
    p_ref, s4_ref = oracle.quantize_weight_int4_pc(W)
    p, s4 = cider.cider_pack_weight_int4_pc(Wd)
    np.testing.assert_array_equal(s4.cpu().numpy().view(np.uint32), s4_ref.view(np.uint32))
    np.testing.assert_array_equal(p.cpu().numpy(), p_ref)


@pytest.mark.parametrize("gs", [64, 128])
@pytest.mark.parametrize("N,K", [(8, 256), (136, 2560), (5, 1920), (3, 128 * 7), (2560, 10240)])
def test_quantize_weight_pg_bitexact(N, K, gs):
    W = synth.weights(N, K, seed=3 * N + K)
    w_ref, s_ref = oracle.quantize_weight_pg(W, gs)
    w, s = cider.cider_quantize_weight_pg(dev(W), gs)
    np.testing.assert_array_equal(s.cpu().numpy(), s_ref.T)  # GPU scales are group-major [G][N]
    np.testing.assert_array_equal(w.cpu().numpy(), w_ref)


@pytest.mark.parametrize("gs", [64, 128])
@pytest.mark.parametrize("N,K", [(8, 128), (136, 4096), (5, 640), (12288, 4096)])
def test_pack_weight_int4_bitexact(N, K, gs):
    W = synth.weights(N, K, seed=5 * N + K)
    W[0, :gs] = 0.0  # an all-zero group
    p_ref, s_ref = oracle.quantize_weight_int4_pg(W, gs)
    p, s = cider.cider_pack_weight_int4_pg(dev(W), gs)
    np.testing.assert_array_equal(s.cpu().numpy(), s_ref.T)
    np.testing.assert_array_equal(p.cpu().numpy(), p_ref)


def test_unpack_int4_all_bytes():
    packed = np.tile(np.arange(256, dtype=np.uint8), 4).reshape(32, 32)  # K = 64
    w = cider.cider_test_unpack_int4(dev(packed), 64)
    np.testing.assert_array_equal(w.cpu().numpy(), oracle.unpack_int4(packed, 64))


# ---------------------------------------------------------------- INT32 accumulators

def _codes(M, N, K, seed):
    rng = np.random.default_rng(seed)
    q = rng.integers(-127, 128, size=(M, K), dtype=np.int64).astype(np.int8)
    w = rng.integers(-128, 128, size=(N, K), dtype=np.int64).astype(np.int8)
    return q, w


@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (1, 8, 16), (129, 264, 272), (300, 520, 1040),
                                   (256, 1024, 2560), (64, 136, 4096),
                                   (1280, 4096, 256), (1283, 4104, 272)])  # the last two use BN=256
def test_gemm_i32_bitexact(M, N, K):
    q, w = _codes(M, N, K, seed=M + N + K)
    acc = cider.cider_test_gemm_i32(dev(q), dev(w))
    np.testing.assert_array_equal(acc.cpu().numpy(), oracle.gemm_i32(q, w))


def test_gemm_i32_extremes():
    """All-(-128) weights against all-127 codes at the largest K: |acc| = 127*128*K."""
    M, N, K = 130, 136, 16384
    q = np.full((M, K), 127, np.int8)
    q[1::2] = -127
    w = np.full((N, K), -128, np.int8)
    acc = cider.cider_test_gemm_i32(dev(q), dev(w)).cpu().numpy()
    np.testing.assert_array_equal(acc[0], np.full(N, -127 * 128 * K, np.int64))
    np.testing.assert_array_equal(acc[1], np.full(N, 127 * 128 * K, np.int64))


@pytest.mark.parametrize("gs", [64, 128])
@pytest.mark.parametrize("M,N,K", [(130, 136, 256), (128, 256, 1024), (3, 8, 128), (257, 392, 640)])
def test_gemm_i32_grouped_bitexact(M, N, K, gs):
    if K % gs:
        pytest.skip("gs must divide K")
    q, w = _codes(M, N, K, seed=2 * M + N + K + gs)
    acc_g = cider.cider_test_gemm_i32_grouped(dev(q), dev(w), gs)
    np.testing.assert_array_equal(acc_g.cpu().numpy(), oracle.gemm_i32_grouped(q, w, gs))


def test_gemm_i32_grouped_odd_group_count():
    """K = 192 with gs = 64: the last 128-wide stage holds one group only."""
    q, w = _codes(129, 264, 192, seed=11)
    acc_g = cider.cider_test_gemm_i32_grouped(dev(q), dev(w), 64)
    np.testing.assert_array_equal(acc_g.cpu().numpy(), oracle.gemm_i32_grouped(q, w, 64))


# ---------------------------------------------------------------- whole linears

PC_SHAPES = [(16, 128, 256), (1, 512, 2560), (2, 264, 1024), (4, 128, 512), (5, 264, 2560),
             (17, 520, 1040), (128, 1024, 2560), (300, 1032, 4096), (1283, 4104, 272)]


def _pc_inputs(M, N, K, dt, seed):
    x = act(M, K, seed, dt)
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed))
    return x, qw, sw


@pytest.mark.parametrize("M,N,K", PC_SHAPES)
@pytest.mark.parametrize("xdt,ydt", [(F16, F16), (BF16, BF16), (F16, BF16)])
def test_linear_pc(M, N, K, xdt, ydt):
    x, qw, sw = _pc_inputs(M, N, K, xdt, seed=M * 31 + N + K)
    y_ref = oracle.linear_pc(x, qw, sw, xdt=xdt, ydt=ydt)
    y = cider.cider_w8a8_linear_pc(dev_bits(x, xdt), dev(qw), dev(sw),
                                   out_dtype=torch.float16 if ydt == F16 else torch.bfloat16)
    check_y(y, y_ref, ydt)


@pytest.mark.parametrize("M", [1, 2, 3, 4, 8, 16])
def test_linear_pc_small_m_and_tensor_core_paths_agree(M, small_m):
    N, K = 264, 2560
    x, qw, sw = _pc_inputs(M, N, K, F16, seed=M)
    y_ref = oracle.linear_pc(x, qw, sw)
    small_m(16)
    y_small = cider.cider_w8a8_linear_pc(dev_bits(x, F16), dev(qw), dev(sw))
    small_m(0)
    y_tc = cider.cider_w8a8_linear_pc(dev_bits(x, F16), dev(qw), dev(sw))
    check_y(y_small, y_ref, F16)
    check_y(y_tc, y_ref, F16)


def test_linear_pc_zero_token_and_empty():
    M, N, K = 6, 136, 512
    x, qw, sw = _pc_inputs(M, N, K, F16, seed=99)
    x[2] = 0
    y = cider.cider_w8a8_linear_pc(dev_bits(x, F16), dev(qw), dev(sw))
    check_y(y, oracle.linear_pc(x, qw, sw), F16)
    assert not y[2].any()
    y0 = cider.cider_w8a8_linear_pc(torch.empty((0, K), dtype=torch.float16, device="cuda"), dev(qw), dev(sw))
    assert y0.shape == (0, N)


PG_SHAPES = [(1, 256, 1024), (3, 136, 2560), (16, 128, 256), (129, 264, 1280), (300, 520, 2560)]


@pytest.mark.parametrize("gs", [64, 128])
@pytest.mark.parametrize("M,N,K", PG_SHAPES)
@pytest.mark.parametrize("xdt", [F16, BF16])
def test_linear_pg(M, N, K, gs, xdt):
    x = act(M, K, seed=M + N + K + gs, dt=xdt)
    qw, sw = oracle.quantize_weight_pg(synth.weights(N, K, seed=N + gs), gs)
    y_ref = oracle.linear_pg(x, qw, sw, gs, xdt=xdt, ydt=xdt)
    y = cider.cider_w8a8_linear_pg(dev_bits(x, xdt), dev(qw), dev(np.ascontiguousarray(sw.T)), gs)
    check_y(y, y_ref, xdt)


@pytest.mark.parametrize("gs", [64, 128])
@pytest.mark.parametrize("M,N,K", PG_SHAPES + [(130, 264, 192)])
def test_w4a8_linear_pg(M, N, K, gs):
    if K % gs:
        pytest.skip("gs must divide K")
    x = act(M, K, seed=3 * M + N + K + gs)
    packed, sw = oracle.quantize_weight_int4_pg(synth.weights(N, K, seed=2 * N + gs), gs)
    y_ref = oracle.w4a8_linear_pg(x, packed, sw, gs)
    y = cider.cider_w4a8_linear_pg(dev_bits(x, F16), dev(packed), dev(np.ascontiguousarray(sw.T)), gs)
    check_y(y, y_ref, F16)


@pytest.mark.parametrize("mode", ["pg", "w4"])
@pytest.mark.parametrize("M", [1, 2, 4, 16])
def test_grouped_small_m_and_tensor_core_paths_agree(mode, M, small_m):
    N, K, gs = 264, 1280, 64
    x = act(M, K, seed=M + 5)
    W = synth.weights(N, K, seed=M)
    if mode == "pg":
        qw, sw = oracle.quantize_weight_pg(W, gs)
        y_ref = oracle.linear_pg(x, qw, sw, gs)
        run = lambda: cider.cider_w8a8_linear_pg(dev_bits(x, F16), dev(qw), dev(np.ascontiguousarray(sw.T)), gs)
    else:
        packed, sw = oracle.quantize_weight_int4_pg(W, gs)
        y_ref = oracle.w4a8_linear_pg(x, packed, sw, gs)
        run = lambda: cider.cider_w4a8_linear_pg(dev_bits(x, F16), dev(packed), dev(np.ascontiguousarray(sw.T)), gs)
    small_m(16)
    check_y(run(), y_ref, F16)
    small_m(0)
    check_y(run(), y_ref, F16)


def test_gemm_q_entry_points_match_linears():
    """The pre-quantized entry points run the same arithmetic as the linears,
    bit for bit.  The per-group linears would split K here (6 tiles), which
    adds fp32 piece sums in another order, so splitting is turned off; the
    split path has its own tests against the oracle."""
    cider.cider_test_set_split_k(1)
    try:
        _gemm_q_entry_points_match_linears()
    finally:
        cider.cider_test_set_split_k(0)


def _gemm_q_entry_points_match_linears():
    M, N, K, gs = 200, 264, 1024, 128
    x = act(M, K, seed=1)
    xd = dev_bits(x, F16)
    q, s = cider.cider_quantize_act(xd)
    W = synth.weights(N, K, seed=1)
    qw, sw = oracle.quantize_weight_pc(W)
    torch.testing.assert_close(cider.cider_w8a8_gemm_pc_q(q, s, dev(qw), dev(sw)),
                               cider.cider_w8a8_linear_pc(xd, dev(qw), dev(sw)), rtol=0, atol=0)
    qg, sg = oracle.quantize_weight_pg(W, gs)
    sgt = dev(np.ascontiguousarray(sg.T))
    torch.testing.assert_close(cider.cider_w8a8_gemm_pg_q(q, s, dev(qg), sgt, gs),
                               cider.cider_w8a8_linear_pg(xd, dev(qg), sgt, gs), rtol=0, atol=0)
    p4, s4 = oracle.quantize_weight_int4_pg(W, gs)
    s4t = dev(np.ascontiguousarray(s4.T))
    torch.testing.assert_close(cider.cider_w4a8_gemm_pg_q(q, s, dev(p4), s4t, gs),
                               cider.cider_w4a8_linear_pg(xd, dev(p4), s4t, gs), rtol=0, atol=0)


# ---------------------------------------------------------------- decoder MLP producer

@pytest.mark.parametrize("dt", [F16, BF16])
@pytest.mark.parametrize("M,F", [(3, 256), (17, 12288), (2, 4112)])
def test_silu_mul_quantize(M, F, dt):
    g = act(M, F, seed=M + F, dt=dt)
    u = act(M, F, seed=M + F + 1, dt=dt)
    q, s, a = cider.cider_silu_mul_quantize(dev_bits(g, dt), dev_bits(u, dt), want_a=True)
    a_bits = host_bits(a)
    # a within one unit in the last place of the oracle's fp64-evaluated value
    a_ref = oracle.silu_mul(g, u, dt)
    ulp_gap = np.abs(a_bits.view(np.int16).astype(np.int32) - a_ref.view(np.int16).astype(np.int32))
    assert ulp_gap.max() <= 1
    # the codes are exactly the quantization of the kernel's own a (teacher forcing)
    q_ref, s_ref = oracle.quantize_act(a_bits, dt)
    np.testing.assert_array_equal(s.cpu().numpy(), s_ref)
    np.testing.assert_array_equal(q.cpu().numpy(), q_ref)
    # and the same without writing a
    q2, s2, _ = cider.cider_silu_mul_quantize(dev_bits(g, dt), dev_bits(u, dt))
    assert torch.equal(q2, q) and torch.equal(s2, s)
