"""Decode attention on the GPU (Cider README, section "优化 SDPA（解码注意
力）") against the float64 oracle: the pages' configurations (MHA, GQA4, GQA8
at D = 128) up to N = 32K, ragged sequence lengths (one key, fewer keys than
a chunk's streams, chunk tails), other group sizes, bf16, peaked weights
(queries scaled by 8, outputs of order one), a maximum that arrives in the
last chunk, and the argument checks.

Tolerance (tests/sdpa_tolerance.py): element by element, one unit of the
output format at the output itself plus a bound on the kernels' fp32 error
that scales with sum_j p_j |v_j| and with the depth of the kernels'
summation, derived from the arithmetic they do.  tests/test_sdpa_tolerance.py
shows on the host that this bound rejects a dropped chunk, an unrescaled
chunk partial and a dropped key stream.  The pages report a maximum
difference of 1.22e-4 (fp16) against their reference; the largest
difference seen here is printed by test_sdpa_max_difference_report."""
import numpy as np
import pytest
import torch

import oracle
from oracle import sdpa
import w8a8_activation_quantized_b200 as cider
from tests.parity import dev_bits, host_bits
from tests import sdpa_tolerance as tl

pytestmark = pytest.mark.gpu
D = 128
MAX_DIFF = {}


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    cider.cider_device_status()


def _num_sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _check(H_q, H_kv, N, seed, dt=oracle.F16, kind="diffuse"):
    q, k, v = tl.make_inputs(kind, H_q, H_kv, N, seed, dt)
    out = cider.cider_sdpa_decode(dev_bits(q, dt), dev_bits(k, dt), dev_bits(v, dt))
    got = host_bits(out)
    ref = sdpa.sdpa_decode(q, k, v, dt)
    assert np.all(np.isfinite(oracle.as_float(got, dt)))
    n_bad, max_diff = tl.violations(ref, got, q, k, v, dt, _num_sms())
    MAX_DIFF[(kind, H_q, H_kv, N, dt)] = max_diff
    assert n_bad == 0, f"{n_bad} outputs out of tolerance; max |diff| = {max_diff:.3g}"
    return out


def test_sdpa_tc_operand_layout_probe():
    """The tensor-core kernel reads V as an MN-major operand; of the two orders
    of the descriptor's offset fields (mode 2: atoms along MN in the leading
    field; mode 3: exchanged) exactly one reproduces the oracle.  The default
    (mode 0) uses mode 2's order, so this test also pins the default."""
    q, k, v = tl.make_inputs("peaked", 32, 8, 1024, seed=11)
    ref = sdpa.sdpa_decode(q, k, v, oracle.F16)
    ok = {}
    for mode in (2, 3):
        cider.cider_test_set_sdpa_kernel(mode)
        try:
            out = cider.cider_sdpa_decode(dev_bits(q, oracle.F16), dev_bits(k, oracle.F16), dev_bits(v, oracle.F16))
            torch.cuda.synchronize()
        finally:
            cider.cider_test_set_sdpa_kernel(0)
        n_bad, _ = tl.violations(ref, host_bits(out), q, k, v, oracle.F16, _num_sms())
        ok[mode] = n_bad == 0
    print(f"\ntensor-core V descriptor: mode 2 {'ok' if ok[2] else 'wrong'}, mode 3 {'ok' if ok[3] else 'wrong'}")
    assert ok[2] and not ok[3]


@pytest.mark.parametrize("kernel", [1, 2])
@pytest.mark.parametrize("H_kv,N", [(8, 4096), (4, 32768), (16, 3001)])
def test_sdpa_both_kernels(kernel, H_kv, N):
    """GQA shapes on the CUDA-core kernels (1) and the tensor-core kernel (2)."""
    cider.cider_test_set_sdpa_kernel(kernel)
    try:
        _check(32, H_kv, N, seed=17 * kernel + N, kind="last_max")
    finally:
        cider.cider_test_set_sdpa_kernel(0)


@pytest.mark.parametrize("H_kv", [32, 8, 4])
@pytest.mark.parametrize("N", [1024, 4096, 32768])
def test_sdpa_pages_configs(H_kv, N):
    _check(32, H_kv, N, seed=H_kv + N)


@pytest.mark.parametrize("N", [1, 2, 15, 16, 17, 77, 1025, 3001])
@pytest.mark.parametrize("H_q,H_kv", [(32, 8), (32, 32), (8, 1), (6, 3), (3, 1)])
def test_sdpa_ragged(H_q, H_kv, N):
    _check(H_q, H_kv, N, seed=N * 7 + H_q + H_kv)


@pytest.mark.parametrize("kind", ["peaked", "last_max"])
@pytest.mark.parametrize("H_kv", [32, 8, 4])
@pytest.mark.parametrize("N", [1024, 4096, 32768])
def test_sdpa_concentrated(H_kv, N, kind):
    _check(32, H_kv, N, seed=3 * N + H_kv, kind=kind)


@pytest.mark.parametrize("kind", ["diffuse", "last_max"])
@pytest.mark.parametrize("H_kv", [32, 4])
def test_sdpa_bf16_kinds(H_kv, kind):
    _check(32, H_kv, 2049, seed=H_kv + 1, dt=oracle.BF16, kind=kind)


@pytest.mark.parametrize("H_kv", [32, 4])
def test_sdpa_bf16(H_kv):
    _check(32, H_kv, 2049, seed=H_kv, dt=oracle.BF16)


def test_sdpa_single_key_is_its_value_exactly():
    q, k, v = tl.make_inputs("diffuse", 32, 8, 1, seed=5)
    out = cider.cider_sdpa_decode(dev_bits(q, oracle.F16), dev_bits(k, oracle.F16), dev_bits(v, oracle.F16))
    np.testing.assert_array_equal(host_bits(out), np.repeat(v[:, 0, :], 4, axis=0))


def test_sdpa_argument_checks():
    q, k, v = tl.make_inputs("diffuse", 32, 8, 64, seed=6)
    qd, kd, vd = (dev_bits(a, oracle.F16) for a in (q, k, v))
    with pytest.raises(cider.CiderError):  # H_kv must divide H_q
        cider.cider_sdpa_decode(dev_bits(tl.make_inputs("diffuse", 30, 8, 64, 1)[0], oracle.F16), kd, vd)
    with pytest.raises(cider.CiderError):  # D = 128 only
        cider.cider_sdpa_decode(qd[:, :64].contiguous(), kd[:, :, :64].contiguous(), vd[:, :, :64].contiguous())
    with pytest.raises(cider.CiderError):  # workspace too small
        cider.cider_sdpa_decode(qd, kd, vd, workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))


def test_sdpa_max_difference_report():
    """The largest |GPU - oracle| over the fp16 cases of this module, beside the
    pages' 1.22e-4 (fp16, against their reference implementation)."""
    f16 = {key: d for key, d in MAX_DIFF.items() if key[-1] == oracle.F16}
    if not f16:
        pytest.skip("no fp16 case ran in this session")
    worst = max(f16, key=f16.get)
    print(f"\nsdpa fp16 max |diff| over {len(f16)} cases: {f16[worst]:.3g} at {worst[:4]} (pages: 1.22e-4)")
    pages = [d for key, d in f16.items() if key[0] == "diffuse" and key[1] == 32 and key[3] in (1024, 4096, 32768)]
    if pages:
        print(f"sdpa fp16 max |diff| over the pages' nine configurations: {max(pages):.3g}")
