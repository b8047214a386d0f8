"""Parity at the benchmarked shapes themselves: every linear row that bench.py
times is run here at its own M x N x K, with the same seeded inputs and the
same workspace (cider_workspace_bytes_mnk, so the same tile schedule and
split-K plan), and sampled output rows are compared with the oracle.

Token rows are independent, so the oracle on a subset of rows gives exactly
those rows of the full product.  The sample holds the first and last rows,
the rows on both sides of each 128- and 256-row tile edge inside the first
two tiles, and seeded random rows over the whole range, so that every
persistent round of the GEMM's schedule and the split tail is visited.

Shapes (Cider README, section "性能（Apple M5 Pro）/ 单算子延迟": N = 10240,
K = 2560 per channel and N = 2560, K = 10240 per group, M from 1 to 8192; the
W4A8 workload of 2048 x 12288 x 4096 with gs = 64)."""
import numpy as np
import pytest
import torch

import oracle
import w8a8_activation_quantized_b200 as cider
from w8a8_activation_quantized_b200 import synth
from tests.parity import check_y, dev

pytestmark = pytest.mark.gpu
F16 = oracle.F16


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    cider.cider_device_status()


def sample_rows(M, seed, n_random=24):
    fixed = [0, 1, 126, 127, 128, 129, 254, 255, 256, 257, M - 2, M - 1]
    rnd = np.random.default_rng(seed).choice(M, size=min(M, n_random), replace=False)
    rows = np.unique(np.concatenate([np.array([r for r in fixed if 0 <= r < M], np.int64), rnd]))
    return rows


def _check_rows(y, rows, y_ref_bits):
    idx = torch.from_numpy(rows).to(y.device)
    return check_y(y.index_select(0, idx), y_ref_bits, F16)


@pytest.fixture(scope="module")
def pc_weights():
    # bench.py's per-channel rows: synth.weights(10240, 2560, seed=1001)
    return oracle.quantize_weight_pc(synth.weights(10240, 2560, 1001))


@pytest.mark.parametrize("M", [1, 128, 1024, 4096, 8192])
def test_w8a8_linear_pc_bench_shape(M, pc_weights):
    N, K = 10240, 2560
    qw, sw = pc_weights
    x = synth.activations(M, K, 1000 + M)
    y = cider.cider_w8a8_linear_pc(dev(x), dev(qw), dev(sw))
    torch.cuda.synchronize()
    rows = sample_rows(M, seed=M)
    _check_rows(y, rows, oracle.linear_pc(x[rows], qw, sw))


@pytest.fixture(scope="module")
def pg_weights():
    # bench.py's per-group rows: synth.weights(2560, 10240, seed=2001)
    W = synth.weights(2560, 10240, 2001)
    return {gs: oracle.quantize_weight_pg(W, gs) for gs in (128, 64)}


@pytest.mark.parametrize("gs", [128, 64])
@pytest.mark.parametrize("M", [1, 128, 1024, 4096, 8192])
def test_w8a8_linear_pg_bench_shape(M, gs, pg_weights):
    N, K = 2560, 10240
    qw, sw = pg_weights[gs]  # oracle layout [N][K/gs]; the library takes [K/gs][N]
    x = synth.activations(M, K, 2000 + M)
    y = cider.cider_w8a8_linear_pg(dev(x), dev(qw), dev(np.ascontiguousarray(sw.T)), gs)
    torch.cuda.synchronize()
    rows = sample_rows(M, seed=M + gs)
    _check_rows(y, rows, oracle.linear_pg(x[rows], qw, sw, gs))


def test_w4a8_linear_pg_bench_shape():
    M, N, K, gs = 2048, 12288, 4096, 64
    packed, sw = oracle.quantize_weight_int4_pg(synth.weights(N, K, 3001), gs)
    x = synth.activations(M, K, 3000 + M)
    y = cider.cider_w4a8_linear_pg(dev(x), dev(packed), dev(np.ascontiguousarray(sw.T)), gs)
    torch.cuda.synchronize()
    rows = sample_rows(M, seed=4)
    _check_rows(y, rows, oracle.w4a8_linear_pg(x[rows], packed, sw, gs))


def test_w4a8_linear_pc_bench_shape():
    M, N, K = 2048, 12288, 4096
    packed, sw = oracle.quantize_weight_int4_pc(synth.weights(N, K, 3001))
    x = synth.activations(M, K, 3000 + M)
    y = cider.cider_w4a8_linear_pc(dev(x), dev(packed), dev(sw))
    torch.cuda.synchronize()
    rows = sample_rows(M, seed=5)
    _check_rows(y, rows, oracle.w4a8_linear_pc(x[rows], packed, sw))


def test_w8a16_mv_pc_bench_shape(pc_weights):
    N, K = 10240, 2560
    qw, sw = pc_weights
    x = synth.activations(1, K, 1001)
    y = cider.cider_w8a16_mv_pc(dev(x), dev(qw), dev(sw))
    torch.cuda.synchronize()
    check_y(y, oracle.w8a16_linear_pc(x, qw, sw), F16)


@pytest.mark.parametrize("gs", [128, 64])
def test_w8a16_mv_pg_bench_shape(gs, pg_weights):
    N, K = 2560, 10240
    qw, sw = pg_weights[gs]
    x = synth.activations(1, K, 2001)
    y = cider.cider_w8a16_mv_pg(dev(x), dev(qw), dev(np.ascontiguousarray(sw.T)), gs)
    torch.cuda.synchronize()
    check_y(y, oracle.w8a16_linear_pg(x, qw, sw, gs), F16)
