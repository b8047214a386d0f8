"""The 8B-class decoder linear stack (36 layers, 2048 tokens): every linear of
layers 0, 17 and 35 against the oracle with teacher forcing.

Each linear is checked on its own input as the GPU produced it (copied back
to the host), on sampled token rows (rows are independent).  The weights are
regenerated from their seeds and quantized by the oracle itself.  The fused
SiLU(gate)*up -> quantize output is checked the same way: its activation
within one unit in the last place of the oracle's, and the down projection
against the oracle on the GPU's own activation.
"""
import numpy as np
import pytest
import torch

import oracle
import w8a8_activation_quantized_b200 as cider
from w8a8_activation_quantized_b200 import stack, synth
from tests.parity import check_y, host_bits

pytestmark = pytest.mark.gpu

M = 2048
ROWS = np.array([0, 511, 1024, 2047])


@pytest.fixture(scope="module")
def stk():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return stack.DecoderLinearStack(layers=36)


@pytest.fixture(scope="module")
def hidden():
    x = synth.activations(M, stack.HIDDEN, seed=4000 + M, outlier_frac=0.005, outlier_scale=100.0)
    return torch.from_numpy(x).cuda()


@pytest.mark.parametrize("layer", [0, 17, 35])
def test_stack_layer_teacher_forced(stk, hidden, layer):
    out = stk.layer(layer, hidden, keep=True)
    torch.cuda.synchronize()
    inputs = {"q": "h", "k": "h", "v": "h", "o": "q", "gate": "o", "up": "o", "down": "a"}
    for i, (name, n, k) in enumerate(stack.LINEARS):
        W = synth.weights_device(n, k, stack.layer_weight_seed(layer, i)).cpu().numpy()
        qw, sw = oracle.quantize_weight_pc(W)
        x_rows = host_bits(out[inputs[name]])[ROWS]
        check_y(out[name], oracle.linear_pc(x_rows, qw, sw), oracle.F16, rows=ROWS)
    # the fused SiLU(gate) * up: within one ulp of the oracle on the GPU's own gate/up
    g_rows = host_bits(out["gate"])[ROWS]
    u_rows = host_bits(out["up"])[ROWS]
    a_ref = oracle.silu_mul(g_rows, u_rows)
    a_gpu = host_bits(out["a"])[ROWS]
    gap = np.abs(a_gpu.view(np.int16).astype(np.int32) - a_ref.view(np.int16).astype(np.int32))
    assert gap.max() <= 1
    cider.cider_device_status()


def test_stack_forward_runs_every_layer(stk, hidden):
    d = stk.forward(hidden)
    torch.cuda.synchronize()
    assert d.shape == (M, stack.HIDDEN) and torch.isfinite(d.float()).all()
    # every layer sees the same hidden state, so the last output equals layer 35's
    ref = stk.layer(35, hidden)
    assert torch.equal(d, ref)
