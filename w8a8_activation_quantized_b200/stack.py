"""The linear stack of an 8B-class decoder, W8A8 per-channel throughout.

Per layer (hidden 4096, kv 1024, ffn 12288): q_proj 4096->4096, k_proj and
v_proj 4096->1024, o_proj 4096->4096, gate/up 4096->12288, down 12288->4096,
with SiLU(gate) * up between the MLP linears.  Attention, norms and residuals
are not part of this workload.  o_proj takes q_proj's output in attention's
place, and every layer takes the same synthetic hidden state.

All arithmetic runs in the library's kernels through the C ABI:
- the hidden state is quantized once and shared by q/k/v;
- the q output is quantized and fed to o_proj;
- the o output is quantized once and shared by gate and up;
- SiLU(gate) * up and its quantization are one kernel feeding down_proj.

Sharing one quantized input among the projections that read it follows the
Cider README, section "ANE+GPU 异构张量并行", where Q/K/V and Gate/Up share one
input preparation.
"""
import torch

import w8a8_activation_quantized_b200 as cider
from w8a8_activation_quantized_b200 import synth

HIDDEN, KV, FFN = 4096, 1024, 12288
LINEARS = (("q", HIDDEN, HIDDEN), ("k", KV, HIDDEN), ("v", KV, HIDDEN), ("o", HIDDEN, HIDDEN),
           ("gate", FFN, HIDDEN), ("up", FFN, HIDDEN), ("down", HIDDEN, FFN))


def layer_weight_seed(layer: int, idx: int) -> int:
    return 5_000_000 + 100 * layer + idx


def ops_per_layer(M: int) -> float:
    return sum(2.0 * M * n * k for _, n, k in LINEARS)


class DecoderLinearStack:
    """Quantized weights of `layers` layers, resident on `device`."""

    def __init__(self, layers: int = 36, device="cuda", std: float = 0.02):
        self.layers = []
        for l in range(layers):
            ws = {}
            for i, (name, n, k) in enumerate(LINEARS):
                W = synth.weights_device(n, k, layer_weight_seed(l, i), std, device)
                ws[name] = cider.cider_quantize_weight_pc(W)
                del W
            self.layers.append(ws)

    def layer(self, l, h, keep=False):
        """One layer on hidden state h [M, 4096] fp16.  With keep=True returns
        every linear's input and output (for checks); else the down output."""
        w = self.layers[l]
        qh, sh = cider.cider_quantize_act(h)
        q = cider.cider_w8a8_gemm_pc_q(qh, sh, *w["q"])
        k = cider.cider_w8a8_gemm_pc_q(qh, sh, *w["k"])
        v = cider.cider_w8a8_gemm_pc_q(qh, sh, *w["v"])
        qq, sq = cider.cider_quantize_act(q)
        o = cider.cider_w8a8_gemm_pc_q(qq, sq, *w["o"])
        qo, so = cider.cider_quantize_act(o)
        g = cider.cider_w8a8_gemm_pc_q(qo, so, *w["gate"])
        u = cider.cider_w8a8_gemm_pc_q(qo, so, *w["up"])
        qa, sa, a = cider.cider_silu_mul_quantize(g, u, want_a=keep)
        d = cider.cider_w8a8_gemm_pc_q(qa, sa, *w["down"])
        if keep:
            return dict(h=h, q=q, k=k, v=v, o=o, gate=g, up=u, a=a, down=d)
        return d

    def forward(self, h):
        """Every layer on the same hidden state; returns the last layer's output."""
        out = None
        for l in range(len(self.layers)):
            out = self.layer(l, h)
        return out

    # launches of this library per layer: 3 quantize + 1 fused SiLU-quantize + 7 GEMMs
    LAUNCHES_PER_LAYER = 11
