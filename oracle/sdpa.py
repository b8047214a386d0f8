"""Decode attention -- scaled dot-product attention for one query token with
no mask -- in float64.

TEST INFRASTRUCTURE ONLY: like the rest of this package, only ``tests/``,
``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` may import it.
It shares nothing with the CUDA library.

What it computes (Cider README, section "优化 SDPA（解码注意力）": attention
for autoregressive decode with Q_seq = 1 and no mask, several query heads
sharing one KV head; head dimension D = 128 in the pages' measurements):
for query head h and its KV head g = h // (H_q / H_kv),

    s_j   = (q_h . k_{g,j}) / sqrt(D)                  j = 0 .. N-1
    p_j   = exp(s_j - max s) / sum_j exp(s_j - max s)
    out_h = sum_j p_j v_{g,j}

on the exactly widened fp16 / bf16 inputs, rounded once to the input format.
Layouts: q [H_q][D]; K and V [H_kv][N][D] (a head-major cache); out [H_q][D].
"""
import numpy as np

from . import F16, narrow, widen


def sdpa_decode_f64(q, k, v, dt=F16):
    """-> float64 [H_q, D], before the final rounding."""
    qf = widen(q, dt).astype(np.float64)
    kf = widen(k, dt).astype(np.float64)
    vf = widen(v, dt).astype(np.float64)
    H_q, D = qf.shape
    H_kv, N, Dk = kf.shape
    if H_q % H_kv or Dk != D or vf.shape != kf.shape or N < 1:
        raise ValueError("shapes: q [H_q][D], k and v [H_kv][N][D], H_kv dividing H_q, N >= 1")
    G = H_q // H_kv
    out = np.empty((H_q, D), np.float64)
    for h in range(H_q):
        g = h // G
        s = kf[g] @ qf[h] / np.sqrt(D)
        e = np.exp(s - s.max())
        out[h] = (e / e.sum()) @ vf[g]
    return out


def sdpa_decode(q, k, v, dt=F16):
    """-> fp16 / bf16 bit patterns [H_q, D]."""
    return narrow(sdpa_decode_f64(q, k, v, dt), dt)
