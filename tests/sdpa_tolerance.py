"""Element-wise tolerance of the decode-attention parity tests, derived from
the arithmetic the GPU kernels do (Cider README, section "优化 SDPA（解码注意
力）": one query token per head, no mask, D = 128).

The GPU result o' of one output element and the exact result o (what the
float64 oracle computes before its single rounding) differ by

    |round(o') - round(o)| <= ulp(out) + |o' - o|,

so the bound is one unit of the output format at the larger of the two
values, plus F, a bound on the fp32 error |o' - o|:

    F = eps_rel * sum_j p_j |v_j|          (p_j the exact softmax weights)

    eps_rel = 2 ln2 (E_s + u S) + 4 depth 2^-21

* E_s: error of one score in the log2 domain.  The CUDA-core kernel rounds
  q * log2(e) / sqrt(D) once per element, sums 8 products with fused
  multiply-adds and 4 shuffle additions (13 roundings); the tensor-core
  kernel forms the D exact products of 16-bit values and adds them in fp32
  in an order of its own (at most D - 1 roundings), then scales once.  Both
  are within D + 2 roundings: E_s <= (D + 2) u c max_j sum_d |q_d k_jd| with
  c = log2(e) / sqrt(D) and u = 2^-24.  The subtraction s - max adds u S,
  S = the largest |s_j - max s|.  A weight's relative error is at most ln2
  times its exponent's error, and normalising by the sum of the weights at
  most doubles it.  (The tensor-core kernel hands P to its second product as
  a sum of 16-bit parts exact to 2^-22 of each weight, inside the 2^-21 per
  step below.)
* The rest: every hardware exp2 (relative error below 2^-22), every rescale
  of the running state, every fp32 addition of the running sums and every
  merge of streams and chunks costs at most 2^-21 relative; along any path
  from a key to the output there are at most depth = (keys per stream) +
  (chunks) + 12 such steps, counted for the running sum of the weights and
  for the weighted values, and once more for the final division.

The bound scales with the actual outputs and with sum_j p_j |v_j|, not with
max |V|: dropping a chunk, mis-weighting a chunk's partial or skipping a
rescale changes outputs by far more than F, which tests/test_sdpa_tolerance.py
checks on the host for planted mistakes.
"""
import math

import numpy as np

import oracle

D = 128
U = 2.0 ** -24
C = math.log2(math.e) / math.sqrt(D)
MANT = {oracle.F16: 10, oracle.BF16: 7}
MIN_EXP = {oracle.F16: -14, oracle.BF16: -126}


def ulp(x, dt):
    """One unit in the last place of the format at |x| (subnormal spacing below)."""
    a = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, MIN_EXP[dt])
    return np.exp2(e - MANT[dt])


def fp32_bound(q, k, v, dt, keys_per_stream, chunks):
    """F [H_q, D]: bound on the kernel's fp32 error, per output element."""
    qf = oracle.widen(q, dt).astype(np.float64)
    kf = oracle.widen(k, dt).astype(np.float64)
    vf = oracle.widen(v, dt).astype(np.float64)
    H_q = qf.shape[0]
    H_kv = kf.shape[0]
    G = H_q // H_kv
    depth = keys_per_stream + chunks + 12
    out = np.empty((H_q, D), np.float64)
    for h in range(H_q):
        g = h // G
        s = (kf[g] @ qf[h]) * C                      # scores in the log2 domain
        e_s = (D + 2) * U * C * np.max(np.abs(kf[g]) @ np.abs(qf[h]))
        spread = float(s.max() - s.min())
        eps_rel = 2 * math.log(2) * (e_s + U * spread) + 4 * depth * 2.0 ** -21
        p = np.exp2(s - s.max())
        p /= p.sum()
        out[h] = eps_rel * (p @ np.abs(vf[g]))
    return out


def plan_depths(H_q, H_kv, N, num_sms):
    """(keys per stream, chunks) of the kernel's cut of the sequence."""
    import w8a8_activation_quantized_b200 as cider
    _, _, chunk, chunks = cider.cider_test_sdpa_plan(H_q, H_kv, N, num_sms)
    return -(-chunk // 16), chunks, chunk


def tolerance(ref_bits, got_bits, q, k, v, dt, num_sms):
    """Per-element tolerance: ulp at max(|ref|, |got|) plus the fp32 bound."""
    H_q, H_kv, N = q.shape[0], k.shape[0], k.shape[1]
    kps, chunks, _ = plan_depths(H_q, H_kv, N, num_sms)
    r = oracle.as_float(ref_bits, dt)
    g = oracle.as_float(got_bits, dt)
    return ulp(np.maximum(np.abs(r), np.abs(g)), dt) + fp32_bound(q, k, v, dt, kps, chunks)


def violations(ref_bits, got_bits, q, k, v, dt, num_sms):
    """(number of elements out of tolerance, max |got - ref|)."""
    r = oracle.as_float(ref_bits, dt)
    g = oracle.as_float(got_bits, dt)
    err = np.abs(g - r)
    tol = tolerance(ref_bits, got_bits, q, k, v, dt, num_sms)
    return int(np.count_nonzero(~(err <= tol))), float(np.max(err))


# ---- seeded inputs of the decode-attention tests --------------------------------

def make_inputs(kind, H_q, H_kv, N, seed, dt=oracle.F16):
    """q [H_q, D], k and v [H_kv, N, D] as bit patterns.

    kind "diffuse": q, k, v ~ N(0, 1), scores ~ N(0, 1) spread over ~N/e keys.
    kind "peaked": q ~ N(0, 8^2): a few keys carry most of each head's weight,
    so outputs are O(1).
    kind "last_max": q ~ N(0, 4^2); in each KV head one key of the sequence's
    last 16 is set along its query heads' mean so that its score exceeds every
    other score of those heads by 3: the maximum arrives last and every
    earlier chunk and stream must be rescaled to it."""
    rng = np.random.default_rng(seed)
    qs = {"diffuse": 1.0, "peaked": 8.0, "last_max": 4.0}[kind]
    q = oracle.narrow(rng.normal(0, qs, size=(H_q, D)), dt)
    k64 = rng.normal(0, 1, size=(H_kv, N, D))
    v = oracle.narrow(rng.normal(0, 1, size=(H_kv, N, D)), dt)
    if kind == "last_max":
        G = H_q // H_kv
        qf = oracle.widen(q, dt).astype(np.float64)
        kf = oracle.widen(oracle.narrow(k64, dt), dt).astype(np.float64)
        j_star = N - 1 - int(rng.integers(0, min(16, N)))
        for g in range(H_kv):
            qg = qf[g * G:(g + 1) * G]
            qbar = qg.mean(axis=0)
            others = np.delete(kf[g], j_star, axis=0) @ qg.T / math.sqrt(D)
            t = (others.max() + 3.0) * math.sqrt(D) / np.min(qg @ qbar)
            k64[g, j_star] = t * qbar
    return q, oracle.narrow(k64, dt), v


def chunked_f64(q, k, v, dt, chunk, drop_chunks=(), unrescaled_chunks=(), drop_stream=None):
    """The decode-attention output computed in float64 chunk by chunk, the way
    the two-pass kernels combine partial results -- with optional planted
    mistakes: chunks left out of the merge, chunks whose partial result is
    added without its 2^(m_c - M) rescale, or one of the 16 key streams of
    every chunk left out.  Returns bit patterns of the format."""
    qf = oracle.widen(q, dt).astype(np.float64)
    kf = oracle.widen(k, dt).astype(np.float64)
    vf = oracle.widen(v, dt).astype(np.float64)
    H_q, H_kv, N = qf.shape[0], kf.shape[0], kf.shape[1]
    G = H_q // H_kv
    out = np.empty((H_q, D), np.float64)
    n_chunks = -(-N // chunk)
    for h in range(H_q):
        s = kf[h // G] @ qf[h] / math.sqrt(D)
        keep = np.ones(N, bool)
        if drop_stream is not None:
            keep &= (np.arange(N) % chunk) % 16 != drop_stream
        parts = []
        for c in range(n_chunks):
            if c in drop_chunks:
                continue
            idx = np.arange(c * chunk, min(N, (c + 1) * chunk))
            idx = idx[keep[idx]]
            if idx.size == 0:
                continue
            m_c = s[idx].max()
            e = np.exp(s[idx] - m_c)
            parts.append((c, m_c, e.sum(), e @ vf[h // G][idx]))
        M = max(p[1] for p in parts)
        L, A = 0.0, np.zeros(D)
        for c, m_c, l_c, a_c in parts:
            w = 1.0 if c in unrescaled_chunks else math.exp(m_c - M)
            L += w * l_c
            A += w * a_c
        out[h] = A / L
    return oracle.narrow(out, dt)


def kernel_order_f32(q, k, v, dt, chunk):
    """The two-pass decode attention evaluated in float32 in the kernels'
    order: q pre-scaled by log2(e)/sqrt(D), 16 key streams per chunk with an
    online softmax in the log2 domain, streams merged, then chunks.  Lets the
    host check that the tolerance admits fp32 arithmetic of that structure."""
    f32 = np.float32
    qf = oracle.widen(q, dt).astype(f32) * f32(C)
    kf = oracle.widen(k, dt).astype(f32)
    vf = oracle.widen(v, dt).astype(f32)
    H_q, H_kv, N = qf.shape[0], kf.shape[0], kf.shape[1]
    G = H_q // H_kv
    n_chunks = -(-N // chunk)
    per = chunk // 16
    pad = n_chunks * chunk - N
    out = np.empty((H_q, D), f32)
    for h in range(H_q):
        s = (kf[h // G] @ qf[h]).astype(f32)
        s = np.concatenate([s, np.full(pad, -np.inf, f32)]).reshape(n_chunks, per, 16)
        vv = np.concatenate([vf[h // G], np.zeros((pad, D), f32)]).reshape(n_chunks, per, 16, D)
        m = np.full((n_chunks, 16), -np.inf, f32)
        l = np.zeros((n_chunks, 16), f32)
        a = np.zeros((n_chunks, 16, D), f32)
        for i in range(per):
            si = s[:, i, :]
            up = si > m
            corr = np.where(up, np.exp2(np.where(up, m - si, 0)).astype(f32), f32(1))
            l = (l * corr).astype(f32)
            a = (a * corr[..., None]).astype(f32)
            m = np.where(up, si, m)
            p = np.where(np.isfinite(si), np.exp2(si - m), 0).astype(f32)
            l = (l + p).astype(f32)
            a = (p[..., None].astype(np.float64) * vv[:, i] + a).astype(f32)
        Mc = m.max(axis=1)
        sc = np.where(np.isfinite(m), np.exp2(m - Mc[:, None]), 0).astype(f32)
        Lc = (l * sc).sum(axis=1, dtype=f32)
        Ac = (a * sc[..., None]).sum(axis=1, dtype=f32)
        M = Mc.max()
        w = np.exp2(Mc - M).astype(f32)
        out[h] = (Ac * w[:, None]).sum(axis=0, dtype=f32) / (Lc * w).sum(dtype=f32)
    return oracle.narrow(out.astype(np.float64), dt)
