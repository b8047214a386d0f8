"""CPU oracle for the W8A8 / W4A8 activation-quantized linear.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package.  It is a thin ctypes
wrapper around ``cider_oracle.c`` (plain C, one IEEE operation per step, no
blocking or fusion) and shares no code with the CUDA library.

What it computes, with sources (page title, then section):

* per-token symmetric INT8 activation quantization,
  ``scale = max|x|/127``, ``q = clamp(round(x/scale), -128, 127)`` --
  juejin post "在Mac上跑大模型，MLX 不是终点", section "W8A8 对称量化：Cider 的选择";
  Cider README, table "量化" (activations: symmetric INT8, per token);
* offline weight quantization (per output channel, per group of gs along K,
  INT4 packed two per byte) -- Cider README, section "底层 API"
  (``quantize_weight_int8``, ``pack_weight_int4``) and table "量化";
* the INT8 x INT8 -> INT32 product -- juejin post, section "INT8 TensorOps 内核设计";
* the dequant ``y = acc * scale_x * scale_w`` (per channel) and the per-group
  piecewise rescale -- juejin post, sections "W8A8 对称量化" and "三种量化粒度的实现".

Bit patterns of fp16 / bf16 data travel as ``np.uint16`` arrays; ``F16`` and
``BF16`` name the format.  Every function here has its pins in
``tests/test_oracle_*.py`` (hand-worked examples under ``tests/golden/``,
exhaustive format checks against numpy/torch, brute force on tiny inputs,
invariants).
"""
import ctypes

import numpy as np

from .build import LIB, build_oracle

F16 = 0
BF16 = 1

_i64 = ctypes.c_int64
_int = ctypes.c_int
_ptr = ctypes.c_void_p
_lib = None


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(build_oracle())
    return _lib


def _bind(path):
    """Load an oracle library from ``path`` and declare its C signatures."""
    lib = ctypes.CDLL(path)
    sig = {
        "oracle_f16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
        "oracle_bf16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
        "oracle_f64_to_f16_rne": (ctypes.c_uint16, [ctypes.c_double]),
        "oracle_f64_to_bf16_rne": (ctypes.c_uint16, [ctypes.c_double]),
        "oracle_round_half_away": (ctypes.c_float, [ctypes.c_float]),
        "oracle_quantize_act": (None, [_ptr, _int, _i64, _i64, _ptr, _ptr]),
        "oracle_quantize_weight_pc": (None, [_ptr, _i64, _i64, _ptr, _ptr]),
        "oracle_quantize_weight_pg": (None, [_ptr, _i64, _i64, _i64, _ptr, _ptr]),
        "oracle_quantize_weight_int4_pg": (None, [_ptr, _i64, _i64, _i64, _ptr, _ptr]),
        "oracle_quantize_weight_pc_clip": (None, [_ptr, _i64, _i64, ctypes.c_double, _ptr, _ptr]),
        "oracle_quantize_weight_pg_clip": (None, [_ptr, _i64, _i64, _i64, ctypes.c_double, _ptr, _ptr]),
        "oracle_percentile_position": (None, [ctypes.c_double, _i64, _ptr, _ptr]),
        "oracle_unpack_int4": (None, [_ptr, _i64, _i64, _ptr]),
        "oracle_gemm_i32": (_int, [_ptr, _ptr, _i64, _i64, _i64, _ptr]),
        "oracle_gemm_i32_grouped": (_int, [_ptr, _ptr, _i64, _i64, _i64, _i64, _ptr]),
        "oracle_dequant_pc": (None, [_ptr, _ptr, _ptr, _i64, _i64, _int, _ptr]),
        "oracle_dequant_pg": (None, [_ptr, _ptr, _ptr, _i64, _i64, _i64, _int, _ptr]),
        "oracle_linear_pc": (_int, [_ptr, _int, _i64, _i64, _ptr, _ptr, _i64, _int, _ptr]),
        "oracle_w8a16_linear_pc": (_int, [_ptr, _int, _i64, _i64, _ptr, _ptr, _i64, _int, _ptr]),
        "oracle_w8a16_linear_pg": (_int, [_ptr, _int, _i64, _i64, _ptr, _ptr, _i64, _i64, _int, _ptr]),
        "oracle_linear_pg": (_int, [_ptr, _int, _i64, _i64, _ptr, _ptr, _i64, _i64, _int, _ptr]),
        "oracle_w4a8_linear_pg": (_int, [_ptr, _int, _i64, _i64, _ptr, _ptr, _i64, _i64, _int,
                                         _ptr, _ptr]),
        "oracle_silu_mul": (None, [_ptr, _ptr, _int, _i64, _ptr]),
        "oracle_num_threads": (_int, []),
        "oracle_widen_array": (None, [_ptr, _int, _i64, _ptr]),
        "oracle_narrow_array": (None, [_ptr, _int, _i64, _ptr]),
        "oracle_round_half_away_array": (None, [_ptr, _i64, _ptr]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def _c(a, dtype):
    """Contiguous array of exactly ``dtype`` (no silent value conversion)."""
    a = np.asarray(a)
    if a.dtype != np.dtype(dtype):
        raise TypeError(f"oracle expects {np.dtype(dtype)}, got {a.dtype}")
    return np.ascontiguousarray(a)


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _bits(x, dt):
    """fp16 arrays are viewed as their bit patterns; bf16 must already be uint16 bits."""
    x = np.asarray(x)
    if x.dtype == np.float16:
        if dt != F16:
            raise TypeError("float16 array given with a non-F16 dtype tag")
        x = x.view(np.uint16)
    return _c(x, np.uint16)


def num_threads() -> int:
    return _load().oracle_num_threads()


# ---- number formats -------------------------------------------------------

def widen(bits, dt) -> np.ndarray:
    """fp16/bf16 bit patterns -> exact float32 values."""
    b = _bits(bits, dt)
    out = np.empty(b.shape, np.float32)
    _load().oracle_widen_array(_p(b), dt, b.size, _p(out))
    return out


def narrow(values, dt) -> np.ndarray:
    """float64 values -> fp16/bf16 bit patterns, round to nearest even."""
    v = _c(np.asarray(values, dtype=np.float64), np.float64)
    out = np.empty(v.shape, np.uint16)
    _load().oracle_narrow_array(_p(v), dt, v.size, _p(out))
    return out


def round_half_away(t) -> np.ndarray:
    t = _c(np.asarray(t, dtype=np.float32), np.float32)
    out = np.empty(t.shape, np.float32)
    _load().oracle_round_half_away_array(_p(t), t.size, _p(out))
    return out


# ---- activation quantization ----------------------------------------------

def quantize_act(x, dt=F16):
    """x [M,K] (fp16 array, or uint16 bits with ``dt``) -> (q int8 [M,K], scale_x f32 [M])."""
    b = _bits(x, dt)
    M, K = b.shape
    q = np.empty((M, K), np.int8)
    sx = np.empty((M,), np.float32)
    _load().oracle_quantize_act(_p(b), dt, M, K, _p(q), _p(sx))
    return q, sx


# ---- offline weight quantization ------------------------------------------

def quantize_weight_pc(W):
    """W f32 [N,K] -> (qw int8 [N,K], sw f32 [N])."""
    W = _c(W, np.float32)
    N, K = W.shape
    qw = np.empty((N, K), np.int8)
    sw = np.empty((N,), np.float32)
    _load().oracle_quantize_weight_pc(_p(W), N, K, _p(qw), _p(sw))
    return qw, sw


def quantize_weight_pg(W, gs):
    """W f32 [N,K] -> (qw int8 [N,K], sw f32 [N, K/gs])."""
    W = _c(W, np.float32)
    N, K = W.shape
    if K % gs:
        raise ValueError("gs must divide K")
    qw = np.empty((N, K), np.int8)
    sw = np.empty((N, K // gs), np.float32)
    _load().oracle_quantize_weight_pg(_p(W), N, K, gs, _p(qw), _p(sw))
    return qw, sw


def percentile_position(p, n):
    """-> (i, t): the p-th percentile of n ascending values lies a fraction t
    of the way from the i-th to the (i+1)-th (t is fp32)."""
    i = ctypes.c_int64()
    t = ctypes.c_float()
    _load().oracle_percentile_position(float(p), int(n), ctypes.byref(i), ctypes.byref(t))
    return i.value, np.float32(t.value)


def quantize_weight_pc_clip(W, p):
    """Percentile-clipped per-channel weights (Cider README, section "说明",
    clip_percentile): W f32 [N,K] -> (qw int8 [N,K] in [-127,127], sw f32 [N])."""
    W = _c(W, np.float32)
    N, K = W.shape
    qw = np.empty((N, K), np.int8)
    sw = np.empty((N,), np.float32)
    _load().oracle_quantize_weight_pc_clip(_p(W), N, K, float(p), _p(qw), _p(sw))
    return qw, sw


def quantize_weight_pg_clip(W, gs, p):
    """Percentile-clipped per-group weights: W f32 [N,K] -> (qw int8 [N,K],
    sw f32 [N, K/gs])."""
    W = _c(W, np.float32)
    N, K = W.shape
    if K % gs:
        raise ValueError("gs must divide K")
    qw = np.empty((N, K), np.int8)
    sw = np.empty((N, K // gs), np.float32)
    _load().oracle_quantize_weight_pg_clip(_p(W), N, K, gs, float(p), _p(qw), _p(sw))
    return qw, sw


def quantize_weight_int4_pg(W, gs):
    """W f32 [N,K] -> (packed uint8 [N, K/2], sw f32 [N, K/gs])."""
    W = _c(W, np.float32)
    N, K = W.shape
    if K % gs or K % 2 or gs % 2:
        raise ValueError("gs must divide K; K and gs even")
    packed = np.zeros((N, K // 2), np.uint8)
    sw = np.empty((N, K // gs), np.float32)
    _load().oracle_quantize_weight_int4_pg(_p(W), N, K, gs, _p(packed), _p(sw))
    return packed, sw


def quantize_weight_int4_pc(W):
    """INT4 weights with one scale per output channel (Cider README, table
    "量化": W4A8 weights symmetric INT4, zp = 8, per column) -- the per-group
    definition with a single group spanning K.  W f32 [N,K] -> (packed uint8
    [N, K/2], sw f32 [N])."""
    W = _c(W, np.float32)
    packed, sw = quantize_weight_int4_pg(W, W.shape[1])
    return packed, np.ascontiguousarray(sw[:, 0])


def unpack_int4(packed, K):
    packed = _c(packed, np.uint8)
    N = packed.shape[0]
    w = np.empty((N, K), np.int8)
    _load().oracle_unpack_int4(_p(packed), N, K, _p(w))
    return w


# ---- integer product and dequant ------------------------------------------

def gemm_i32(q, w):
    """q int8 [M,K], w int8 [N,K] -> acc int32 [M,N]."""
    q, w = _c(q, np.int8), _c(w, np.int8)
    M, K = q.shape
    N = w.shape[0]
    acc = np.empty((M, N), np.int32)
    if _load().oracle_gemm_i32(_p(q), _p(w), M, N, K, _p(acc)) != 0:
        raise OverflowError("INT32 accumulator overflow")
    return acc


def gemm_i32_grouped(q, w, gs):
    """-> acc_g int32 [K/gs, M, N], one INT32 partial per K group."""
    q, w = _c(q, np.int8), _c(w, np.int8)
    M, K = q.shape
    N = w.shape[0]
    acc = np.empty((K // gs, M, N), np.int32)
    if _load().oracle_gemm_i32_grouped(_p(q), _p(w), M, N, K, gs, _p(acc)) != 0:
        raise OverflowError("INT32 accumulator overflow")
    return acc


def dequant_pc(acc, sx, sw, ydt=F16):
    acc, sx, sw = _c(acc, np.int32), _c(sx, np.float32), _c(sw, np.float32)
    M, N = acc.shape
    y = np.empty((M, N), np.uint16)
    _load().oracle_dequant_pc(_p(acc), _p(sx), _p(sw), M, N, ydt, _p(y))
    return y


def dequant_pg(acc_g, sx, sw, ydt=F16):
    acc_g, sx, sw = _c(acc_g, np.int32), _c(sx, np.float32), _c(sw, np.float32)
    G, M, N = acc_g.shape
    y = np.empty((M, N), np.uint16)
    _load().oracle_dequant_pg(_p(acc_g), _p(sx), _p(sw), M, N, G, ydt, _p(y))
    return y


# ---- whole linears ----------------------------------------------------------

def linear_pc(x, w, sw, xdt=F16, ydt=F16):
    """W8A8 per-channel linear.  Returns y as fp16/bf16 bit patterns [M,N]."""
    b = _bits(x, xdt)
    w, sw = _c(w, np.int8), _c(sw, np.float32)
    M, K = b.shape
    N = w.shape[0]
    y = np.empty((M, N), np.uint16)
    if _load().oracle_linear_pc(_p(b), xdt, M, K, _p(w), _p(sw), N, ydt, _p(y)) != 0:
        raise OverflowError("INT32 accumulator overflow")
    return y


def w8a16_linear_pc(x, w, sw, xdt=F16, ydt=F16):
    """W8A16 decode product (no activation quantization): y = round(sw[n] *
    sum_k x[m,k] * w[n,k]) in fp64.  Returns fp16/bf16 bit patterns [M,N]."""
    b = _bits(x, xdt)
    w, sw = _c(w, np.int8), _c(sw, np.float32)
    M, K = b.shape
    N = w.shape[0]
    y = np.empty((M, N), np.uint16)
    _load().oracle_w8a16_linear_pc(_p(b), xdt, M, K, _p(w), _p(sw), N, ydt, _p(y))
    return y


def w8a16_linear_pg(x, w, sw, gs, xdt=F16, ydt=F16):
    """W8A16 decode product with per-group weight scales (sw [N, K/gs]), no
    activation quantization: y = round(sum_g sw[n,g] * sum_{k in g} x[m,k] *
    w[n,k]) in fp64.  Returns fp16/bf16 bit patterns [M,N]."""
    b = _bits(x, xdt)
    w, sw = _c(w, np.int8), _c(sw, np.float32)
    M, K = b.shape
    N = w.shape[0]
    if gs < 1 or K % gs or sw.shape != (N, K // gs):
        raise ValueError("gs must divide K and sw must be [N, K/gs]")
    y = np.empty((M, N), np.uint16)
    _load().oracle_w8a16_linear_pg(_p(b), xdt, M, K, _p(w), _p(sw), N, gs, ydt, _p(y))
    return y


def linear_pg(x, w, sw, gs, xdt=F16, ydt=F16):
    """W8A8 per-group linear (sw [N, K/gs])."""
    b = _bits(x, xdt)
    w, sw = _c(w, np.int8), _c(sw, np.float32)
    M, K = b.shape
    N = w.shape[0]
    y = np.empty((M, N), np.uint16)
    if _load().oracle_linear_pg(_p(b), xdt, M, K, _p(w), _p(sw), N, gs, ydt, _p(y)) != 0:
        raise OverflowError("INT32 accumulator overflow")
    return y


def w4a8_linear_pg(x, packed, sw, gs, xdt=F16, ydt=F16):
    """W4A8 per-group linear (packed uint8 [N, K/2], sw [N, K/gs])."""
    b = _bits(x, xdt)
    packed, sw = _c(packed, np.uint8), _c(sw, np.float32)
    M, K = b.shape
    N = packed.shape[0]
    y = np.empty((M, N), np.uint16)
    scratch = np.empty((N, K), np.int8)
    if _load().oracle_w4a8_linear_pg(_p(b), xdt, M, K, _p(packed), _p(sw), N, gs, ydt,
                                     _p(y), _p(scratch)) != 0:
        raise OverflowError("INT32 accumulator overflow")
    return y


def w4a8_linear_pc(x, packed, sw, xdt=F16, ydt=F16):
    """W4A8 linear with per-output-channel scales (sw [N]): the per-group
    linear with one group spanning K, y = round(acc * scale_x * sw[n])."""
    K = _bits(x, xdt).shape[1]
    return w4a8_linear_pg(x, packed, _c(sw, np.float32).reshape(-1, 1), K, xdt, ydt)


def silu_mul(g, u, dt=F16):
    """a = round_dt(silu(g) * u), evaluated in fp64."""
    gb, ub = _bits(g, dt), _bits(u, dt)
    if gb.shape != ub.shape:
        raise ValueError("shape mismatch")
    a = np.empty(gb.shape, np.uint16)
    _load().oracle_silu_mul(_p(gb), _p(ub), dt, gb.size, _p(a))
    return a


def as_float(bits, dt) -> np.ndarray:
    """Bit patterns -> float64 values (for comparisons in the tests)."""
    return widen(bits, dt).astype(np.float64)


__all__ = [n for n in dir() if not n.startswith("_")] + ["LIB"]
