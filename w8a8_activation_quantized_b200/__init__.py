"""B200-native W8A8 / W4A8 activation-quantized linear.

Every step runs in the sm_100a CUDA kernels of ``libcider.so`` (built from
``csrc/`` by ``_build.py``); this module only marshals torch tensors into the
C ABI declared in ``include/cider.h`` and raises on a non-zero status.  The
Python names are the C entry points' names.  There is no CPU fallback: if the
library is missing, or the device is not sm_100-family, the calls raise.

PyTorch provides device memory and the current stream; outputs that the
caller does not pass are allocated with ``torch.empty`` on the input's device.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcider.so")

F16, BF16 = 0, 1
_DT = {torch.float16: F16, torch.bfloat16: BF16}
_TORCH_DT = {F16: torch.float16, BF16: torch.bfloat16}

STATUS = {0: "CIDER_OK", 1: "CIDER_ERR_INVALID_ARG", 2: "CIDER_ERR_UNSUPPORTED",
          3: "CIDER_ERR_CUDA", 4: "CIDER_ERR_TIMEOUT"}


class CiderError(RuntimeError):
    def __init__(self, fn, status, message):
        self.status = status
        self.message = message
        super().__init__(f"{fn} failed with {STATUS.get(status, status)}: {message}")


_P, _I64, _INT, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
_SIGNATURES = {
    "cider_is_available": (_INT, []),
    "cider_status_string": (ctypes.c_char_p, [_INT]),
    "cider_last_error": (ctypes.c_char_p, []),
    "cider_device_status": (_INT, [_P]),
    "cider_workspace_bytes": (_SZ, [_I64, _I64]),
    "cider_workspace_bytes_mnk": (_SZ, [_I64, _I64, _I64]),
    "cider_set_small_m_threshold": (_INT, [_I64]),
    "cider_get_small_m_threshold": (_I64, []),
    "cider_quantize_act": (_INT, [_P, _INT, _I64, _I64, _I64, _P, _I64, _P, _P]),
    "cider_w8a8_linear_pc": (_INT, [_P, _INT, _I64, _I64, _P, _P, _I64, _P, _INT, _P, _SZ, _P]),
    "cider_w8a16_mv_pc": (_INT, [_P, _INT, _I64, _I64, _P, _P, _I64, _P, _INT, _P]),
    "cider_w8a16_mv_pg": (_INT, [_P, _INT, _I64, _I64, _P, _P, _I64, _I64, _P, _INT, _P]),
    "cider_w8a8_linear_pg": (_INT, [_P, _INT, _I64, _I64, _P, _P, _I64, _I64, _P, _INT, _P, _SZ, _P]),
    "cider_w4a8_linear_pg": (_INT, [_P, _INT, _I64, _I64, _P, _P, _I64, _I64, _P, _INT, _P, _SZ, _P]),
    "cider_w4a8_linear_pc": (_INT, [_P, _INT, _I64, _I64, _P, _P, _I64, _P, _INT, _P, _SZ, _P]),
    "cider_workspace_bytes_w4a8_pc": (_SZ, [_I64, _I64, _I64]),
    "cider_sdpa_decode_workspace_bytes": (_SZ, [_I64, _I64, _I64, _I64]),
    "cider_sdpa_decode": (_INT, [_P, _P, _P, _INT, _I64, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "cider_test_sdpa_plan": (_INT, [_I64, _I64, _I64, _I64, _P]),
    "cider_w8a8_linear_pc_noalloc": (_INT, [_P, _INT, _I64, _I64, _P, _P, _I64, _P, _INT, _P]),
    "cider_w8a8_gemm_pc_q": (_INT, [_P, _P, _I64, _I64, _P, _P, _I64, _P, _INT, _P]),
    "cider_w8a8_gemm_pg_q": (_INT, [_P, _P, _I64, _I64, _P, _P, _I64, _I64, _P, _INT, _P]),
    "cider_w4a8_gemm_pg_q": (_INT, [_P, _P, _I64, _I64, _P, _P, _I64, _I64, _P, _INT, _P]),
    "cider_w4a8_gemm_pc_q": (_INT, [_P, _P, _I64, _I64, _P, _P, _I64, _P, _INT, _P]),
    "cider_silu_mul_quantize": (_INT, [_P, _P, _INT, _I64, _I64, _P, _P, _P, _P]),
    "cider_quantize_weight_pc": (_INT, [_P, _I64, _I64, _P, _P, _P]),
    "cider_quantize_weight_pg": (_INT, [_P, _I64, _I64, _I64, _P, _P, _P]),
    "cider_quantize_weight_pc_clip": (_INT, [_P, _I64, _I64, ctypes.c_double, _P, _P, _P]),
    "cider_quantize_weight_pg_clip": (_INT, [_P, _I64, _I64, _I64, ctypes.c_double, _P, _P, _P]),
    "cider_pack_weight_int4_pg": (_INT, [_P, _I64, _I64, _I64, _P, _P, _P]),
    "cider_pack_weight_int4_pc": (_INT, [_P, _I64, _I64, _P, _P, _P]),
    "cider_test_gemm_i32": (_INT, [_P, _P, _I64, _I64, _I64, _P, _P]),
    "cider_test_gemm_i32_grouped": (_INT, [_P, _P, _I64, _I64, _I64, _I64, _P, _P]),
    "cider_test_unpack_int4": (_INT, [_P, _I64, _I64, _P, _P]),
    "cider_test_set_gemm_variant": (_INT, [_INT]),
    "cider_test_set_split_k": (_INT, [_INT]),
    "cider_test_set_fused_quantize": (_INT, [_INT]),
    "cider_test_set_small_m_kernel": (_INT, [_INT]),
    "cider_test_set_sdpa_kernel": (_INT, [_INT]),
    "cider_test_bounded_wait": (_INT, [_I64, _P]),
}
EXPORTS = tuple(_SIGNATURES)

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C library.  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libcider.so not found at {LIB_PATH}: build it with "
                              "`python -m w8a8_activation_quantized_b200._build` "
                              "(there is no CPU fallback)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _check(fn, status):
    if status != 0:
        raise CiderError(fn, status, lib().cider_last_error().decode(errors="replace"))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _contig(t, name):
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


# ---- availability, diagnostics, configuration -----------------------------

def cider_is_available() -> bool:
    return bool(lib().cider_is_available())


def cider_device_status(stream=None, device=None):
    _check("cider_device_status", lib().cider_device_status(_stream(stream, device)))


def cider_workspace_bytes(M: int, K: int) -> int:
    return int(lib().cider_workspace_bytes(M, K))


def cider_workspace_bytes_mnk(M: int, N: int, K: int) -> int:
    return int(lib().cider_workspace_bytes_mnk(M, N, K))


def cider_workspace_bytes_w4a8_pc(M: int, N: int, K: int) -> int:
    return int(lib().cider_workspace_bytes_w4a8_pc(M, N, K))


def cider_set_small_m_threshold(threshold: int):
    _check("cider_set_small_m_threshold", lib().cider_set_small_m_threshold(threshold))


def cider_get_small_m_threshold() -> int:
    return int(lib().cider_get_small_m_threshold())


# ---- the operations -----------------------------------------------------------

def cider_quantize_act(x, q=None, scale_x=None, stream=None):
    """x [M, K] fp16/bf16 -> (q int8 [M, K], scale_x fp32 [M]).  x and q may be
    row-strided views (unit stride along K); their row strides are passed on."""
    M, K = x.shape
    if x.stride(1) != 1 or (q is not None and q.stride(1) != 1):
        raise ValueError("x and q need unit stride along K")
    q = torch.empty((M, K), dtype=torch.int8, device=x.device) if q is None else q
    scale_x = torch.empty((M,), dtype=torch.float32, device=x.device) if scale_x is None else scale_x
    _check("cider_quantize_act", lib().cider_quantize_act(
        _ptr(x), _DT[x.dtype], M, K, x.stride(0) if M > 1 else K, _ptr(q), q.stride(0) if M > 1 else K,
        _ptr(scale_x), _stream(stream, x.device)))
    return q, scale_x


def _workspace(M, K, device, workspace, N=0):
    need = cider_workspace_bytes_mnk(M, N, K) if N else cider_workspace_bytes(M, K)
    if workspace is None and need:
        workspace = torch.empty((need,), dtype=torch.uint8, device=device)
    return workspace, (0 if workspace is None else workspace.numel() * workspace.element_size())


def _out(y, M, N, dtype, device):
    return torch.empty((M, N), dtype=dtype, device=device) if y is None else y


def cider_w8a8_linear_pc(x, w, scale_w, y=None, out_dtype=None, workspace=None, stream=None):
    """W8A8 per-channel linear: x [M, K], w int8 [N, K], scale_w fp32 [N] -> y [M, N]."""
    _contig(x, "x"), _contig(w, "w")
    M, K = x.shape
    N = w.shape[0]
    y = _out(y, M, N, out_dtype or x.dtype, x.device)
    ws, ws_bytes = _workspace(M, K, x.device, workspace, N)
    _check("cider_w8a8_linear_pc", lib().cider_w8a8_linear_pc(
        _ptr(x), _DT[x.dtype], M, K, _ptr(w), _ptr(scale_w), N, _ptr(y), _DT[y.dtype],
        _ptr(ws), ws_bytes, _stream(stream, x.device)))
    return y


def cider_w8a16_mv_pc(x, w, scale_w, y=None, out_dtype=None, stream=None):
    """W8A16 decode product (1 <= M <= 4): y = scale_w[n] * sum_k x[m,k] * w[n,k]
    with fp16/bf16 x used as is (no activation quantization)."""
    _contig(x, "x"), _contig(w, "w")
    M, K = x.shape
    N = w.shape[0]
    y = _out(y, M, N, out_dtype or x.dtype, x.device)
    _check("cider_w8a16_mv_pc", lib().cider_w8a16_mv_pc(
        _ptr(x), _DT[x.dtype], M, K, _ptr(w), _ptr(scale_w), N, _ptr(y), _DT[y.dtype], _stream(stream, x.device)))
    return y


def cider_w8a16_mv_pg(x, w, scale_w, gs, y=None, out_dtype=None, stream=None):
    """W8A16 decode product with per-group weight scales (1 <= M <= 4):
    y = sum_g scale_w[g, n] * sum_{k in g} x[m,k] * w[n,k], fp16/bf16 x used
    as is; scale_w fp32 [K/gs, N] (group-major)."""
    _contig(x, "x"), _contig(w, "w")
    M, K = x.shape
    N = w.shape[0]
    y = _out(y, M, N, out_dtype or x.dtype, x.device)
    _check("cider_w8a16_mv_pg", lib().cider_w8a16_mv_pg(
        _ptr(x), _DT[x.dtype], M, K, _ptr(w), _ptr(scale_w), N, gs, _ptr(y), _DT[y.dtype],
        _stream(stream, x.device)))
    return y


def cider_w8a8_linear_pg(x, w, scale_w, gs, y=None, out_dtype=None, workspace=None, stream=None):
    """W8A8 per-group linear: scale_w fp32 [K/gs, N] (group-major)."""
    _contig(x, "x"), _contig(w, "w")
    M, K = x.shape
    N = w.shape[0]
    y = _out(y, M, N, out_dtype or x.dtype, x.device)
    ws, ws_bytes = _workspace(M, K, x.device, workspace, N)
    _check("cider_w8a8_linear_pg", lib().cider_w8a8_linear_pg(
        _ptr(x), _DT[x.dtype], M, K, _ptr(w), _ptr(scale_w), N, gs, _ptr(y), _DT[y.dtype],
        _ptr(ws), ws_bytes, _stream(stream, x.device)))
    return y


def cider_w4a8_linear_pg(x, w_packed, scale_w, gs, y=None, out_dtype=None, workspace=None, stream=None):
    """W4A8 per-group linear: w_packed uint8 [N, K/2], scale_w fp32 [K/gs, N]."""
    _contig(x, "x"), _contig(w_packed, "w_packed")
    M, K = x.shape
    N = w_packed.shape[0]
    y = _out(y, M, N, out_dtype or x.dtype, x.device)
    ws, ws_bytes = _workspace(M, K, x.device, workspace, N)
    _check("cider_w4a8_linear_pg", lib().cider_w4a8_linear_pg(
        _ptr(x), _DT[x.dtype], M, K, _ptr(w_packed), _ptr(scale_w), N, gs, _ptr(y), _DT[y.dtype],
        _ptr(ws), ws_bytes, _stream(stream, x.device)))
    return y


def cider_w4a8_linear_pc(x, w_packed, scale_w, y=None, out_dtype=None, workspace=None, stream=None):
    """W4A8 linear with one scale per output channel: w_packed uint8 [N, K/2],
    scale_w fp32 [N]."""
    _contig(x, "x"), _contig(w_packed, "w_packed")
    M, K = x.shape
    N = w_packed.shape[0]
    y = _out(y, M, N, out_dtype or x.dtype, x.device)
    if workspace is None:
        need = cider_workspace_bytes_w4a8_pc(M, N, K)
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=x.device)
    ws, ws_bytes = workspace, workspace.numel() * workspace.element_size()
    _check("cider_w4a8_linear_pc", lib().cider_w4a8_linear_pc(
        _ptr(x), _DT[x.dtype], M, K, _ptr(w_packed), _ptr(scale_w), N, _ptr(y), _DT[y.dtype],
        _ptr(ws), ws_bytes, _stream(stream, x.device)))
    return y


def cider_w8a8_linear_pc_noalloc(x, w, scale_w, y=None, out_dtype=None, stream=None):
    """The per-channel linear without a workspace, for callers that cannot
    allocate device memory: its scratch is a fixed 32 MiB array inside the
    library, shared by every call on the device (calls that overlap on the GPU
    race on it).  Raises CiderError when M*K is too large for that scratch."""
    _contig(x, "x"), _contig(w, "w")
    M, K = x.shape
    N = w.shape[0]
    y = _out(y, M, N, out_dtype or x.dtype, x.device)
    _check("cider_w8a8_linear_pc_noalloc", lib().cider_w8a8_linear_pc_noalloc(
        _ptr(x), _DT[x.dtype], M, K, _ptr(w), _ptr(scale_w), N, _ptr(y), _DT[y.dtype],
        _stream(stream, x.device)))
    return y


def cider_w8a8_gemm_pc_q(q, scale_x, w, scale_w, y=None, out_dtype=torch.float16, stream=None):
    M, K = q.shape
    N = w.shape[0]
    y = _out(y, M, N, out_dtype, q.device)
    _check("cider_w8a8_gemm_pc_q", lib().cider_w8a8_gemm_pc_q(
        _ptr(q), _ptr(scale_x), M, K, _ptr(w), _ptr(scale_w), N, _ptr(y), _DT[y.dtype],
        _stream(stream, q.device)))
    return y


def cider_w8a8_gemm_pg_q(q, scale_x, w, scale_w, gs, y=None, out_dtype=torch.float16, stream=None):
    M, K = q.shape
    N = w.shape[0]
    y = _out(y, M, N, out_dtype, q.device)
    _check("cider_w8a8_gemm_pg_q", lib().cider_w8a8_gemm_pg_q(
        _ptr(q), _ptr(scale_x), M, K, _ptr(w), _ptr(scale_w), N, gs, _ptr(y), _DT[y.dtype],
        _stream(stream, q.device)))
    return y


def cider_w4a8_gemm_pg_q(q, scale_x, w_packed, scale_w, gs, y=None, out_dtype=torch.float16, stream=None):
    M, K = q.shape
    N = w_packed.shape[0]
    y = _out(y, M, N, out_dtype, q.device)
    _check("cider_w4a8_gemm_pg_q", lib().cider_w4a8_gemm_pg_q(
        _ptr(q), _ptr(scale_x), M, K, _ptr(w_packed), _ptr(scale_w), N, gs, _ptr(y), _DT[y.dtype],
        _stream(stream, q.device)))
    return y


def cider_w4a8_gemm_pc_q(q, scale_x, w_packed, scale_w, y=None, out_dtype=torch.float16, stream=None):
    M, K = q.shape
    N = w_packed.shape[0]
    y = _out(y, M, N, out_dtype, q.device)
    _check("cider_w4a8_gemm_pc_q", lib().cider_w4a8_gemm_pc_q(
        _ptr(q), _ptr(scale_x), M, K, _ptr(w_packed), _ptr(scale_w), N, _ptr(y), _DT[y.dtype],
        _stream(stream, q.device)))
    return y


def cider_silu_mul_quantize(gate, up, want_a=False, q=None, scale_x=None, stream=None):
    """-> (q int8 [M, F], scale_x fp32 [M], a [M, F] or None)."""
    _contig(gate, "gate"), _contig(up, "up")
    M, F = gate.shape
    q = torch.empty((M, F), dtype=torch.int8, device=gate.device) if q is None else q
    scale_x = torch.empty((M,), dtype=torch.float32, device=gate.device) if scale_x is None else scale_x
    a = torch.empty_like(gate) if want_a else None
    _check("cider_silu_mul_quantize", lib().cider_silu_mul_quantize(
        _ptr(gate), _ptr(up), _DT[gate.dtype], M, F, _ptr(q), _ptr(scale_x), _ptr(a),
        _stream(stream, gate.device)))
    return q, scale_x, a


def cider_quantize_weight_pc(W, stream=None):
    """W fp32 [N, K] -> (w int8 [N, K], scale_w fp32 [N])."""
    N, K = W.shape
    w = torch.empty((N, K), dtype=torch.int8, device=W.device)
    s = torch.empty((N,), dtype=torch.float32, device=W.device)
    _check("cider_quantize_weight_pc", lib().cider_quantize_weight_pc(
        _ptr(_contig(W, "W")), N, K, _ptr(w), _ptr(s), _stream(stream, W.device)))
    return w, s


def cider_quantize_weight_pg(W, gs, stream=None):
    """W fp32 [N, K] -> (w int8 [N, K], scale_w fp32 [K/gs, N])."""
    N, K = W.shape
    w = torch.empty((N, K), dtype=torch.int8, device=W.device)
    s = torch.empty((K // gs, N), dtype=torch.float32, device=W.device)
    _check("cider_quantize_weight_pg", lib().cider_quantize_weight_pg(
        _ptr(_contig(W, "W")), N, K, gs, _ptr(w), _ptr(s), _stream(stream, W.device)))
    return w, s


def cider_quantize_weight_pc_clip(W, clip_percentile, stream=None):
    """Percentile-clipped per channel: W fp32 [N, K] -> (w int8 [N, K] in
    [-127, 127], scale_w fp32 [N])."""
    N, K = W.shape
    w = torch.empty((N, K), dtype=torch.int8, device=W.device)
    s = torch.empty((N,), dtype=torch.float32, device=W.device)
    _check("cider_quantize_weight_pc_clip", lib().cider_quantize_weight_pc_clip(
        _ptr(_contig(W, "W")), N, K, float(clip_percentile), _ptr(w), _ptr(s), _stream(stream, W.device)))
    return w, s


def cider_quantize_weight_pg_clip(W, gs, clip_percentile, stream=None):
    """Percentile-clipped per group: W fp32 [N, K] -> (w int8 [N, K],
    scale_w fp32 [K/gs, N])."""
    N, K = W.shape
    w = torch.empty((N, K), dtype=torch.int8, device=W.device)
    s = torch.empty((K // gs, N), dtype=torch.float32, device=W.device)
    _check("cider_quantize_weight_pg_clip", lib().cider_quantize_weight_pg_clip(
        _ptr(_contig(W, "W")), N, K, gs, float(clip_percentile), _ptr(w), _ptr(s), _stream(stream, W.device)))
    return w, s


def cider_pack_weight_int4_pg(W, gs, stream=None):
    """W fp32 [N, K] -> (packed uint8 [N, K/2], scale_w fp32 [K/gs, N])."""
    N, K = W.shape
    p = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    s = torch.empty((K // gs, N), dtype=torch.float32, device=W.device)
    _check("cider_pack_weight_int4_pg", lib().cider_pack_weight_int4_pg(
        _ptr(_contig(W, "W")), N, K, gs, _ptr(p), _ptr(s), _stream(stream, W.device)))
    return p, s


def cider_pack_weight_int4_pc(W, stream=None):
    """W fp32 [N, K] -> (packed uint8 [N, K/2], scale_w fp32 [N])."""
    N, K = W.shape
    p = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    s = torch.empty((N,), dtype=torch.float32, device=W.device)
    _check("cider_pack_weight_int4_pc", lib().cider_pack_weight_int4_pc(
        _ptr(_contig(W, "W")), N, K, _ptr(p), _ptr(s), _stream(stream, W.device)))
    return p, s


def cider_sdpa_decode_workspace_bytes(H_q: int, H_kv: int, N: int, D: int = 128) -> int:
    return int(lib().cider_sdpa_decode_workspace_bytes(H_q, H_kv, N, D))


def cider_test_sdpa_plan(H_q, H_kv, N, num_sms):
    """-> (query heads per CTA, head tiles per KV group, keys per chunk, chunks)."""
    out = (ctypes.c_int32 * 4)()
    _check("cider_test_sdpa_plan", lib().cider_test_sdpa_plan(H_q, H_kv, N, num_sms, out))
    return tuple(out)


def cider_sdpa_decode(q, k, v, out=None, workspace=None, stream=None):
    """Decode attention: q [H_q, D], k and v [H_kv, N, D] (fp16 or bf16, D = 128)
    -> out [H_q, D]: softmax(q . k / sqrt(D)) v per head, H_q / H_kv query
    heads per KV head."""
    _contig(q, "q"), _contig(k, "k"), _contig(v, "v")
    H_q, D = q.shape
    H_kv, N, _ = k.shape
    out = torch.empty((H_q, D), dtype=q.dtype, device=q.device) if out is None else out
    if workspace is None:
        need = int(lib().cider_sdpa_decode_workspace_bytes(H_q, H_kv, N, D))
        workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=q.device)
    _check("cider_sdpa_decode", lib().cider_sdpa_decode(
        _ptr(q), _ptr(k), _ptr(v), _DT[q.dtype], H_q, H_kv, N, D, _ptr(out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream, q.device)))
    return out


# ---- test exports ---------------------------------------------------------------

def cider_test_gemm_i32(q, w, acc=None, stream=None):
    M, K = q.shape
    N = w.shape[0]
    acc = torch.empty((M, N), dtype=torch.int32, device=q.device) if acc is None else acc
    _check("cider_test_gemm_i32", lib().cider_test_gemm_i32(
        _ptr(q), _ptr(w), M, N, K, _ptr(acc), _stream(stream, q.device)))
    return acc


def cider_test_gemm_i32_grouped(q, w, gs, acc_g=None, stream=None):
    M, K = q.shape
    N = w.shape[0]
    acc_g = torch.empty((K // gs, M, N), dtype=torch.int32, device=q.device) if acc_g is None else acc_g
    _check("cider_test_gemm_i32_grouped", lib().cider_test_gemm_i32_grouped(
        _ptr(q), _ptr(w), M, N, K, gs, _ptr(acc_g), _stream(stream, q.device)))
    return acc_g


def cider_test_set_gemm_variant(variant: int):
    """0 automatic, 1 single-CTA 128x128, 2 single-CTA 128x256, 3 CTA-pair 256x256, 4 single-CTA 128x80,
    5 CTA-pair 256x192."""
    _check("cider_test_set_gemm_variant", lib().cider_test_set_gemm_variant(variant))


def cider_test_set_sdpa_kernel(kernel: int):
    """0 automatic, 1 CUDA cores only, 2 tensor cores, 3 tensor cores with the V descriptor fields swapped."""
    _check("cider_test_set_sdpa_kernel", lib().cider_test_set_sdpa_kernel(kernel))


def cider_test_set_small_m_kernel(kernel: int):
    """0 automatic, 1 register ring, 2 bulk-staged, 3 bulk-staged within half of shared memory, 4 one-shot."""
    _check("cider_test_set_small_m_kernel", lib().cider_test_set_small_m_kernel(kernel))


def cider_test_set_fused_quantize(mode: int):
    """0 automatic, 1 always the separate quantize kernel, 2 always inside the GEMM launch."""
    _check("cider_test_set_fused_quantize", lib().cider_test_set_fused_quantize(mode))


def cider_test_set_split_k(splits: int):
    """0 automatic split-K of the per-group GEMM, 1 never, 2..16 forced pieces."""
    _check("cider_test_set_split_k", lib().cider_test_set_split_k(splits))


def cider_test_bounded_wait(limit_ns: int, stream=None, device=None):
    """Runs the bounded-wait self-test kernel (see include/cider.h)."""
    _check("cider_test_bounded_wait", lib().cider_test_bounded_wait(limit_ns, _stream(stream, device)))


def cider_test_unpack_int4(w_packed, K, w=None, stream=None):
    N = w_packed.shape[0]
    w = torch.empty((N, K), dtype=torch.int8, device=w_packed.device) if w is None else w
    _check("cider_test_unpack_int4", lib().cider_test_unpack_int4(
        _ptr(w_packed), N, K, _ptr(w), _stream(stream, w_packed.device)))
    return w
