"""CPU-side checks of the C-ABI boundary: the library builds and loads, exports
every entry point that include/cider.h declares, and rejects bad arguments on
the host before touching a device (so these run without a GPU)."""
import ctypes
import os
import re

import pytest

import w8a8_activation_quantized_b200 as cider
from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "cider.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"CIDER_API[^;]*?\b(cider_\w+)\s*\(", text, flags=re.S)))


@pytest.fixture(scope="module")
def lib():
    from w8a8_activation_quantized_b200._build import build_library
    build_library()
    return cider.lib()


def test_header_declares_the_four_operations():
    names = _declared()
    for op in ("cider_quantize_act", "cider_w8a8_linear_pc", "cider_w8a8_linear_pg", "cider_w4a8_linear_pg"):
        assert op in names


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 20
    for n in names:
        assert hasattr(lib, n), f"{n} declared in cider.h but not exported"
    assert sorted(cider.EXPORTS) == names  # the binding covers exactly the header


def test_status_strings(lib):
    for s in range(5):
        assert lib.cider_status_string(s)


P = ctypes.c_void_p(256)  # a 16-byte aligned, never dereferenced address


def _lin_pc(lib, **kw):
    a = dict(x=P, xdt=0, M=4, K=64, w=ctypes.c_void_p(4096), sw=ctypes.c_void_p(8192), N=16,
             y=ctypes.c_void_p(1 << 20), ydt=0, ws=None, wsb=0, st=None)
    a.update(kw)
    return lib.cider_w8a8_linear_pc(a["x"], a["xdt"], a["M"], a["K"], a["w"], a["sw"], a["N"], a["y"],
                                    a["ydt"], a["ws"], a["wsb"], a["st"])


@pytest.mark.parametrize("kw,why", [
    (dict(K=40), "K % 16"),
    (dict(N=12), "N % 8"),
    (dict(M=-1), "M < 0"),
    (dict(K=0), "K < 1"),
    (dict(K=131072 + 16), "K too large"),
    (dict(xdt=7), "dtype"),
    (dict(x=None), "NULL"),
    (dict(x=ctypes.c_void_p(258)), "misaligned"),
    (dict(y=ctypes.c_void_p(256 + 64)), "y overlaps x"),
])
def test_invalid_arguments_rejected_on_host(lib, kw, why):
    assert _lin_pc(lib, **kw) == 1, why
    assert lib.cider_last_error()


def test_empty_input_is_a_noop(lib):
    assert _lin_pc(lib, M=0) == 0


def test_group_size_checks(lib):
    f = lib.cider_w8a8_linear_pg
    base = (P, 0, 4, 256, ctypes.c_void_p(4096), ctypes.c_void_p(8192), 16)
    assert f(*base, 32, ctypes.c_void_p(1 << 20), 0, None, 0, None) == 1       # gs not 64/128
    assert f(P, 0, 4, 192, ctypes.c_void_p(4096), ctypes.c_void_p(8192), 16, 128,
             ctypes.c_void_p(1 << 20), 0, None, 0, None) == 1                   # gs does not divide K
    g = lib.cider_w4a8_linear_pg
    assert g(P, 0, 4, 192, ctypes.c_void_p(4096), ctypes.c_void_p(8192), 16, 128,
             ctypes.c_void_p(1 << 20), 0, None, 0, None) == 1                   # gs does not divide K
    assert lib.cider_set_small_m_threshold(17) == 1
    assert lib.cider_set_small_m_threshold(-1) == 1


def test_workspace_size(lib):
    thr = lib.cider_get_small_m_threshold()
    assert lib.cider_workspace_bytes(1, 2560) == 0 if thr >= 1 else True
    M, K = 4096, 2560
    assert lib.cider_workspace_bytes(M, K) == M * K + ((M * 4 + 255) // 256) * 256
    assert lib.cider_workspace_bytes(0, 64) == 0


def test_no_device_means_unsupported_or_cuda_error(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert lib.cider_is_available() == 0
    # valid arguments, no device: the call must fail loudly, never compute on the CPU
    st = _lin_pc(lib)
    assert st in (2, 3)


# ---- the entry points added for the pages' other forms: host-side checks ----

def _sdpa(lib, **kw):
    a = dict(q=P, k=ctypes.c_void_p(4096), v=ctypes.c_void_p(1 << 16), dt=0, H_q=32, H_kv=8, N=64, D=128,
             out=ctypes.c_void_p(1 << 20), ws=ctypes.c_void_p(1 << 22), wsb=1 << 20, st=None)
    a.update(kw)
    return lib.cider_sdpa_decode(a["q"], a["k"], a["v"], a["dt"], a["H_q"], a["H_kv"], a["N"], a["D"], a["out"],
                                 a["ws"], a["wsb"], a["st"])


@pytest.mark.parametrize("kw,why", [
    (dict(D=64), "D must be 128"),
    (dict(H_q=30), "H_kv must divide H_q"),
    (dict(H_kv=0), "H_kv >= 1"),
    (dict(N=0), "N >= 1"),
    (dict(N=(1 << 30) + 1), "N <= 2^30"),
    (dict(dt=7), "dtype"),
    (dict(v=None), "NULL"),
    (dict(k=ctypes.c_void_p(4100)), "misaligned"),
])
def test_sdpa_arguments_rejected_on_host(lib, kw, why):
    assert _sdpa(lib, **kw) == 1, why
    assert lib.cider_last_error()


def test_sdpa_without_a_device_fails_loudly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _sdpa(lib) in (2, 3)


@pytest.mark.parametrize("H_q,H_kv", [(32, 32), (32, 8), (32, 4), (8, 1), (6, 3), (3, 1), (64, 2)])
@pytest.mark.parametrize("N", [1, 15, 16, 17, 1000, 1024, 4096, 32768, 1 << 20])
@pytest.mark.parametrize("sms", [148, 132, 1])
@pytest.mark.parametrize("kernel", [0, 1])
def test_sdpa_plan_covers_every_key(H_q, H_kv, N, sms, kernel):
    """kernel 1: the CUDA-core kernels' cut (head tiles of 1, 2 or 4 query
    heads, chunks of whole 16-key streams); kernel 0 (automatic) takes the
    tensor-core cut for 2 <= H_q / H_kv <= 16 (one CTA per KV head and chunk
    of 1 .. 15 whole 128-key tiles: the fewest tiles that put every CTA in one
    wave of one CTA per SM) when its chunks fit the merge."""
    cider.cider_test_set_sdpa_kernel(kernel)
    try:
        th, tiles, chunk, chunks = cider.cider_test_sdpa_plan(H_q, H_kv, N, sms)
    finally:
        cider.cider_test_set_sdpa_kernel(0)
    G = H_q // H_kv
    tc = kernel == 0 and 2 <= G <= 16 and -(-N // 1920) <= 1024
    assert 1 <= chunks <= 1024
    assert (chunks - 1) * chunk < N <= chunks * chunk  # every chunk has a key; every key has a chunk
    if tc:
        assert th == G and tiles == 1
        assert chunk % 128 == 0 and 128 <= chunk <= 1920
        tiles, t = -(-N // 128), 1
        while t < 15 and H_kv * -(-tiles // t) > sms:
            t += 1
        assert chunk == 128 * t
        assert H_kv * chunks <= sms or t == 15
    else:
        assert th in (1, 2, 4) and th * tiles == G
        assert th == (4 if G % 4 == 0 else 2 if G % 2 == 0 else 1)
        assert chunk % 16 == 0 and chunk >= 16
        # enough CTAs to fill the device, unless the keys or the merge's chunk limit run out first
        assert H_kv * tiles * chunks >= min(4 * sms, H_kv * tiles * -(-N // 16)) or chunks >= 1024 or \
            chunks == -(-N // chunk)


def test_sdpa_plan_rejects_bad_shapes(lib):
    with pytest.raises(cider.CiderError):
        cider.cider_test_sdpa_plan(30, 8, 64, 148)
    with pytest.raises(cider.CiderError):
        cider.cider_test_sdpa_plan(32, 8, 64, 0)


def test_clip_and_w4pc_arguments_rejected_on_host(lib):
    W, out, sw = P, ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 21)
    for p in (-0.5, 100.5, float("nan")):
        assert lib.cider_quantize_weight_pc_clip(W, 8, 64, p, out, sw, None) == 1
    assert lib.cider_quantize_weight_pg_clip(W, 8, 256, 32, 99.9, out, sw, None) == 1      # gs not 64/128
    assert lib.cider_pack_weight_int4_pc(W, 8, 63, out, sw, None) == 1                      # odd K
    assert lib.cider_w4a8_linear_pc(P, 0, 4, 48, ctypes.c_void_p(4096), ctypes.c_void_p(8192), 16,
                                    ctypes.c_void_p(1 << 20), 0, None, 0, None) == 1          # K % 32


def test_w4pc_workspace_covers_small_m(lib):
    # the per-column W4A8 form has no decode kernel: even M = 1 needs q and scale_x
    assert lib.cider_workspace_bytes_w4a8_pc(1, 256, 1024) >= 1024 + 256
    assert lib.cider_workspace_bytes_w4a8_pc(0, 256, 1024) == 0


def _quant(lib, **kw):
    a = dict(x=P, xdt=0, M=4, K=64, ldx=64, q=ctypes.c_void_p(1 << 20), ldq=64, sx=ctypes.c_void_p(1 << 21), st=None)
    a.update(kw)
    return lib.cider_quantize_act(a["x"], a["xdt"], a["M"], a["K"], a["ldx"], a["q"], a["ldq"], a["sx"], a["st"])


@pytest.mark.parametrize("kw,why", [
    (dict(ldx=48), "ldx < K"),
    (dict(ldq=32), "ldq < K"),
    (dict(ldx=68), "ldx not a multiple of 8"),
    (dict(ldq=72), "ldq not a multiple of 16"),
    (dict(K=40, ldx=40, ldq=48), "K % 16"),
    (dict(ldx=128, q=ctypes.c_void_p(256 + 3 * 128 * 2)), "q inside the strided span of x"),
])
def test_quantize_act_stride_checks(lib, kw, why):
    assert _quant(lib, **kw) == 1, why
    assert lib.cider_last_error()


def test_quantize_act_strided_span_allows_q_past_it(lib):
    # x rows 0..3 at stride 128 span (3 * 128 + 64) * 2 bytes from 256; q right after is legal,
    # and the call then fails only for want of a device (not an argument error)
    q = ctypes.c_void_p(256 + (3 * 128 + 64) * 2 + 16 * 40)
    assert _quant(lib, ldx=128, q=q) in (2, 3)
