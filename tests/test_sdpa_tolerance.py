"""The decode-attention tolerance (tests/sdpa_tolerance.py) can fail: on the
host, planted mistakes in the two-pass combination of chunk results -- a
chunk left out of the merge, a chunk's partial added without its rescale to
the common maximum, one of the 16 key streams left out -- are recomputed in
float64 from the same seeded inputs the GPU tests use, and the bound must
reject each of them.  The same inputs evaluated in float32 in the kernels'
order must pass it, so the bound is not tighter than fp32 arithmetic of that
structure.  Chunk sizes come from the kernels' own plan for a 148-SM B200
(cider_test_sdpa_plan, which needs no device)."""
import numpy as np
import pytest

import oracle
from oracle import sdpa
from tests import sdpa_tolerance as tl

NUM_SMS = 148
F16 = oracle.F16

CASES = [
    ("diffuse", 4, 4, 32768),
    ("diffuse", 4, 1, 4096),
    ("peaked", 8, 2, 8192),
    ("last_max", 8, 2, 8192),
    ("last_max", 4, 4, 32768),
]


@pytest.fixture(scope="module", params=CASES, ids=lambda c: "-".join(map(str, c)))
def case(request):
    kind, H_q, H_kv, N = request.param
    q, k, v = tl.make_inputs(kind, H_q, H_kv, N, seed=N + H_q)
    ref = sdpa.sdpa_decode(q, k, v, F16)
    kps, chunks, chunk = tl.plan_depths(H_q, H_kv, N, NUM_SMS)
    return dict(q=q, k=k, v=v, ref=ref, chunk=chunk, chunks=chunks, kind=kind)


def _n_bad(case, got):
    n, _ = tl.violations(case["ref"], got, case["q"], case["k"], case["v"], F16, NUM_SMS)
    return n


def test_chunked_f64_without_mistakes_equals_the_oracle(case):
    got = tl.chunked_f64(case["q"], case["k"], case["v"], F16, case["chunk"])
    assert np.count_nonzero(got != case["ref"]) <= 2  # float64 order only; within one unit
    assert _n_bad(case, got) == 0


def test_fp32_in_kernel_order_passes(case):
    got = tl.kernel_order_f32(case["q"], case["k"], case["v"], F16, case["chunk"])
    assert _n_bad(case, got) == 0


def _top_key(case):
    """Index of head 0's highest-scoring key (the key a peaked head rests on)."""
    qf = oracle.widen(case["q"], F16).astype(np.float64)
    kf = oracle.widen(case["k"], F16).astype(np.float64)
    return int(np.argmax(kf[0] @ qf[0]))


def test_dropped_middle_chunk_is_rejected(case):
    assert case["chunks"] >= 3
    # a middle chunk; with peaked weights, the chunk that holds head 0's top key
    c = case["chunks"] // 2 if case["kind"] == "diffuse" else _top_key(case) // case["chunk"]
    got = tl.chunked_f64(case["q"], case["k"], case["v"], F16, case["chunk"], drop_chunks=(c,))
    assert _n_bad(case, got) > 0


def test_dropped_last_chunk_is_rejected(case):
    if case["kind"] == "peaked":
        pytest.skip("peaked weights rest on a few keys; the last chunk need not hold any")
    got = tl.chunked_f64(case["q"], case["k"], case["v"], F16, case["chunk"], drop_chunks=(case["chunks"] - 1,))
    assert _n_bad(case, got) > 0


def test_unrescaled_chunk_partial_is_rejected(case):
    # the first chunk whose maximum is below the common one, added as if it were not
    got = tl.chunked_f64(case["q"], case["k"], case["v"], F16, case["chunk"], unrescaled_chunks=(0,))
    assert _n_bad(case, got) > 0


def test_dropped_key_stream_is_rejected(case):
    stream = 5 if case["kind"] == "diffuse" else (_top_key(case) % case["chunk"]) % 16
    got = tl.chunked_f64(case["q"], case["k"], case["v"], F16, case["chunk"], drop_stream=stream)
    assert _n_bad(case, got) > 0


def test_last_max_is_in_the_last_chunk():
    q, k, v = tl.make_inputs("last_max", 8, 2, 8192, seed=1)
    _, _, chunk = tl.plan_depths(8, 2, 8192, NUM_SMS)
    qf = oracle.widen(q, F16).astype(np.float64)
    kf = oracle.widen(k, F16).astype(np.float64)
    for h in range(8):
        s = kf[h // 4] @ qf[h]
        j = int(np.argmax(s))
        assert j // chunk == (8192 - 1) // chunk
        assert (s[j] - np.partition(s, -2)[-2]) / np.sqrt(128) >= 2.9
