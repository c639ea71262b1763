"""The host-buffer GEMV that allocates no device memory (needs a B200).

stagq_gemv_host_noalloc serves callers that must not allocate device memory
while they run (a fixed budget owned by another allocator, or a phase where
allocation is forbidden): it stages x and y through the library's static
device array instead of a buffer allocated on first use. Its y must equal the
allocating entry point's on consecutive calls -- the array keeps the previous
call's contents, which must not leak into the next result.

This file is collected last on purpose, and also passes on its own in a fresh
process (the first call on the device sets up the array's address).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import quantized_gemv_stagq_b200 as Q
from oracle import stagq as O
from quantized_gemv_stagq_b200 import synth
from tests.helpers import check_close

pytestmark = pytest.mark.gpu


def test_noalloc_host_gemv_matches_host_gemv_on_consecutive_calls():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    out, inp = 1024, 4096
    P = Q.stagq_encode(synth.weights(out, inp, seed=77), 128, 2, 0.005, "fast")
    m = Q.stagq_load(Q.stagq_pack(P), 0)
    rng = np.random.default_rng(78)
    # two calls in a row with different x (and n): the second must not see the first's leftovers
    for call, (n, bits) in enumerate([(4, 4), (1, 2)]):
        x = (rng.standard_normal((n, inp)) * (1.0 + call)).astype(np.float16)
        y_ref = np.empty((n, out), np.float16)
        y = np.full((n, out), np.float16(np.nan))
        Q.stagq_gemv_host(m, bits, x, y_ref, n=n)
        Q.stagq_gemv_host_noalloc(m, bits, x, y, n=n)
        assert np.all(np.isfinite(y)), f"call {call}: y not fully written"
        check_close(y.astype(np.float64), y_ref.astype(np.float64), f"call {call} p{bits} n{n}")
        assert np.array_equal(y.view(np.uint16), y_ref.view(np.uint16)), f"call {call}: not bit-identical"
    Q.stagq_check(m)
    m.free()


def test_noalloc_host_gemv_on_a_large_matrix():
    """A matrix of more than 2^24 weights, where n = 1 runs the single-vector
    kernel: its reads of x from the static array match the allocating call."""
    out, inp = 14336, 4096
    P = Q.stagq_encode(synth.weights(out, inp, seed=81), 128, 2, 0.005, "fast")
    m = Q.stagq_load(Q.stagq_pack(P), 0)
    rng = np.random.default_rng(82)
    for call, bits in enumerate((4, 2)):
        x = rng.standard_normal((1, inp)).astype(np.float16)
        y_ref = np.empty((1, out), np.float16)
        y = np.full((1, out), np.float16(np.nan))
        Q.stagq_gemv_host(m, bits, x, y_ref)
        Q.stagq_gemv_host_noalloc(m, bits, x, y)
        assert np.all(np.isfinite(y)), f"call {call}: y not fully written"
        check_close(y.astype(np.float64), y_ref.astype(np.float64), f"large call {call} p{bits}")
        assert np.array_equal(y.view(np.uint16), y_ref.view(np.uint16)), f"large call {call}: not bit-identical"
    Q.stagq_check(m)
    m.free()


def test_noalloc_host_gemv_rejects_outputs_beyond_the_static_area():
    out, inp = 8192, 128
    P = Q.stagq_encode(synth.weights(out, inp, seed=79), 64, 1, 0.0, "fast")
    m = Q.stagq_load(Q.stagq_pack(P), 0)
    # n * out * 2 bytes = 64 KiB fits; the limit is STAGQ_NOALLOC_STAGE_BYTES - 256 KiB
    x = np.zeros((4, inp), np.float16)
    y = np.empty((4, out), np.float16)
    Q.stagq_gemv_host_noalloc(m, 2, x, y, n=4)
    assert not np.any(y.astype(np.float32))
    m.free()
    # at n = 4, y of more than (2 MiB - 256 KiB) / 8 = 229376 rows does not fit
    big_out = 229384
    P = Q.stagq_encode(synth.weights(big_out, 128, seed=80), 64, 1, 0.0, "fast")
    mb = Q.stagq_load(Q.stagq_pack(P), 0)
    with pytest.raises(Q.StagqError) as e:
        Q.stagq_gemv_host_noalloc(mb, 2, np.zeros((4, 128), np.float16), np.empty((4, big_out), np.float16), n=4)
    assert e.value.status == 1
    y1 = np.empty((1, big_out), np.float16)  # the same matrix at n = 1 fits
    Q.stagq_gemv_host_noalloc(mb, 2, np.zeros((1, 128), np.float16), y1, n=1)
    assert not np.any(y1.astype(np.float32))
    mb.free()
