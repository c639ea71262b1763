"""Host side of libstagq.so (CPU only): exported symbols, encoder and packer
against the oracle, the byte-scaling property of the layout, error paths."""
import ctypes
import os
import re

import numpy as np
import pytest

import quantized_gemv_stagq_b200 as Q
from oracle import stagq as O
from quantized_gemv_stagq_b200 import synth
from tests.helpers import fields_equal, to_lib_fields

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "stagq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(stagq_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_function():
    names = _declared_functions()
    assert len(names) >= 18
    L = Q.lib()
    for n in names:
        assert hasattr(L, n), f"libstagq.so does not export {n}"


@pytest.mark.parametrize("out,inp,g,npl,dens,mode", [
    (64, 512, 128, 2, 0.005, "search"),
    (48, 256, 64, 4, 0.01, "search"),
    (32, 256, 64, 0, 0.0, "search"),
    (16, 256, 16, 2, 0.02, "search"),
    (256, 1024, 128, 2, 0.005, "fast"),
    (40, 384, 128, 3, 1.0, "search"),
    (8, 128, 64, 1, 0.3, "fast"),
])
def test_encoder_matches_oracle_bit_exactly(out, inp, g, npl, dens, mode):
    W = synth.weights(out, inp, seed=out * 7 + inp)
    F = O.encode(W, group=g, n_planes=npl, density=dens, mode=mode)
    P = Q.stagq_encode(W, group=g, n_planes=npl, density=dens, mode=mode, n_threads=3)
    eq = fields_equal(F, P)
    assert all(eq.values()), eq


@pytest.mark.parametrize("out,inp,g,npl,T,post,mode", [
    (64, 512, 64, 2, 4.0, True, "fast"),
    (48, 256, 16, 4, 4.0, True, "search"),
    (40, 384, 32, 3, 2.0, True, "fast"),
    (16, 256, 128, 2, 8.0, False, "search"),
    (8, 128, 64, 1, 4.0, True, "fast"),
])
def test_guarded_encoder_matches_oracle_bit_exactly(out, inp, g, npl, T, post, mode):
    """The paper's guards (pre-grid ratio criterion, post-grid per-row guard):
    every field, the post-grid flags in the columns and the residuals."""
    W = synth.weights(out, inp, seed=out * 5 + inp)
    W[3, 5] = np.float16(0.9)                 # a dominant entry: the ratio guard takes it
    F = O.encode(W, group=g, n_planes=npl, mode=mode, guard="ratio", ratio_T=T, post_guard=post)
    P = Q.stagq_encode(W, group=g, n_planes=npl, mode=mode, guard="ratio", ratio_T=T, post_guard=post, n_threads=3)
    eq = fields_equal(F, P)
    assert all(eq.values()), eq
    assert F.post_flags.sum() == (out if post else 0)
    assert ((P.col & Q.STAGQ_SIDE_POST) != 0).sum() == F.post_flags.sum()


@pytest.mark.parametrize("out,inp,g,npl,mode,dens", [
    (24, 256, 32, 2, "search", 0.0),
    (24, 256, 32, 3, "fast", 0.01),
    (16, 512, 64, 0, "fast", 0.0),       # no planes: the fallback keeps uniform placement
    (40, 384, 16, 2, "search", 0.02),
])
def test_codebook_rules_encoder_matches_oracle_bit_exactly(out, inp, g, npl, mode, dens):
    """Appendix E's codebook rules (Lloyd / anchored Lloyd / uniform, the
    nine-combination choice, the fallback): every field bit for bit."""
    from tests.test_oracle_pins import _weights_with_spread_scales
    W = _weights_with_spread_scales(out, inp, out + g)
    F = O.encode(W, g, npl, dens, mode, codebooks="appendix_e")
    P = Q.stagq_encode(W, g, npl, dens, mode, codebooks="appendix_e", n_threads=3)
    eq = fields_equal(F, P)
    assert all(eq.values()), eq
    U = O.encode(W, g, npl, dens, mode)
    assert np.array_equal(F.cb_log2s, U.cb_log2s) == (npl == 0)


def test_guarded_stream_packs_and_rereads():
    W = synth.weights(24, 640, seed=7)
    F = O.encode(W, group=32, n_planes=2, mode="fast", guard="ratio", ratio_T=4.0)
    S = Q.stagq_pack(to_lib_fields(F))
    for M in (2, 3, 4):
        assert np.array_equal(Q.stagq_unpack_levels_host(S, M), O.decode_levels(F, M)), M


def test_encoder_handles_constant_and_zero_groups():
    W = np.zeros((4, 256), np.float16)
    W[1, :128] = np.float16(0.25)
    W[2] = synth.weights(1, 256, seed=3)[0]
    for mode in ("search", "fast"):
        F = O.encode(W, group=128, n_planes=2, density=0.01, mode=mode)
        P = Q.stagq_encode(W, group=128, n_planes=2, density=0.01, mode=mode)
        eq = fields_equal(F, P)
        assert all(eq.values()), (mode, eq)


@pytest.mark.parametrize("npl,g", [(0, 64), (1, 128), (2, 128), (3, 64), (4, 64), (2, 16), (3, 32)])
def test_packed_levels_reread_on_host_equal_oracle_levels(npl, g):
    W = synth.weights(24, 640, seed=npl)
    F = O.encode(W, group=g, n_planes=npl, density=0.01, mode="fast")
    S = Q.stagq_pack(to_lib_fields(F))
    assert S.planes.size == 24 * 640 * (2 + npl) // 8
    for M in range(2, 3 + npl):
        assert np.array_equal(Q.stagq_unpack_levels_host(S, M), O.decode_levels(F, M)), M


def test_p_bit_read_touches_only_the_first_p_minus_2_planes():
    """Section 3.3: a shallower read skips the deeper planes. Overwriting every
    plane deeper than p leaves the p-bit read unchanged; overwriting plane p
    changes it."""
    W = synth.weights(16, 512, seed=5)
    F = O.encode(W, group=128, n_planes=4, density=0.005, mode="fast")
    S = Q.stagq_pack(to_lib_fields(F))
    out, inp = 16, 512
    rng = np.random.default_rng(0)
    for p in range(2, 7):
        ref = Q.stagq_unpack_levels_host(S, p)
        end = out * inp // 4 + (p - 2) * (out * inp // 8)    # bytes a p-read may touch
        T = Q.HostStream(**{**S.__dict__, "planes": S.planes.copy()})
        T.planes[end:] = rng.integers(0, 256, T.planes.size - end, dtype=np.uint8)
        assert np.array_equal(Q.stagq_unpack_levels_host(T, p), ref)
        if p > 2:
            T2 = Q.HostStream(**{**S.__dict__, "planes": S.planes.copy()})
            T2.planes[end - out * inp // 8:end] ^= 0xFF
            assert not np.array_equal(Q.stagq_unpack_levels_host(T2, p), ref)


def test_plane_bytes_and_side_record_count():
    assert Q.stagq_stream_plane_bytes(14336, 4096, 2) == 14336 * 4096 // 4 + 2 * 14336 * 4096 // 8
    assert Q.stagq_side_record_count(14336, 4096, 0.005) == O.side_record_count(14336, 4096, 0.005) == 293601
    assert Q.stagq_side_record_count(512, 512, 0.005) == 1311


def _stream(out=8, inp=256, npl=2, dens=0.02):
    W = synth.weights(out, inp, seed=1)
    return Q.stagq_pack(Q.stagq_encode(W, group=128, n_planes=npl, density=dens, mode="fast"))


def test_error_paths_return_status_codes():
    W = synth.weights(8, 192, seed=1)
    with pytest.raises(Q.StagqError) as e:   # in not a multiple of 128
        Q.stagq_pack(Q.stagq_encode(W, group=64, n_planes=2, density=0.0, mode="fast"))
    assert e.value.status == 1
    with pytest.raises(Q.StagqError) as e:   # group below 16
        Q.stagq_pack(Q.stagq_encode(synth.weights(8, 256, seed=1), group=8, n_planes=2, density=0.0, mode="fast"))
    assert e.value.status == 1
    S = _stream()
    with pytest.raises(Q.StagqError) as e:
        Q.stagq_unpack_levels_host(S, 5)          # bits > 2 + n_planes
    assert e.value.status == 1
    bad = Q.HostStream(**{**S.__dict__, "row_ptr": S.row_ptr.copy()})
    bad.row_ptr[3] = bad.row_ptr[4] + 1           # not monotone
    with pytest.raises(Q.StagqError) as e:
        Q.stagq_load(bad, 0)
    assert e.value.status == 2
    bad = Q.HostStream(**{**S.__dict__, "col": S.col.copy()})
    bad.col[0] = 256                              # col >= in
    with pytest.raises(Q.StagqError) as e:
        Q.stagq_save(bad, "/tmp/never_written.stagq")
    assert e.value.status == 2
    with pytest.raises(Q.StagqError) as e:
        Q.stagq_save(S, "/nonexistent_dir/x.stagq")
    assert e.value.status == 5


def test_stream_file_header(tmp_path):
    S = _stream()
    p = str(tmp_path / "m.stagq")
    Q.stagq_save(S, p)
    raw = open(p, "rb").read()
    assert raw[:8] == b"STAGQS1\0"
    assert len(raw) == 8 + 4 * 4 + 8 + 64 + S.planes.size + S.pair_idx.size + 4 * (S.out + 1) + 4 * S.nnz


def test_load_file_rejects_bad_files_before_any_allocation(tmp_path):
    """Host-side failures of the file loader return status codes, before any
    device work: a missing file, a wrong magic, a truncated file, a header that
    declares more than the file holds (a hostile header asking for terabytes is
    refused by size, not by an allocation attempt), a null path."""
    S = _stream()
    good = str(tmp_path / "good.stagq")
    Q.stagq_save(S, good)
    raw = open(good, "rb").read()
    cases = {
        "missing": (str(tmp_path / "nope.stagq"), None, 5),
        "magic": (str(tmp_path / "magic.stagq"), b"NOTSTAGQ" + raw[8:], 2),
        "truncated": (str(tmp_path / "trunc.stagq"), raw[:-7], 2),
        "trailing": (str(tmp_path / "long.stagq"), raw + b"\0" * 16, 2),
    }
    import struct
    huge = bytearray(raw)
    struct.pack_into("<iiii", huge, 8, 1 << 30, 32768, 128, 4)   # 2^30 x 32768 at 6 bits: ~24 TB of planes
    cases["huge"] = (str(tmp_path / "huge.stagq"), bytes(huge), 2)
    for name, (path, data, status) in cases.items():
        if data is not None:
            open(path, "wb").write(data)
        with pytest.raises(Q.StagqError) as e:
            Q.stagq_load_file(path, 0)
        assert e.value.status == status, (name, e.value.status)
    assert Q.lib().stagq_load_file(None, 0, None) == 1
    # the intact file passes every host check; what remains is the device
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:
        has_gpu = False
    if has_gpu:
        Q.stagq_load_file(good, 0).free()
    else:
        with pytest.raises(Q.StagqError) as e:
            Q.stagq_load_file(good, 0)
        assert e.value.status in (4, 6), e.value.status   # STAGQ_ECUDA / STAGQ_ENODEV: the device step


def test_encoder_output_does_not_depend_on_thread_count():
    """Every floating-point step runs in a fixed order inside one group or
    row, so 1 and 7 encoder threads give the same fields, in every mode."""
    from tests.test_oracle_pins import _weights_with_spread_scales
    W = _weights_with_spread_scales(40, 512, 77)
    for kw in (dict(density=0.01, mode="search"),
               dict(density=0.0, mode="fast", guard="ratio", ratio_T=4.0),
               dict(density=0.0, mode="search", codebooks="appendix_e")):
        a = Q.stagq_encode(W, group=32, n_planes=3, n_threads=1, **kw)
        b = Q.stagq_encode(W, group=32, n_planes=3, n_threads=7, **kw)
        for k in ("q", "planes", "pair_idx", "cb_log2s", "cb_lo_over_s", "row_ptr", "col", "val"):
            assert np.array_equal(getattr(a, k), getattr(b, k)), (kw, k)


def test_guarded_encoder_error_paths():
    W = synth.weights(8, 256, seed=3)
    with pytest.raises(Q.StagqError) as e:            # T below 1
        Q.stagq_encode(W, group=64, n_planes=2, mode="fast", guard="ratio", ratio_T=0.5)
    assert e.value.status == 1
    with pytest.raises(Q.StagqError) as e:            # unknown pair-mode bits
        F = Q.Fields(8, 256, 64, 2, q=np.empty((8, 256), np.uint8), planes=np.empty((2, 8, 256), np.uint8),
                     pair_idx=np.empty((8, 4), np.uint8), cb_log2s=np.zeros(16, np.uint16),
                     cb_lo_over_s=np.zeros(16, np.uint16), row_ptr=np.empty(9, np.int32),
                     col=np.empty(Q.stagq_guard_capacity(8, 256, 64) - 1, np.uint16),
                     val=np.empty(Q.stagq_guard_capacity(8, 256, 64) - 1, np.uint16))
        cf = F._c()
        st = Q.lib().stagq_encode_guarded(np.ascontiguousarray(W).ctypes.data, 4.0, 1, Q.STAGQ_PAIR_FAST, 1, ctypes.byref(cf))
        if st:
            raise Q.StagqError(st, "capacity")
    assert e.value.status == 1                        # capacity one short of stagq_guard_capacity
    assert Q.stagq_guard_capacity(8, 256, 64) == 8 * 4 + 8


def test_stream_with_digits_under_the_side_record_is_refused(tmp_path):
    """The GEMV's side-record correction needs the zero-digit convention
    (Section 3.6): a pre-grid position stores q = 0 and zero planes, a
    post-grid position zero planes (its base digit stays). A stream that
    breaks it is refused with STAGQ_EFORMAT by stagq_save and stagq_load."""
    W = synth.weights(16, 256, seed=5)
    F = O.encode(W, 64, 2, 0.02, "fast")
    r = int(np.argmax(np.diff(F.row_ptr) > 0))
    c = int(F.col[F.row_ptr[r]])
    path = str(tmp_path / "x.stagq")
    Q.stagq_save(Q.stagq_pack(to_lib_fields(F)), path)            # the convention holds: accepted
    for what in ("q", "plane3", "plane4"):
        L = to_lib_fields(F)
        if what == "q":
            L.q[r, c] = 2
        else:
            L.planes[int(what[-1]) - 3, r, c] = 1
        S = Q.stagq_pack(L)
        for call in (lambda: Q.stagq_save(S, path), lambda: Q.stagq_load(S, 0)):
            with pytest.raises(Q.StagqError) as e:
                call()
            assert e.value.status == 2, what
    # post-grid entries keep their base digit but no plane digit
    G = O.encode(synth.weights(8, 256, seed=6), 64, 2, mode="fast", guard="ratio", ratio_T=4.0, post_guard=True)
    e = int(np.flatnonzero(G.post_flags)[0])
    r = int(np.searchsorted(G.row_ptr, e, side="right") - 1)
    c = int(G.col[e])
    L = to_lib_fields(G)
    L.q[r, c] = 3
    Q.stagq_save(Q.stagq_pack(L), path)                           # a base digit is allowed
    L.planes[0, r, c] = 1
    with pytest.raises(Q.StagqError) as e:
        Q.stagq_save(Q.stagq_pack(L), path)
    assert e.value.status == 2


def test_binding_refuses_tensors_that_do_not_fit_the_call():
    """The binding checks every x / y / u against the handle's shape before a
    pointer reaches the C ABI (a short y would be written out of bounds on the
    device). No GPU is needed: each bad argument fails before the device check."""
    import torch
    m = Q.Matrix.__new__(Q.Matrix)              # a handle's shape without a device
    m.handle, m.out, m.inp, m.device = None, 64, 512, 0
    x = torch.zeros(1, 512, dtype=torch.float16)
    y_short = torch.zeros(1, 63, dtype=torch.float16)
    with pytest.raises(ValueError, match="y holds 63"):
        Q.stagq_gemv(m, 2, x, y_short)
    with pytest.raises(ValueError, match="x holds 512 elements; the call needs 1024"):
        Q.stagq_gemv_n(m, 2, x, 2, torch.zeros(2, 64, dtype=torch.float16))
    with pytest.raises(TypeError, match="x must be float16"):
        Q.stagq_gemv(m, 2, x.float(), torch.zeros(1, 64, dtype=torch.float16))
    with pytest.raises(TypeError, match="y must be float32"):    # STAGQ_Y_F32 asks for an fp32 y
        Q.stagq_gemv_ex(m, 2, x, torch.zeros(1, 64, dtype=torch.float16), flags=Q.STAGQ_Y_F32)
    with pytest.raises(ValueError, match="contiguous"):
        Q.stagq_gemv(m, 2, torch.zeros(512, 2, dtype=torch.float16).t()[:1], torch.zeros(1, 64, dtype=torch.float16))
    with pytest.raises(ValueError, match="cuda:0"):              # right type and size, wrong device
        Q.stagq_gemv(m, 2, x, torch.zeros(1, 64, dtype=torch.float16))
    with pytest.raises(ValueError, match="u_dev holds"):
        Q.stagq_decode_levels(m, 2, torch.zeros(64, 511, dtype=torch.uint8))
    with pytest.raises(ValueError, match="y_host holds"):
        Q.stagq_gemv_host(m, 2, np.zeros((1, 512), np.float16), np.zeros((1, 32), np.float16))
    with pytest.raises(TypeError, match="x_host"):
        Q.stagq_gemv_host_noalloc(m, 2, np.zeros((1, 512), np.float32), np.zeros((1, 64), np.float16))
    # several GEMVs with host buffers: one entry per GEMV in every list, each
    # buffer checked against its own handle and n
    xh, yh = np.zeros((1, 512), np.float16), np.zeros((1, 64), np.float16)
    with pytest.raises(ValueError, match="one entry per GEMV"):
        Q.stagq_gemv_host_many([m, m], [2], [xh, xh], [yh, yh])
    with pytest.raises(ValueError, match="y_host holds 64 elements; the call needs 256"):
        Q.stagq_gemv_host_many([m, m], [2, 3], [xh, np.zeros((4, 512), np.float16)], [yh, yh], ns=[1, 4])
    with pytest.raises(TypeError, match="x_host"):
        Q.stagq_gemv_host_many([m], [2], [xh.astype(np.float32)], [yh])


def test_stacked_load_checks_its_members():
    """stagq_load_stack (members applied to one x) refuses bad counts and
    members that differ in in / group / n_planes before any device work."""
    a = _stream()
    b = Q.stagq_pack(Q.stagq_encode(synth.weights(8, 512, seed=3), 128, 2, 0.0, "fast"))
    with pytest.raises(Q.StagqError) as e:
        Q.stagq_load_stack([], 0)
    assert e.value.status == 1
    with pytest.raises(Q.StagqError) as e:
        Q.stagq_load_stack([a] * 5, 0)
    assert e.value.status == 1
    c = Q.stagq_pack(Q.stagq_encode(synth.weights(8, a.inp, seed=4), a.group, a.n_planes + 1, 0.0, "fast"))
    with pytest.raises(Q.StagqError) as e:              # n_planes differ
        Q.stagq_load_stack([a, c], 0)
    assert e.value.status == 1
    if a.inp != b.inp:
        with pytest.raises(Q.StagqError) as e:
            Q.stagq_load_stack([a, b], 0)
        assert e.value.status == 1
    bad = Q.HostStream(**{**a.__dict__, "row_ptr": a.row_ptr.copy()})
    bad.row_ptr[2] = bad.row_ptr[3] + 1
    with pytest.raises(Q.StagqError) as e:              # a malformed member
        Q.stagq_load_stack([a, bad], 0)
    assert e.value.status == 2


def test_host_many_refuses_bad_arguments_before_any_device_work():
    """stagq_gemv_host_many checks its count and arrays through the C ABI
    before it touches a device, so this runs without a GPU (status 1 =
    STAGQ_EINVAL)."""
    import ctypes
    L = Q.lib()
    one = (ctypes.c_void_p * 1)(None)
    bits = (ctypes.c_int * 1)(2)
    ns = (ctypes.c_int * 1)(1)
    assert L.stagq_gemv_host_many(0, one, bits, one, ns, one, None) == 1
    assert L.stagq_gemv_host_many(Q.STAGQ_MAX_MANY + 1, one, bits, one, ns, one, None) == 1
    assert L.stagq_gemv_host_many(1, None, bits, one, ns, one, None) == 1
    assert L.stagq_gemv_host_many(1, one, None, one, ns, one, None) == 1
    assert L.stagq_gemv_host_many(1, one, bits, one, ns, one, None) == 1  # null handle
