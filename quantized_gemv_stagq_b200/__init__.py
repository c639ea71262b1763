"""StagQ multi-precision batch-one GEMV on B200 (sm_100a).

Thin ctypes binding of ``libstagq.so`` (see ``include/stagq.h``): the
functions below carry the C ABI's names and only marshal arguments. Every
step of the GEMV runs in the library's CUDA kernels; PyTorch is used only for
device memory and streams. If the library is missing this package raises --
there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libstagq.so")

STAGQ_OK = 0
STAGQ_PAIR_SEARCH = 0
STAGQ_PAIR_FAST = 1
STAGQ_Y_F32 = 1
STAGQ_KERNEL_GENERAL = 2
STAGQ_KERNEL_SINGLE = 4
STAGQ_SIDE_POST = 0x8000
STAGQ_CODEBOOK_RULES = 0x100
STAGQ_MAX_PLANES = 4
STAGQ_MAX_BATCH = 4
STAGQ_MAX_STACK = 4
STAGQ_MAX_MANY = 1024

_c_p = ctypes.c_void_p
_i32, _i64, _u32, _dbl = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_double


class _Fields(ctypes.Structure):
    _fields_ = [("out", _i32), ("in_", _i32), ("group", _i32), ("n_planes", _i32), ("nnz", _i64),
                ("codebook_log2s", ctypes.c_uint16 * 16), ("codebook_lo_over_s", ctypes.c_uint16 * 16),
                ("q", _c_p), ("planes", _c_p), ("pair_idx", _c_p), ("row_ptr", _c_p),
                ("col", _c_p), ("val", _c_p)]


class _HostStream(ctypes.Structure):
    _fields_ = [("out", _i32), ("in_", _i32), ("group", _i32), ("n_planes", _i32), ("nnz", _i64),
                ("codebook_log2s", ctypes.c_uint16 * 16), ("codebook_lo_over_s", ctypes.c_uint16 * 16),
                ("planes", _c_p), ("pair_idx", _c_p), ("row_ptr", _c_p), ("col", _c_p), ("val", _c_p)]


class _SideLayout(ctypes.Structure):
    _fields_ = [("grid", _i32), ("stride", _i32), ("ent_off", _i32), ("row_groups", _i32), ("k_slices", _i32),
                ("class_rows", _i32), ("grid1", _i32), ("stride1", _i32), ("ent_off1", _i32)]


class _Info(ctypes.Structure):
    _fields_ = [("out", _i32), ("in_", _i32), ("group", _i32), ("n_planes", _i32), ("nnz", _i64),
                ("device", _i32), ("device_bytes", _i64)]


_SIGNATURES = {
    "stagq_side_record_count": (_i64, [_i32, _i32, _dbl]),
    "stagq_encode": (ctypes.c_int, [_c_p, _dbl, _i32, _i32, ctypes.POINTER(_Fields)]),
    "stagq_guard_capacity": (_i64, [_i32, _i32, _i32]),
    "stagq_encode_guarded": (ctypes.c_int, [_c_p, _dbl, _i32, _i32, _i32, ctypes.POINTER(_Fields)]),
    "stagq_stream_plane_bytes": (_i64, [_i32, _i32, _i32]),
    "stagq_pack": (ctypes.c_int, [ctypes.POINTER(_Fields), _c_p]),
    "stagq_unpack_levels_host": (ctypes.c_int, [ctypes.POINTER(_HostStream), ctypes.c_int, _c_p]),
    "stagq_save": (ctypes.c_int, [ctypes.POINTER(_HostStream), ctypes.c_char_p]),
    "stagq_load_file": (ctypes.c_int, [ctypes.c_char_p, ctypes.c_int, ctypes.POINTER(_c_p)]),
    "stagq_load": (ctypes.c_int, [ctypes.POINTER(_HostStream), ctypes.c_int, ctypes.POINTER(_c_p)]),
    "stagq_load_stack": (ctypes.c_int, [ctypes.POINTER(ctypes.POINTER(_HostStream)), ctypes.c_int, ctypes.c_int,
                                        ctypes.POINTER(_c_p)]),
    "stagq_gemv": (ctypes.c_int, [_c_p, ctypes.c_int, _c_p, _c_p, _c_p]),
    "stagq_gemv_n": (ctypes.c_int, [_c_p, ctypes.c_int, _c_p, ctypes.c_int, _c_p, _c_p]),
    "stagq_gemv_ex": (ctypes.c_int, [_c_p, ctypes.c_int, _c_p, ctypes.c_int, _c_p, _u32, _c_p]),
    "stagq_gemv_scaled": (ctypes.c_int, [_c_p, ctypes.c_int, _c_p, ctypes.c_int, _c_p, _c_p, _u32, _c_p]),
    "stagq_gemv_host": (ctypes.c_int, [_c_p, ctypes.c_int, _c_p, ctypes.c_int, _c_p, _c_p]),
    "stagq_gemv_host_many": (ctypes.c_int, [ctypes.c_int, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p]),
    "stagq_gemv_host_noalloc": (ctypes.c_int, [_c_p, ctypes.c_int, _c_p, ctypes.c_int, _c_p, _c_p]),
    "stagq_decode_levels": (ctypes.c_int, [_c_p, ctypes.c_int, _c_p, _c_p]),
    "stagq_bytes": (_i64, [_c_p, ctypes.c_int, ctypes.c_int]),
    "stagq_info": (ctypes.c_int, [_c_p, ctypes.POINTER(_Info)]),
    "stagq_check": (ctypes.c_int, [_c_p]),
    "stagq_debug_stall": (ctypes.c_int, [_c_p, _u32]),
    "stagq_debug_side_record": (ctypes.c_int, [_c_p, ctypes.POINTER(_SideLayout), _c_p, _i64, _c_p, _i64]),
    "stagq_free": (None, [_c_p]),
    "stagq_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    "stagq_last_error": (ctypes.c_char_p, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libstagq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m quantized_gemv_stagq_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


class StagqError(RuntimeError):
    def __init__(self, status: int, where: str):
        L = lib()
        msg = L.stagq_strerror(status).decode()
        detail = L.stagq_last_error().decode()
        super().__init__(f"{where}: {msg} ({detail})")
        self.status = status


def _check(status: int, where: str) -> None:
    if status != STAGQ_OK:
        raise StagqError(status, where)


def _ptr(a) -> int:
    return a.ctypes.data if a is not None and a.size else 0


# ------------------------------------------------------------------ host side

@dataclass
class Fields:
    """Logical fields of an encoded matrix (numpy, host)."""
    out: int
    inp: int
    group: int
    n_planes: int
    q: np.ndarray            # uint8 [out, inp]
    planes: np.ndarray       # uint8 [n_planes, out, inp]
    pair_idx: np.ndarray     # uint8 [out, inp // group]
    cb_log2s: np.ndarray     # uint16 [16] fp16 bits
    cb_lo_over_s: np.ndarray  # uint16 [16] fp16 bits
    row_ptr: np.ndarray      # int32 [out + 1]
    col: np.ndarray          # uint16 [nnz]
    val: np.ndarray          # uint16 [nnz] fp16 bits

    @property
    def nnz(self) -> int:
        return int(self.col.shape[0])

    def _c(self) -> _Fields:
        f = _Fields(self.out, self.inp, self.group, self.n_planes, self.nnz)
        f.codebook_log2s[:] = [int(v) for v in self.cb_log2s]
        f.codebook_lo_over_s[:] = [int(v) for v in self.cb_lo_over_s]
        f.q, f.planes, f.pair_idx = _ptr(self.q), _ptr(self.planes), _ptr(self.pair_idx)
        f.row_ptr, f.col, f.val = _ptr(self.row_ptr), _ptr(self.col), _ptr(self.val)
        return f


@dataclass
class HostStream:
    """Packed plane-major stream (numpy, host)."""
    out: int
    inp: int
    group: int
    n_planes: int
    planes: np.ndarray       # uint8, stagq_stream_plane_bytes bytes
    pair_idx: np.ndarray
    cb_log2s: np.ndarray
    cb_lo_over_s: np.ndarray
    row_ptr: np.ndarray
    col: np.ndarray
    val: np.ndarray

    @property
    def nnz(self) -> int:
        return int(self.col.shape[0])

    def _c(self) -> _HostStream:
        s = _HostStream(self.out, self.inp, self.group, self.n_planes, self.nnz)
        s.codebook_log2s[:] = [int(v) for v in self.cb_log2s]
        s.codebook_lo_over_s[:] = [int(v) for v in self.cb_lo_over_s]
        s.planes, s.pair_idx, s.row_ptr = _ptr(self.planes), _ptr(self.pair_idx), _ptr(self.row_ptr)
        s.col, s.val = _ptr(self.col), _ptr(self.val)
        return s


def stagq_side_record_count(out: int, inp: int, density: float) -> int:
    return int(lib().stagq_side_record_count(out, inp, density))


def stagq_stream_plane_bytes(out: int, inp: int, n_planes: int) -> int:
    return int(lib().stagq_stream_plane_bytes(out, inp, n_planes))


def stagq_guard_capacity(out: int, inp: int, group: int) -> int:
    return int(lib().stagq_guard_capacity(out, inp, group))


def stagq_encode(w: np.ndarray, group: int = 128, n_planes: int = 2, density: float = 0.005,
                 mode: str = "search", n_threads: int = 0, guard: str = "density", ratio_T: float = 4.0,
                 post_guard: bool = True, codebooks: str = "uniform") -> Fields:
    """Encode an fp16 [out, inp] matrix (library encoder, host). guard
    "density": global top-|w| record of `density` (stagq_encode); "ratio": the
    pre-grid ratio guard with `ratio_T` and, if post_guard, the post-grid guard
    (stagq_encode_guarded; post-grid columns carry STAGQ_SIDE_POST). codebooks
    "uniform" or "appendix_e" (STAGQ_CODEBOOK_RULES)."""
    w = np.ascontiguousarray(w, dtype=np.float16)
    out, inp = w.shape
    if guard == "density":
        nnz = stagq_side_record_count(out, inp, density)
    elif guard == "ratio":
        nnz = stagq_guard_capacity(out, inp, group)
    else:
        raise ValueError("guard must be 'density' or 'ratio'")
    F = Fields(out, inp, group, n_planes,
               q=np.empty((out, inp), np.uint8),
               planes=np.empty((n_planes, out, inp), np.uint8),
               pair_idx=np.empty((out, inp // group), np.uint8),
               cb_log2s=np.zeros(16, np.uint16), cb_lo_over_s=np.zeros(16, np.uint16),
               row_ptr=np.empty(out + 1, np.int32), col=np.empty(nnz, np.uint16),
               val=np.empty(nnz, np.uint16))
    cf = F._c()
    m = {"search": STAGQ_PAIR_SEARCH, "fast": STAGQ_PAIR_FAST}[mode]
    if codebooks == "appendix_e":
        m |= STAGQ_CODEBOOK_RULES
    elif codebooks != "uniform":
        raise ValueError("codebooks must be 'uniform' or 'appendix_e'")
    if guard == "density":
        _check(lib().stagq_encode(w.ctypes.data, density, m, n_threads, ctypes.byref(cf)), "stagq_encode")
    else:
        _check(lib().stagq_encode_guarded(w.ctypes.data, ratio_T, int(post_guard), m, n_threads, ctypes.byref(cf)),
               "stagq_encode_guarded")
        F.col = F.col[:cf.nnz].copy()
        F.val = F.val[:cf.nnz].copy()
    F.cb_log2s = np.array(cf.codebook_log2s[:], dtype=np.uint16)
    F.cb_lo_over_s = np.array(cf.codebook_lo_over_s[:], dtype=np.uint16)
    return F


def stagq_pack(F: Fields) -> HostStream:
    """Lay the digits of F out plane-major (library packer, host)."""
    planes = np.empty(stagq_stream_plane_bytes(F.out, F.inp, F.n_planes), np.uint8)
    q = np.ascontiguousarray(F.q, dtype=np.uint8)
    pl = np.ascontiguousarray(F.planes, dtype=np.uint8)
    G = Fields(F.out, F.inp, F.group, F.n_planes, q, pl, F.pair_idx, F.cb_log2s, F.cb_lo_over_s,
               F.row_ptr, F.col, F.val)
    cf = G._c()
    _check(lib().stagq_pack(ctypes.byref(cf), planes.ctypes.data), "stagq_pack")
    return HostStream(F.out, F.inp, F.group, F.n_planes, planes,
                      np.ascontiguousarray(F.pair_idx, np.uint8),
                      np.asarray(F.cb_log2s, np.uint16), np.asarray(F.cb_lo_over_s, np.uint16),
                      np.ascontiguousarray(F.row_ptr, np.int32), np.ascontiguousarray(F.col, np.uint16),
                      np.ascontiguousarray(F.val, np.uint16))


def stagq_unpack_levels_host(S: HostStream, bits: int) -> np.ndarray:
    u = np.empty((S.out, S.inp), np.uint8)
    cs = S._c()
    _check(lib().stagq_unpack_levels_host(ctypes.byref(cs), bits, u.ctypes.data), "stagq_unpack_levels_host")
    return u


def stagq_save(S: HostStream, path: str) -> None:
    cs = S._c()
    _check(lib().stagq_save(ctypes.byref(cs), path.encode()), "stagq_save")


# ------------------------------------------------------------------ GPU side

def _stream_ptr(stream) -> int:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


class Matrix:
    """A stream loaded onto one GPU (owns a stagq_handle)."""

    def __init__(self, handle: int):
        self.handle = ctypes.c_void_p(handle)
        info = _Info()
        _check(lib().stagq_info(self.handle, ctypes.byref(info)), "stagq_info")
        self.out, self.inp, self.group = info.out, info.in_, info.group
        self.n_planes, self.nnz, self.device = info.n_planes, info.nnz, info.device
        self.device_bytes = info.device_bytes

    def free(self) -> None:
        if self.handle is not None and self.handle.value:
            lib().stagq_free(self.handle)
        self.handle = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def stagq_load(S: HostStream, device: int = 0) -> Matrix:
    h = ctypes.c_void_p()
    cs = S._c()
    _check(lib().stagq_load(ctypes.byref(cs), device, ctypes.byref(h)), "stagq_load")
    return Matrix(h.value)


def stagq_load_stack(streams, device: int = 0) -> Matrix:
    """One handle for several matrices applied to the same x (q/k/v, gate/up):
    their rows stacked in order, each with its own codebooks. y of a GEMV is
    the members' outputs one after the other."""
    cs = [S._c() for S in streams]
    arr = (ctypes.POINTER(_HostStream) * len(cs))(*[ctypes.pointer(c) for c in cs])
    h = ctypes.c_void_p()
    _check(lib().stagq_load_stack(arr, len(cs), device, ctypes.byref(h)), "stagq_load_stack")
    return Matrix(h.value)


def stagq_load_file(path: str, device: int = 0) -> Matrix:
    h = ctypes.c_void_p()
    _check(lib().stagq_load_file(path.encode(), device, ctypes.byref(h)), "stagq_load_file")
    return Matrix(h.value)


def _check_device_tensor(t, name: str, dtype_name: str, numel: int, device: int) -> None:
    """The C ABI takes raw pointers and sizes from the handle: a tensor of the
    wrong type, layout or size would be read or written out of bounds on the
    device, so it is refused here (and one on the wrong GPU by
    _check_on_device)."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    want = getattr(torch, dtype_name)
    if t.dtype != want:
        raise TypeError(f"{name} must be {dtype_name}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements; the call needs {numel}")


def _check_on_device(t, name: str, device: int) -> None:
    import torch
    if not t.is_cuda or (t.device.index if t.device.index is not None else torch.cuda.current_device()) != device:
        raise ValueError(f"{name} must be on cuda:{device} (the matrix's GPU), got {t.device}")


def _check_host_array(a, name: str, numel: int) -> None:
    if not isinstance(a, np.ndarray) or a.dtype != np.float16:
        raise TypeError(f"{name} must be a float16 numpy array")
    if not a.flags["C_CONTIGUOUS"]:
        raise ValueError(f"{name} must be C-contiguous")
    if a.size < numel:
        raise ValueError(f"{name} holds {a.size} elements; the call needs {numel}")


def _check_gemv_args(m: Matrix, x, y, n: int, f32: bool) -> None:
    # (n itself is checked by the library: STAGQ_EINVAL outside 1..STAGQ_MAX_BATCH)
    _check_device_tensor(x, "x", "float16", n * m.inp, m.device)
    _check_device_tensor(y, "y", "float32" if f32 else "float16", n * m.out, m.device)
    _check_on_device(x, "x", m.device)
    _check_on_device(y, "y", m.device)


def stagq_gemv_ex(m: Matrix, bits: int, x, y, n: int = 1, flags: int = 0, stream=None) -> None:
    """x, y: CUDA tensors (x fp16 [n, inp]; y fp16 or fp32 [n, out])."""
    _check_gemv_args(m, x, y, n, bool(flags & STAGQ_Y_F32))
    _check(lib().stagq_gemv_ex(m.handle, bits, x.data_ptr(), n, y.data_ptr(), flags,
                               _stream_ptr(stream)), "stagq_gemv_ex")


def stagq_gemv_scaled(m: Matrix, bits: int, x, in_scale, y, n: int = 1, flags: int = 0, stream=None) -> None:
    """y = W_hat (x * in_scale): in_scale a CUDA fp32 tensor [inp] (the
    inverse activation scale 1/a), x fp16 [n, inp], y fp16 or fp32 [n, out]."""
    _check_gemv_args(m, x, y, n, bool(flags & STAGQ_Y_F32))
    _check_device_tensor(in_scale, "in_scale", "float32", m.inp, m.device)
    _check_on_device(in_scale, "in_scale", m.device)
    _check(lib().stagq_gemv_scaled(m.handle, bits, x.data_ptr(), n, in_scale.data_ptr(), y.data_ptr(), flags,
                                   _stream_ptr(stream)), "stagq_gemv_scaled")


def stagq_gemv(m: Matrix, bits: int, x, y, stream=None) -> None:
    _check_gemv_args(m, x, y, 1, False)
    _check(lib().stagq_gemv(m.handle, bits, x.data_ptr(), y.data_ptr(), _stream_ptr(stream)), "stagq_gemv")


def stagq_gemv_n(m: Matrix, bits: int, x, n: int, y, stream=None) -> None:
    _check_gemv_args(m, x, y, n, False)
    _check(lib().stagq_gemv_n(m.handle, bits, x.data_ptr(), n, y.data_ptr(), _stream_ptr(stream)),
           "stagq_gemv_n")


def stagq_gemv_host(m: Matrix, bits: int, x_host: np.ndarray, y_host: np.ndarray, n: int = 1,
                    stream=None) -> None:
    """Host buffers (pinned or pageable numpy arrays): copies in and out, synchronous."""
    _check_host_array(x_host, "x_host", n * m.inp)
    _check_host_array(y_host, "y_host", n * m.out)
    _check(lib().stagq_gemv_host(m.handle, bits, x_host.ctypes.data, n, y_host.ctypes.data,
                                 _stream_ptr(stream)), "stagq_gemv_host")


def stagq_gemv_host_many(mats, bits, x_hosts, y_hosts, ns=None, stream=None) -> None:
    """Several GEMVs with host buffers and one synchronization: every x copied
    in, every GEMV run, every y copied out, in that order on one stream."""
    count = len(mats)
    ns = [1] * count if ns is None else list(ns)
    if not (len(bits) == len(x_hosts) == len(y_hosts) == len(ns) == count):
        raise ValueError("mats, bits, x_hosts, y_hosts and ns must have one entry per GEMV")
    for m, x, y, n in zip(mats, x_hosts, y_hosts, ns):
        _check_host_array(x, "x_host", n * m.inp)
        _check_host_array(y, "y_host", n * m.out)
    H = (ctypes.c_void_p * count)(*[m.handle.value for m in mats])
    B = (ctypes.c_int * count)(*bits)
    X = (ctypes.c_void_p * count)(*[x.ctypes.data for x in x_hosts])
    N = (ctypes.c_int * count)(*ns)
    Y = (ctypes.c_void_p * count)(*[y.ctypes.data for y in y_hosts])
    _check(lib().stagq_gemv_host_many(count, H, B, X, N, Y, _stream_ptr(stream)), "stagq_gemv_host_many")


def stagq_gemv_host_noalloc(m: Matrix, bits: int, x_host: np.ndarray, y_host: np.ndarray, n: int = 1,
                            stream=None) -> None:
    """As stagq_gemv_host, staging through the library's static device array
    instead of a device buffer allocated on first use (no device allocation).
    Calls must not overlap on the GPU; see include/stagq.h."""
    _check_host_array(x_host, "x_host", n * m.inp)
    _check_host_array(y_host, "y_host", n * m.out)
    _check(lib().stagq_gemv_host_noalloc(m.handle, bits, x_host.ctypes.data, n, y_host.ctypes.data,
                                         _stream_ptr(stream)), "stagq_gemv_host_noalloc")


def stagq_decode_levels(m: Matrix, bits: int, u_dev, stream=None) -> None:
    _check_device_tensor(u_dev, "u_dev", "uint8", m.out * m.inp, m.device)
    _check_on_device(u_dev, "u_dev", m.device)
    _check(lib().stagq_decode_levels(m.handle, bits, u_dev.data_ptr(), _stream_ptr(stream)),
           "stagq_decode_levels")


def stagq_bytes(m: Matrix, bits: int, n: int = 1) -> int:
    return int(lib().stagq_bytes(m.handle, bits, n))


def stagq_check(m: Matrix) -> None:
    """Synchronise the handle's device and raise on any pending CUDA error."""
    _check(lib().stagq_check(m.handle), "stagq_check")


def stagq_debug_stall(m: Matrix, stall_ns: int) -> None:
    """Test hook: launches on m take one bounded wait of stall_ns that runs out (0: off)."""
    _check(lib().stagq_debug_stall(m.handle, int(stall_ns)), "stagq_debug_stall")


def stagq_debug_side_record(m: Matrix):
    """Test hook: the layout of the two device cuts of the side record and
    their bytes, copied to host memory: (layout dict, cut, cut1)."""
    lay = _SideLayout()
    _check(lib().stagq_debug_side_record(m.handle, ctypes.byref(lay), None, 0, None, 0), "stagq_debug_side_record")
    cut = np.empty(lay.grid * lay.stride, np.uint8)
    cut1 = np.empty(lay.grid1 * lay.stride1, np.uint8)
    _check(lib().stagq_debug_side_record(m.handle, ctypes.byref(lay), cut.ctypes.data, cut.size, cut1.ctypes.data,
                                         cut1.size), "stagq_debug_side_record")
    return {k: getattr(lay, k) for k, _ in _SideLayout._fields_}, cut, cut1


def stagq_free(m: Matrix) -> None:
    m.free()
