"""Shared test helpers: oracle fields -> library fields, tolerance checks."""
import numpy as np

import quantized_gemv_stagq_b200 as Q

# Tolerance of the GEMV against the fp64 oracle (fp32 accumulation, fp16 x).
REL_L2_TOL = 1e-3
MAX_ABS_TOL = 5e-3   # times max|y_ref|


def to_lib_fields(F) -> "Q.Fields":
    """The oracle's logical fields in the library's Fields container."""
    return Q.Fields(out=F.out, inp=F.inp, group=F.group, n_planes=F.n_planes,
                    q=np.ascontiguousarray(F.q, np.uint8),
                    planes=np.ascontiguousarray(F.planes, np.uint8),
                    pair_idx=np.ascontiguousarray(F.pair_idx, np.uint8),
                    cb_log2s=F.cb_log2s.view(np.uint16).copy(),
                    cb_lo_over_s=F.cb_lo_over_s.view(np.uint16).copy(),
                    row_ptr=F.row_ptr.astype(np.int32), col=lib_columns(F),
                    val=F.val.view(np.uint16).copy())


def lib_columns(F) -> np.ndarray:
    """The oracle's side-record columns as the library stores them: bit 15
    (STAGQ_SIDE_POST) marks a post-grid entry."""
    return (F.col.astype(np.uint16) | (F.post_flags.astype(np.uint16) << 15)).astype(np.uint16)


def fields_equal(F, P) -> dict:
    """Field-by-field equality of oracle fields F and library fields P."""
    return dict(
        codebooks=bool(np.array_equal(F.cb_log2s.view(np.uint16), P.cb_log2s)
                       and np.array_equal(F.cb_lo_over_s.view(np.uint16), P.cb_lo_over_s)),
        pair_idx=bool(np.array_equal(F.pair_idx, P.pair_idx)),
        q=bool(np.array_equal(F.q, P.q)),
        planes=bool(np.array_equal(F.planes, P.planes)),
        side_record=bool(np.array_equal(F.row_ptr, P.row_ptr) and np.array_equal(lib_columns(F), P.col)
                         and np.array_equal(F.val.view(np.uint16), P.val)),
    )


def check_close(y, y_ref, what=""):
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    scale = np.abs(y_ref).max()
    rel = np.linalg.norm(y - y_ref) / max(np.linalg.norm(y_ref), 1e-300)
    mabs = np.abs(y - y_ref).max() if y.size else 0.0
    assert rel <= REL_L2_TOL, f"{what}: rel L2 {rel:.3e} > {REL_L2_TOL}"
    assert mabs <= MAX_ABS_TOL * max(scale, 1e-300), f"{what}: max abs {mabs:.3e} > {MAX_ABS_TOL} * {scale:.3e}"
    return rel, mabs


# The single-vector kernel holds one warp per 2048-weight K slice plus its
# producer warp in the register file: it plans K up to 15 slices (30720).
SINGLE_MAX_IN = 15 * 2048


def n1_kernels(inp, include_default=False):
    """The n = 1 kernels that can serve a matrix with K = inp (flags)."""
    ks = ([0] if include_default else []) + [Q.STAGQ_KERNEL_GENERAL]
    if inp <= SINGLE_MAX_IN:
        ks.append(Q.STAGQ_KERNEL_SINGLE)
    return tuple(ks)


# With several vectors a lane of the single-vector kernel takes half a chunk:
# it plans K up to 15 slices of 1024 weights, for groups of 64 or more.
SINGLE_MAX_IN_NB = 15 * 1024


def nb_kernels(inp, group):
    """The kernels that can serve n = 2..4 vectors of a matrix with K = inp."""
    ks = [Q.STAGQ_KERNEL_GENERAL]
    if inp <= SINGLE_MAX_IN_NB and group >= 64:
        ks.append(Q.STAGQ_KERNEL_SINGLE)
    return tuple(ks)
