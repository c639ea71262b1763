"""CPU oracle for the StagQ multi-precision GEMV -- TEST INFRASTRUCTURE ONLY.

This module is the plain, slow, fp64 statement of what the StagQ format
computes, written from the StagQ paper ("StagQ: Constraint-Driven
Multi-Precision Weight Quantization for LLMs", arXiv 2610.05977). Only the
test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import it; the product (the CUDA library and its Python
binding) never does, and it shares no code with them.

It covers three things:

* the encoder of Sections 3.1-3.6 (+ Appendices B and E) for synthetic
  weights: side record (the workloads' global top-|w| density, or the
  paper's pre-grid ratio guard plus the post-grid guard), clipping, initial
  pair, codebooks (uniform, or Appendix E's choice among uniform, Lloyd and
  anchored Lloyd placement with its fallback), per-group pair choice by
  Eq. (5)-(6),
  nearest-rounding base, sign planes (Eq. (7));
* the decoder: composite integer Eq. (8), affine map Eq. (10) (with the
  additive form Eq. (9) kept as a cross-check), complete reconstruction
  Eq. (4);
* the GEMV ``y = W_hat x`` as an fp64 dot product.

Every place where the paper is silent and a reading had to be taken is
marked "Reading:" below. Parity status of each function: all functions are
pinned by the ``-m "not gpu"`` tests (Figure 1 worked example, closed forms,
invariants, brute force); the Eq. (5) pair search is pinned only by brute
force on tiny groups, because the paper prints no fitted pair values.

Array conventions: ``W`` is [out, inp] (row = output channel, K = inp),
groups are runs of ``group`` consecutive entries along K inside one row.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

# Appendix B: the initial pair places four levels symmetrically, the outer
# two 6 % in from each end of the group range.
INIT_EDGE_FRACTION = 0.06
# Section 3.1: weight of the floor term in Eq. (5).
FLOOR_LAMBDA = 4.0
# Section 3.1: two sixteen-entry codebooks per matrix.
CODEBOOK_SIZE = 16
# Appendix E, Lloyd's rule: Reading -- at most this many assignment steps.
LLOYD_MAX_STEPS = 100
# Appendix E: a matrix whose deepest-precision error exceeds this fraction of
# its two-bit error under the chosen codebooks falls back to uniform placement.
FALLBACK_RATIO = 0.1
# Reading: a group whose clipped range is zero has no initial step; it gets
# this placeholder, stays out of the codebook fit and takes its pair by the
# Eq. (5) search in every mode.
DEGENERATE_STEP = 2.0 ** -24


@dataclass
class Fields:
    """Logical fields of one encoded matrix (no physical layout)."""

    out: int
    inp: int
    group: int
    n_planes: int               # refinement planes stored: b_3 .. b_{2+n_planes}
    q: np.ndarray               # uint8 [out, inp], base digit 0..3
    planes: np.ndarray          # uint8 [n_planes, out, inp], b_k in {0, 1}
    pair_idx: np.ndarray        # uint8 [out, inp // group]; hi nibble = log2(s) index
    cb_log2s: np.ndarray        # float16 [16]
    cb_lo_over_s: np.ndarray    # float16 [16]
    row_ptr: np.ndarray         # int64 [out + 1]  (side record, CSR)
    col: np.ndarray             # int64 [nnz], sorted inside each row
    val: np.ndarray             # float16 [nnz]: the recorded value (pre-grid) or residual (post-grid)
    post: np.ndarray = None     # bool [nnz]: entry held out by the post-grid guard (None: none)

    @property
    def depth(self) -> int:
        """Stream depth N of Section 3: base + planes, i.e. the top precision."""
        return 2 + self.n_planes

    @property
    def nnz(self) -> int:
        return int(self.col.shape[0])

    @property
    def post_flags(self) -> np.ndarray:
        return np.zeros(self.nnz, dtype=bool) if self.post is None else np.asarray(self.post, dtype=bool)


# --------------------------------------------------------------------------
# Grid algebra (Sections 3.2-3.4)
# --------------------------------------------------------------------------

def half_step(s, k: int):
    """Eq. (7): refinement half-step t_k = alpha_k = s / 2^(k-1), k >= 3."""
    return s / 2.0 ** (k - 1)


def grid_at(lo, s, M: int):
    """Eq. (10): origin lo_M and spacing s_M of the precision-M grid.

    s_M = s / 2^(M-2) and lo_M = lo - s (2^(M-2) - 1) / 2^(M-1).
    """
    s_M = s / 2.0 ** (M - 2)
    lo_M = lo - s * (2.0 ** (M - 2) - 1.0) / 2.0 ** (M - 1)
    return lo_M, s_M


def reach(s, N: int):
    """Eq. (6): rho = s * sum_{k=3}^{N} 2^-(k-1), the furthest the planes move
    the base reconstruction."""
    return s * sum(2.0 ** -(k - 1) for k in range(3, N + 1))


def composite_level(q, planes, M: int):
    """Eq. (8): u_M = q 2^(M-2) + sum_{k=3}^{M} b_k 2^(M-k).

    ``planes`` is a sequence whose entry k-3 holds b_k; only b_3..b_M are read.
    """
    u = np.asarray(q, dtype=np.int64) * (1 << (M - 2))
    for k in range(3, M + 1):
        u = u + np.asarray(planes[k - 3], dtype=np.int64) * (1 << (M - k))
    return u


def reconstruct_additive(lo, s, q, planes, M: int):
    """Eq. (9): lo + s q + sum_{k=3}^{M} (2 b_k - 1) s / 2^(k-1).

    Kept as an independent statement of the main stream; Eq. (10) is what the
    decoder uses, and the tests check that the two agree.
    """
    w = lo + s * np.asarray(q, dtype=np.float64)
    for k in range(3, M + 1):
        b = np.asarray(planes[k - 3], dtype=np.float64)
        w = w + (2.0 * b - 1.0) * half_step(s, k)
    return w


def reconstruct_affine(lo, s, u, M: int):
    """Eq. (10): W_main^(M) = lo_M + s_M u_M."""
    lo_M, s_M = grid_at(lo, s, M)
    return lo_M + s_M * np.asarray(u, dtype=np.float64)


# --------------------------------------------------------------------------
# Digit encoding of one value under a fixed pair (Sections 3.3 and 3.6)
# --------------------------------------------------------------------------

def base_digit(w, lo, s):
    """Appendix E: the base code is nearest rounding onto the four levels
    lo + s q, q in {0..3}.

    Reading: round half up, q = clamp(floor((w - lo)/s + 1/2), 0, 3).
    """
    q = np.floor((np.asarray(w, dtype=np.float64) - lo) / s + 0.5)
    return np.clip(q, 0, 3).astype(np.int64)


def encode_digits(w, lo, s, N: int):
    """Base digit, then each refinement plane k = 3..N stores the sign of the
    residual left by the preceding prefix (Section 3.6), with sign(0) := +1
    (Section 3.3); plane k moves the reconstruction by +-t_k (Eq. (7)).

    Returns (q, [b_3..b_N], [W^(2)..W^(N)]) with the reconstructions computed
    step by step as the encoder walks the prefix.
    """
    w = np.asarray(w, dtype=np.float64)
    q = base_digit(w, lo, s)
    recon = lo + s * q.astype(np.float64)
    recons = [recon]
    bits = []
    for k in range(3, N + 1):
        r = w - recon
        b = (r >= 0.0).astype(np.int64)
        recon = recon + (2.0 * b - 1.0) * half_step(s, k)
        bits.append(b)
        recons.append(recon)
    return q, bits, recons


# --------------------------------------------------------------------------
# Encoder stages (Sections 3.1, 3.5, 3.6; Appendices B and E)
# --------------------------------------------------------------------------

def side_record_count(out: int, inp: int, density: float) -> int:
    """Reading: the record holds round(density * out * inp) entries (half up)."""
    return int(np.floor(density * out * inp + 0.5))


def select_side_record(W: np.ndarray, density: float) -> np.ndarray:
    """Pre-grid hold-out for the synthetic workloads: the largest-|w| entries.

    Reading: the workloads name a global top-|w| density in place of the
    paper's per-group ratio / gain criteria (Section 3.5); ties in |w| go to
    the smaller flat row-major index. Returns a bool mask [out, inp].
    """
    out, inp = W.shape
    k = side_record_count(out, inp, density)
    mask = np.zeros(out * inp, dtype=bool)
    if k == 0:
        return mask.reshape(out, inp)
    a = np.abs(W.astype(np.float64)).reshape(-1)
    if k >= a.size:
        mask[:] = True
        return mask.reshape(out, inp)
    # threshold = k-th largest |w|; everything above it is in, ties at it are
    # filled in increasing flat index.
    thr = np.partition(a, a.size - k)[a.size - k]
    above = np.flatnonzero(a > thr)
    tied = np.flatnonzero(a == thr)
    mask[above] = True
    mask[tied[: k - above.size]] = True
    return mask.reshape(out, inp)


def select_ratio_guard(W: np.ndarray, group: int, T: float) -> np.ndarray:
    """Section 3.5, pre-grid guard under the ratio criterion: in each group,
    the largest-|w| entry is held out when its magnitude exceeds T times the
    second largest magnitude of the group (T = 4 on Llama-3.1-8B, Table 6).

    Reading: "largest" is the first index of the maximum |w|; the second
    largest is the maximum over the group's other entries, so two equal
    largest magnitudes hold nothing out. Returns a bool mask [out, inp].
    """
    out, inp = W.shape
    ng = inp // group
    A = np.abs(W.astype(np.float64)).reshape(out, ng, group)
    j1 = np.argmax(A, axis=2)                                    # first maximum
    a1 = np.take_along_axis(A, j1[:, :, None], axis=2)[:, :, 0]
    others = A.copy()
    np.put_along_axis(others, j1[:, :, None], -np.inf, axis=2)
    a2 = others.max(axis=2) if group > 1 else np.zeros_like(a1)
    take = a1 > T * a2
    mask = np.zeros((out, ng, group), dtype=bool)
    np.put_along_axis(mask, j1[:, :, None], take[:, :, None], axis=2)
    return mask.reshape(out, inp)


def select_post_guard(W: np.ndarray, W2: np.ndarray, held: np.ndarray) -> np.ndarray:
    """Appendix E, post-grid guard of a ratio-criterion matrix: after the grid
    is fixed, the one position per output row with the largest
    activation-weighted two-bit error E_c (W - W_hat^(2))^2.

    Reading: E_c = 1 as in Eq. (5) (x ~ N(0,1), no calibration set); ties go
    to the smallest column; positions already held out by the pre-grid guard
    are not candidates, and a row with none takes nothing. Returns a bool mask.
    """
    err = (W.astype(np.float64) - W2) ** 2
    err = np.where(held, -np.inf, err)
    mask = np.zeros(W.shape, dtype=bool)
    rows = np.flatnonzero(~np.all(held, axis=1))
    mask[rows, np.argmax(err[rows], axis=1)] = True
    return mask


def clip_held_out(W: np.ndarray, mask: np.ndarray, group: int):
    """Section 3.1: in the pair fit, every held-out entry is clipped to the next
    value inward.

    Reading: the next value inward is the group's largest retained value for a
    held-out entry >= 0 and its smallest retained value for one < 0 (a held-out
    entry is never inside the retained range, since the record takes the
    largest |w|). Returns (clipped values [out, inp] fp64, bool [out, ngroups]
    marking groups with no retained entry).
    """
    out, inp = W.shape
    ng = inp // group
    V = W.astype(np.float64).reshape(out, ng, group)
    M = mask.reshape(out, ng, group)
    mx = np.where(M, -np.inf, V).max(axis=2)
    mn = np.where(M, np.inf, V).min(axis=2)
    empty = ~np.any(~M, axis=2)
    repl = np.where(V >= 0.0, mx[:, :, None], mn[:, :, None])
    Vc = np.where(M, repl, V)
    Vc = np.where(empty[:, :, None], 0.0, Vc)
    return Vc.reshape(out, inp), empty


def initial_pairs(Vc: np.ndarray, group: int):
    """Appendix B: the initial pair puts four levels symmetrically, the outer
    two 6 % in from the group's ends (a step of 0.29 of the range).

    lo0 = min + 0.06 R, top = max - 0.06 R, s0 = (top - lo0) / 3, R = max - min.
    Reading: a group of zero range gets s0 = 2^-24 and is flagged. Returns
    (lo0, s0, flat), each [out, ngroups]; flat marks the zero-range groups.
    """
    out, inp = Vc.shape
    G = Vc.reshape(out, inp // group, group)
    mn = G.min(axis=2)
    mx = G.max(axis=2)
    R = mx - mn
    lo0 = mn + INIT_EDGE_FRACTION * R
    top = mx - INIT_EDGE_FRACTION * R
    s0 = (top - lo0) / 3.0
    flat = ~(R > 0.0)
    s0 = np.where(flat, DEGENERATE_STEP, s0)
    return lo0, s0, flat


def uniform_codebook(values: np.ndarray) -> np.ndarray:
    """Appendix E, uniform placement: sixteen evenly spaced points over the
    range of the initial pairs, stored as fp16 (Section 3.1 / Appendix E).

    c_i = vmin + i (vmax - vmin) / 15, rounded to fp16 (nearest even).
    Reading: with no values at all the codebook is all zeros.
    """
    if values.size == 0:
        return np.zeros(CODEBOOK_SIZE, dtype=np.float16)
    vmin = float(values.min())
    vmax = float(values.max())
    cb = [vmin + i * (vmax - vmin) / (CODEBOOK_SIZE - 1) for i in range(CODEBOOK_SIZE)]
    return np.array(cb, dtype=np.float64).astype(np.float16)


def lloyd_codebook(values: np.ndarray, anchored: bool) -> np.ndarray:
    """Appendix E, Lloyd's rule (and Lloyd's rule with its ends anchored at
    the range of the initial pairs): sixteen points, each the mean of the
    values nearest to it, as fp16.

    Reading: the points start at the uniform placement (fp64); a step assigns
    every value to its nearest point (ties to the lower index) and moves each
    point to the mean of its values, summed in index order; a point with no
    value stays; anchored, points 0 and 15 stay at the range ends. The steps
    stop when no assignment changes, or after LLOYD_MAX_STEPS. With no values
    the codebook is all zeros.
    """
    if values.size == 0:
        return np.zeros(CODEBOOK_SIZE, dtype=np.float16)
    v = np.asarray(values, dtype=np.float64).reshape(-1)
    vmin, vmax = float(v.min()), float(v.max())
    c = np.array([vmin + i * (vmax - vmin) / (CODEBOOK_SIZE - 1) for i in range(CODEBOOK_SIZE)])
    assign = None
    for _ in range(LLOYD_MAX_STEPS):
        a = np.argmin(np.abs(v[:, None] - c[None, :]), axis=1)
        if assign is not None and np.array_equal(a, assign):
            break
        assign = a
        for i in range(CODEBOOK_SIZE):
            if anchored and i in (0, CODEBOOK_SIZE - 1):
                continue
            sel = v[a == i]
            if sel.size:
                c[i] = _sum_in_order(sel) / sel.size
    return c.astype(np.float16)


CODEBOOK_RULES = ("uniform", "lloyd", "anchored")


def codebook_by_rule(values: np.ndarray, rule: str) -> np.ndarray:
    if rule == "uniform":
        return uniform_codebook(values)
    return lloyd_codebook(values, anchored=(rule == "anchored"))


def first_term_min(Vc: np.ndarray, group: int, N: int, lo_tab, s_tab, skip,
                   chunk: int = 256) -> np.ndarray:
    """Per group: the smallest first term of Eq. (5) (the distortion averaged
    over M = 2..N, no floor term) over the 256 pairs; groups in ``skip`` give 0."""
    out, inp = Vc.shape
    G = Vc.reshape(out * (inp // group), group)
    best = np.empty(G.shape[0])
    for c0 in range(0, G.shape[0], chunk):
        V = G[c0:c0 + chunk][:, None, :]
        _, _, recons = encode_digits(V, lo_tab[None, :, None], s_tab[None, :, None], N)
        first = 0.0
        for rec in recons:
            first = first + _sum_in_order((V - rec) ** 2)
        best[c0:c0 + chunk] = (first / (N - 1)).min(axis=1)
    return np.where(skip.reshape(-1), 0.0, best)


def choose_codebook_rules(Vc, group: int, N: int, lo0, s0, skip, empty):
    """Appendix E: of the nine combinations of a rule for the log2(s)
    codebook and a rule for the lo/s codebook, the one whose per-group best
    first term of Eq. (5), summed over the matrix (group order), is smallest.
    Reading: ties go to the first combination, s-rule outer, in the order
    uniform, Lloyd, anchored Lloyd. The codebooks are fitted to the groups
    not in ``skip``; every group with a retained entry (not ``empty``) counts
    in the sum. Returns (rule_s, rule_lo)."""
    keep = ~skip
    ls, rl = np.log2(s0[keep]), lo0[keep] / s0[keep]
    best, arg = None, None
    for rs in CODEBOOK_RULES:
        for rr in CODEBOOK_RULES:
            lo_tab, s_tab = pair_table(codebook_by_rule(ls, rs), codebook_by_rule(rl, rr))
            tot = _sum_in_order(first_term_min(Vc, group, N, lo_tab, s_tab, empty))
            if best is None or tot < best:
                best, arg = tot, (rs, rr)
    return arg


def precision_errors(Vc, group: int, N: int, pair_idx, lo_tab, s_tab, skip):
    """Sum over the matrix (group order, then index order) of the two-bit and
    the deepest-precision (M = N) errors sum_c (V_c - W_c^(M))^2 of the
    clipped groups under their pairs; groups in ``skip`` count 0."""
    out, inp = Vc.shape
    G = Vc.reshape(out * (inp // group), group)
    p = pair_idx.reshape(-1).astype(np.int64)
    _, _, recons = encode_digits(G, lo_tab[p][:, None], s_tab[p][:, None], N)
    e2 = np.where(skip.reshape(-1), 0.0, _sum_in_order((G - recons[0]) ** 2))
    eN = np.where(skip.reshape(-1), 0.0, _sum_in_order((G - recons[-1]) ** 2))
    return _sum_in_order(e2), _sum_in_order(eN)


def fit_codebooks(lo0: np.ndarray, s0: np.ndarray, skip: np.ndarray):
    """Section 3.1: one codebook in log2(s) and one in lo/s per matrix, fitted
    to the initial pairs of the groups not marked in ``skip`` (Reading: groups
    with no retained entry or zero range have no initial pair to fit)."""
    keep = ~skip
    cb_log2s = uniform_codebook(np.log2(s0[keep]))
    cb_lo_over_s = uniform_codebook(lo0[keep] / s0[keep])
    return cb_log2s, cb_lo_over_s


def pair_table(cb_log2s: np.ndarray, cb_lo_over_s: np.ndarray):
    """The 256 (lo, s) combinations of Section 3.1, indexed a*16 + b with
    a = log2(s) index (high nibble) and b = lo/s index (low nibble).

    s = 2^(cb_log2s[a]), lo = cb_lo_over_s[b] * s, in fp64 from the fp16
    codebook values. Reading: nibble order high = log2(s).
    """
    a = np.repeat(np.arange(CODEBOOK_SIZE), CODEBOOK_SIZE)
    b = np.tile(np.arange(CODEBOOK_SIZE), CODEBOOK_SIZE)
    s = np.exp2(cb_log2s.astype(np.float64)[a])
    lo = cb_lo_over_s.astype(np.float64)[b] * s
    return lo, s


def pair_cost(V: np.ndarray, lo, s, N: int):
    """Eq. (5) with E_c = 1 (x ~ N(0,1) gives unit channel mean squares):

    D = 1/(N-1) sum_{M=2}^{N} sum_c (V_c - W_c^(M))^2
        + lambda sum_c max(|V_c - W_c^(2)| - rho, 0)^2          (Eq. (6))

    with W^(M) the digit encoding of ``encode_digits`` under (lo, s) and rho
    from ``reach``. ``V`` is [..., g] (the clipped group), lo and s broadcast
    against V[..., 0]. Returns D with V's leading shape.
    """
    lo = np.asarray(lo, dtype=np.float64)[..., None]
    s = np.asarray(s, dtype=np.float64)[..., None]
    _, _, recons = encode_digits(V, lo, s, N)
    first = 0.0
    for rec in recons:                       # M = 2 .. N
        first = first + _sum_in_order((V - rec) ** 2)
    first = first / (N - 1)
    rho = reach(s, N)
    floor = _sum_in_order(np.maximum(np.abs(V - recons[0]) - rho, 0.0) ** 2)
    return first + FLOOR_LAMBDA * floor


def _sum_in_order(a):
    """Sum over the last axis in index order c = 0, 1, ... (a fixed rounding
    order, so that any other implementation of Eq. (5) can reproduce it)."""
    return np.cumsum(a, axis=-1)[..., -1]


def choose_pairs(Vc: np.ndarray, group: int, N: int, lo_tab, s_tab, empty,
                 mode: str = "search", lo0=None, s0=None, cb_log2s=None,
                 cb_lo_over_s=None, flat=None, chunk: int = 256) -> np.ndarray:
    """Per-group pair choice.

    mode "search" (Section 3.1): the combination minimising Eq. (5) over all
    256; Reading: ties go to the smallest index a*16+b.
    mode "fast" (a labelled shortcut for very large stacks, not the paper's
    rule): the nearest codebook entry to log2(s0) and to lo0/s0 separately,
    ties to the smaller index.
    Groups with no retained entry get pair 0 (their digits are all zero);
    zero-range groups (``flat``) are searched in both modes.
    """
    out, inp = Vc.shape
    ng = inp // group
    if mode == "fast":
        ls = np.log2(s0)
        r = lo0 / s0
        da = np.abs(cb_log2s.astype(np.float64)[None, None, :] - ls[:, :, None])
        db = np.abs(cb_lo_over_s.astype(np.float64)[None, None, :] - r[:, :, None])
        a = np.argmin(da, axis=2)
        b = np.argmin(db, axis=2)
        idx = (a * CODEBOOK_SIZE + b).astype(np.uint8)
        if flat is not None and np.any(flat & ~empty):
            sel = flat & ~empty
            searched = choose_pairs(Vc, group, N, lo_tab, s_tab, empty, mode="search")
            idx = np.where(sel, searched, idx)
    elif mode == "search":
        G = Vc.reshape(out * ng, group)
        idx = np.empty(out * ng, dtype=np.uint8)
        for s0_ in range(0, G.shape[0], chunk):
            Vg = G[s0_:s0_ + chunk][:, None, :]                 # [c, 1, g]
            D = pair_cost(Vg, lo_tab[None, :], s_tab[None, :], N)   # [c, 256]
            idx[s0_:s0_ + chunk] = np.argmin(D, axis=1).astype(np.uint8)
        idx = idx.reshape(out, ng)
    else:
        raise ValueError(f"unknown pair mode {mode!r}")
    return np.where(empty, 0, idx).astype(np.uint8)


def encode(W: np.ndarray, group: int = 128, n_planes: int = 2,
           density: float = 0.005, mode: str = "search", rows=None,
           row_block: int = 512, guard: str = "density", ratio_T: float = 4.0,
           post_guard: bool = True, codebooks: str = "uniform") -> Fields:
    """Figure 3's encoder for synthetic weights (no AWQ scale: with x ~ N(0,1)
    every channel scale is equal):

    1. side record: with ``guard="density"`` the top-|w| entries
       (``select_side_record``, the workloads' reading); with ``guard="ratio"``
       the pre-grid ratio guard of Section 3.5 (``select_ratio_guard``, T =
       ``ratio_T``); P = fp16 value;
    2. clip held-out entries inward for the fit (``clip_held_out``);
    3. initial pairs (Appendix B), 4. codebooks: ``codebooks="uniform"``
       places both uniformly (Appendix E's first rule); ``"appendix_e"``
       picks one of the nine rule combinations (``choose_codebook_rules``)
       and falls back to uniform placement when the deepest precision's error
       exceeds FALLBACK_RATIO of the two-bit error under the chosen codebooks
       and the final pair choice (Reading: "six-bit" is the stream's deepest
       precision N; with N = 2 the test always falls back);
    5. pair per group (Eq. (5) search, or the labelled fast rule),
    6. base by nearest rounding, 7. sign planes k = 3..N; held-out positions
       store zero digits (Reading: the planes skip them, Section 3.6, and the
       paper gives no stored value -- zeros make the main stream decode to
       lo_M there, which Eq. (4) then masks).

    8. with ``guard="ratio"`` and ``post_guard``, the post-grid guard
       (``select_post_guard``): per row the position with the largest two-bit
       error. Its base digit stays; its planes are zero; it records the fp16
       residual r = fp16(w - W_hat^(2)), and Eq. (4) takes P = W_hat^(2) + r
       there (Section 3, Eq. (4): the two-bit reconstruction plus the
       residual, the same for every M).

    Steps 1-4 look at the whole matrix (global record, per-matrix codebooks).
    With ``rows`` given, steps 5-7 run only for those rows and the returned
    Fields hold just them (out = len(rows)); the encoding of a row depends on
    nothing else. Rows are processed ``row_block`` at a time to bound memory.
    """
    W = np.asarray(W)
    if W.dtype != np.float16:
        raise TypeError("W must be fp16")
    out, inp = W.shape
    if group <= 0 or inp % group:
        raise ValueError("group must divide the input dimension")
    N = 2 + n_planes
    ng = inp // group

    if guard == "density":
        mask = select_side_record(W, density)
    elif guard == "ratio":
        mask = select_ratio_guard(W, group, ratio_T)
    else:
        raise ValueError("guard must be 'density' or 'ratio'")
    with_post = guard == "ratio" and post_guard
    Vc, empty = clip_held_out(W, mask, group)
    lo0, s0, flat = initial_pairs(Vc, group)
    cb_log2s, cb_lo_over_s = fit_codebooks(lo0, s0, empty | flat)
    if codebooks == "appendix_e":
        rs, rr = choose_codebook_rules(Vc, group, N, lo0, s0, empty | flat, empty)
        keep = ~(empty | flat)
        cand = (codebook_by_rule(np.log2(s0[keep]), rs), codebook_by_rule(lo0[keep] / s0[keep], rr))
        lo_c, s_c = pair_table(*cand)
        pidx = choose_pairs(Vc, group, N, lo_c, s_c, empty, mode=mode, lo0=lo0, s0=s0,
                            cb_log2s=cand[0], cb_lo_over_s=cand[1], flat=flat)
        e2, eN = precision_errors(Vc, group, N, pidx, lo_c, s_c, empty)
        if not eN > FALLBACK_RATIO * e2:
            cb_log2s, cb_lo_over_s = cand
    elif codebooks != "uniform":
        raise ValueError("codebooks must be 'uniform' or 'appendix_e'")
    lo_tab, s_tab = pair_table(cb_log2s, cb_lo_over_s)

    rows = np.arange(out) if rows is None else np.asarray(rows, dtype=np.int64)
    n = rows.size
    pair_idx = np.empty((n, ng), dtype=np.uint8)
    q = np.empty((n, inp), dtype=np.uint8)
    planes = np.empty((n_planes, n, inp), dtype=np.uint8)
    post = np.zeros((n, inp), dtype=bool)
    resid = np.zeros((n, inp), dtype=np.float16)
    for b0 in range(0, n, row_block):
        rb = rows[b0:b0 + row_block]
        sl = slice(b0, b0 + rb.size)
        pair_idx[sl] = choose_pairs(Vc[rb], group, N, lo_tab, s_tab, empty[rb], mode=mode,
                                    lo0=lo0[rb], s0=s0[rb], cb_log2s=cb_log2s,
                                    cb_lo_over_s=cb_lo_over_s, flat=flat[rb])
        lo_w = np.repeat(lo_tab[pair_idx[sl].astype(np.int64)], group, axis=1)
        s_w = np.repeat(s_tab[pair_idx[sl].astype(np.int64)], group, axis=1)
        Wb = W[rb].astype(np.float64)
        qb, bits, _ = encode_digits(Wb, lo_w, s_w, N)
        m = mask[rb]
        pb = np.zeros_like(m)
        if with_post:
            W2 = lo_w + s_w * qb                          # Eq. (10) at M = 2: lo + s q
            pb = select_post_guard(W[rb], W2, m)
            resid[sl] = np.where(pb, Wb - W2, 0.0).astype(np.float16)
        post[sl] = pb
        q[sl] = np.where(m, 0, qb)                        # post-grid positions keep their base digit
        for k in range(n_planes):
            planes[k, sl] = np.where(m | pb, 0, bits[k])

    sub = mask[rows] | post
    r_idx, cols = np.nonzero(sub)                         # row-major order
    row_ptr = np.zeros(n + 1, dtype=np.int64)
    np.add.at(row_ptr, r_idx + 1, 1)
    row_ptr = np.cumsum(row_ptr)
    is_post = post[r_idx, cols]
    val = np.where(is_post, resid[r_idx, cols], W[rows[r_idx], cols]).astype(np.float16)
    return Fields(out=n, inp=inp, group=group, n_planes=n_planes, q=q,
                  planes=planes, pair_idx=pair_idx,
                  cb_log2s=cb_log2s, cb_lo_over_s=cb_lo_over_s,
                  row_ptr=row_ptr, col=cols.astype(np.int64), val=val,
                  post=is_post if with_post else None)


# --------------------------------------------------------------------------
# Decoder and GEMV (Eq. (4), (8), (10))
# --------------------------------------------------------------------------

def held_out_mask(F: Fields, rows=None) -> np.ndarray:
    """The mask m of Eq. (4), rebuilt from the CSR side record."""
    rows = np.arange(F.out) if rows is None else np.asarray(rows)
    m = np.zeros((rows.size, F.inp), dtype=bool)
    for i, r in enumerate(rows):
        m[i, F.col[F.row_ptr[r]:F.row_ptr[r + 1]]] = True
    return m


def check_precision(F: Fields, M: int) -> None:
    """A p_M read needs the base plus planes 3..M of the stored stream."""
    if not (2 <= M <= F.depth):
        raise ValueError(f"precision {M} outside 2..{F.depth}")


def decode_levels(F: Fields, M: int, rows=None) -> np.ndarray:
    """Eq. (8) per weight: the integer u_M read from the first M-2 planes."""
    check_precision(F, M)
    sl = slice(None) if rows is None else np.asarray(rows)
    return composite_level(F.q[sl], [F.planes[k][sl] for k in range(F.n_planes)], M)


def group_pairs(F: Fields, rows=None):
    """fp64 (lo, s) of every group, from the 8-bit pair index and codebooks."""
    lo_tab, s_tab = pair_table(F.cb_log2s, F.cb_lo_over_s)
    idx = F.pair_idx if rows is None else F.pair_idx[np.asarray(rows)]
    return lo_tab[idx.astype(np.int64)], s_tab[idx.astype(np.int64)]


def decode(F: Fields, M: int, rows=None) -> np.ndarray:
    """Eq. (4): W_hat^(M) = (1 - m) * (lo_M + s_M u_M) + P, fp64 [rows, inp].
    P is the recorded value at a pre-grid entry and the two-bit
    reconstruction lo + s q plus the recorded residual at a post-grid entry
    (Section 3, below Eq. (4))."""
    u = decode_levels(F, M, rows)
    lo_g, s_g = group_pairs(F, rows)
    lo_w = np.repeat(lo_g, F.group, axis=1)
    s_w = np.repeat(s_g, F.group, axis=1)
    main = reconstruct_affine(lo_w, s_w, u, M)
    rows_ = np.arange(F.out) if rows is None else np.asarray(rows)
    q = F.q if rows is None else F.q[rows_]
    w2 = lo_w + s_w * q.astype(np.float64)               # two-bit reconstruction, Eq. (10) at M = 2
    m = held_out_mask(F, rows_)
    post = F.post_flags
    P = np.zeros_like(main)
    for i, r in enumerate(rows_):
        sl = slice(F.row_ptr[r], F.row_ptr[r + 1])
        c = F.col[sl]
        v = F.val[sl].astype(np.float64)
        P[i, c] = np.where(post[sl], w2[i, c] + v, v)
    return np.where(m, 0.0, main) + P


def gemv(F: Fields, M: int, x: np.ndarray, rows=None, in_scale=None) -> np.ndarray:
    """y = W_hat^(M) x in fp64 for x [n, inp] (fp16 values taken exactly);
    returns [n, len(rows)] (all rows by default).

    ``in_scale`` [inp] (fp32 values taken exactly): the run-time inverse
    activation scale of Section 4 / Appendix E -- the quantizer saw W diag(a),
    so the decoder multiplies channel c of x by 1/a_c (given here) before the
    product: y = W_hat (x * in_scale)."""
    x = np.atleast_2d(np.asarray(x)).astype(np.float64)
    if in_scale is not None:
        x = x * np.asarray(in_scale, dtype=np.float64)[None, :]
    What = decode(F, M, rows)
    return x @ What.T


def model_bytes(out: int, inp: int, group: int, nnz: int, M: int, n: int = 1) -> int:
    """Bytes a p_M GEMV must move: the base and M-2 planes (M bits per weight),
    one pair byte per group, the CSR record (4 B per entry + 4 B per row
    pointer), x and y in fp16."""
    return (out * inp * M) // 8 + (out * inp) // group + 4 * nnz + 4 * (out + 1) \
        + 2 * n * inp + 2 * n * out
