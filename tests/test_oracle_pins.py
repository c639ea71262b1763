"""Pins of the CPU oracle against what the StagQ paper and plain mathematics
fix, independent of the oracle's own formulas (CPU only)."""
import itertools
import math
import os

import numpy as np
import pytest

from oracle import stagq as O
from quantized_gemv_stagq_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    d = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *v = line.split()
            d[k] = [float(t) for t in v]
    return d


# ---------------------------------------------------------------- Figure 1

def test_figure1_worked_example():
    """Figure 1 caption: w = 2.15 -> q=2, b3=1, b4=0, b5=1, b6=0."""
    g = _read_golden("fig1_worked_example.txt")
    q, bits, recons = O.encode_digits(np.array([g["w"][0]]), g["lo"][0], g["s"][0], int(g["N"][0]))
    assert int(q[0]) == int(g["q"][0])
    assert [int(b[0]) for b in bits] == [int(v) for v in g["b"]]


def test_figure1_every_prefix_is_a_grid_point():
    """Each prefix of the Figure 1 stream decodes, via Eq. (10), to the point
    of its own uniform grid that holds 2.15 (the caption's claim that every
    precision is again a uniform grid)."""
    q, bits, recons = O.encode_digits(np.array([2.15]), 0.0, 1.0, 6)
    for M in range(2, 7):
        lo_M, s_M = O.grid_at(0.0, 1.0, M)
        u = O.composite_level(q, bits, M)
        w = O.reconstruct_affine(0.0, 1.0, u, M)
        assert w[0] == recons[M - 2][0]
        # the point is the nearest grid point to 2.15 (exact dyadic arithmetic)
        grid = lo_M + s_M * np.arange(2 ** M)
        assert w[0] == grid[np.argmin(np.abs(grid - 2.15))]


# ------------------------------------------------------- closed forms

def test_eq9_equals_eq10_all_digit_patterns():
    """Section 3.4: the additive form Eq. (9) collapses to lo_M + s_M u_M."""
    rng = np.random.default_rng(3)
    for M in range(2, 7):
        for lo, s in [(0.0, 1.0), (-0.75, 0.125)] + [tuple(rng.normal(size=2) * [0.05, 0.01] + [0, 0.02]) for _ in range(3)]:
            for q in range(4):
                for pat in itertools.product([0, 1], repeat=M - 2):
                    planes = [np.array([b]) for b in pat]
                    a = O.reconstruct_additive(lo, s, np.array([q]), planes, M)[0]
                    u = O.composite_level(np.array([q]), planes, M)
                    b = O.reconstruct_affine(lo, s, u, M)[0]
                    assert abs(a - b) <= 1e-12 * max(1.0, abs(a))


def test_reach_equals_top_level_overhang():
    """Eq. (6): rho is how far the planes move the top base level lo + 3s; it
    equals the top grid point at depth N, lo_N + s_N (2^N - 1), minus lo + 3s."""
    for N in range(2, 9):
        lo, s = -0.3, 0.07
        lo_N, s_N = O.grid_at(lo, s, N)
        assert math.isclose(lo_N + s_N * (2 ** N - 1), lo + 3 * s + O.reach(s, N), rel_tol=1e-13)
        # and in closed form s (1/2 - 2^-(N-1))
        assert math.isclose(O.reach(s, N), s * (0.5 - 2.0 ** -(N - 1)) if N > 2 else 0.0, abs_tol=1e-15)


def test_midpoint_split_is_the_mmse_split():
    """Appendix C, Eq. (12): splitting a uniform cell [a, b] at the midpoint with
    reconstructions (3a+b)/4 and (a+3b)/4 is optimal; the p3 reconstructions of
    the two halves of every base cell must be exactly these."""
    lo, s = 0.25, 0.5
    for q in range(4):
        a = lo + s * (q - 0.5)
        b = a + s
        lo3, s3 = O.grid_at(lo, s, 3)
        left = lo3 + s3 * (2 * q)
        right = lo3 + s3 * (2 * q + 1)
        assert left == (3 * a + b) / 4 and right == (a + 3 * b) / 4
    # Eq. (13): D(theta) is minimised at the midpoint (numeric brute force)
    a, b = 0.0, 1.0
    th = np.linspace(0.01, 0.99, 981)
    D = ((th - a) ** 3 + (b - th) ** 3) / (12 * (b - a))
    assert abs(th[np.argmin(D)] - 0.5) < 1e-9


def test_initial_pair_matches_appendix_b_constants():
    """Appendix B: four symmetric levels, outer two 6 % in from each end, a step
    of 0.29 of the group range."""
    V = np.array([[0.0, 0.3, 0.7, 1.0] * 2])
    lo0, s0, flat = O.initial_pairs(V, 8)
    R = 1.0
    assert math.isclose(lo0[0, 0], 0.06 * R)
    assert math.isclose(lo0[0, 0] + 3 * s0[0, 0], R - 0.06 * R)
    assert abs(s0[0, 0] / R - 0.29) < 0.005


def test_rate_of_pair_and_planes():
    """Section 4.2: one 8-bit pair per group of 32 costs 0.25 bpw; Section 4.1:
    each refinement plane adds exactly 1 bpw."""
    out, inp = 64, 1024
    fixed = 4 * (out + 1)
    b2 = O.model_bytes(out, inp, 32, 0, 2, n=0) - fixed
    b3 = O.model_bytes(out, inp, 32, 0, 3, n=0) - fixed
    assert (b2 * 8) / (out * inp) == 2.25
    assert ((b3 - b2) * 8) / (out * inp) == 1.0


# --------------------------------------------------------- invariants

def test_every_precision_is_a_uniform_grid():
    """Figure 1 / Eq. (10): the reachable set at precision M is
    {lo_M + s_M u : u = 0..2^M-1}, evenly spaced by s_M."""
    lo, s = -0.037, 0.0113
    for M in range(2, 7):
        vals = set()
        for q in range(4):
            for pat in itertools.product([0, 1], repeat=M - 2):
                vals.add(O.reconstruct_additive(lo, s, np.array([q]), [np.array([b]) for b in pat], M)[0])
        v = np.array(sorted(vals))
        assert v.size == 2 ** M
        lo_M, s_M = O.grid_at(lo, s, M)
        assert np.allclose(v, lo_M + s_M * np.arange(2 ** M), rtol=0, atol=1e-15)


def test_shallow_read_is_midpoint_of_merged_cells():
    """Section 2.1: each shallower read reconstructs at the midpoint of the
    two deeper cells it merges."""
    lo, s = 0.011, 0.0031
    for M in range(2, 6):
        for u in range(2 ** M):
            a = O.reconstruct_affine(lo, s, 2 * u, M + 1)
            b = O.reconstruct_affine(lo, s, 2 * u + 1, M + 1)
            c = O.reconstruct_affine(lo, s, u, M)
            assert math.isclose(c, (a + b) / 2, rel_tol=1e-13, abs_tol=1e-16)


def test_sign_planes_equal_nearest_level_rounding():
    """The base by nearest rounding plus sign-of-residual planes lands on the
    nearest point of the precision-M grid (a textbook uniform quantiser with
    half-open cells), including the clamped ends."""
    rng = np.random.default_rng(7)
    lo, s = -0.05, 0.031
    w = rng.uniform(lo - 3 * s, lo + 6 * s, size=20000)
    N = 6
    q, bits, _ = O.encode_digits(w, lo, s, N)
    for M in range(2, N + 1):
        lo_M, s_M = O.grid_at(lo, s, M)
        t = (w - lo_M) / s_M + 0.5
        ok = np.abs(t - np.round(t)) > 1e-9             # stay off exact cell edges
        ref = np.clip(np.floor(t), 0, 2 ** M - 1)
        u = O.composite_level(q, bits, M)
        assert np.array_equal(u[ok], ref[ok])


def test_prefix_read_equals_truncated_stream():
    """Sections 1 and 3.3: a p-bit read of a deep stream equals reading the
    stream cut after plane p."""
    W = synth.weights(16, 256, seed=11)
    F = O.encode(W, group=64, n_planes=4, density=0.01, mode="search")
    x = synth.activations(1, 256, seed=12)
    for p in range(2, 7):
        T = O.Fields(**{**F.__dict__, "n_planes": p - 2, "planes": F.planes[: p - 2]})
        assert np.array_equal(O.decode_levels(F, p), O.decode_levels(T, p))
        assert np.array_equal(O.gemv(F, p, x), O.gemv(T, p, x))


# ---------------------------------------------------- side record, Eq. (4)

def test_side_record_top_abs_with_index_tiebreak():
    W = np.array([[0.5, -0.5, 0.1, 0.25], [0.5, 0.0, -0.25, 0.3]], dtype=np.float16)
    m = O.select_side_record(W, 3 / 8)
    # |w| = 0.5 appears three times: flat indices 0, 1, 4 -> all in
    assert m.reshape(-1).nonzero()[0].tolist() == [0, 1, 4]
    m = O.select_side_record(W, 2 / 8)
    assert m.reshape(-1).nonzero()[0].tolist() == [0, 1]


def test_clip_to_next_value_inward():
    W = np.array([[-0.1, 5.0, 0.05, 0.2, -3.0, 0.0, 0.1, -0.05]], dtype=np.float16)
    m = np.zeros_like(W, dtype=bool)
    m[0, 1] = m[0, 4] = True
    Vc, empty = O.clip_held_out(W, m, 8)
    f16 = lambda v: float(np.float16(v))
    assert Vc[0, 1] == f16(0.2) and Vc[0, 4] == f16(-0.1)
    assert not empty[0, 0]


def test_density_zero_is_the_main_stream_alone():
    W = synth.weights(8, 128, seed=1)
    F = O.encode(W, group=64, n_planes=2, density=0.0, mode="search")
    assert F.nnz == 0
    x = synth.activations(1, 128, seed=2).astype(np.float64)
    lo, s = O.group_pairs(F)
    for M in (2, 3, 4):
        u = O.decode_levels(F, M)
        Wm = np.empty((8, 128))
        for r in range(8):
            for c in range(128):
                lo_M, s_M = O.grid_at(lo[r, c // 64], s[r, c // 64], M)
                Wm[r, c] = lo_M + s_M * u[r, c]
        assert np.allclose(O.gemv(F, M, x)[0], Wm @ x[0], rtol=1e-12, atol=1e-12)


def test_everything_held_out_is_a_dense_fp16_gemv():
    """Eq. (4) with m = 1 everywhere: W_hat = P = W, so y = W x exactly."""
    W = synth.weights(12, 256, seed=5)
    F = O.encode(W, group=128, n_planes=2, density=1.0, mode="search")
    assert F.nnz == W.size and not F.q.any() and not F.planes.any()
    x = synth.activations(2, 256, seed=6)
    ref = x.astype(np.float64) @ W.astype(np.float64).T
    for M in (2, 3, 4):
        assert np.allclose(O.gemv(F, M, x), ref, rtol=1e-13, atol=1e-13)


def test_held_out_positions_store_zero_digits():
    W = synth.weights(32, 256, seed=9)
    F = O.encode(W, group=128, n_planes=2, density=0.02, mode="fast")
    m = O.held_out_mask(F)
    assert m.sum() == F.nnz == O.side_record_count(32, 256, 0.02)
    assert not F.q[m].any() and not F.planes[:, m].any()
    assert np.array_equal(F.val, W[m])


# ----------------------------------------------------------- brute force

def _brute_force_gemv(F, M, x):
    """Scalar Python loops straight from Eq. (8), (10) and (4)."""
    y = [0.0] * F.out
    cbs = [float(v) for v in F.cb_log2s]
    cbr = [float(v) for v in F.cb_lo_over_s]
    for r in range(F.out):
        held = {}
        for e in range(F.row_ptr[r], F.row_ptr[r + 1]):
            held[int(F.col[e])] = float(F.val[e])
        acc = 0.0
        for c in range(F.inp):
            if c in held:
                w = held[c]
            else:
                p = int(F.pair_idx[r, c // F.group])
                s = 2.0 ** cbs[p >> 4]
                lo = cbr[p & 15] * s
                u = int(F.q[r, c]) << (M - 2)
                for k in range(3, M + 1):
                    u += int(F.planes[k - 3, r, c]) << (M - k)
                s_M = s / 2 ** (M - 2)
                lo_M = lo - s * (2 ** (M - 2) - 1) / 2 ** (M - 1)
                w = lo_M + s_M * u
            acc += w * float(x[c])
        y[r] = acc
    return np.array(y)


@pytest.mark.parametrize("M", [2, 3, 4])
def test_gemv_against_scalar_brute_force(M):
    W = synth.weights(6, 256, seed=21)
    F = O.encode(W, group=64, n_planes=2, density=0.02, mode="search")
    x = synth.activations(1, 256, seed=22)
    y = O.gemv(F, M, x)[0]
    assert np.allclose(y, _brute_force_gemv(F, M, x[0]), rtol=1e-12, atol=1e-14)


def _brute_force_pair(V, cbs, cbr, N):
    best, best_i = None, None
    for a in range(16):
        for b in range(16):
            s = 2.0 ** float(cbs[a])
            lo = float(cbr[b]) * s
            rho = sum(s / 2 ** (k - 1) for k in range(3, N + 1))
            first, floor = 0.0, 0.0
            for v in V:
                q = min(3, max(0, math.floor((v - lo) / s + 0.5)))
                rec = lo + s * q
                e2 = v - rec
                first += e2 * e2
                floor += max(abs(e2) - rho, 0.0) ** 2
                for k in range(3, N + 1):
                    rec = rec + (s / 2 ** (k - 1) if v - rec >= 0 else -s / 2 ** (k - 1))
                    first += (v - rec) ** 2
            D = first / (N - 1) + 4.0 * floor
            if best is None or D < best:
                best, best_i = D, a * 16 + b
    return best_i


def test_pair_search_matches_brute_force_argmin():
    """Eq. (5)-(6) with E_c = 1: the searched pair is the brute-force argmin
    (parity of the search itself is otherwise unpinned by the paper)."""
    W = synth.weights(3, 64, seed=31)
    N = 4
    F = O.encode(W, group=16, n_planes=N - 2, density=0.0, mode="search")
    Vc = W.astype(np.float64)
    for r in range(3):
        for g in range(4):
            V = [float(v) for v in Vc[r, g * 16:(g + 1) * 16]]
            assert F.pair_idx[r, g] == _brute_force_pair(V, F.cb_log2s, F.cb_lo_over_s, N)


def test_codebooks_are_uniform_over_initial_pair_range():
    W = synth.weights(16, 512, seed=41)
    F = O.encode(W, group=128, n_planes=2, density=0.005, mode="fast")
    m = O.select_side_record(W, 0.005)
    Vc, empty = O.clip_held_out(W, m, 128)
    lo0, s0, flat = O.initial_pairs(Vc, 128)
    ls = np.log2(s0)
    assert F.cb_log2s[0] == np.float16(ls.min()) and F.cb_log2s[-1] == np.float16(ls.max())
    exact = ls.min() + np.arange(16) * (ls.max() - ls.min()) / 15
    ulp = float(np.spacing(np.float16(np.abs(ls).max())))
    assert np.all(np.abs(F.cb_log2s.astype(np.float64) - exact) <= ulp / 2)


# ------------------------------------------------ guards (Section 3.5, Appendix E)

def _brute_ratio_guard(W, group, T):
    out, inp = W.shape
    m = np.zeros((out, inp), dtype=bool)
    for r in range(out):
        for g0 in range(0, inp, group):
            a = [abs(float(W[r, g0 + j])) for j in range(group)]
            j1 = 0
            for j in range(1, group):
                if a[j] > a[j1]:
                    j1 = j
            second = max([a[j] for j in range(group) if j != j1], default=0.0)
            if a[j1] > T * second:
                m[r, g0 + j1] = True
    return m


def test_ratio_guard_matches_brute_force():
    rng = np.random.default_rng(4)
    W = (rng.standard_normal((6, 64)) * 0.02).astype(np.float16)
    W[0, 3] = 0.5                 # dominant: > 4x the rest of its group
    W[1, 17:19] = 0.4             # two equal largest: nothing held out
    W[2, 32:48] = 0.0
    W[2, 40] = 0.01               # the only nonzero of its group
    W[3, 48:64] = 0.0             # all-zero group: nothing held out
    for T in (4.0, 2.0, 8.0):
        m = O.select_ratio_guard(W, 16, T)
        assert np.array_equal(m, _brute_ratio_guard(W, 16, T)), T
    m = O.select_ratio_guard(W, 16, 4.0)
    assert m[0, 3] and not m[1, 16:32].any() and m[2, 40] and not m[3, 48:64].any()
    assert (m.reshape(6, 4, 16).sum(axis=2) <= 1).all()   # at most one entry per group


def test_post_guard_is_the_row_argmax_of_two_bit_error():
    """Each row's post-grid entry is the non-held position with the largest
    (w - (lo + s q))^2 (first on ties), recomputed here with scalar loops from
    the stored digits and pairs; its base digit is the grid's, its planes 0."""
    W = synth.weights(10, 256, seed=31)
    F = O.encode(W, group=64, n_planes=2, mode="fast", guard="ratio", ratio_T=4.0)
    post = F.post_flags
    cbs = [float(v) for v in F.cb_log2s]
    cbr = [float(v) for v in F.cb_lo_over_s]
    for r in range(F.out):
        sl = slice(F.row_ptr[r], F.row_ptr[r + 1])
        pre_cols = set(int(c) for c, p in zip(F.col[sl], post[sl]) if not p)
        post_cols = [int(c) for c, p in zip(F.col[sl], post[sl]) if p]
        best, best_c = -1.0, None
        for c in range(F.inp):
            if c in pre_cols:
                continue
            p = int(F.pair_idx[r, c // F.group])
            s = 2.0 ** cbs[p >> 4]
            lo = cbr[p & 15] * s
            w = float(W[r, c])
            q = min(3, max(0, math.floor((w - lo) / s + 0.5)))   # nearest rounding under the fixed grid
            e = (w - (lo + s * q)) ** 2
            if e > best:
                best, best_c = e, c
        assert post_cols == [best_c], r
        assert F.planes[:, r, best_c].sum() == 0
        p = int(F.pair_idx[r, best_c // F.group])
        s = 2.0 ** cbs[p >> 4]
        lo = cbr[p & 15] * s
        assert int(F.q[r, best_c]) == min(3, max(0, math.floor((float(W[r, best_c]) - lo) / s + 0.5)))


def test_post_entries_reconstruct_w_at_every_precision():
    """At a post-grid entry P = two-bit reconstruction + fp16 residual: the
    same at every M, and within the residual's fp16 rounding of w; pre-grid
    entries return the recorded fp16 value exactly."""
    W = synth.weights(16, 512, seed=33)
    F = O.encode(W, group=32, n_planes=4, mode="fast", guard="ratio", ratio_T=4.0)
    post = F.post_flags
    assert post.sum() == 16 and (~post).sum() > 0
    r = np.repeat(np.arange(F.out), np.diff(F.row_ptr))
    w = W[r, F.col].astype(np.float64)
    got = [O.decode(F, M)[r, F.col] for M in range(2, 7)]
    for g in got[1:]:
        assert np.array_equal(g, got[0])
    res = np.abs(F.val[post].astype(np.float64))
    assert np.all(np.abs(got[0][post] - w[post]) <= res * 2.0 ** -11 + 1e-12)
    assert np.array_equal(got[0][~post], w[~post])


def test_ratio_guard_without_hold_outs_is_the_main_stream():
    """T = infinity and no post-grid guard hold nothing out: the stream equals
    the density-0 encoding field for field."""
    W = synth.weights(8, 256, seed=35)
    A = O.encode(W, group=64, n_planes=2, density=0.0, mode="fast")
    B = O.encode(W, group=64, n_planes=2, mode="fast", guard="ratio", ratio_T=math.inf, post_guard=False)
    assert B.nnz == 0
    for k in ("q", "planes", "pair_idx", "cb_log2s", "cb_lo_over_s"):
        assert np.array_equal(getattr(A, k), getattr(B, k)), k


def test_gemv_with_guards_against_scalar_brute_force():
    W = synth.weights(6, 256, seed=37)
    F = O.encode(W, group=64, n_planes=2, mode="search", guard="ratio", ratio_T=4.0)
    x = synth.activations(1, 256, seed=38)[0]
    cbs = [float(v) for v in F.cb_log2s]
    cbr = [float(v) for v in F.cb_lo_over_s]
    for M in (2, 3, 4):
        y = O.gemv(F, M, x[None])[0]
        ref = []
        for r in range(F.out):
            acc = 0.0
            ent = {int(F.col[e]): (float(F.val[e]), bool(F.post_flags[e]))
                   for e in range(F.row_ptr[r], F.row_ptr[r + 1])}
            for c in range(F.inp):
                p = int(F.pair_idx[r, c // F.group])
                s = 2.0 ** cbs[p >> 4]
                lo = cbr[p & 15] * s
                if c in ent and not ent[c][1]:
                    w = ent[c][0]
                elif c in ent:
                    w = lo + s * int(F.q[r, c]) + ent[c][0]
                else:
                    u = int(F.q[r, c]) << (M - 2)
                    for k in range(3, M + 1):
                        u += int(F.planes[k - 3, r, c]) << (M - k)
                    w = lo - s * (2 ** (M - 2) - 1) / 2 ** (M - 1) + s / 2 ** (M - 2) * u
                acc += w * float(x[c])
            ref.append(acc)
        assert np.allclose(y, ref, rtol=1e-12, atol=1e-14), M


# ------------------------------------------- codebook rules (Appendix E)

def _clusters(rng, centers, counts, spread=1e-3):
    return np.concatenate([c + spread * rng.standard_normal(n) for c, n in zip(centers, counts)])


def test_lloyd_points_are_the_cluster_means():
    """Sixteen tight clusters near the uniform points: Lloyd's rule moves each
    point to the mean of its cluster (fp16 of the exact mean); anchored, the
    two end points stay at the range ends."""
    rng = np.random.default_rng(1)
    centers = np.linspace(-3.0, 2.0, 16) + rng.uniform(-0.05, 0.05, 16)
    counts = rng.integers(3, 40, 16)
    v = _clusters(rng, centers, counts)
    groups = np.split(v, np.cumsum(counts)[:-1])
    means = np.array([math.fsum(gv) / gv.size for gv in groups])
    c = O.lloyd_codebook(v, anchored=False)
    assert np.array_equal(c, means.astype(np.float16))
    a = O.lloyd_codebook(v, anchored=True)
    assert a[0] == np.float16(v.min()) and a[15] == np.float16(v.max())
    assert np.array_equal(a[1:15], means[1:15].astype(np.float16))


def _distortion(v, c):
    c = c.astype(np.float64)
    return float(np.sum(np.min((v[:, None] - c[None, :]) ** 2, axis=1)))


def test_lloyd_never_worse_than_uniform():
    """Lloyd's rule starts at the uniform points and never raises the
    quantisation distortion of the values (up to the fp16 rounding of the
    points)."""
    rng = np.random.default_rng(2)
    for trial in range(5):
        v = np.concatenate([rng.standard_normal(300) * 0.3, rng.standard_normal(40) * 2.0 + 3.0])
        u = O.uniform_codebook(v)
        for anchored in (False, True):
            l = O.lloyd_codebook(v, anchored)
            assert _distortion(v, l) <= _distortion(v, u) * (1 + 1e-3) + 1e-9, (trial, anchored)


def _weights_with_spread_scales(out, inp, seed):
    rng = np.random.default_rng(seed)
    scale = np.exp(rng.standard_normal((out, 1)) * 1.5) * 0.02
    scale[:3] *= 30
    return (rng.standard_normal((out, inp)) * scale).astype(np.float16)


def test_codebook_rule_choice_matches_brute_force():
    """The nine combinations scored with scalar loops: per group the smallest
    first term of Eq. (5) over the 256 pairs (digits of R8, Eq. (7)), summed
    over the matrix; the oracle picks the same combination."""
    W = _weights_with_spread_scales(6, 64, 5)
    g, N = 16, 3
    Vc, empty = O.clip_held_out(W, np.zeros_like(W, dtype=bool), g)
    lo0, s0, flat = O.initial_pairs(Vc, g)
    keep = ~(empty | flat)
    ls, rl = np.log2(s0[keep]), lo0[keep] / s0[keep]
    best, arg = None, None
    for rs in ("uniform", "lloyd", "anchored"):
        for rr in ("uniform", "lloyd", "anchored"):
            cbs = [float(x) for x in O.codebook_by_rule(ls, rs)]
            cbr = [float(x) for x in O.codebook_by_rule(rl, rr)]
            total = 0.0
            for r in range(W.shape[0]):
                for g0 in range(0, W.shape[1], g):
                    V = [float(x) for x in Vc[r, g0:g0 + g]]
                    gb = None
                    for p in range(256):
                        s = 2.0 ** cbs[p >> 4]
                        lo = cbr[p & 15] * s
                        first = 0.0
                        errs = [0.0] * (N - 1)
                        for v in V:
                            q = min(3, max(0, math.floor((v - lo) / s + 0.5)))
                            rec = lo + s * q
                            errs[0] += (v - rec) ** 2
                            for k in range(3, N + 1):
                                rec += s / 2 ** (k - 1) if v - rec >= 0 else -s / 2 ** (k - 1)
                                errs[k - 2] += (v - rec) ** 2
                        first = sum(errs) / (N - 1)
                        gb = first if gb is None else min(gb, first)
                    total += gb
            if best is None or total < best * (1 - 1e-12):
                best, arg = total, (rs, rr)
    assert O.choose_codebook_rules(Vc, g, N, lo0, s0, empty | flat, empty) == arg


def test_codebook_rules_keep_lloyd_or_fall_back():
    """Spread group scales: a Lloyd rule wins and the deep-precision test keeps
    it (its error is below a tenth of the two-bit error); with no planes the
    deepest precision is two bits, so the matrix falls back to uniform."""
    W = _weights_with_spread_scales(24, 256, 0)
    A = O.encode(W, 32, 2, 0.0, "search", codebooks="appendix_e")
    U = O.encode(W, 32, 2, 0.0, "search")
    assert not np.array_equal(A.cb_log2s, U.cb_log2s)
    Vc, empty = O.clip_held_out(W, np.zeros_like(W, dtype=bool), 32)
    lo_t, s_t = O.pair_table(A.cb_log2s, A.cb_lo_over_s)
    e2, e4 = O.precision_errors(Vc, 32, 4, A.pair_idx, lo_t, s_t, empty)
    assert e4 <= 0.1 * e2
    assert ((O.decode(A, 2) - W) ** 2).sum() < ((O.decode(U, 2) - W) ** 2).sum()
    A0 = O.encode(W, 32, 0, 0.0, "fast", codebooks="appendix_e")
    U0 = O.encode(W, 32, 0, 0.0, "fast")
    assert np.array_equal(A0.cb_log2s, U0.cb_log2s) and np.array_equal(A0.cb_lo_over_s, U0.cb_lo_over_s)


# ------------------------------------- run-time inverse activation scale

def test_input_scale_is_a_column_scaling_of_w_hat():
    """y = W_hat (x * s) equals (W_hat diag(s)) x, and power-of-two scales
    equal the GEMV of the scaled x exactly; all-ones is the plain GEMV."""
    W = synth.weights(12, 256, seed=41)
    F = O.encode(W, group=64, n_planes=2, density=0.01, mode="fast")
    x = synth.activations(2, 256, seed=42)
    rng = np.random.default_rng(43)
    s = rng.uniform(0.25, 4.0, 256).astype(np.float32)
    p2 = (2.0 ** rng.integers(-3, 4, 256)).astype(np.float32)
    for M in (2, 3, 4):
        D = O.decode(F, M)
        assert np.allclose(O.gemv(F, M, x, in_scale=s), x.astype(np.float64) @ (D * s.astype(np.float64)[None, :]).T,
                           rtol=1e-12, atol=1e-13)
        xs = (x.astype(np.float64) * p2.astype(np.float64)).astype(np.float64)
        assert np.array_equal(O.gemv(F, M, x, in_scale=p2), xs @ D.T)
        assert np.array_equal(O.gemv(F, M, x, in_scale=np.ones(256, np.float32)), O.gemv(F, M, x))


# ------------------------------------- the labelled fast pair rule (Section 3.1)

def _nearest_entry(cb, v):
    """Index of the codebook entry nearest to v, ties to the smaller index
    (a scalar scan)."""
    best = 0
    for i in range(1, len(cb)):
        if abs(float(cb[i]) - v) < abs(float(cb[best]) - v):
            best = i
    return best


def _scalar_fast_pairs(W, held, group, cb_log2s, cb_lo_over_s, N):
    """The fast rule restated with scalar loops per group: clip held-out
    entries to the group's retained max (w >= 0) or min (w < 0), take
    Appendix B's initial pair (lo0 = min + 0.06 R, s0 = (max - 0.06 R - lo0)
    / 3), then the nearest log2(s) entry (high nibble) and the nearest lo/s
    entry (low nibble). A group with nothing retained takes pair 0; a group of
    zero range is searched (Eq. (5) brute force)."""
    out, inp = W.shape
    idx = np.zeros((out, inp // group), dtype=np.int64)
    for r in range(out):
        for g in range(inp // group):
            cols = range(g * group, (g + 1) * group)
            kept = [float(W[r, c]) for c in cols if not held[r, c]]
            if not kept:
                idx[r, g] = 0
                continue
            hi, lo = max(kept), min(kept)
            vals = [float(W[r, c]) if not held[r, c] else (hi if float(W[r, c]) >= 0.0 else lo) for c in cols]
            mn, mx = min(vals), max(vals)
            if mx == mn:
                idx[r, g] = _brute_force_pair(vals, cb_log2s, cb_lo_over_s, N)
                continue
            R = mx - mn
            lo0 = mn + 0.06 * R
            s0 = (mx - 0.06 * R - lo0) / 3.0
            a = _nearest_entry(cb_log2s, math.log2(s0))
            b = _nearest_entry(cb_lo_over_s, lo0 / s0)
            idx[r, g] = 16 * a + b
    return idx


def _fast_rule_weights():
    W = synth.weights(8, 128, seed=57)
    W[0, 0:16] = np.float16(0.01)                           # a zero-range group: searched
    W[1, 16:32] = (np.arange(16) * 0.01 + 1.0).astype(np.float16)  # all held out: pair 0
    return W


def test_fast_pair_rule_matches_scalar_nearest_entries():
    """The fast rule (used by the large workloads) against its statement in
    scalar loops, on groups with held-out entries, a zero-range group and a
    fully held-out group."""
    W = _fast_rule_weights()
    density = 24 / W.size
    for n_planes in (2, 4):
        F = O.encode(W, group=16, n_planes=n_planes, density=density, mode="fast")
        held = np.zeros(W.shape, dtype=bool)
        for r in range(F.out):
            for e in range(F.row_ptr[r], F.row_ptr[r + 1]):
                held[r, F.col[e]] = True
        assert held[1, 16:32].all() and held.sum() == 24
        want = _scalar_fast_pairs(W, held, 16, F.cb_log2s, F.cb_lo_over_s, 2 + n_planes)
        assert want[1, 1] == 0
        assert np.array_equal(F.pair_idx.astype(np.int64), want)
        # the rule is not the search: on these groups at least one pair differs
        S = O.encode(W, group=16, n_planes=n_planes, density=density, mode="search")
        assert not np.array_equal(S.pair_idx, F.pair_idx)
