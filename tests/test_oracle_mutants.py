"""Planted mistakes in the oracle (CPU only): each plausible slip -- a dropped
term, a wrong sign, a wrong exponent, swapped nibbles -- must make at least
one pin in test_oracle_pins fail."""
import dataclasses

import numpy as np
import pytest

from oracle import stagq as O
import tests.test_oracle_pins as P


def _fails(fn, *args):
    try:
        fn(*args)
    except AssertionError:
        return True
    return False


def _grid_wrong_sign(lo, s, M):
    s_M = s / 2.0 ** (M - 2)
    return lo + s * (2.0 ** (M - 2) - 1.0) / 2.0 ** (M - 1), s_M


def _grid_wrong_spacing(lo, s, M):
    s_M = s / 2.0 ** (M - 1)
    return lo - s * (2.0 ** (M - 2) - 1.0) / 2.0 ** (M - 1), s_M


def _half_step_wrong(s, k):
    return s / 2.0 ** (k - 2)


def _composite_dropped_plane(q, planes, M):
    u = np.asarray(q, dtype=np.int64) * (1 << (M - 2))
    for k in range(3, M):          # b_M dropped
        u = u + np.asarray(planes[k - 3], dtype=np.int64) * (1 << (M - k))
    return u


def _pair_table_swapped(cb_log2s, cb_lo_over_s):
    a = np.tile(np.arange(16), 16)             # nibbles swapped
    b = np.repeat(np.arange(16), 16)
    s = np.exp2(cb_log2s.astype(np.float64)[a])
    return cb_lo_over_s.astype(np.float64)[b] * s, s


def _base_digit_truncating(w, lo, s):
    return np.clip(np.floor((np.asarray(w, dtype=np.float64) - lo) / s), 0, 3).astype(np.int64)


_select_post_guard = O.select_post_guard


def _lloyd_median(values, anchored):
    """Moves points to the median of their values instead of the mean."""
    v = np.asarray(values, dtype=np.float64).reshape(-1)
    c = np.linspace(v.min(), v.max(), 16)
    for _ in range(100):
        a = np.argmin(np.abs(v[:, None] - c[None, :]), axis=1)
        for i in range(16):
            if anchored and i in (0, 15):
                continue
            if np.any(a == i):
                c[i] = np.median(v[a == i])
    return c.astype(np.float16)


def _lloyd_unanchored(values, anchored):
    return _lloyd_codebook(values, False)


_lloyd_codebook = O.lloyd_codebook
_decode = O.decode


def _decode_post_as_recorded_value(F, M, rows=None):
    """Takes a post-grid residual as if it were a recorded value (drops the
    two-bit reconstruction from P)."""
    return _decode(dataclasses.replace(F, post=None), M, rows)


def _post_guard_wrong_error(W, W2, held):
    """Scores |w| instead of the two-bit error (the reconstruction dropped)."""
    return _select_post_guard(W, np.zeros_like(W2), held)


def _ratio_guard_second_excluded_wrongly(W, group, T):
    out, inp = W.shape
    A = np.abs(W.astype(np.float64)).reshape(out, inp // group, group)
    j1 = np.argmax(A, axis=2)
    a1 = np.take_along_axis(A, j1[:, :, None], axis=2)[:, :, 0]
    a2 = np.sort(A, axis=2)[:, :, -1]            # compares with the largest itself, not the second
    mask = np.zeros(A.shape, dtype=bool)
    np.put_along_axis(mask, j1[:, :, None], (a1 > T * a2)[:, :, None], axis=2)
    return mask.reshape(out, inp)


_choose_pairs = O.choose_pairs


def _fast_pairs_nibbles_swapped(Vc, group, N, lo_tab, s_tab, empty, mode="search", **kw):
    """The fast rule with the log2(s) index in the low nibble."""
    idx = _choose_pairs(Vc, group, N, lo_tab, s_tab, empty, mode=mode, **kw).astype(np.int64)
    if mode == "fast":
        idx = (idx & 15) * 16 + (idx >> 4)
    return idx.astype(np.uint8)


def _fast_pairs_lo_not_divided(Vc, group, N, lo_tab, s_tab, empty, mode="search", lo0=None, s0=None, **kw):
    """The fast rule matching lo0 itself instead of lo0 / s0 against the lo/s codebook."""
    if mode == "fast":
        return _choose_pairs(Vc, group, N, lo_tab, s_tab, empty, mode=mode, lo0=lo0 * s0, s0=s0, **kw)
    return _choose_pairs(Vc, group, N, lo_tab, s_tab, empty, mode=mode, lo0=lo0, s0=s0, **kw)


@pytest.mark.parametrize("name,mutant,pins", [
    ("choose_pairs", _fast_pairs_nibbles_swapped, ["test_fast_pair_rule_matches_scalar_nearest_entries"]),
    ("choose_pairs", _fast_pairs_lo_not_divided, ["test_fast_pair_rule_matches_scalar_nearest_entries"]),
    ("grid_at", _grid_wrong_sign, ["test_eq9_equals_eq10_all_digit_patterns", "test_figure1_every_prefix_is_a_grid_point"]),
    ("grid_at", _grid_wrong_spacing, ["test_every_precision_is_a_uniform_grid", "test_midpoint_split_is_the_mmse_split"]),
    ("half_step", _half_step_wrong, ["test_figure1_worked_example", "test_sign_planes_equal_nearest_level_rounding"]),
    ("composite_level", _composite_dropped_plane, ["test_eq9_equals_eq10_all_digit_patterns"]),
    ("pair_table", _pair_table_swapped, ["test_gemv_against_scalar_brute_force"]),
    ("base_digit", _base_digit_truncating, ["test_sign_planes_equal_nearest_level_rounding"]),
    ("select_ratio_guard", _ratio_guard_second_excluded_wrongly, ["test_ratio_guard_matches_brute_force"]),
    ("select_post_guard", _post_guard_wrong_error, ["test_post_guard_is_the_row_argmax_of_two_bit_error"]),
    ("lloyd_codebook", _lloyd_median, ["test_lloyd_points_are_the_cluster_means"]),
    ("lloyd_codebook", _lloyd_unanchored, ["test_lloyd_points_are_the_cluster_means"]),
    ("decode", _decode_post_as_recorded_value, ["test_post_entries_reconstruct_w_at_every_precision",
                                                "test_gemv_with_guards_against_scalar_brute_force"]),
])
def test_planted_mistake_is_caught(monkeypatch, name, mutant, pins):
    monkeypatch.setattr(O, name, mutant)
    for pin in pins:
        fn = getattr(P, pin)
        args = (2,) if pin == "test_gemv_against_scalar_brute_force" else ()
        assert _fails(fn, *args), f"{pin} did not catch the mutant of {name}"
