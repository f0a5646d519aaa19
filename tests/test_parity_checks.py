"""The selection check used by the GPU parity tests rejects what it must
(runs on CPU): a selection from independently rounded scores may differ from
the oracle's top-k only among positions tied within 1e-3 of the k-th score."""
import numpy as np

from parity import selection_agrees_outside_tie_band


def _scores():
    s = np.linspace(1.0, 2.0, 1000)
    s[500:510] = 1.5          # ten positions tied at what becomes the k-th score
    return s


def test_exact_top_k_is_accepted():
    s = _scores()
    k = 300
    top = np.argsort(-s, kind="stable")[:k]
    assert selection_agrees_outside_tie_band(top, s, k)


def test_a_swap_inside_the_tie_band_is_accepted():
    s = _scores()
    k = int((s > 1.5).sum()) + 5          # five of the ten tied positions are taken
    base = np.flatnonzero(s > 1.5)
    assert selection_agrees_outside_tie_band(np.concatenate([base, [500, 502, 504, 506, 508]]), s, k)
    assert selection_agrees_outside_tie_band(np.concatenate([base, [501, 503, 505, 507, 509]]), s, k)


def test_a_swap_outside_the_band_is_rejected():
    s = _scores()
    k = int((s > 1.5).sum()) + 5
    base = np.flatnonzero(s > 1.5)
    sel = np.concatenate([base, [500, 502, 504, 506, 508]])
    sel[0] = 10                           # a clearly lower score instead of a clearly higher one
    assert not selection_agrees_outside_tie_band(sel, s, k)


def test_duplicates_and_short_selections_are_rejected():
    s = _scores()
    top = np.argsort(-s, kind="stable")[:100]
    assert not selection_agrees_outside_tie_band(np.concatenate([top[:-1], top[:1]]), s, 100)
    assert not selection_agrees_outside_tie_band(top[:-1], s, 100)
    assert selection_agrees_outside_tie_band(np.arange(50), s[:50], 100)     # fewer keys than k: all of them
    assert not selection_agrees_outside_tie_band(np.arange(49), s[:50], 100)
