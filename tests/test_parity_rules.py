"""The tie rule used by the parity tests, checked on constructed selections (CPU)."""
import numpy as np

from oracle import bsa_oracle as O
from tests.parity import selection_verdict


def _sel(S, p, k_max, n_sink=1, n_local=1):
    return O.select_decode(np.asarray(S, dtype=np.float64), n_sink, n_local, p, k_max)


def test_exact_match():
    S = [9, 5, 4, 3, 2, 1, 9]
    sel = _sel(S, 1.0, 2)
    assert selection_verdict(sel, sel.kept, 1.0) == "exact"


def test_equal_mass_swap_is_tie():
    # blocks 2 and 3 have masses within 1e-7 relative; the cap cuts between them
    S = [9, 5, 4.0, 4.0 - 1e-8, 1, 1, 9]
    sel = _sel(S, 1.0, 2)
    assert sel.kept == [0, 1, 2, 6]
    assert selection_verdict(sel, [0, 1, 3, 6], 1.0) == "tie"


def test_clear_swap_is_mismatch():
    S = [9, 5, 4.0, 3.0, 1, 1, 9]
    sel = _sel(S, 1.0, 2)
    assert selection_verdict(sel, [0, 1, 3, 6], 1.0).startswith("mismatch")


def test_count_off_by_one_needs_cumulative_at_p():
    # two equal candidates: cumulative after the first is exactly 0.5
    S = [9, 1.0, 1.0, 9]
    sel = _sel(S, 0.5, 8)
    assert sel.k == 1
    assert selection_verdict(sel, [0, 1, 2, 3], 0.5) == "tie"       # cum 0.5 == p
    sel2 = _sel(S, 0.3, 8)
    assert sel2.k == 1
    assert selection_verdict(sel2, [0, 1, 2, 3], 0.3).startswith("mismatch")


def test_missing_reserved_is_mismatch():
    S = [9, 5, 4, 3, 2, 1, 9]
    sel = _sel(S, 1.0, 2)
    assert selection_verdict(sel, [1, 2, 6], 1.0).startswith("mismatch")
