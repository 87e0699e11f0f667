"""The parity check's acceptance rule for tie rows (tests/gpu_util.py), on the CPU:
another valid answer on a tie row passes, a wrong one (not a ranked prefix, short of
p, not minimal, a floor from the wrong end of the ranking) fails."""
import numpy as np

import oracle as O
from gpu_util import valid_tie_topk, valid_tie_topp


def _row(P):
    L = np.log(np.asarray(P, dtype=np.float64))
    return L, O.row_softmax(L[None])[0]


def _mask(nb, ids):
    m = np.zeros(nb, dtype=np.uint8)
    m[list(ids)] = 1
    return m


def test_mass_tie_accepts_both_cuts_and_rejects_wrong_sets():
    L, P = _row([0.5, 0.3, 0.2])          # cumulative 0.5, 0.8, 1.0: p = 0.8 sits on a cut
    p = 0.8
    assert abs(P[0] + P[1] - p) < 1e-12
    assert valid_tie_topp(L, P, _mask(3, [0, 1]), p)
    assert valid_tie_topp(L, P, _mask(3, [0, 1, 2]), p)   # one block past the cut: mass within tol
    assert not valid_tie_topp(L, P, _mask(3, [0]), p)       # short of p
    assert not valid_tie_topp(L, P, _mask(3, [0, 2]), p)    # not a ranked prefix
    assert not valid_tie_topp(L, P, _mask(3, [1, 2]), p)    # skips the best block
    assert not valid_tie_topp(L, P, _mask(3, []), p)


def test_non_minimal_set_is_rejected_away_from_the_band():
    L, P = _row([0.6, 0.25, 0.1, 0.05])   # p = 0.85 is reached at 2 blocks exactly
    assert valid_tie_topp(L, P, _mask(4, [0, 1]), 0.85)
    assert valid_tie_topp(L, P, _mask(4, [0, 1, 2]), 0.85)      # 3rd block: dropping it leaves 0.85 < p + tol
    assert not valid_tie_topp(L, P, _mask(4, [0, 1, 2, 3]), 0.85)   # dropping the 4th still leaves 0.95


def test_keep_all_is_valid_when_the_total_sits_at_p():
    L = np.zeros(4)
    P = np.full(4, 0.25 - 1e-7)            # total mass a hair below 1 (rounding)
    assert valid_tie_topp(L, P, _mask(4, range(4)), 1.0 - 1e-6)


def test_near_equal_logits_may_swap_at_the_cut():
    L = np.array([2.0, 1.0, 1.0 + 3e-6, -1.0])
    P = O.row_softmax(L[None])[0]
    p = float(P[0] + P[2]) - 1e-9          # oracle: {0, 2}; {0, 1} differs only by the near-tie
    assert valid_tie_topp(L, P, _mask(4, [0, 2]), p)
    assert valid_tie_topp(L, P, _mask(4, [0, 1]), p)
    assert not valid_tie_topp(L, P, _mask(4, [0, 3]), p)


def test_floor_validity():
    L = np.array([1.0, 3.0, 3.0 + 1e-7, 0.5])
    assert valid_tie_topk(L, [2], 1)
    assert valid_tie_topk(L, [1], 1)                 # within the tie band of the best
    assert not valid_tie_topk(L, [0], 1)
    assert valid_tie_topk(L, [1, 2], 2)
    assert not valid_tie_topk(L, [2, 1], 2)          # not ascending
    assert not valid_tie_topk(L, [0, 3], 2)          # the floor from the wrong end
    assert not valid_tie_topk(L, [1, 1], 2)
    assert not valid_tie_topk(L, [1], 2)             # wrong size
