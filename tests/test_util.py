"""The list comparison the GPU parity tests use (CPU): near-ties of the k-th score, and
padded blocks forced into every list."""
import numpy as np

from tests._util import TIE_REL_TOL, rows_agree_up_to_ties


def test_equal_lists_agree():
    assert rows_agree_up_to_ties([1, 3, 5], [1, 3, 5], np.arange(8.0), 3)


def test_a_swap_at_the_kth_score_is_a_tie():
    s = np.array([0.9, 0.5, 0.2, 0.2 * (1 + 0.5 * TIE_REL_TOL), 0.1])
    # the k-th (k = 3) score is 0.2*(1+eps); blocks 2 and 3 are within the tie tolerance
    assert rows_agree_up_to_ties([0, 1, 2], [0, 1, 3], s, 3)


def test_a_swap_away_from_the_kth_score_is_not():
    s = np.array([0.9, 0.5, 0.3, 0.2, 0.1])
    assert not rows_agree_up_to_ties([0, 1, 4], [0, 1, 2], s, 3)


def test_forced_blocks_must_be_in_both_lists():
    s = np.array([0.1, 0.9, 0.8, 0.7, 0.0])
    # block 4 is padded: forced in, whatever its score
    assert rows_agree_up_to_ties([1, 2, 4], [1, 2, 4], s, 3, forced=[4])
    assert not rows_agree_up_to_ties([1, 2, 3], [1, 2, 4], s, 3, forced=[4])


def test_forced_blocks_leave_k_minus_forced_free_places():
    # k = 3 with one forced block: the threshold is the 2nd largest free score (0.8), so a
    # swap of block 2 (0.8) and block 3 (0.8 * (1 + eps)) is a tie, but not of 1 and 3
    eps = 0.5 * TIE_REL_TOL
    s = np.array([0.1, 0.9, 0.8, 0.8 * (1 + eps), 0.0])
    assert rows_agree_up_to_ties([1, 2, 4], [1, 3, 4], s, 3, forced=[4])
    s2 = np.array([0.1, 0.9, 0.8, 0.5, 0.0])
    assert not rows_agree_up_to_ties([3, 2, 4], [1, 2, 4], s2, 3, forced=[4])
