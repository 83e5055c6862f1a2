"""CPU checks of the near-tie validity rules (tests/validity.py): each accepts a true near-tie
and rejects a clearly wrong answer."""
import numpy as np
import pytest

import oracle
import validity


@pytest.fixture(autouse=True)
def _keep_session_log_clean():
    """These checks exercise the rules on made-up cases; their entries leave the session log."""
    before = (validity.NEAR_TIES.copy(), list(validity.LOG))
    yield
    validity.NEAR_TIES.clear()
    validity.NEAR_TIES.update(before[0])
    validity.LOG[:] = before[1]


def test_labels_accept_ties_and_reject_far_labels():
    # two identical centroids: the distances tie exactly, so either label is correct
    x = np.array([[0.5, 0.25], [3.0, 3.0]], dtype=np.float32)
    cent = np.array([[1.0, 1.0], [1.0, 1.0], [3.0, 3.0]], dtype=np.float32)
    assert validity.labels_valid(x, cent, np.array([1, 2]), "tie") == 1
    with pytest.raises(AssertionError):
        validity.labels_valid(x, cent, np.array([2, 2]), "far")     # row 0 is far from centroid 2
    # a gap below the fp32 error bound of the kernel's formula (see the oracle's exactness pin)
    x = np.array([[1.0 + 3 * 2.0 ** -23]], dtype=np.float32)
    cent = np.array([[1.0], [1.0 + 2.0 ** -21]], dtype=np.float32)
    assert oracle.kmeans_assign(x, cent)[0][0] == 1
    assert validity.labels_valid(x, cent, np.array([0]), "fp32 tie") == 1


def test_topk_accepts_boundary_swaps_only():
    score = np.array([[5.0, 3.0, 3.0, 1.0], [0.0, 4.0, 2.0, 1.0], [1.0, 2.0, 3.0, 4.0], [4.0, 3.0, 2.0, 1.0]])
    keep_o = np.array([[1, 1, 0, 0], [1, 1, 0, 0], [0, 0, 1, 1], [1, 0, 0, 1]], dtype=bool)
    keep_g = keep_o.copy()
    keep_g[0] = [1, 0, 1, 0]                   # the k-th and (k+1)-th scores tie: accepted
    assert validity.topk_rows_valid(keep_g, keep_o, score, 2, "tie") == 1
    keep_g = keep_o.copy()
    keep_g[1] = [1, 0, 1, 0]                   # drops score 4 for score 2: rejected
    with pytest.raises(AssertionError):
        validity.topk_rows_valid(keep_g, keep_o, score, 2, "far")


def test_topp_accepts_equal_weights_only():
    w = np.array([[3.0, 2.0, 2.0, 1.0]])
    keep_o = np.array([[1, 1, 0, 0]], dtype=bool)   # top_p 0.6 of 8 -> 4.8 reached by 3 + 2
    assert validity.topp_rows_valid(np.array([[1, 0, 1, 0]], dtype=bool), keep_o, w, 0.6, "tie") == 1
    with pytest.raises(AssertionError):
        validity.topp_rows_valid(np.array([[1, 0, 0, 1]], dtype=bool), keep_o, w, 0.6, "short")
    with pytest.raises(AssertionError):
        validity.topp_rows_valid(np.array([[1, 1, 1, 0]], dtype=bool), keep_o, w, 0.6, "long")


def test_kind_accepts_close_errors_only():
    assert validity.kind_valid(1, 0, [1.0, 1.0 + 1e-5], "close")
    assert not validity.kind_valid(0, 0, [1.0, 2.0], "same")
    with pytest.raises(AssertionError):
        validity.kind_valid(1, 0, [1.0, 1.5], "far")
