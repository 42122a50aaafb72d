"""Pins of the retrieval oracle (oracle.retrieval) against facts that do not
come from the oracle itself: pure-Python loops on tiny inputs, closed forms,
tie order, and invariances a wrong index or sign would break."""
import numpy as np
import pytest

from oracle import retrieval as R


def _brute(E, H, K):
    """Explicit loops: every (user, item) dot product, then repeatedly take
    the best remaining item (highest score, then lowest id)."""
    out_v, out_i = [], []
    for h in H:
        s = []
        for m, e in enumerate(E):
            acc = 0.0
            for k in range(len(h)):
                acc += float(e[k]) * float(h[k])
            s.append(acc)
        taken, vals, ids = set(), [], []
        for _ in range(K):
            best = None
            for m in range(len(s)):
                if m in taken:
                    continue
                if best is None or s[m] > s[best]:
                    best = m
            taken.add(best)
            vals.append(s[best])
            ids.append(best)
        out_v.append(vals)
        out_i.append(ids)
    return np.array(out_v), np.array(out_i)


def test_matches_brute_force_loops():
    rng = np.random.default_rng(0)
    for (U, M, d, K) in [(1, 5, 3, 1), (2, 9, 4, 3), (3, 17, 5, 17), (4, 30, 8, 7)]:
        E = rng.normal(size=(M, d))
        H = rng.normal(size=(U, d))
        v, i = R.retrieve(E, H, K)
        bv, bi = _brute(E, H, K)
        np.testing.assert_array_equal(i, bi)
        np.testing.assert_allclose(v, bv, rtol=0, atol=1e-12)


def test_ties_go_to_the_smaller_id():
    # items 1, 3 and 6 are the same vector; 4 and 5 the same smaller one
    E = np.array([[0, 0], [2, 1], [0, 1], [2, 1], [1, 1], [1, 1], [2, 1], [-1, 0]], float)
    H = np.array([[1.0, 1.0], [-1.0, -1.0]])
    v, i = R.retrieve(E, H, 6)
    assert i[0].tolist() == [1, 3, 6, 4, 5, 2]
    assert v[0].tolist() == [3, 3, 3, 2, 2, 1]
    assert i[1].tolist() == [7, 0, 2, 4, 5, 1]


def test_identity_catalog_returns_the_largest_components():
    # E = I: the score of item m is the m-th component of h
    d = 12
    h = np.array([[0.5, -2, 7, 7, 1, 0, 3, -1, 7, 2, 0.25, 4]])
    v, i = R.retrieve(np.eye(d), h, 5)
    assert i[0].tolist() == [2, 3, 8, 11, 6]
    assert v[0].tolist() == [7, 7, 7, 4, 3]


def test_item_permutation_permutes_ids_and_scale_keeps_order():
    rng = np.random.default_rng(3)
    E = rng.integers(-3, 4, size=(40, 6)).astype(float)
    H = rng.integers(-3, 4, size=(3, 6)).astype(float)
    v, i = R.retrieve(E, H, 10)
    perm = rng.permutation(40)
    E2 = E[perm]                      # item m of E2 is item perm[m] of E
    S2 = R.scores(E2, H)
    np.testing.assert_array_equal(S2, R.scores(E, H)[:, perm])
    v3, i3 = R.retrieve(E, 2.5 * H, 10)
    np.testing.assert_array_equal(i3, i)
    np.testing.assert_array_equal(v3, 2.5 * v)


def test_user_vectors_take_the_last_row_and_zero_for_empty_users():
    Y = np.arange(20, dtype=float).reshape(10, 2)
    H = R.user_vectors(Y, [0, 3, 3, 10])
    np.testing.assert_array_equal(H, [[4, 5], [0, 0], [18, 19]])
    # an empty user scores every item 0: the first K ids
    v, i = R.retrieve(np.ones((6, 2)), H[1:2], 4)
    assert i[0].tolist() == [0, 1, 2, 3] and not v.any()


def test_k_bounds():
    with pytest.raises(ValueError):
        R.topk(np.zeros((1, 3)), 4)
    with pytest.raises(ValueError):
        R.topk(np.zeros((1, 3)), 0)


def test_planted_mistakes_are_caught():
    """Mistakes a retrieval implementation could make (ascending order, ties
    by larger id, a transposed catalog) give different answers on pin inputs."""
    E = np.array([[0, 0], [2, 1], [0, 1], [2, 1], [1, 1], [1, 1], [2, 1], [-1, 0]], float)
    H = np.array([[1.0, 1.0]])
    _, good = R.retrieve(E, H, 6)
    S = R.scores(E, H)[0]
    asc = np.lexsort((np.arange(8), S))[:6]
    big_id = np.lexsort((-np.arange(8), -S))[:6]
    assert not np.array_equal(asc, good[0])
    assert not np.array_equal(big_id, good[0])
    # square, non-symmetric catalog: item m's score is row m of E times h,
    # not column m
    Es = np.array([[1.0, 4.0, 0.0], [0.0, 1.0, 0.0], [2.0, 0.0, 3.0]])
    h = np.array([[1.0, 2.0, 3.0]])
    assert R.scores(Es, h)[0].tolist() == [9.0, 2.0, 11.0]
    assert (Es.T @ h[0]).tolist() == [7.0, 6.0, 9.0]
    assert R.retrieve(Es, h, 1)[1][0, 0] == 2
