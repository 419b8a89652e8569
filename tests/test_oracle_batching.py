"""Pins of the oracle's multi-adapter batch and shared-input projection group
(no GPU): hand-worked examples, reduction to the single-adapter layer, row
permutations, an equivalent single layer of rank P*r, and exact finite
differences of the backward."""
import numpy as np
import pytest

import oracle


def rand(rng, *shape, scale=1.0):
    return rng.standard_normal(shape) * scale


def test_multi_hand_example():
    """Two adapters, two rows, r = 1, alpha = 2 (s = 2), W = [[1, 0], [0, 1]]:
    row 0 = (1, 2) uses adapter 0 (A = [[1, 0]], B = [[1], [0]]): A x = 1,
    y = (1, 2) + 2 (1, 0) = (3, 2); row 1 = (1, 2) uses adapter 1 (A = [[0, 1]],
    B = [[0], [1]]): A x = 2, y = (1, 2) + 2 (0, 2) = (1, 6)."""
    X = np.array([[1.0, 2.0], [1.0, 2.0]])
    W = np.eye(2)
    As = np.array([[[1.0, 0.0]], [[0.0, 1.0]]])
    Bs = np.array([[[1.0], [0.0]], [[0.0], [1.0]]])
    Y = oracle.forward_multi(X, W, As, Bs, [0, 1], alpha=2.0, r=1)
    assert Y.tolist() == [[3.0, 2.0], [1.0, 6.0]]


def test_multi_with_one_adapter_is_the_layer():
    rng = np.random.default_rng(20)
    M, N, K, r, P = 9, 12, 16, 4, 3
    X, W, dY = rand(rng, M, K), rand(rng, N, K), rand(rng, M, N)
    As, Bs = rand(rng, P, r, K), rand(rng, P, N, r)
    for k in range(P):
        ids = np.full(M, k)
        Y, _ = oracle.forward(X, W, As[k], Bs[k], 8.0, r)
        assert np.array_equal(oracle.forward_multi(X, W, As, Bs, ids, 8.0, r), Y)
        dX, dA, dB = oracle.backward(dY, X, W, As[k], Bs[k], 8.0, r)
        gX, gA, gB = oracle.backward_multi(dY, X, W, As, Bs, ids, 8.0, r)
        assert np.array_equal(gX, dX) and np.array_equal(gA[k], dA) and np.array_equal(gB[k], dB)
        others = [j for j in range(P) if j != k]
        assert not gA[others].any() and not gB[others].any()


def test_multi_row_permutation():
    rng = np.random.default_rng(21)
    M, N, K, r, P = 11, 8, 16, 4, 3
    X, W = rand(rng, M, K), rand(rng, N, K)
    As, Bs = rand(rng, P, r, K), rand(rng, P, N, r)
    ids = rng.integers(0, P, M)
    perm = rng.permutation(M)
    Y = oracle.forward_multi(X, W, As, Bs, ids, 8.0, r)
    Yp = oracle.forward_multi(X[perm], W, As, Bs, ids[perm], 8.0, r)
    assert np.array_equal(Yp, Y[perm])


def test_multi_matches_per_row_definition():
    """Against a per-row loop of the formula, written here independently."""
    rng = np.random.default_rng(22)
    M, N, K, r, P = 7, 6, 8, 2, 4
    X, W = rand(rng, M, K), rand(rng, N, K)
    As, Bs = rand(rng, P, r, K), rand(rng, P, N, r)
    ids = rng.integers(0, P, M)
    Y = oracle.forward_multi(X, W, As, Bs, ids, 6.0, r)
    for m in range(M):
        k = ids[m]
        want = W @ X[m] + (6.0 / r) * (Bs[k] @ (As[k] @ X[m]))
        assert np.allclose(Y[m], want, rtol=1e-13, atol=1e-13)


def test_multi_backward_finite_differences():
    """The forward is linear in X, in each A_k and in each B_k, so a finite
    difference along any direction equals the directional derivative up to
    fp64 rounding."""
    rng = np.random.default_rng(23)
    M, N, K, r, P = 10, 6, 8, 2, 3
    X, W, dY = rand(rng, M, K), rand(rng, N, K), rand(rng, M, N)
    As, Bs = rand(rng, P, r, K), rand(rng, P, N, r)
    ids = rng.integers(0, P, M)
    ids[:P] = np.arange(P)
    f = lambda X_, As_, Bs_: np.sum(dY * oracle.forward_multi(X_, W, As_, Bs_, ids, 4.0, r))  # noqa: E731
    dX, dAs, dBs = oracle.backward_multi(dY, X, W, As, Bs, ids, 4.0, r)
    E = rand(rng, M, K)
    assert np.isclose(f(X + E, As, Bs) - f(X, As, Bs), np.sum(dX * E), rtol=1e-10)
    EA = rand(rng, P, r, K)
    assert np.isclose(f(X, As + EA, Bs) - f(X, As, Bs), np.sum(dAs * EA), rtol=1e-10)
    EB = rand(rng, P, N, r)
    assert np.isclose(f(X, As, Bs + EB) - f(X, As, Bs), np.sum(dBs * EB), rtol=1e-10)


def test_multi_rejects_bad_ids():
    X, W = np.zeros((2, 4)), np.zeros((4, 4))
    As, Bs = np.zeros((2, 1, 4)), np.zeros((2, 4, 1))
    with pytest.raises(ValueError):
        oracle.forward_multi(X, W, As, Bs, [0, 2], 2.0, 1)
    with pytest.raises(ValueError):
        oracle.forward_multi(X, W, As, Bs, [-1, 0], 2.0, 1)


def test_group_is_one_layer_of_rank_p_r():
    """Gate and up (or q, k, v) side by side are one layer: the weights stacked
    along N, the down-projections stacked along the rank ([A_1; A_2], rank
    P*r) and the up-projections block-diagonal, with alpha scaled by P so that
    the scale alpha/r is unchanged."""
    rng = np.random.default_rng(24)
    M, K, r = 5, 16, 4
    Ns = [8, 12, 8]
    X = rand(rng, M, K)
    Ws = [rand(rng, n, K) for n in Ns]
    As = [rand(rng, r, K) for _ in Ns]
    Bs = [rand(rng, n, r) for n in Ns]
    Y = oracle.forward_group(X, Ws, As, Bs, 16.0, r)
    P = len(Ns)
    Bbd = np.zeros((sum(Ns), P * r))
    row = 0
    for i, n in enumerate(Ns):
        Bbd[row:row + n, i * r:(i + 1) * r] = Bs[i]
        row += n
    Y1, _ = oracle.forward(X, np.concatenate(Ws), np.concatenate(As), Bbd, 16.0 * P, P * r)
    assert np.allclose(Y, Y1, rtol=1e-13, atol=1e-13)
    assert Y.shape == (M, sum(Ns))
