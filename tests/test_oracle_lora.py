"""Pins of the CPU oracle's forward/backward (fp64) against a hand-worked
example, closed forms and exact finite differences (no GPU)."""
import numpy as np

import oracle


def test_hand_example_scaling_and_orientation():
    """waylandz ch.26, 26.2.4: y = W x + (alpha/r) B (A x).
    x = (1, 2), W = [[1, 0], [3, 1]], A = [[1, 1]] (r = 1), B = [[1], [0]],
    alpha = 2: W x = (1, 5), A x = 3, B (A x) = (3, 0), y = (1 + 6, 5) = (7, 5).
    The asymmetric W catches a transposed weight; alpha/r catches a dropped
    scale."""
    X = np.array([[1.0, 2.0]])
    W = np.array([[1.0, 0.0], [3.0, 1.0]])
    A = np.array([[1.0, 1.0]])
    B = np.array([[1.0], [0.0]])
    Y, T = oracle.forward(X, W, A, B, alpha=2.0, r=1)
    assert Y.tolist() == [[7.0, 5.0]]
    assert T.tolist() == [[3.0]]
    # r = 2 with the same update split over two ranks halves the scale
    A2 = np.array([[1.0, 1.0], [0.0, 0.0]])
    B2 = np.array([[1.0, 0.0], [0.0, 0.0]])
    Y2, _ = oracle.forward(X, W, A2, B2, alpha=2.0, r=2)
    assert Y2.tolist() == [[4.0, 5.0]]


def test_hand_example_backward():
    """Same layer, upstream gradient dy = (1, 10):
    dx = W^T dy + s A^T (B^T dy) = (1 + 30, 10) + 2 * (1, 1) * 1 = (33, 12);
    dA = s (B^T dy) x^T = 2 * 1 * (1, 2) = (2, 4); dB = s dy (A x)^T = 2 * 3 * (1, 10)."""
    X = np.array([[1.0, 2.0]])
    W = np.array([[1.0, 0.0], [3.0, 1.0]])
    A = np.array([[1.0, 1.0]])
    B = np.array([[1.0], [0.0]])
    dY = np.array([[1.0, 10.0]])
    dX, dA, dB = oracle.backward(dY, X, W, A, B, alpha=2.0, r=1)
    assert dX.tolist() == [[33.0, 12.0]]
    assert dA.tolist() == [[2.0, 4.0]]
    assert dB.tolist() == [[6.0], [60.0]]


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def test_backward_is_gradient_of_forward():
    """<dY, Y> is linear in each of X, A and B separately, so a unit step in
    one entry changes it by exactly that entry's gradient (up to fp64
    rounding): a central-difference check with no truncation error."""
    rng = np.random.default_rng(0)
    M, N, K, r, alpha = 5, 6, 7, 3, 6.0
    X, W, A, B, dY = _rand(rng, M, K), _rand(rng, N, K), _rand(rng, r, K), _rand(rng, N, r), _rand(rng, M, N)

    def f(X_, A_, B_):
        return float(np.sum(dY * oracle.forward(X_, W, A_, B_, alpha, r)[0]))

    dX, dA, dB = oracle.backward(dY, X, W, A, B, alpha, r)
    for name, P, G in (("X", X, dX), ("A", A, dA), ("B", B, dB)):
        for idx in np.ndindex(P.shape):
            E = np.zeros_like(P)
            E[idx] = 1.0
            args = {"X": X, "A": A, "B": B}
            plus = dict(args, **{name: P + E})
            minus = dict(args, **{name: P - E})
            fd = (f(plus["X"], plus["A"], plus["B"]) - f(minus["X"], minus["A"], minus["B"])) / 2
            if name == "X":
                assert abs(fd - G[idx]) < 1e-9 * (1 + abs(G[idx]))
            else:
                # bilinear in (A, B): still exact for a step in one of them
                assert abs(fd - G[idx]) < 1e-9 * (1 + abs(G[idx]))


def test_zero_b_reduces_to_base_layer():
    """waylandz ch.26, 26.2.3: B starts at zero so B A = 0 and the layer equals
    W at the start; then dA is exactly zero and dB = s dY^T (X A^T)."""
    rng = np.random.default_rng(1)
    M, N, K, r = 4, 8, 16, 2
    X, W, A, dY = _rand(rng, M, K), _rand(rng, N, K), _rand(rng, r, K), _rand(rng, M, N)
    B = np.zeros((N, r))
    Y, _ = oracle.forward(X, W, A, B, 4.0, r)
    assert np.array_equal(Y, X @ W.T)
    dX, dA, dB = oracle.backward(dY, X, W, A, B, 4.0, r)
    assert np.all(dA == 0)
    assert np.array_equal(dX, dY @ W)
    assert np.allclose(dB, 2.0 * dY.T @ (X @ A.T), rtol=1e-14, atol=0)


def test_lora_parameter_counts(golden):
    """ta-paperlens explainer: 4096x4096, r = 16 -> 131,072 trainable numbers;
    waylandz 26.2.1: N=1024, D=512, r=32 -> 49,152."""
    assert oracle.lora_param_count(4096, 4096, 16) == golden["lora_params_4096sq_r16"]["value"]
    assert oracle.lora_param_count(1024, 512, 32) == golden["lora_params_1024x512_r32"]["value"]


def test_rel_err_metric():
    assert oracle.rel_err([1.0, 2.0], [1.0, 2.0]) == 0.0
    assert oracle.rel_err([1.0, 2.5], [1.0, 2.0]) == 0.25
    assert oracle.rel_err([0.0], [0.0]) == 0.0


def test_alpha_scaling_is_linear_and_b_zero_is_the_base_layer():
    """Y(alpha) - Y(0) grows linearly with alpha ([p2] 26.2.4: the update is
    scaled by alpha/r), and B = 0 leaves the base layer X W^T with dA = 0 and
    dB = s dY^T (X A^T)."""
    rng = np.random.default_rng(40)
    M, N, K, r = 6, 10, 12, 4
    X, W, A, B, dY = (rng.standard_normal(s) for s in ((M, K), (N, K), (r, K), (N, r), (M, N)))
    Y0, _ = oracle.forward(X, W, A, B, 0.0, r)
    Y1, _ = oracle.forward(X, W, A, B, 8.0, r)
    Y3, _ = oracle.forward(X, W, A, B, 24.0, r)
    assert np.allclose(Y3 - Y0, 3.0 * (Y1 - Y0), rtol=1e-12, atol=1e-12)
    assert np.allclose(Y0, X @ W.T, rtol=1e-13, atol=1e-13)
    Zb = np.zeros_like(B)
    Yb, _ = oracle.forward(X, W, A, Zb, 8.0, r)
    assert np.array_equal(Yb, X @ W.T + 0.0)
    dX, dA, dB = oracle.backward(dY, X, W, A, Zb, 8.0, r)
    assert not dA.any()
    assert np.allclose(dB, (8.0 / r) * dY.T @ (X @ A.T), rtol=1e-13, atol=1e-13)
    assert np.allclose(dX, dY @ W, rtol=1e-13, atol=1e-13)
