"""Pins of the oracle's storage without double quantisation and of the adapter
merge (no GPU). Independent of the oracle's own code: the glossary's printed
MSE, torch's bf16 cast, exact-rational brute force over every bf16 value, a
hand-worked merge, and the forward pass of the layer."""
import bisect
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle


# ------------------------------------------- no double quantisation --------

def test_nodq_reproduces_printed_mse(golden):
    """The glossary's snippet keeps one fp32 absmax per row of 64 and restores
    in fp32: randn(4096, 64) * 0.02 with seed 0 gives NF4 MSE 3.395e-06. With
    K = 64 every flat block of the storage without double quantisation is one
    such row, so its quantiser and fp32 restore must print the same number."""
    torch.manual_seed(0)
    w = (torch.randn(4096, 64) * 0.02).numpy()
    q = oracle.quantize_nf4_nodq(w)
    assert np.array_equal(q["absmax"], np.abs(w).max(axis=1))
    restored = oracle.dequant_f32_nodq(q["codes"], q["absmax"], 4096, 64)
    mse = float(np.mean((restored.astype(np.float64) - w) ** 2))
    assert float(f"{mse:.3e}") == golden["nf4_mse"]["value"]


def test_nodq_bf16_is_torch_cast_of_fp32_restore():
    rng = np.random.default_rng(11)
    W = (rng.standard_normal((48, 192)) * 0.02).astype(np.float32)
    W[3, 64:128] = 0.0
    q = oracle.quantize_nf4_nodq(W)
    f = oracle.dequant_f32_nodq(q["codes"], q["absmax"], 48, 192)
    bits = oracle.dequant_bf16_bits_nodq(q["codes"], q["absmax"], 48, 192)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, ref)
    # the zero block restores to +0 everywhere (code 7 times c = 0)
    assert np.all(bits[3, 64:128] == 0)


def test_nodq_codes_equal_double_quant_codes_and_storage(golden):
    """Double quantisation changes only the constants, never the codes; the
    storage is 4 + 32/64 bits per weight."""
    rng = np.random.default_rng(12)
    W = (rng.standard_normal((64, 512)) * 0.02).astype(np.float32)
    a = oracle.quantize_nf4_nodq(W)
    b = oracle.quantize_nf4(W)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.array_equal(a["absmax"], b["absmax"])
    n = 64 * 512
    assert 8 * (a["codes"].nbytes + a["absmax"].nbytes) / n == golden["bits_per_param_no_dq"]["value"]


# ----------------------------------------------------------- fp64 -> bf16 --

def _bf16_values():
    """Every non-negative finite bf16 value as an exact Fraction, with its bit
    pattern, in increasing order, then +inf's pattern at 2^128 (the first
    value past the largest finite one, which overflow rounds to)."""
    vals, pats = [], []
    for p in range(0x7F80):
        u = np.array([p << 16], np.uint32).view(np.float32)[0]
        vals.append(Fraction(float(u)))
        pats.append(p)
    vals.append(Fraction(2) ** 128)
    pats.append(0x7F80)
    return vals, pats


_BF16 = None


def _brute_bf16(x) -> int:
    """Nearest bf16 to x (a float or an exact Fraction) by exact comparison,
    ties to the even pattern."""
    global _BF16
    if _BF16 is None:
        _BF16 = _bf16_values()
    vals, pats = _BF16
    if isinstance(x, Fraction):
        a, sign = abs(x), (0x8000 if x < 0 else 0)
    else:
        a, sign = Fraction(abs(x)), (0x8000 if np.signbit(x) else 0)
    if a >= vals[-1]:
        return sign | 0x7F80
    i = bisect.bisect_left(vals, a)
    if vals[i] == a:
        return sign | pats[i]
    lo, hi = i - 1, i
    dl, dh = a - vals[lo], vals[hi] - a
    if dl < dh:
        return sign | pats[lo]
    if dh < dl:
        return sign | pats[hi]
    return sign | (pats[lo] if pats[lo] % 2 == 0 else pats[hi])


def test_f64_to_bf16_brute_force():
    rng = np.random.default_rng(13)
    xs = list(rng.standard_normal(400) * np.exp2(rng.integers(-140, 128, 400)))
    # exact ties between neighbours and the doubles just beside them
    for p in (0x3F80, 0x3F81, 0x0001, 0x0080, 0x7F7E, 0x7F7F, 0x4049, 0x2000):
        v0 = float(np.array([p << 16], np.uint32).view(np.float32)[0])
        v1 = float(np.array([(p + 1) << 16], np.uint32).view(np.float32)[0]) if p < 0x7F7F else 2.0 ** 128
        mid = (v0 + v1) / 2
        xs += [mid, np.nextafter(mid, 0.0), np.nextafter(mid, np.inf), -mid]
    xs += [0.0, -0.0, 2.0 ** -134, 2.0 ** -133, 3 * 2.0 ** -134, 1e300, -1e300]
    got = oracle.f64_to_bf16_bits(np.array(xs))
    want = np.array([_brute_bf16(float(x)) for x in xs], np.uint16)
    assert np.array_equal(got, want)


def test_f64_to_bf16_of_fp32_values_matches_torch_cast():
    """On values exactly representable in fp32 there is no double rounding, so
    the one-step rounding must equal torch's fp32 -> bf16 cast."""
    rng = np.random.default_rng(14)
    x = (rng.standard_normal(5000) * np.exp2(rng.integers(-120, 120, 5000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f64_to_bf16_bits(x.astype(np.float64)), ref)


# ------------------------------------------------------------ adapter merge --

def test_merge_hand_example():
    """W = [[1, 2], [3, 4]], B = [[1], [0]] (N x r), A = [[0.5, -1]] (r x K),
    alpha = 2, r = 1: s = 2, s B A = [[1, -2], [0, 0]], W + s B A =
    [[2, 0], [3, 4]]. An A B product, a B^T or a dropped scale gives another
    matrix."""
    W = np.array([[1.0, 2.0], [3.0, 4.0]])
    B = np.array([[1.0], [0.0]])
    A = np.array([[0.5, -1.0]])
    assert oracle.merge_lora(W, A, B, alpha=2.0, r=1).tolist() == [[2.0, 0.0], [3.0, 4.0]]


def test_merge_agrees_with_the_layer_forward():
    """The merged weight must give the layer's output with no adapter:
    X W_merged^T = X What^T + s (X A^T) B^T for every X ([p2] 26.2.2, zero
    inference overhead after the merge). The forward pass is written
    independently of the merge."""
    rng = np.random.default_rng(15)
    N, K, r, M = 96, 128, 16, 7
    What = oracle.bf16_bits_to_f64(oracle.f64_to_bf16_bits(rng.standard_normal((N, K)) * 0.02))
    A = rng.standard_normal((r, K)) * np.sqrt(2 / r)
    B = rng.standard_normal((N, r)) * 0.01
    X = rng.standard_normal((M, K))
    Wm = oracle.merge_lora(What, A, B, alpha=32.0, r=r)
    Y, _ = oracle.forward(X, What, A, B, alpha=32.0, r=r)
    Ym, _ = oracle.forward(X, Wm, A, np.zeros_like(B), alpha=32.0, r=r)
    assert np.max(np.abs(Ym - Y)) <= 1e-12 * np.max(np.abs(Y))


def test_merge_with_zero_update_is_the_dequantised_weight():
    rng = np.random.default_rng(16)
    W = (rng.standard_normal((32, 256)) * 0.02).astype(np.float32)
    q = oracle.quantize_nf4(W)
    bits = oracle.dequant_bf16_bits(q["codes"], q["qabsmax"], q["s2"], q["mean"], 32, 256)
    What = oracle.bf16_bits_to_f64(bits)
    A = rng.standard_normal((8, 256))
    B = rng.standard_normal((32, 8))
    assert np.array_equal(oracle.merge_lora_bf16_bits(What, A, np.zeros_like(B), 16.0, 8), bits)
    assert np.array_equal(oracle.merge_lora_bf16_bits(What, A, B, 0.0, 8), bits)


@pytest.mark.parametrize("seed", [0, 1])
def test_merge_rounding_brute_force(seed):
    """Each merged entry is the exact W + s B A (Fractions) rounded once."""
    rng = np.random.default_rng(17 + seed)
    N, K, r = 4, 6, 8
    What = oracle.bf16_bits_to_f64(oracle.f64_to_bf16_bits(rng.standard_normal((N, K)) * 0.02))
    A = oracle.bf16_bits_to_f64(oracle.f64_to_bf16_bits(rng.standard_normal((r, K))))
    B = oracle.bf16_bits_to_f64(oracle.f64_to_bf16_bits(rng.standard_normal((N, r)) * 0.01))
    got = oracle.merge_lora_bf16_bits(What, A, B, alpha=16.0, r=r)
    s = Fraction(16, r)
    for n in range(N):
        for k in range(K):
            exact = Fraction(What[n, k]) + s * sum(Fraction(B[n, j]) * Fraction(A[j, k]) for j in range(r))
            assert got[n, k] == _brute_bf16(exact), (n, k)


def test_requantised_merge_loses_the_update():
    """The explainer's 落とし穴: an adapter update added to the 4-bit weight and
    quantised again is mostly lost, so the merge goes to 16 bits. With an
    update of 5 % of the weights' rms, the bf16 merge keeps it to within 10 %,
    while quantising the merged weight to NF4 again leaves an error as large as
    the update itself."""
    rng = np.random.default_rng(30)
    N, K, r = 256, 512, 16
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    z = oracle.quantize_nf4(W)
    What = oracle.bf16_bits_to_f64(oracle.dequant_bf16_bits(z["codes"], z["qabsmax"], z["s2"], z["mean"], N, K))
    A = rng.standard_normal((r, K)) * np.sqrt(2 / r)
    B = rng.standard_normal((N, r))
    B *= 0.05 * 0.02 / np.sqrt(np.mean((B @ A) ** 2))  # alpha = r: s = 1
    update = oracle.merge_lora(What, A, B, float(r), r) - What
    Wm = oracle.bf16_bits_to_f64(oracle.merge_lora_bf16_bits(What, A, B, float(r), r))
    z2 = oracle.quantize_nf4(Wm.astype(np.float32))
    Wrq = oracle.bf16_bits_to_f64(oracle.dequant_bf16_bits(z2["codes"], z2["qabsmax"], z2["s2"], z2["mean"], N, K))
    err16 = np.linalg.norm(Wm - What - update) / np.linalg.norm(update)
    err4 = np.linalg.norm(Wrq - What - update) / np.linalg.norm(update)
    assert err16 < 0.1
    assert err4 > 0.9
