"""Pins of the CPU oracle's quantisation half against what the pages and the
mathematics fix (no GPU). Every check here is independent of the oracle's own
code path: printed numbers, the stdlib inverse normal CDF, exact-arithmetic
brute force, closed forms and invariants."""
import math
import statistics
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle


def f32(x):
    return np.float32(x)


def next_up(x):
    return np.nextafter(np.float32(x), np.float32(np.inf))


def next_down(x):
    return np.nextafter(np.float32(x), np.float32(-np.inf))


# ------------------------------------------------------------------ levels --

def test_levels_match_stdlib_normal_quantiles():
    """NF4 levels (QLoRA glossary, NF4 snippet): quantiles of N(0,1) at
    linspace(0.9677083, 0.5, 9)[:-1] and -quantiles at linspace(.., 8)[:-1],
    plus zero, sorted, divided by the max. Python's statistics.NormalDist is an
    independent inverse-CDF implementation."""
    nd = statistics.NormalDist()
    p0 = 0.9677083
    v = [nd.inv_cdf(p0 - k * ((p0 - 0.5) / 8)) for k in range(8)]
    v += [-nd.inv_cdf(p0 - k * ((p0 - 0.5) / 7)) for k in range(7)]
    v = sorted(v + [0.0])
    ref = np.array([x / v[-1] for x in v])
    l64, l32 = oracle.nf4_levels()
    assert np.max(np.abs(l64 - ref)) < 1e-14
    ulp = np.spacing(np.abs(ref).astype(np.float32))
    assert np.all(np.abs(l32.astype(np.float64) - ref) <= ulp)


def test_levels_invariants():
    """ta-paperlens explainer, NF4: zero is exact and the ends are exactly -1
    and +1; the snippet gives 7 negative and 8 positive levels."""
    _, L = oracle.nf4_levels()
    assert L.shape == (16,)
    assert np.all(np.diff(L) > 0)
    assert L[0] == -1.0 and L[7] == 0.0 and L[15] == 1.0
    assert np.sum(L < 0) == 7 and np.sum(L > 0) == 8
    # denser near zero than near the ends
    gaps = np.diff(L.astype(np.float64))
    assert gaps[7] < gaps[0] and gaps[7] < gaps[14]


def test_levels_close_to_torch_fp32_construction():
    """The glossary builds the levels in torch fp32; our fp64-then-round reading
    must agree with that to a few fp32 ulps."""
    normal = torch.distributions.Normal(0.0, 1.0)
    pos = normal.icdf(torch.linspace(0.9677083, 0.5, 9)[:-1])
    neg = -normal.icdf(torch.linspace(0.9677083, 0.5, 8)[:-1])
    t = torch.cat([neg, torch.zeros(1), pos]).sort().values
    t = (t / t.max()).numpy()
    _, L = oracle.nf4_levels()
    ulp = np.spacing(np.maximum(np.abs(L), np.float32(1e-30)))
    assert np.all(np.abs(t - L) <= 8 * ulp)


def test_icdf_closed_forms():
    assert abs(oracle.normal_icdf(0.5)) < 1e-15
    # symmetric, and Phi(1.959963984540054) = 0.975
    assert abs(oracle.normal_icdf(0.975) - 1.959963984540054) < 1e-13
    assert abs(oracle.normal_icdf(0.25) + oracle.normal_icdf(0.75)) < 1e-15


# -------------------------------------------------------------- midpoints --

def _brute_nearest(v, L):
    """argmin_k |v - L[k]| in exact rational arithmetic, first index on ties."""
    fv = Fraction(float(v))
    d = [abs(fv - Fraction(float(x))) for x in L]
    m = min(d)
    return d.index(m)


def test_midpoints_bracket_exact_midpoint():
    _, L = oracle.nf4_levels()
    M = oracle.midpoints(L)
    for k in range(15):
        exact = (Fraction(float(L[k])) + Fraction(float(L[k + 1]))) / 2
        assert Fraction(float(M[k])) <= exact < Fraction(float(next_up(M[k])))


def _encode_values(vals, L=None):
    """Encode a list of v in [-1, 1] as one block whose absmax is exactly 1."""
    vals = list(vals)
    codes = []
    for i in range(0, len(vals), 63):
        chunk = vals[i:i + 63]
        blk = np.zeros(64, np.float32)
        blk[0] = 1.0
        blk[1:1 + len(chunk)] = chunk
        _, c = oracle.encode_blocks(blk, 64, L)
        assert c[0] == (15 if L is None else len(L) - 1)
        codes += list(c[1:1 + len(chunk)])
    return codes


def test_encode_at_every_threshold_matches_brute_force():
    """Nearest level in exact arithmetic, at each decision threshold and its
    fp32 neighbours (QLoRA glossary snippet: argmin over |x/absmax - level|)."""
    _, L = oracle.nf4_levels()
    M = oracle.midpoints(L)
    vals = []
    for m in M:
        vals += [m, next_up(m), next_down(m), next_up(next_up(m)), next_down(next_down(m))]
    vals += list(L) + [next_up(x) for x in L[:-1]] + [next_down(x) for x in L[1:]]
    vals += [np.float32(0.0), np.float32(-0.0), np.float32(1e-40), np.float32(-1e-40)]
    codes = _encode_values(vals)
    for v, c in zip(vals, codes):
        assert c == _brute_nearest(v, L), (v, c)


def test_encode_random_blocks_match_brute_force():
    _, L = oracle.nf4_levels()
    rng = np.random.default_rng(7)
    w = (rng.standard_normal((40, 64)) * 0.02).astype(np.float32)
    w[3] *= 1e-38  # subnormal-range block
    w[5, 10] = 5.0  # outlier
    absmax, codes = oracle.encode_blocks(w)
    codes = codes.reshape(40, 64)
    for b in range(40):
        c = np.float32(np.max(np.abs(w[b])))
        assert absmax[b] == c
        v = (w[b] / c).astype(np.float32)  # one IEEE fp32 division each
        for i in range(64):
            assert codes[b, i] == _brute_nearest(v[i], L)


def test_encode_special_blocks():
    """Zero block -> all zero-level (index 7); one nonzero -> 15 or 0, the rest
    7; the absmax element always lands on an end (+-1 exactly)."""
    z = np.zeros(64, np.float32)
    a, c = oracle.encode_blocks(z)
    assert a[0] == 0 and np.all(c == 7)
    one = np.zeros(64, np.float32)
    one[17] = -0.3
    a, c = oracle.encode_blocks(one)
    assert a[0] == np.float32(0.3) and c[17] == 0 and np.all(np.delete(c, 17) == 7)
    neg0 = np.full(64, -0.0, np.float32)
    _, c = oracle.encode_blocks(neg0)
    assert np.all(c == 7)
    rng = np.random.default_rng(3)
    w = rng.standard_normal((50, 64)).astype(np.float32)
    _, c = oracle.encode_blocks(w)
    c = c.reshape(50, 64)
    idx = np.argmax(np.abs(w), axis=1)
    ends = c[np.arange(50), idx]
    assert np.all((ends == 0) | (ends == 15))


def test_pack_nibble_order():
    """Reading of the two-codes-per-byte layout: element 2j high nibble."""
    codes = np.array([1, 2, 3, 4, 15, 0, 7, 9], np.uint8)
    p = oracle.pack_nibbles(codes)
    assert list(p) == [0x12, 0x34, 0xF0, 0x79]
    assert list(oracle.unpack_nibbles(p)) == list(codes)


def test_printed_mse_nf4_vs_int4(golden):
    """The glossary's printed result: NF4 MSE 3.395e-06 vs uniform 4.053e-06 on
    torch.manual_seed(0), randn(4096, 64) * 0.02, one absmax per 64, no double
    quantisation, fp32 restore. The input tensor is drawn here with torch; all
    quantisation arithmetic is the oracle's."""
    torch.manual_seed(0)
    w = (torch.randn(4096, 64) * 0.02).numpy()
    _, nf4 = oracle.nf4_levels()
    int4 = torch.linspace(-1, 1, 16).numpy()
    out = {}
    for name, lev, zc in (("nf4", nf4, 7), ("int4", int4, 0)):
        absmax, codes = oracle.encode_blocks(w, 64, lev, zero_code=zc)
        restored = lev[codes.reshape(4096, 64)] * absmax[:, None]  # fp32 products
        out[name] = float(np.mean((restored.astype(np.float64) - w) ** 2))
    for name in ("nf4", "int4"):
        want = golden[f"{name}_mse"]["value"]
        assert float(f"{out[name]:.3e}") == want, (name, out[name])
    assert 0.15 < 1 - out["nf4"] / out["int4"] < 0.17  # "about 16 %"


# -------------------------------------------------------------------- E4M3 --

def _e4m3_closed_form(q):
    s = -1.0 if q & 0x80 else 1.0
    e = (q >> 3) & 15
    m = q & 7
    if e == 15 and m == 7:
        return math.nan
    if e == 0:
        return s * m / 8 * 2.0 ** -6
    return s * (1 + m / 8) * 2.0 ** (e - 7)


def test_e4m3_decode_all_codes():
    for q in range(256):
        a, b = oracle.e4m3_decode(q), _e4m3_closed_form(q)
        assert (math.isnan(a) and math.isnan(b)) or a == b
    assert oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9
    assert math.isnan(oracle.e4m3_decode(0x7F)) and math.isnan(oracle.e4m3_decode(0xFF))


def test_e4m3_encode_against_torch_float8():
    """torch's float8_e4m3fn cast is an independent round-to-nearest-even
    implementation of the same OCP format (in range it needs no saturation)."""
    vals = [oracle.e4m3_decode(q) for q in range(0x7F)]
    probes = []
    for a, b in zip(vals[:-1], vals[1:]):
        mid = np.float32((a + b) / 2)
        probes += [mid, next_up(mid), next_down(mid), np.float32(a), np.float32(b)]
    rng = np.random.default_rng(11)
    probes += list(np.float32(rng.uniform(-448, 448, 4000)))
    probes += list(np.float32(np.exp(rng.uniform(-14, 6, 4000))))
    probes = np.array(probes, np.float32)
    probes = np.concatenate([probes, -probes])
    ref = torch.from_numpy(probes).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(x)) for x in probes], np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_encode_saturates_and_ties_to_even():
    assert oracle.e4m3_encode(1000.0) == 0x7E
    assert oracle.e4m3_encode(-1e30) == 0xFE
    assert oracle.e4m3_encode(460.0) == 0x7E
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00   # half the smallest subnormal: tie -> even
    assert oracle.e4m3_encode(3 * 2.0 ** -10) == 0x02  # 1.5 ulp: tie between 1 and 2 -> 2
    assert oracle.e4m3_encode(-0.0) == 0x80


# ------------------------------------------------------------ double quant --

def test_mean_tree_order_and_fsum():
    """Reading: fp64 stride-doubling pairwise sum. [2^53, 1, 1, 1] sums to
    2^53 + 2 by the tree ((2^53+1) + (1+1)), while a left-to-right fp64 sum
    gives 2^53."""
    m, s = oracle.dq_mean(np.array([2.0 ** 53, 1, 1, 1], np.float32))
    assert s == 2.0 ** 53 + 2
    rng = np.random.default_rng(5)
    for n in (1, 7, 256, 1000, 4099):
        c = np.abs(rng.standard_normal(n)).astype(np.float32) * 0.05
        m, s = oracle.dq_mean(c)
        exact = f32(math.fsum(float(x) for x in c) / n)
        assert abs(m - exact) <= np.spacing(exact)
    m, _ = oracle.dq_mean(np.full(777, 0.125, np.float32))
    assert m == np.float32(0.125)


def test_double_quant_invariants():
    """ta-paperlens explainer, 二重量子化: constants centred by their mean,
    8-bit floats in groups of 256 with one fp32 constant per group. With the
    reading 'group absmax -> E4M3 max 448', the largest entry of each group
    decodes to exactly +-448, and every constant comes back within half an
    E4M3 step of its centred value."""
    rng = np.random.default_rng(9)
    nb = 256 * 5 + 77  # short last group
    c = (np.abs(rng.standard_normal(nb)) * 0.02 + 0.01).astype(np.float32)
    c[300] = 0.4
    q, s2, mu = oracle.double_quant(c)
    assert s2.shape == (6,)
    assert mu == oracle.dq_mean(c)[0]
    for g in range(6):
        sl = slice(g * 256, min(nb, g * 256 + 256))
        d = (c[sl] - mu).astype(np.float32)
        assert s2[g] == np.float32(np.max(np.abs(d)) / np.float32(448.0))
        dec = np.array([oracle.e4m3_decode(x) for x in q[sl]])
        assert np.max(np.abs(dec)) == 448.0
        for i, qq in enumerate(q[sl]):
            cp = oracle.dq_constant(qq, s2[g], mu)
            err = abs(float(cp) - float(c[sl][i]))
            bound = max(abs(float(d[i])) / 16, 2.0 ** -10 * float(s2[g]))
            assert err <= bound * (1 + 1e-5) + 4 * float(np.spacing(c[sl][i]))


def test_double_quant_constant_group_and_zero():
    c = np.full(300, 0.05, np.float32)
    q, s2, mu = oracle.double_quant(c)
    assert mu == np.float32(0.05) and np.all(s2 == 0) and np.all(q == 0)
    assert oracle.dq_constant(0, 0.0, mu) == np.float32(0.05)


def test_storage_bits(golden):
    """Bits per parameter: 4 + 8/64 + 32/(64*256) (+ the one fp32 mean) with
    double quantisation, 4 + 32/64 without."""
    N = K = 8192
    bits_dq = 8 * oracle.storage_bytes(N, K, True) / (N * K)
    bits_no = 8 * oracle.storage_bytes(N, K, False) / (N * K)
    assert abs(bits_dq - golden["bits_per_param_dq"]["value"]) < golden["bits_per_param_dq"]["tol"]
    assert bits_no == golden["bits_per_param_no_dq"]["value"]
    assert abs((bits_no - bits_dq) - golden["dq_saving_bits"]["value"]) < 5e-4
    assert abs((bits_dq - 4) - golden["dq_overhead_bits"]["value"]) < 5e-4
    # 65e9 parameters: 4-bit weights 32.5 GB, fp32 constants 4.06 GB
    assert 65e9 * 4 / 8 / 1e9 == golden["weights_4bit_65b_gb"]["value"]
    assert abs(65e9 * (bits_no - 4) / 8 / 1e9 - golden["constants_no_dq_65b_gb"]["value"]) < 0.005


# --------------------------------------------------------------- dequant ----

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.standard_normal(3000).astype(np.float32),
                        np.float32([0.0, -0.0, 1e-40, -1e-40, 3.0e38, 1.00390625, 1.01171875])])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.f32_to_bf16_bits(float(v)) for v in x], np.uint16)
    assert np.array_equal(got, ref)


def test_dequant_round_trip_and_zero_sign():
    rng = np.random.default_rng(4)
    W = (rng.standard_normal((64, 256)) * 0.02).astype(np.float32)
    W[0, :64] = 0.0
    q = oracle.quantize_nf4(W)
    bits = oracle.dequant_bf16_bits(q["codes"], q["qabsmax"], q["s2"], q["mean"], 64, 256)
    What = oracle.bf16_bits_to_f64(bits)
    codes = oracle.unpack_nibbles(q["codes"]).reshape(64, 256)
    _, L = oracle.nf4_levels()
    nb = 64 * 256 // 64
    cprime = np.array([oracle.dq_constant(q["qabsmax"][b], q["s2"][b // 256], q["mean"])
                       for b in range(nb)], np.float32).reshape(64, 4)
    # exact-zero level restores to a zero whose sign is the sign of c'
    z = codes == 7
    for i, j in zip(*np.nonzero(z)):
        assert What[i, j] == 0.0
        assert (bits[i, j] >> 15) == (1 if cprime[i, j // 64] < 0 else 0)
    # the two ends restore to -c' and +c' rounded to bf16
    for i, j in zip(*np.nonzero(codes == 15)):
        assert bits[i, j] == oracle.f32_to_bf16_bits(float(cprime[i, j // 64]))
    # every weight restores within half the widest level gap of its block scale
    gap = np.max(np.diff(L.astype(np.float64))) / 2
    blk = np.repeat(q["absmax"].reshape(64, 4), 64, axis=1)
    cp = np.repeat(cprime.astype(np.float64).reshape(64, 4), 64, axis=1)
    err = np.abs(What - W)
    assert np.all(err <= blk * gap + np.abs(cp - blk) + np.abs(W) * 2 ** -8 + 1e-12)


def test_no_negative_decoded_constant_on_the_workloads():
    """Reading: a decoded constant c' = E4M3(q) s2 + mean is not clamped, so
    a tiny block next to a large mean could get c' < 0. Count it over every
    block of every workload weight: none. The sign is taken from the exact
    sum (E4M3 times s2 is exact in fp64, and adding the fp32 mean cannot flip
    the sign of a nonzero value), which is the sign of the fp32 fma."""
    import synth
    e4 = np.array([oracle.e4m3_decode(v) for v in range(256)])
    for cfg in (synth.TINY, synth.ATTN7B, *synth.MLP7B, *synth.L65B):
        z = oracle.quantize_nf4(synth.weight(cfg).numpy())
        nb = z["qabsmax"].size
        cp = e4[z["qabsmax"]] * z["s2"].astype(np.float64)[np.arange(nb) // 256] + np.float64(z["mean"])
        assert np.count_nonzero(cp <= 0) == 0, cfg.name
