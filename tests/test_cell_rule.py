"""The encoder's nearest-level rule, checked on the CPU.

The GPU encoder does not search the 15 decision thresholds per weight: it
reads a table over a uniform grid of 129 cells of width 1/64 on [-1, 1].
Cell j = RN(64 v + 64) covers [(j - 64.5)/64, (j - 63.5)/64] and stores the
number of thresholds below the cell and the single threshold inside it, so
code = base_j + [v > t_j]. This is exact only if no cell holds two
thresholds; these tests pin that property on the oracle's thresholds and
replay the rule, with its fp32 cell index, against the oracle's own count
of thresholds below v (the definition of the nearest level with the lower
level on ties)."""
import numpy as np

import oracle


def thresholds():
    _, L = oracle.nf4_levels()
    return oracle.midpoints(L).astype(np.float32)


def cell_table(M):
    lo = (np.arange(130) - 64.5) / 64.0
    base = np.array([int(np.sum(M.astype(np.float64) < lo[j])) for j in range(129)])
    inside = np.full(129, 2.0, np.float32)
    for j in range(129):
        hit = [m for m in M.astype(np.float64) if lo[j] <= m < lo[j + 1]]
        assert len(hit) <= 1, f"cell {j} holds {len(hit)} thresholds"
        if hit:
            inside[j] = np.float32(hit[0])
    return base, inside


def cell_code(v, base, inside):
    # one fp32 fma with 1.5*2^23 + 64: the sum is exact in fp64, then rounded once
    t = np.float32(np.float64(v) * 64.0 + 12582976.0)
    j = int(t.view(np.int32) - np.int32(0x4B400000))
    assert 0 <= j <= 128
    return int(base[j] + (1 if np.float32(v) > inside[j] else 0))


def neighbours(x, k):
    out = [np.float32(x)]
    up = down = np.float32(x)
    for _ in range(k):
        up = np.nextafter(up, np.float32(2))
        down = np.nextafter(down, np.float32(-2))
        out += [up, down]
    return [y for y in out if -1 <= y <= 1]


def test_at_most_one_threshold_per_cell():
    M = thresholds()
    gaps = np.diff(M.astype(np.float64))
    assert gaps.min() > 1 / 64, gaps.min()
    cell_table(M)


def test_cell_rule_equals_threshold_count_everywhere_it_can_differ():
    """Every threshold and every cell edge +-40 ulps, both ends and zeros,
    plus 100k random values: the rule equals #(thresholds < v)."""
    M = thresholds()
    base, inside = cell_table(M)
    vals = [np.float32(-1), np.float32(1), np.float32(0), np.float32(-0.0)]
    for m in M:
        vals += neighbours(m, 40)
    for j in range(130):
        vals += neighbours((j - 64.5) / 64.0, 40)
    rng = np.random.default_rng(7)
    vals += list(rng.uniform(-1, 1, 50000).astype(np.float32))
    vals += list(np.clip(rng.standard_normal(50000) * 0.25, -1, 1).astype(np.float32))
    bad = [v for v in vals if cell_code(v, base, inside) != int(np.sum(np.float32(v) > M))]
    assert not bad, bad[:5]
