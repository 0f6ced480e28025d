"""Pins of the oracle's RoPE-pair energy ("EliteKV - RoPE频率选择与低秩投影"
§3.1, frequency energy analysis: E_i = sum over cached keys of
|K_{2i}|^2 + |K_{2i+1}|^2), kept exactly as an integer number of 2^-48.
Checked against exact rational arithmetic, RoPE invariance (a rotation
preserves each pair's norm) and the ranking rule."""
from fractions import Fraction

import numpy as np

UNIT = Fraction(1, 1 << 48)


def _exact(x):
    """Brute force: sum of squares of the fp16 values as exact rationals."""
    B, H, T, D = x.shape
    E = [[Fraction(0)] * (D // 2) for _ in range(H)]
    for b in range(B):
        for h in range(H):
            for t in range(T):
                for i in range(D // 2):
                    a, c = Fraction(float(x[b, h, t, 2 * i])), Fraction(float(x[b, h, t, 2 * i + 1]))
                    E[h][i] += a * a + c * c
    return E


def test_matches_exact_rationals(orc):
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((2, 3, 4, 8)) * rng.choice([1e-6, 1e-2, 1.0, 300.0], size=(2, 3, 4, 8))).astype(np.float16)
    x[0, 0, 0, 0] = np.float16(65504.0)   # largest half
    x[1, 2, 3, 7] = np.float16(6e-8)      # smallest subnormal
    e, _ = orc.pair_energy(x.view(np.uint16))
    got = orc.energy_ints(e)
    want = _exact(x)
    for h in range(3):
        for i in range(4):
            assert want[h][i] / UNIT == got[h][i]  # an exact integer number of 2^-48


def test_every_finite_half_squares_exactly(orc):
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16)
    finite = bits[np.isfinite(vals)]
    x = np.zeros((1, 1, finite.size, 2), np.uint16)
    x[0, 0, :, 0] = finite
    e, _ = orc.pair_energy(x)
    total = sum(Fraction(float(v)) ** 2 for v in finite.view(np.float16))
    assert orc.energy_ints(e)[0][0] == total / UNIT
    # one value at a time, a sample spanning subnormals, normals and the top binade
    for b in (0x0001, 0x03FF, 0x0400, 0x3C00, 0x3C01, 0x7BFF, 0x8001, 0xFBFF):
        y = np.zeros((1, 1, 1, 2), np.uint16)
        y[0, 0, 0, 1] = b
        e1, _ = orc.pair_energy(y)
        v = Fraction(float(np.array([b], np.uint16).view(np.float16)[0]))
        assert orc.energy_ints(e1)[0][0] == v * v / UNIT


def test_rope_invariance(orc):
    rng = np.random.default_rng(9)
    B, H, T, D = 1, 2, 33, 128
    x = rng.standard_normal((B, H, T, D)).astype(np.float16)
    e, _ = orc.pair_energy(x.view(np.uint16))
    got = np.array(orc.energy_ints(e), dtype=np.float64) * 2.0 ** -48
    rot = np.zeros((H, D // 2))
    for h in range(H):
        for t in range(T):
            y = orc.rope_f64(x[0, h, t].astype(np.float64), t)
            rot[h] += y[0::2] ** 2 + y[1::2] ** 2
    assert np.allclose(got, rot, rtol=1e-12, atol=0)


def test_ranking_rule(orc):
    rng = np.random.default_rng(2)
    x = rng.standard_normal((2, 2, 10, 16)).astype(np.float16)
    x[:, 1, :, 10] *= 20          # pair 5 of head 1 dominates
    x[:, 0, :, 4:6] = x[:, 0, :, 8:10]  # pairs 2 and 4 of head 0 tie exactly
    e, rank = orc.pair_energy(x.view(np.uint16))
    E = orc.energy_ints(e)
    assert rank[1, 0] == 5
    for h in range(2):
        assert sorted(rank[h].tolist()) == list(range(8))
        seq = [E[h][i] for i in rank[h]]
        assert all(a >= b for a, b in zip(seq, seq[1:]))
        for j in range(7):
            if seq[j] == seq[j + 1]:
                assert rank[h, j] < rank[h, j + 1]
    assert E[0][2] == E[0][4] and list(rank[0]).index(2) < list(rank[0]).index(4)
