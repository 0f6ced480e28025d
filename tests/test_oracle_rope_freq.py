"""Pins of the oracle's frequency-aware RoPE table (KV-Latent page,
"frequency-aware RoPE": skip the highest frequencies, sample the low ones
more densely, so that low-dimensional heads keep a smoothly decaying
autocorrelation). Checked against the page's stated properties, not by
retyping its formula: the autocorrelation of the all-ones vector stays
positive at head dim 16 where the standard table's goes negative, the top
frequency is dropped and the bottom one extended, and the relative-position
identity holds for the new frequencies too."""
import numpy as np

BASE = 10000.0


def _thetas(orc, d, mode):
    return np.array([orc.rope_theta(i, d, BASE, mode) for i in range(d // 2)])


def _autocorr(th, lags):
    # 1^T R(p) 1 / d for the all-ones vector: the mean of cos(p theta_i) over the pairs
    return np.cos(np.outer(lags, th)).mean(axis=1)


def test_standard_mode_is_the_usual_table(orc):
    for d in (64, 128):
        th = _thetas(orc, d, orc.ROPE_STD)
        assert th[0] == 1.0 and np.all(np.diff(th) < 0)
        assert np.isclose(th[-1], BASE ** (-(d - 2) / d), rtol=1e-15)


def test_autocorrelation_stays_positive_at_low_dim(orc):
    lags = np.arange(1, 4097)
    for d in (16, 32, 64, 128):
        std = _autocorr(_thetas(orc, d, orc.ROPE_STD), lags)
        fa = _autocorr(_thetas(orc, d, orc.ROPE_FREQ_AWARE), lags)
        assert np.all(fa > 0), d
        if d <= 32:
            assert np.mean(std < 0) > 0.2  # the failure the page describes for d < 32


def test_skips_high_and_densifies_low(orc):
    for d in (16, 64, 128):
        std, fa = _thetas(orc, d, orc.ROPE_STD), _thetas(orc, d, orc.ROPE_FREQ_AWARE)
        assert fa.max() < std.max() and fa.min() < std.min()
        assert np.all(np.diff(fa) < 0)  # still one frequency per pair, strictly decreasing
        # more pairs below the standard table's median frequency: denser low end
        assert np.sum(fa < np.median(std)) > np.sum(std < np.median(std))


def test_relative_position_identity(orc):
    rng = np.random.default_rng(3)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    for m, n in ((5, 2), (300, 297), (40000, 39997)):
        a = orc.rope_f64(q, m, mode=orc.ROPE_FREQ_AWARE) @ orc.rope_f64(k, n, mode=orc.ROPE_FREQ_AWARE)
        b = orc.rope_f64(q, m - n, mode=orc.ROPE_FREQ_AWARE) @ k
        assert np.isclose(a, b, rtol=1e-9, atol=1e-9)
    # the fp32 table agrees with the fp64 rotation
    c, s = orc.rope_cs(777, 128, mode=orc.ROPE_FREQ_AWARE)
    th = _thetas(orc, 128, orc.ROPE_FREQ_AWARE)
    assert np.array_equal(c, np.cos(777 * th).astype(np.float32))
    assert np.array_equal(s, np.sin(777 * th).astype(np.float32))
