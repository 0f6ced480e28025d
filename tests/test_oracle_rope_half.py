"""Pins of the oracle's half-split RoPE pairing ("EliteKV - RoPE频率选择与低秩投影",
§7.1: the page's apply_rope pairs channel i with i + d/2, rotating the pair
by the angle m * theta_i of the rotation matrix of §2.1). Checked against
the interleaved rotation (pinned elsewhere) through an explicit channel
reordering, and against the rotation's own algebra."""
import math

import numpy as np
import pytest

HALF = 4


def _pi(d):
    """y = x[idx]: interleaved slot 2i holds channel i, slot 2i+1 holds i + d/2."""
    idx = np.empty(d, np.int64)
    idx[0::2] = np.arange(d // 2)
    idx[1::2] = np.arange(d // 2) + d // 2
    return idx


@pytest.mark.parametrize("d,table", [(128, 1), (64, 1), (128, 2)])
def test_half_split_is_interleaved_on_reordered_channels(orc, d, table):
    """Bit for bit in fp32 (the same operations on every pair) and in fp64."""
    rng = np.random.default_rng(d + table)
    idx = _pi(d)
    for m in (0, 1, 7, 4095, 32768):
        x = rng.standard_normal(d).astype(np.float32)
        c, s = orc.rope_cs(m, d, mode=table)
        half = orc.rope_f32(x, c, s, mode=table + HALF)
        inter = orc.rope_f32(x[idx], c, s, mode=table)
        back = np.empty_like(inter)
        back[idx] = inter
        assert np.array_equal(half.view(np.uint32), back.view(np.uint32))
        xd = x.astype(np.float64)
        h64 = orc.rope_f64(xd, m, mode=table + HALF)
        i64 = orc.rope_f64(xd[idx], m, mode=table)
        b64 = np.empty_like(i64)
        b64[idx] = i64
        assert np.array_equal(h64, b64)


def test_half_split_explicit_pair(orc):
    """Channel i and i + d/2 turn by m theta_i, theta_i = 10000^(-2i/d)."""
    d, m = 128, 37
    x = np.zeros(d)
    x[5], x[5 + 64] = 1.0, 0.5
    y = orc.rope_f64(x, m, mode=1 + HALF)
    a = m * 10000.0 ** (-2 * 5 / d)
    assert math.isclose(y[5], math.cos(a) - 0.5 * math.sin(a), abs_tol=1e-15)
    assert math.isclose(y[5 + 64], math.sin(a) + 0.5 * math.cos(a), abs_tol=1e-15)
    assert np.count_nonzero(y) == 2


def test_half_split_group_property(orc):
    """R(a) R(b) = R(a + b), R(0) = I, norm preserved, R(-m) inverts R(m)."""
    d = 128
    rng = np.random.default_rng(3)
    x = rng.standard_normal(d)
    assert np.array_equal(orc.rope_f64(x, 0, mode=1 + HALF), x)
    for a, b in ((3, 5), (100, 2000), (1, 32767)):
        ab = orc.rope_f64(orc.rope_f64(x, a, mode=1 + HALF), b, mode=1 + HALF)
        assert np.allclose(ab, orc.rope_f64(x, a + b, mode=1 + HALF), atol=1e-10)
        y = orc.rope_f64(x, a, mode=1 + HALF)
        assert math.isclose(np.linalg.norm(y), np.linalg.norm(x), rel_tol=1e-12)
        assert np.allclose(orc.rope_f64(y, a, mode=1 + HALF, inverse=True), x, atol=1e-12)


def test_half_split_relative_position(orc):
    """<R_m q, R_n k> depends only on m - n."""
    d = 64
    rng = np.random.default_rng(4)
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    for m, n, shift in ((10, 3, 100), (0, 40, 7), (500, 499, 1234)):
        s0 = orc.rope_f64(q, m, mode=1 + HALF) @ orc.rope_f64(k, n, mode=1 + HALF)
        s1 = orc.rope_f64(q, m + shift, mode=1 + HALF) @ orc.rope_f64(k, n + shift, mode=1 + HALF)
        assert math.isclose(s0, s1, rel_tol=1e-9, abs_tol=1e-9)


def test_half_split_encode_decode(orc):
    """Head-variant encode with half-split RoPE decodes back (the inverse RoPE
    uses the same pairs) within the quantizer's error."""
    import workloads as W
    w = W.Workload("half", B=1, H=2, T=9, D=128, bits=4, group=128)
    x = W.kv_tensor(w, "k")
    kw = dict(rot=orc.ROT_FWHT_HEAD, bits=4, group=128, rope=1 + HALF)
    pk = orc.encode(x.view(np.uint16), np.arange(9), **kw)
    dec = orc.decode(pk, np.arange(9), x.shape, **kw)
    err = np.abs(dec - x.astype(np.float64))
    kw1 = dict(kw, rope=1)
    dec1 = orc.decode(orc.encode(x.view(np.uint16), np.arange(9), **kw1), np.arange(9), x.shape, **kw1)
    # the same size of error as with interleaved pairs (the rotation is orthogonal either way)
    assert err.max() < 4 * np.abs(dec1 - x.astype(np.float64)).max() + 1e-3
