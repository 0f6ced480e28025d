"""Pins of the oracle's attention-sink handling ("RotateKV: Accurate and
Robust 2-Bit KV Cache Quantization for LLMs via Outlier-Aware Adaptive
Rotations", abstract (iii) and 关键设计: sinks are identified from the
activations, by their massive magnitude, and kept at high precision).
Detection is checked against constructed sequences, a numpy brute force of
the stated rule (per-token max |x|, lower median, strict tau threshold, the
largest first with ties to the earlier token, ascending output), the cap
and the exact threshold; the sink-position list against the prefix form it
generalises."""
import math

import numpy as np
import pytest

import workloads as W


def _x(B, H, T, D, seed):
    return np.random.default_rng(seed).standard_normal((B, H, T, D)).astype(np.float16)


def _brute(x, pos, tau, max_sinks):
    a = np.abs(x.astype(np.float32)).max(axis=(1, 3))  # [B][T]
    out = np.full((x.shape[0], max_sinks), -1, np.int32)
    cnt = np.zeros(x.shape[0], np.int32)
    for b in range(x.shape[0]):
        med = np.sort(a[b])[(a.shape[1] - 1) // 2]
        cand = [t for t in range(a.shape[1]) if float(a[b, t]) > tau * float(med)]
        cand.sort(key=lambda t: (-float(a[b, t]), t))
        pick = sorted(cand[:max_sinks])
        out[b, :len(pick)] = [pos[t] for t in pick]
        cnt[b] = len(pick)
    return out, cnt


def test_detect_known_massive_tokens(orc):
    x = _x(2, 3, 50, 16, 1)
    x[0, 1, 0, 4] = np.float16(300.0)
    x[0, 2, 17, 9] = np.float16(-250.0)
    x[1, 0, 5, 0] = np.float16(400.0)
    sp, cnt = orc.detect_sinks(x.view(np.uint16), np.arange(50), tau=20.0, max_sinks=4)
    assert sp[0].tolist() == [0, 17, -1, -1] and sp[1].tolist() == [5, -1, -1, -1]
    assert cnt.tolist() == [2, 1]


@pytest.mark.parametrize("tau", [1.0, 1.5, 2.5, 8.0])
def test_detect_matches_brute_force(orc, tau):
    x = _x(3, 2, 41, 8, 2)
    x[:, :, ::7] *= np.float16(3.0)
    pos = np.arange(100, 141)
    sp, cnt = orc.detect_sinks(x.view(np.uint16), pos, tau=tau, max_sinks=6)
    want_sp, want_cnt = _brute(x, pos, tau, 6)
    assert np.array_equal(sp, want_sp) and np.array_equal(cnt, want_cnt)


def test_detect_cap_and_ties(orc):
    x = _x(1, 1, 30, 8, 3) * np.float16(0.1)
    for t in (3, 9, 12, 20, 25):
        x[0, 0, t, 2] = np.float16(64.0)  # equal magnitudes: the earlier tokens win
    x[0, 0, 27, 5] = np.float16(128.0)     # the largest is taken first
    sp, cnt = orc.detect_sinks(x.view(np.uint16), np.arange(30), tau=10.0, max_sinks=3)
    assert sp[0].tolist() == [3, 9, 27] and cnt[0] == 3


def test_detect_threshold_is_strict(orc):
    """a_t equal to tau * median is not a sink; one fp16 step above is."""
    T = 9
    x = np.zeros((1, 1, T, 4), np.float16)
    x[0, 0, :, 0] = np.float16(1.0)          # median magnitude 1
    x[0, 0, 2, 0] = np.float16(4.0)          # exactly tau * median
    x[0, 0, 6, 0] = np.float16(4.00390625)   # the next fp16 above 4
    sp, cnt = orc.detect_sinks(x.view(np.uint16), np.arange(T), tau=4.0, max_sinks=4)
    assert sp[0].tolist() == [6, -1, -1, -1] and cnt[0] == 1


def test_detect_median_zero(orc):
    """With a zero median every nonzero token clears the threshold (capped)."""
    x = np.zeros((1, 2, 11, 4), np.float16)
    x[0, 1, 4, 3] = np.float16(1e-3)
    x[0, 0, 9, 0] = np.float16(-2.0)
    sp, cnt = orc.detect_sinks(x.view(np.uint16), np.arange(11), tau=100.0, max_sinks=2)
    assert sp[0].tolist() == [4, 9] and cnt[0] == 2


@pytest.mark.parametrize("rot,kw", [
    ("head", dict(bits=2, group=64, rope=1)),
    ("group", dict(bits=2, group=128, group_heads=4, rope=1)),
    ("none", dict(bits=4, group=32, rope=0)),
])
def test_sink_list_prefix_is_the_prefix_form(orc, rot, kw):
    """An explicit list 0 .. n_sink-1 encodes and decodes bit for bit like the prefix."""
    B, H, T, D, S = 2, 4, 12, 128, 3
    x = _x(B, H, T, D, 4)
    r = {"head": orc.ROT_FWHT_HEAD, "group": orc.ROT_FWHT_GROUP, "none": orc.ROT_NONE}[rot]
    pos = np.arange(T)
    args = dict(rot=r, n_sink=S, **kw)
    a = orc.encode(x.view(np.uint16), pos, **args)
    sp = np.tile(np.arange(S, dtype=np.int32), (B, 1))
    b = orc.encode(x.view(np.uint16), pos, sink_pos=sp, **args)
    for k in ("codes", "sz", "sink"):
        assert np.array_equal(a[k], b[k])
    assert np.array_equal(orc.decode(a, pos, x.shape, **args), orc.decode(b, pos, x.shape, sink_pos=sp, **args))


def test_sink_list_arbitrary_positions(orc):
    """Listed positions keep their fp16 rows in list order (zero codes and
    scale/zero) and decode verbatim; every other token encodes exactly as
    with no sinks at all."""
    B, H, T, D = 2, 2, 30, 128
    x = _x(B, H, T, D, 5)
    pos = np.arange(T)
    kw = dict(rot=orc.ROT_FWHT_HEAD, bits=2, group=64, rope=1)
    sp = np.array([[7, 20, -1], [0, 29, 13]], np.int32)
    e = orc.encode(x.view(np.uint16), pos, n_sink=3, sink_pos=sp, **kw)
    plain = orc.encode(x.view(np.uint16), pos, **kw)
    for b in range(B):
        for k, m in enumerate(sp[b]):
            if m < 0:
                continue
            assert np.array_equal(e["sink"][b, :, k], x[b, :, m].view(np.uint16))
            assert not e["codes"][b, :, m].any() and not e["sz"][b, :, m].any()
        keep = [t for t in range(T) if t not in sp[b]]
        assert np.array_equal(e["codes"][b][:, keep], plain["codes"][b][:, keep])
        assert np.array_equal(e["sz"][b][:, keep], plain["sz"][b][:, keep])
    dec = orc.decode(e, pos, x.shape, n_sink=3, sink_pos=sp, **kw)
    assert np.array_equal(dec[0, :, 20], x[0, :, 20].astype(np.float64))
    assert np.array_equal(dec[1, :, 29], x[1, :, 29].astype(np.float64))


def test_sink_list_score(orc):
    """The score of a listed sink is scale * q . RoPE_n(sink row)."""
    B, H, Hq, T, D = 1, 2, 4, 16, 128
    x = _x(B, H, T, D, 6)
    pos = np.arange(T)
    kw = dict(rot=orc.ROT_FWHT_HEAD, bits=2, group=128, rope=1)
    sp = np.array([[5, 11]], np.int32)
    e = orc.encode(x.view(np.uint16), pos, n_sink=2, sink_pos=sp, **kw)
    q = np.random.default_rng(7).standard_normal((B, Hq, D)).astype(np.float16)
    s = orc.score(q.view(np.uint16), e, np.array([5, 11, 3]), H=H, t_cap=T, scale=0.5, n_sink=2, sink_pos=sp, **kw)
    for i, n in enumerate((5, 11)):
        for qh in range(Hq):
            k = orc.rope_f64(x[0, qh // 2, n].astype(np.float64), n)
            assert math.isclose(s[0, qh, i], 0.5 * (q[0, qh].astype(np.float64) @ k), rel_tol=1e-12, abs_tol=1e-12)
