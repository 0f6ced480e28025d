"""Pins for the CPU oracle: each oracle function is checked against something
other than itself -- closed forms, brute force, library routines, textbook
constants (tests/golden) and invariants stated on the pages.

Pages: [RoPE-KV] "RoPE启发的KV缓存压缩技术解析"; [EliteKV] "EliteKV -
RoPE频率选择与低秩投影"; [IsoQuant] "KV缓存压缩技术：IsoQuant在大语言模型中的应用";
[RotateKV] "RotateKV: Accurate and Robust 2-Bit KV Cache Quantization for LLMs
via Outlier-Aware Adaptive Rotations".
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg
from scipy import integrate, stats
from scipy.spatial.transform import Rotation

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ fp16
def _all_finite_halves():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = h.view(np.float16).astype(np.float64)
    ok = np.isfinite(f)
    return h[ok], f[ok]


def test_half_to_float_exhaustive(orc):
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = h.view(np.float16).astype(np.float32)
    got = np.array([orc.half_to_float(v) for v in h], np.float32)
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin].view(np.uint32), ref[fin].view(np.uint32))
    assert np.all(np.isnan(got[np.isnan(ref)]))
    assert np.array_equal(got[np.isinf(ref)], ref[np.isinf(ref)])


def test_half_rn_matches_numpy(orc):
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 2**32, 60000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    # concentrate extra samples around the half range and its ties
    g = rng.standard_normal(20000).astype(np.float32) * np.float32(1000)
    hs = np.arange(0, 0x7bff, 7, dtype=np.uint16).view(np.float16).astype(np.float32)
    ties = ((hs[:-1].astype(np.float64) + hs[1:].astype(np.float64)) / 2).astype(np.float32)
    special = np.array([0.0, -0.0, 65504, 65519.99, 65520, 65536, 6e-8, 2.98e-8, 2.9802322e-8, -1e-30],
                       np.float32)
    for arr in (f, g, ties, -ties, special):
        ref = arr.astype(np.float16).view(np.uint16)
        got = np.array([orc.float_to_half(v, "rn") for v in arr], np.uint16)
        assert np.array_equal(got, ref)


def test_half_directed_rounding_brute_force(orc):
    hbits, hval = _all_finite_halves()
    order = np.argsort(hval, kind="stable")
    hv, hb = hval[order], hbits[order]
    rng = np.random.default_rng(8)
    xs = np.concatenate([
        rng.standard_normal(20000) * 100,
        rng.standard_normal(5000) * 1e-5,
        hv[::13] + 1e-3 * np.abs(hv[::13]) * rng.standard_normal(hv[::13].size),
        hv[::31],  # exact halves
        [70000.0, -70000.0, 65504.0, -65504.0, 1e-9, -1e-9],
    ]).astype(np.float32)
    for x in xs:
        xd = float(x)
        rd = orc.half_to_float(orc.float_to_half(x, "rd"))
        ru = orc.half_to_float(orc.float_to_half(x, "ru"))
        i = np.searchsorted(hv, xd, side="right") - 1  # largest half <= x
        j = np.searchsorted(hv, xd, side="left")  # smallest half >= x
        assert rd == (-np.inf if i < 0 else hv[i]), x
        assert ru == (np.inf if j >= hv.size else hv[j]), x


# ------------------------------------------------------------------ RoPE
def test_rope_group_property(orc):
    """[RoPE-KV §7.1]: R(t1) R(t2) = R(t1 + t2); R(0) = I; R(-m) R(m) = I."""
    rng = np.random.default_rng(1)
    for d in (64, 128):
        x = rng.standard_normal(d)
        for m1, m2 in ((3, 5), (100, 2000), (31000, 1700)):
            a = orc.rope_f64(orc.rope_f64(x, m2), m1)
            b = orc.rope_f64(x, m1 + m2)
            assert np.allclose(a, b, atol=1e-9)
        assert np.array_equal(orc.rope_f64(x, 0), x)
        assert np.allclose(orc.rope_f64(orc.rope_f64(x, 777), 777, inverse=True), x, atol=1e-12)
        assert math.isclose(np.linalg.norm(orc.rope_f64(x, 12345)), np.linalg.norm(x), rel_tol=1e-12)


def test_rope_relative_position(orc):
    """[EliteKV §2.2]: q_m^rot . k_n^rot depends only on m - n; closed form
    sum_i cos(phi)(q0 k0 + q1 k1) + sin(phi)(q1 k0 - q0 k1), phi = (n - m) theta_i
    (derived from the R_m matrix of [EliteKV §2.1])."""
    rng = np.random.default_rng(2)
    d = 128
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    for m, n, delta in ((5, 9, 100), (4000, 17, 3), (0, 32768, 12)):
        s1 = orc.rope_f64(q, m) @ orc.rope_f64(k, n)
        s2 = orc.rope_f64(q, m + delta) @ orc.rope_f64(k, n + delta)
        th = 10000.0 ** (-2.0 * np.arange(d // 2) / d)
        phi = (n - m) * th
        q0, q1, k0, k1 = q[0::2], q[1::2], k[0::2], k[1::2]
        closed = np.sum(np.cos(phi) * (q0 * k0 + q1 * k1) + np.sin(phi) * (q1 * k0 - q0 * k1))
        assert math.isclose(s1, s2, rel_tol=1e-9, abs_tol=1e-9)
        assert math.isclose(s1, closed, rel_tol=1e-9, abs_tol=1e-9)


def test_rope_table_and_fp32_rotation(orc):
    """cos/sin are the fp32 roundings of the fp64 angle functions; the fp32
    rotation is the documented fmaf order, checked in exact rational
    arithmetic on a sample."""
    d = 128
    for m in (0, 1, 4097, 32768):
        c, s = orc.rope_cs(m, d)
        th = np.array([orc.rope_theta(i, d) for i in range(d // 2)])
        assert np.allclose(th, 10000.0 ** (-2.0 * np.arange(d // 2) / d), rtol=1e-15)
        ang = m * th
        assert np.array_equal(c, np.cos(ang).astype(np.float32)) or np.max(
            np.abs(c.astype(np.float64) - np.cos(ang))) < 6e-8
        assert np.max(np.abs(s.astype(np.float64) - np.sin(ang))) < 6e-8
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(d) * 10).astype(np.float32)
    c, s = orc.rope_cs(31999, d)
    y = orc.rope_f32(x, c, s)

    def rn32(fr):  # round a Fraction to the nearest fp32 (ties to even)
        if fr == 0:
            return 0.0
        sign = -1 if fr < 0 else 1
        a = abs(fr)
        e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
        while Fraction(2) ** e > a:
            e -= 1
        while Fraction(2) ** (e + 1) <= a:
            e += 1
        q = Fraction(2) ** (e - 23)
        n = a / q
        fl = n.numerator // n.denominator
        rem = n - fl
        if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
            fl += 1
        return sign * float(fl * q)

    for i in range(0, d // 2, 5):
        x0, x1 = Fraction(float(x[2 * i])), Fraction(float(x[2 * i + 1]))
        ci, si = Fraction(float(c[i])), Fraction(float(s[i]))
        t1 = Fraction(rn32(x1 * si))
        t2 = Fraction(rn32(x1 * ci))
        assert np.float32(rn32(x0 * ci - t1)) == y[2 * i]
        assert np.float32(rn32(x0 * si + t2)) == y[2 * i + 1]


# ------------------------------------------------------------------ FWHT
def _dense_h(n):
    i = np.arange(n)
    pc = np.vectorize(lambda v: bin(v).count("1"))(i[:, None] & i[None, :])
    return np.where(pc % 2 == 0, 1.0, -1.0)


@pytest.mark.parametrize("n", [2, 4, 8, 16])
def test_fwht_brute_force_small(orc, n):
    """FWHT equals the dense Sylvester matrix H_ij = (-1)^popcount(i & j)
    by brute force; exact on integer input; H H^T = n I."""
    H = _dense_h(n)
    assert np.array_equal(H @ H.T, n * np.eye(n))
    rng = np.random.default_rng(n)
    for _ in range(20):
        xi = rng.integers(-1000, 1000, n).astype(np.float64)
        assert np.array_equal(orc.fwht_f64(xi), H @ xi)
        assert np.array_equal(orc.fwht_f32(xi.astype(np.float32)), (H @ xi).astype(np.float32))
        xr = rng.standard_normal(n)
        assert np.allclose(orc.fwht_f64(xr), H @ xr, rtol=0, atol=1e-12)


@pytest.mark.parametrize("n", [64, 128, 256, 1024])
def test_fwht_matches_library_hadamard(orc, n):
    """Against scipy.linalg.hadamard (Sylvester construction), plus the
    factorisation H_1024 = H_8 (x) H_128 used by the grouped-head rotation."""
    H = scipy.linalg.hadamard(n).astype(np.float64)
    rng = np.random.default_rng(n)
    x = rng.standard_normal(n)
    assert np.allclose(orc.fwht_f64(x), H @ x, atol=1e-10)
    xf = x.astype(np.float32)
    assert np.allclose(orc.fwht_f32(xf), H @ xf.astype(np.float64), atol=1e-4 * math.sqrt(n))
    r = orc.fwht_scale_f32(n)
    assert r == np.float32(1.0 / math.sqrt(n))
    y = orc.fwht_f64(orc.fwht_f64(x)) / n  # involution once normalised
    assert np.allclose(y, x, atol=1e-12)
    if n == 1024:
        H8, H128 = scipy.linalg.hadamard(8), scipy.linalg.hadamard(128)
        assert np.array_equal(np.kron(H8, H128), H)


# ------------------------------------------------------------------ min-max quantizer
def _all_halves_sorted():
    hb, hv = _all_finite_halves()
    o = np.argsort(hv, kind="stable")
    return hv[o]


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_minmax_properties(orc, bits):
    L = (1 << bits) - 1
    hv = _all_halves_sorted()
    rng = np.random.default_rng(bits)
    groups = [rng.standard_normal(64).astype(np.float32) * s + o
              for s, o in ((1, 0), (0.01, 0), (3, 100), (1e-3, 1000), (50, -7), (1e-6, 0.5))]
    groups.append(np.full(32, 1.25, np.float32))  # constant (exactly a half)
    groups.append(np.full(32, 1.2345678, np.float32))  # constant, not a half
    for p in groups:
        codes, s16, z16 = orc.minmax_group(p, bits)
        S = orc.half_to_float(s16)
        Z = orc.half_to_float(z16)
        mn, mx = float(p.min()), float(p.max())
        # Z = largest half <= min (brute force over all halves)
        assert Z == hv[np.searchsorted(hv, mn, side="right") - 1]
        # S = smallest half >= fp32((max - Z) / L)
        q = np.float32(np.float32(mx - np.float32(Z)) / np.float32(L))
        assert S == hv[np.searchsorted(hv, float(q), side="left")]
        assert codes.max() <= L
        if S == 0:
            assert np.all(codes == 0) and mx == mn
            continue
        # every code is the nearest grid point, up to the fp32 rounding of
        # (p - Z) and 1/S; every value lies inside the grid's span
        u = (p.astype(np.float64) - Z) / S
        assert np.all(np.abs(codes - u) <= 0.5 + 1e-5)
        assert np.all(u >= -1e-6) and np.all(u <= L + 1e-5)
        recon = Z + codes.astype(np.float64) * S
        assert np.all(np.abs(recon - p) <= S / 2 * (1 + 1e-5) + 1e-12)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_minmax_brute_force_tiny(orc, bits):
    """Groups of 4 values on a small fp16 grid: each code equals the index of
    the nearest grid point Z + kS (exact rational arithmetic), the tie rule
    being round-half-even of (p - Z) / S."""
    L = (1 << bits) - 1
    rng = np.random.default_rng(10 + bits)
    grid = np.arange(-64, 65, dtype=np.float32) / 16  # exact halves
    for _ in range(300):
        p = rng.choice(grid, 4).astype(np.float32)
        codes, s16, z16 = orc.minmax_group(p, bits)
        S, Z = Fraction(orc.half_to_float(s16)), Fraction(orc.half_to_float(z16))
        for j in range(4):
            if S == 0:
                assert codes[j] == 0
                continue
            u = (Fraction(float(p[j])) - Z) / S
            best = min(range(L + 1), key=lambda k: (abs(u - k), k % 2))
            # the fp32 reciprocal may move a decision by < 2^-20 of a level
            if abs(abs(u - best) - Fraction(1, 2)) > Fraction(1, 2**20):
                assert codes[j] == best, (p, j, u)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_minmax_idempotent(orc, bits):
    """Q(D(c)) = c for a fixed (S, Z): a group whose values sit exactly on the
    grid Z + c S (with codes 0 and L present) re-quantizes to the same codes
    and the same scale/zero."""
    L = (1 << bits) - 1
    rng = np.random.default_rng(20 + bits)
    for S, Z in ((0.25, -1.5), (0.0078125, 3.0), (2.0, -100.0), (0.001953125, 0.0)):
        c = rng.integers(0, L + 1, 64)
        c[0], c[1] = 0, L
        p = (np.float32(Z) + c.astype(np.float32) * np.float32(S)).astype(np.float32)
        codes, s16, z16 = orc.minmax_group(p, bits)
        assert orc.half_to_float(s16) == S and orc.half_to_float(z16) == Z
        assert np.array_equal(codes, c)


# ------------------------------------------------------------------ packing
def _golden_rows(name):
    rows = []
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        rows.append([f.strip() for f in line.split("|")])
    return rows


def test_pack_golden_bytes(orc):
    for bits, codes, hexbytes in _golden_rows("pack_bytes.txt"):
        b = int(bits)
        c = np.array([int(v) for v in codes.split()], np.uint8)
        expect = bytes(int(v, 16) for v in hexbytes.split())
        assert bytes(orc.pack(c, b)) == expect
        assert np.array_equal(orc.unpack(np.frombuffer(expect, np.uint8), c.size, b), c)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_pack_roundtrip(orc, bits):
    rng = np.random.default_rng(bits)
    for n in (8, 64, 128, 256):
        c = rng.integers(0, 1 << bits, n).astype(np.uint8)
        assert np.array_equal(orc.unpack(orc.pack(c, bits), n, bits), c)


# ------------------------------------------------------------------ Lloyd-Max
def test_lloyd_max_textbook(orc):
    """Max (1960) Table I values (tests/golden/lloyd_max_gaussian.txt)."""
    for bits, outs, thr, mse in _golden_rows("lloyd_max_gaussian.txt"):
        b = int(bits)
        lv, m, _ = orc.lloyd_max_normal(b)
        n = 1 << b
        pos = lv[n // 2:]
        assert np.allclose(pos, [float(v) for v in outs.split()], atol=6e-4)
        bnd = 0.5 * (lv[1:] + lv[:-1])
        assert np.allclose(bnd[n // 2 - 1:], [float(v) for v in thr.split()], atol=6e-4)
        assert math.isclose(m, float(mse), rel_tol=1e-3)
        assert np.allclose(lv, -lv[::-1], atol=1e-13)  # symmetric


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_lloyd_max_fixed_point(orc, bits):
    """Centroid condition by numerical integration (scipy.integrate.quad):
    each level is E[X | X in its cell]; boundaries are midpoints."""
    lv, mse, _ = orc.lloyd_max_normal(bits)
    b = np.concatenate([[-np.inf], 0.5 * (lv[1:] + lv[:-1]), [np.inf]])
    total = 0.0
    for k, l in enumerate(lv):
        num = integrate.quad(lambda x: x * stats.norm.pdf(x), b[k], b[k + 1], epsabs=1e-14)[0]
        den = stats.norm.cdf(b[k + 1]) - stats.norm.cdf(b[k])
        assert abs(num / den - l) < 1e-9
        total += integrate.quad(lambda x: (x - l) ** 2 * stats.norm.pdf(x), b[k], b[k + 1], epsabs=1e-14)[0]
    assert math.isclose(total, mse, rel_tol=1e-9)


def test_codebook_scaling(orc):
    lv, _, _ = orc.lloyd_max_normal(3)
    cb = orc.codebook(3, 128)
    assert cb.dtype == np.float32 and np.all(np.diff(cb) > 0)
    assert np.allclose(cb, lv / math.sqrt(128), rtol=1e-7)


# ------------------------------------------------------------------ quaternions
def _qL(a):  # left multiplication matrix: a (x) b = L(a) b
    w, x, y, z = a
    return np.array([[w, -x, -y, -z], [x, w, -z, y], [y, z, w, -x], [z, -y, x, w]])


def _qR(b):  # right multiplication matrix: a (x) b = R(b) a
    w, x, y, z = b
    return np.array([[w, -x, -y, -z], [x, w, z, -y], [y, -z, w, x], [z, y, -x, w]])


def test_quaternion_basis_table(orc):
    """i^2 = j^2 = k^2 = ijk = -1 ([IsoQuant §2.1] quaternion algebra)."""
    one, i, j, k = np.eye(4)
    for f in (orc.quat_mul_f64, orc.quat_mul_f32):
        assert np.array_equal(f(i, i), -one) and np.array_equal(f(j, j), -one)
        assert np.array_equal(f(k, k), -one)
        assert np.array_equal(f(f(i, j), k), -one)
        assert np.array_equal(f(i, j), k) and np.array_equal(f(j, k), i) and np.array_equal(f(k, i), j)
        assert np.array_equal(f(j, i), -k)


def test_quaternion_sandwich(orc):
    """qL v qR equals M v with M = L(qL) R(qR), M orthogonal with det +1;
    (-qL, -qR) gives the same map ([IsoQuant §2.2]); the 3-D sandwich q v q*
    of a pure quaternion matches scipy's rotation; unit quaternions preserve
    norms ([IsoQuant §2.1])."""
    rng = np.random.default_rng(5)
    for _ in range(50):
        a = rng.standard_normal(4)
        b = rng.standard_normal(4)
        assert np.allclose(orc.quat_mul_f64(a, b), _qL(a) @ b, atol=1e-12)
        assert np.allclose(orc.quat_mul_f64(a, b), _qR(b) @ a, atol=1e-12)
        qa, qb = a / np.linalg.norm(a), b / np.linalg.norm(b)
        v = rng.standard_normal(4)
        w = orc.quat_mul_f64(qa, orc.quat_mul_f64(v, qb))
        M = _qL(qa) @ _qR(qb)
        assert np.allclose(w, M @ v, atol=1e-12)
        assert np.allclose(M @ M.T, np.eye(4), atol=1e-12) and abs(np.linalg.det(M) - 1) < 1e-12
        assert np.allclose(orc.quat_mul_f64(-qa, orc.quat_mul_f64(v, -qb)), w, atol=1e-12)
        assert math.isclose(np.linalg.norm(w), np.linalg.norm(v), rel_tol=1e-12)
        p = np.concatenate([[0.0], rng.standard_normal(3)])
        conj = qa * np.array([1, -1, -1, -1])
        r = orc.quat_mul_f64(qa, orc.quat_mul_f64(p, conj))
        ref = Rotation.from_quat([qa[1], qa[2], qa[3], qa[0]]).apply(p[1:])
        assert abs(r[0]) < 1e-12 and np.allclose(r[1:], ref, atol=1e-12)
        wf = orc.quat_mul_f32(qa.astype(np.float32), orc.quat_mul_f32(v.astype(np.float32),
                                                                       qb.astype(np.float32)))
        assert np.allclose(wf, w, atol=1e-5)


# ------------------------------------------------------------------ page numbers
def test_page_numbers():
    for kind, args, val in _golden_rows("page_numbers.txt"):
        a = [int(v) for v in args.split()]
        if kind == "kv_bytes":
            L, N, d, h = a
            assert L * N * d * h * 4 * 2 == int(val)
        elif kind == "dense_rotation_macs":
            assert a[0] * a[0] == int(val)
        elif kind == "blocks3d":
            full, tail = (int(v) for v in val.split())
            assert a[0] // 3 == full and a[0] % 3 == tail
        elif kind == "blocks4d":
            full, tail = (int(v) for v in val.split())
            assert a[0] // 4 == full and a[0] % 4 == tail
