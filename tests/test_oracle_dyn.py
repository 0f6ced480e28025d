"""Pins of the oracle's dynamic IsoQuant codebooks ("KV缓存压缩技术：IsoQuant在
大语言模型中的应用", §4.2: per-channel statistics gathered online, boundaries
set by the KL divergence, twice the codebook for outlier channels).

The scale of channel j is pinned against a numerical minimisation of the KL
divergence from the channel's sample to N(0, s^2) (scipy) and against numpy
moments of the encoder's own rotated values; the outlier rule by brute force;
the codes against the nearest level of the channel's codebook; the layout of
the outlier channels' top bits by a constructed vector; and the special case
of equal scales without outliers against the fixed-codebook encoder."""
import numpy as np
import pytest
from scipy.optimize import minimize_scalar

import workloads as W


def _iso(D, seed, rot="iso"):
    if rot == "iso3":
        return W.iso3_tables(D, seed), None
    return W.unit_quaternions(D // 4, seed, 30), W.unit_quaternions(D // 4, seed, 31)


def _identity(D):
    q = np.zeros((D // 4, 4), np.float32)
    q[:, 0] = 1.0
    return q, q.copy()


def _student(B, H, T, D, seed, scaled=()):
    w = W.Workload("dyn", B=B, H=H, T=T, D=D, dist="student_t", seed=seed)
    x = W.kv_tensor(w, "k").astype(np.float32)
    for c, s in scaled:
        x[..., c] *= s
    return x.astype(np.float16)


def _codes(orc, e, D, bits, wide_row):
    """Full codes [..., D] of one head: low bits plus the outlier channels' top bits."""
    lo = np.stack([orc.unpack(r, D, bits) for r in e["codes"].reshape(-1, D * bits // 8)]).astype(np.int32)
    lo = lo.reshape(*e["codes"].shape[:-1], D)
    wch = [j for j in range(D) if (wide_row[j // 32] >> (j % 32)) & 1]
    for i, j in enumerate(wch):
        lo[..., j] |= ((e["ext"].astype(np.int32) >> i) & 1) << bits
    return lo, wch


@pytest.mark.parametrize("rot", ["iso", "iso3"])
def test_sigma_is_the_kl_minimiser(orc, rot):
    B, H, T, D = 2, 2, 300, 128
    x = _student(B, H, T, D, 1, scaled=[(9, 6.0), (50, 3.0)])
    qL, qR = _iso(D, 2, rot)
    r = orc.ROT_ISO3 if rot == "iso3" else orc.ROT_ISO
    m2, sigma, wide = orc.dyn_calibrate(x.view(np.uint16), np.arange(T), rot=r, qL=qL, qR=qR)
    cb, cbw = orc.codebook(3, 1), orc.codebook(4, 1)
    e = orc.dyn_encode(x.view(np.uint16), np.arange(T), rot=r, bits=3, qL=qL, qR=qR, cb=cb, cbw=cbw,
                       sigma=sigma, wide=wide, want_pre=True)
    w = e["pre"].astype(np.float64)  # [B][H][T][D], the quantizer's input
    np.testing.assert_allclose(m2, (w ** 2).mean(axis=(0, 2)), rtol=1e-12)
    np.testing.assert_allclose(sigma, np.sqrt(m2).astype(np.float32), rtol=0, atol=0)
    for h, j in [(0, 9), (1, 50), (0, 77), (1, 3)]:
        s = w[:, h, :, j].ravel()

        def kl(log_s):  # KL(p || N(0, e^{2 log_s})) up to the entropy of p
            sd = np.exp(log_s)
            return np.mean(0.5 * (s / sd) ** 2 + log_s)
        opt = minimize_scalar(kl, bounds=(-12, 2), method="bounded", options={"xatol": 1e-10})
        assert abs(np.exp(opt.x) / sigma[h, j] - 1) < 1e-6


def test_outlier_rule_brute_force(orc):
    """Identity quaternions leave the channels in place, so scaled input
    channels are the outliers; 20 of them exceed the cap of D/8 = 16."""
    B, H, T, D = 1, 2, 200, 128
    rng = np.random.default_rng(3)
    out_ch = rng.choice(D, size=20, replace=False)
    scaled = [(int(c), float(s)) for c, s in zip(out_ch, rng.uniform(3, 9, size=20))]
    x = _student(B, H, T, D, 4, scaled=scaled)
    x[0, 1] = _student(B, 1, T, D, 5, scaled=scaled[:5])[0, 0]  # head 1: only 5 outliers
    qL, qR = _identity(D)
    _, sigma, wide = orc.dyn_calibrate(x.view(np.uint16), np.arange(T), rot=orc.ROT_ISO, qL=qL, qR=qR)
    for h in range(H):
        s = sigma[h]
        med = np.sort(s)[(D - 1) // 2]
        cand = [j for j in range(D) if s[j] > np.float32(2.0) * med]
        cand.sort(key=lambda j: (-s[j], j))
        want = np.zeros(D // 32, np.uint32)
        for j in cand[:D // 8]:
            want[j // 32] |= np.uint32(1 << (j % 32))
        assert np.array_equal(wide[h], want)
    n0 = sum(bin(int(v)).count("1") for v in wide[0])
    n1 = sum(bin(int(v)).count("1") for v in wide[1])
    assert n0 == 16 and n1 == 5
    got1 = {j for j in range(D) if (wide[1][j // 32] >> (j % 32)) & 1}
    assert got1 == {c for c, _ in scaled[:5]}


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_codes_are_the_nearest_level(orc, bits):
    B, H, T, D = 2, 1, 120, 128
    x = _student(B, H, T, D, 6, scaled=[(1, 8.0), (64, 5.0), (127, 7.0)])
    qL, qR = _iso(D, 7)
    _, sigma, wide = orc.dyn_calibrate(x.view(np.uint16), np.arange(T), rot=orc.ROT_ISO, qL=qL, qR=qR)
    cb, cbw = orc.codebook(bits, 1), orc.codebook(bits + 1, 1)
    e = orc.dyn_encode(x.view(np.uint16), np.arange(T), rot=orc.ROT_ISO, bits=bits, qL=qL, qR=qR, cb=cb, cbw=cbw,
                       sigma=sigma, wide=wide, want_pre=True)
    c, wch = _codes(orc, e, D, bits, wide[0])
    assert wch  # the scaled channels produce outliers after the 4-D blocks mix them
    w = e["pre"].astype(np.float64)
    for j in range(D):
        lv = (sigma[0, j] * (cbw if j in wch else cb)).astype(np.float32).astype(np.float64)
        d = np.abs(w[..., j][..., None] - lv)  # distance to every level
        best = d.min(axis=-1)
        mine = np.take_along_axis(d, c[..., j][..., None], axis=-1)[..., 0]
        mid = 0.5 * (lv[1:] + lv[:-1])
        near_mid = np.min(np.abs(w[..., j][..., None] - mid), axis=-1) <= 1e-6 * np.maximum(np.abs(w[..., j]), 1e-3)
        assert np.all((mine == best) | near_mid), j


def test_ext_layout_constructed(orc):
    """Identity rotation, three outlier channels (3, 40, 77) at a scale of
    0.1: w_40 and w_77 lie far above the top level (top bit 1), w_3 far below
    (top bit 0), so ext = 0b110 and the low bits are all ones / zero."""
    D, bits = 128, 3
    x = np.zeros((1, 1, 1, D), np.float16)
    x[0, 0, 0, 40], x[0, 0, 0, 3], x[0, 0, 0, 77] = 1.0, -0.5, 0.5
    qL, qR = _identity(D)
    sigma = np.full((1, D), 0.1, np.float32)
    wide = np.zeros((1, 4), np.uint32)
    for j in (3, 40, 77):
        wide[0, j // 32] |= np.uint32(1 << (j % 32))
    cb, cbw = orc.codebook(bits, 1), orc.codebook(bits + 1, 1)
    e = orc.dyn_encode(x.view(np.uint16), np.arange(1), rot=orc.ROT_ISO, bits=bits, qL=qL, qR=qR, cb=cb, cbw=cbw,
                       sigma=sigma, wide=wide)
    assert int(e["ext"][0, 0, 0]) == 0b110
    lo = orc.unpack(e["codes"][0, 0, 0], D, bits)
    assert lo[40] == lo[77] == (1 << bits) - 1 and lo[3] == 0
    dec = orc.dyn_decode(e, np.arange(1), x.shape, rot=orc.ROT_ISO, bits=bits, qL=qL, qR=qR, cb=cb, cbw=cbw,
                         sigma=sigma, wide=wide)
    rho = float(e["norm"][0, 0, 0])
    assert dec[0, 0, 0, 40] == pytest.approx(rho * float(np.float32(0.1) * cbw[-1]), rel=1e-12)
    assert dec[0, 0, 0, 3] == pytest.approx(rho * float(np.float32(0.1) * cbw[0]), rel=1e-12)


@pytest.mark.parametrize("rot", ["iso", "iso3"])
def test_equal_scales_reduce_to_the_fixed_codebook(orc, rot):
    """Every sigma equal to s0 and no outlier channel: the codes, norms and
    decode equal the fixed-codebook encoder's with levels fp32(s0 * l_k)."""
    B, H, T, D, bits = 2, 2, 40, 64, 3
    x = _student(B, H, T, D, 8)
    qL, qR = _iso(D, 9, rot)
    r = orc.ROT_ISO3 if rot == "iso3" else orc.ROT_ISO
    s0 = np.float32(0.1234)
    cb, cbw = orc.codebook(bits, 1), orc.codebook(bits + 1, 1)
    sigma = np.full((H, D), s0, np.float32)
    wide = np.zeros((H, D // 32), np.uint32)
    e = orc.dyn_encode(x.view(np.uint16), np.arange(T), rot=r, bits=bits, qL=qL, qR=qR, cb=cb, cbw=cbw,
                       sigma=sigma, wide=wide, n_sink=2)
    fixed = (s0 * cb).astype(np.float32)
    f = orc.encode(x.view(np.uint16), np.arange(T), rot=r, quant=orc.Q_CODEBOOK, bits=bits, qL=qL, qR=qR, cb=fixed,
                   n_sink=2)
    assert np.array_equal(e["codes"], f["codes"]) and np.array_equal(e["norm"], f["norm"])
    assert np.array_equal(e["sink"], f["sink"]) and not e["ext"].any()
    kw = dict(rot=r, bits=bits, qL=qL, qR=qR, n_sink=2)
    a = orc.dyn_decode(e, np.arange(T), x.shape, cb=cb, cbw=cbw, sigma=sigma, wide=wide, **kw)
    b = orc.decode(f, np.arange(T), x.shape, quant=orc.Q_CODEBOOK, cb=fixed, **kw)
    assert np.array_equal(a, b)


def test_dynamic_codebook_raises_snr_on_channel_outliers(orc):
    """On inputs with scaled channels the per-channel codebooks reconstruct
    better than the fixed one (a property the page's +4.2 dB claims)."""
    B, H, T, D, bits = 1, 1, 2000, 128, 3
    x = _student(B, H, T, D, 10, scaled=[(c, 6.0) for c in range(0, 128, 16)])
    qL, qR = _iso(D, 11)
    pos = np.arange(T)
    _, sigma, wide = orc.dyn_calibrate(x.view(np.uint16), pos, rot=orc.ROT_ISO, qL=qL, qR=qR)
    cb, cbw = orc.codebook(bits, 1), orc.codebook(bits + 1, 1)
    e = orc.dyn_encode(x.view(np.uint16), pos, rot=orc.ROT_ISO, bits=bits, qL=qL, qR=qR, cb=cb, cbw=cbw,
                       sigma=sigma, wide=wide)
    dd = orc.dyn_decode(e, pos, x.shape, rot=orc.ROT_ISO, bits=bits, qL=qL, qR=qR, cb=cb, cbw=cbw, sigma=sigma,
                        wide=wide)
    fixed = orc.codebook(bits, D)
    f = orc.encode(x.view(np.uint16), pos, rot=orc.ROT_ISO, quant=orc.Q_CODEBOOK, bits=bits, qL=qL, qR=qR, cb=fixed)
    fd = orc.decode(f, pos, x.shape, rot=orc.ROT_ISO, quant=orc.Q_CODEBOOK, bits=bits, qL=qL, qR=qR, cb=fixed)
    xs = x.astype(np.float64)

    def snr(d):
        return 10 * np.log10((xs ** 2).sum() / ((xs - d) ** 2).sum())
    assert snr(dd) > snr(fd) + 1.0, (snr(dd), snr(fd))
