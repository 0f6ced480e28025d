"""Pins for the oracle's whole-tensor encode / decode / score / calibration.

Invariants used: the rotations are orthonormal, so the reconstruction error
in the input basis equals the quantization error in the rotated basis, which
min-max quantization bounds by S/2 per element; sinks are stored verbatim
([RotateKV] attention-sink-aware quantization); the score is the plain dot
product of the query with the attention-space key ([EliteKV §2.2]).
"""
import math

import numpy as np
import pytest

import workloads as W


def _kv(seed, B, H, T, D, scale=1.0):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((B, H, T, D)) * scale).astype(np.float16)
    x[:, :, :, 3] *= 20  # an outlier channel
    return x


def _bound(orc, packed, D, group):
    sz = packed["sz"].astype(np.uint16)
    S = sz[..., 0].view(np.float16).astype(np.float64)  # [B,H,T,ng]
    return np.sqrt(np.sum(group * (S / 2) ** 2, axis=-1))  # per vector


@pytest.mark.parametrize("bits,group,rope,use_perm,n_sink", [
    (4, 128, 1, False, 0), (2, 64, 1, True, 4), (3, 32, 0, True, 2), (2, 128, 1, False, 0)])
def test_head_roundtrip_bound(orc, bits, group, rope, use_perm, n_sink):
    B, H, T, D = 2, 4, 19, 128
    x = _kv(bits * 7 + group, B, H, T, D)
    pos = np.arange(5, 5 + T) if n_sink == 0 else np.arange(T)
    perm = W.random_perm(H, D, 3) if use_perm else None
    kw = dict(rot=orc.ROT_FWHT_HEAD, bits=bits, group=group, rope=rope, n_sink=n_sink, perm=perm)
    pk = orc.encode(x.view(np.uint16), pos, **kw)
    xr = orc.decode(pk, pos, x.shape, **kw)
    xf = x.astype(np.float64)
    err = np.linalg.norm(xr - xf, axis=-1)
    bound = _bound(orc, pk, D, group)
    live = pos >= n_sink
    assert np.all(err[:, :, live] <= bound[:, :, live] * (1 + 1e-5) + 1e-4 * np.linalg.norm(xf, axis=-1)[:, :, live])
    # quantization is not trivially exact
    assert np.mean(err[:, :, live]) > 0
    if n_sink:
        sinkpos = pos[~live]
        assert np.array_equal(pk["sink"][:, :, sinkpos], x.view(np.uint16)[:, :, ~live])
        assert np.array_equal(xr[:, :, ~live], xf[:, :, ~live])
        assert np.all(pk["codes"][:, :, ~live] == 0) and np.all(pk["sz"][:, :, ~live] == 0)


def test_head_rotation_spreads_outliers(orc):
    """The FWHT spreads an outlier channel over all channels: 2-bit error
    with rotation is well below the error without it ([RotateKV] abstract)."""
    B, H, T, D = 1, 2, 64, 128
    x = _kv(11, B, H, T, D)
    pos = np.arange(T)
    errs = {}
    for rot in (orc.ROT_NONE, orc.ROT_FWHT_HEAD):
        kw = dict(rot=rot, bits=2, group=128, rope=1)
        pk = orc.encode(x.view(np.uint16), pos, **kw)
        errs[rot] = np.mean((orc.decode(pk, pos, x.shape, **kw) - x.astype(np.float64)) ** 2)
    assert errs[orc.ROT_FWHT_HEAD] < 0.5 * errs[orc.ROT_NONE]


@pytest.mark.parametrize("hg,bits,group,rope", [(8, 2, 128, 1), (4, 4, 64, 0), (2, 3, 128, 1)])
def test_group_roundtrip_bound(orc, hg, bits, group, rope):
    B, H, T, D = 2, 8, 11, 128
    x = _kv(hg + bits, B, H, T, D)
    pos = np.arange(100, 100 + T)
    kw = dict(rot=orc.ROT_FWHT_GROUP, bits=bits, group=group, group_heads=hg, rope=rope)
    pk = orc.encode(x.view(np.uint16), pos, **kw)
    xr = orc.decode(pk, pos, x.shape, **kw)
    xf = x.astype(np.float64)
    # orthonormal over each group of hg heads: compare squared norms per token-group
    err2 = np.sum((xr - xf) ** 2, axis=-1).reshape(B, H // hg, hg, T).sum(axis=2)
    sz = pk["sz"]
    S = sz[..., 0].view(np.float16).astype(np.float64)
    b2 = np.sum(group * (S / 2) ** 2, axis=-1).reshape(B, H // hg, hg, T).sum(axis=2)
    nx = np.sum(xf ** 2, axis=-1).reshape(B, H // hg, hg, T).sum(axis=2)
    assert np.all(np.sqrt(err2) <= np.sqrt(b2) * (1 + 1e-5) + 1e-4 * np.sqrt(nx))


def test_group_equals_dense_transform(orc):
    """With rope off and 4-bit codes, the grouped rotation is the dense
    normalised H_{hg*D} applied to the concatenated heads: decode of the codes
    matches a dense inverse built from scipy.linalg.hadamard."""
    import scipy.linalg
    B, H, T, D, hg = 1, 4, 3, 64, 4
    x = _kv(5, B, H, T, D)
    pos = np.arange(T)
    kw = dict(rot=orc.ROT_FWHT_GROUP, bits=4, group=64, group_heads=hg, rope=0)
    pk = orc.encode(x.view(np.uint16), pos, **kw)
    Hn = scipy.linalg.hadamard(hg * D) / math.sqrt(hg * D)
    for t in range(T):
        cat = x[0, :, t, :].astype(np.float64).reshape(-1)
        rot = Hn @ cat
        for h in range(H):
            codes = orc.unpack(pk["codes"][0, h, t], D, 4).astype(np.float64)
            S = np.uint16(pk["sz"][0, h, t, 0, 0]).view(np.float16).astype(np.float64)
            Z = np.uint16(pk["sz"][0, h, t, 0, 1]).view(np.float16).astype(np.float64)
            assert np.all(np.abs(Z + codes * S - rot[h * D:(h + 1) * D]) <= S / 2 * (1 + 1e-4) + 1e-6)


def _M(qL, qR):
    def Lm(a):
        w, x, y, z = a
        return np.array([[w, -x, -y, -z], [x, w, -z, y], [y, z, w, -x], [z, -y, x, w]])

    def Rm(b):
        w, x, y, z = b
        return np.array([[w, -x, -y, -z], [x, w, z, -y], [y, -z, w, x], [z, y, -x, w]])
    return Lm(qL.astype(np.float64)) @ Rm(qR.astype(np.float64))


def test_iso_encode_decode(orc):
    """IsoQuant ([IsoQuant §3.1]): norm split, per-block SO(4) rotation,
    Lloyd-Max codes. Codes equal the nearest-level assignment of the fp64
    rotation (away from boundaries); decode inverts the rotation exactly and
    restores the norm."""
    w = W.scaled(W.WORKLOADS["isoquant_batch"], B=2, T=37)
    x = W.kv_tensor(w, "k")
    qL, qR = W.iso_tables(w)
    cb = orc.codebook(3, w.D)
    pos = np.arange(w.T)
    kw = dict(rot=orc.ROT_ISO, quant=orc.Q_CODEBOOK, bits=3, qL=qL, qR=qR, cb=cb)
    pk = orc.encode(x.view(np.uint16), pos, **kw)
    xr = orc.decode(pk, pos, x.shape, **kw)
    beta = 0.5 * (cb[1:].astype(np.float64) + cb[:-1])
    Ms = [_M(qL[k], qR[k]) for k in range(w.D // 4)]
    near = 0
    for b in range(w.B):
        for t in range(w.T):
            xv = x[b, 0, t].astype(np.float64)
            rho = np.linalg.norm(xv)
            assert math.isclose(pk["norm"][b, 0, t], rho, rel_tol=1e-7)
            u = xv / rho
            wv = np.concatenate([Ms[k] @ u[4 * k:4 * k + 4] for k in range(w.D // 4)])
            codes = orc.unpack(pk["codes"][b, 0, t], w.D, 3)
            ref = np.searchsorted(beta, wv, side="left")  # count of beta < w
            dist = np.min(np.abs(wv[:, None] - beta[None, :]), axis=1)
            ok = dist > 1e-6
            near += np.sum(~ok)
            assert np.array_equal(codes[ok], ref[ok])
            # decode: rotating the decoded direction forward gives the levels
            v = xr[b, 0, t] / pk["norm"][b, 0, t]
            wf = np.concatenate([Ms[k] @ v[4 * k:4 * k + 4] for k in range(w.D // 4)])
            assert np.allclose(wf, cb[codes].astype(np.float64), atol=1e-6)
    assert near < 5


def test_score_matches_decode(orc):
    """Score = scale * q . RoPE_n(decoded key); sinks use RoPE_n(sink);
    GQA: query head qh reads KV head qh // (Hq / H)."""
    B, H, Hq, T, D = 2, 2, 4, 12, 128
    n_sink = 3
    x = _kv(21, B, H, T, D)
    perm = W.random_perm(H, D, 9)
    kw = dict(rot=orc.ROT_FWHT_HEAD, bits=2, group=64, rope=1, n_sink=n_sink, perm=perm)
    pos = np.arange(T)
    pk = orc.encode(x.view(np.uint16), pos, **kw)
    rng = np.random.default_rng(4)
    q = rng.standard_normal((B, Hq, D)).astype(np.float16)
    scale = 1 / math.sqrt(D)
    tok = np.array([0, 2, 3, 7, 11])
    s = orc.score(q.view(np.uint16), pk, tok, H=H, t_cap=T, scale=scale, **kw)
    xr = orc.decode(pk, pos, x.shape, **kw)  # input basis (pre-RoPE)
    for b in range(B):
        for qh in range(Hq):
            h = qh // (Hq // H)
            for i, n in enumerate(tok):
                k = orc.rope_f64(xr[b, h, n], n)
                assert math.isclose(s[b, qh, i], scale * (q[b, qh].astype(np.float64) @ k),
                                    rel_tol=1e-9, abs_tol=1e-9)
    # unit query picks one channel of the attention-space key
    e = np.zeros((B, Hq, D), np.float16)
    e[:, :, 5] = 1
    s5 = orc.score(e.view(np.uint16), pk, tok, H=H, t_cap=T, scale=1.0, **kw)
    assert math.isclose(s5[1, 3, 3], orc.rope_f64(xr[1, 1, 7], 7)[5], rel_tol=1e-12, abs_tol=1e-12)


def test_score_grouped_cache_matches_decode(orc):
    """Grouped-head cache ([RotateKV] pre-RoPE grouped-head rotation): the score
    of query head qh at slot n is scale * q . RoPE_n(k), k = head qh // (Hq/H)
    of the group decode (inverse RoPE, FWHT over the group, the head's slice);
    sinks give RoPE_n(sink)."""
    B, H, Hq, T, D, hg = 1, 4, 8, 10, 128, 4
    n_sink = 2
    x = _kv(23, B, H, T, D)
    kw = dict(rot=orc.ROT_FWHT_GROUP, bits=2, group=128, group_heads=hg, rope=1, n_sink=n_sink)
    pos = np.arange(T)
    pk = orc.encode(x.view(np.uint16), pos, **kw)
    rng = np.random.default_rng(5)
    q = rng.standard_normal((B, Hq, D)).astype(np.float16)
    scale = 1 / math.sqrt(D)
    tok = np.array([0, 1, 2, 5, 9])
    s = orc.score(q.view(np.uint16), pk, tok, H=H, t_cap=T, scale=scale, **kw)
    xr = orc.decode(pk, pos, x.shape, **kw)
    for qh in range(Hq):
        h = qh // (Hq // H)
        for i, n in enumerate(tok):
            k = orc.rope_f64(xr[0, h, n], n)
            assert math.isclose(s[0, qh, i], scale * (q[0, qh].astype(np.float64) @ k), rel_tol=1e-9,
                                abs_tol=1e-9)
    # the sink slots return the stored fp16 key itself
    assert np.array_equal(xr[0, :, :n_sink], x[0, :, :n_sink].astype(np.float64))


def test_calibrate_perm(orc):
    B, H, T, D = 2, 3, 17, 128
    x = _kv(31, B, H, T, D)
    x[:, 1, :, 77] *= 3
    pos = np.arange(T)
    perm = orc.calibrate_perm(x.view(np.uint16), pos, rope=1, n_sink=2)
    a = np.zeros((H, D))
    for b in range(B):
        for h in range(H):
            for t in range(2, T):
                c, s = orc.rope_cs(t, D)
                a[h] = np.maximum(a[h], np.abs(orc.rope_f32(x[b, h, t].astype(np.float32), c, s)))
    for h in range(H):
        assert sorted(perm[h].tolist()) == list(range(D))
        seq = a[h, perm[h]]
        assert np.all(np.diff(seq) <= 0)
        # ties keep ascending channel order
        for j in range(D - 1):
            if seq[j] == seq[j + 1]:
                assert perm[h, j] < perm[h, j + 1]
    # the x20 channel 3 dominates; RoPE spreads it over its pair (2, 3)
    assert all(perm[h, 0] in (2, 3) and perm[h, 1] in (2, 3) for h in range(H))
