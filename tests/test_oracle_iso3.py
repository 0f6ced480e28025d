"""Pins of the oracle's 3-D sandwich variant ("KV缓存压缩技术：IsoQuant在大语言模型中的
应用", §2.1: T(v) = q v q* rotates the pure quaternion v by the unit quaternion
q; §1: with 3-channel blocks, d = 128 leaves 42 whole blocks and a 2-D tail).
Each check is against something other than the oracle's own arithmetic:
scipy's rotation of each block, the closed-form planar rotation of the tail,
norm preservation, the block partition, nearest levels in fp64, and the
inverse recovering the input."""
import math

import numpy as np
import pytest

import workloads as W

Rotation = pytest.importorskip("scipy.spatial.transform").Rotation


def _x(B, T, D, seed):
    rng = np.random.default_rng(seed)
    return rng.standard_t(4.0, size=(B, 1, T, D)).astype(np.float16)


def _pre(orc, x, q, bits=3):
    D = x.shape[-1]
    cb = orc.codebook(bits, D)
    out = orc.encode(x.view(np.uint16), np.arange(x.shape[2]), rot=orc.ROT_ISO3, quant=orc.Q_CODEBOOK, bits=bits,
                     qL=q, cb=cb, want_pre=True)
    return out, cb


def _unit(x):
    xf = x.astype(np.float64)
    rho = np.float32(np.sqrt((xf * xf).sum(-1, keepdims=True)))
    return xf / (rho.astype(np.float64) + np.float64(np.float32(1e-8))), rho


@pytest.mark.parametrize("D", [128, 64])
def test_blocks_match_scipy_rotation(orc, D):
    x = _x(2, 5, D, 1)
    q = W.iso3_tables(D, 3)
    out, _ = _pre(orc, x, q)
    u, _ = _unit(x)
    nb = D // 3
    for k in range(nb):
        a, b, c, d = q[k].astype(np.float64)
        R = Rotation.from_quat([b, c, d, a])  # scipy order (x, y, z, w)
        ref = R.apply(u[..., 3 * k:3 * k + 3].reshape(-1, 3)).reshape(u[..., 3 * k:3 * k + 3].shape)
        assert np.allclose(out["pre"][..., 3 * k:3 * k + 3], ref, atol=2e-6, rtol=0), k


def test_tail_is_planar_rotation(orc):
    """d = 128: channels 126, 127 turn by phi = 2 atan2(q_k, q_real) of the tail entry."""
    D = 128
    x = _x(3, 4, D, 2)
    q = W.iso3_tables(D, 5)
    assert q.shape == (43, 4) and q[42, 1] == 0 and q[42, 2] == 0
    out, _ = _pre(orc, x, q)
    u, _ = _unit(x)
    a, d = float(q[42, 0]), float(q[42, 3])
    phi = 2.0 * math.atan2(d, a)
    xs, ys = u[..., 126], u[..., 127]
    assert np.allclose(out["pre"][..., 126], xs * math.cos(phi) - ys * math.sin(phi), atol=2e-6)
    assert np.allclose(out["pre"][..., 127], xs * math.sin(phi) + ys * math.cos(phi), atol=2e-6)


@pytest.mark.parametrize("D,blocks,tail", [(128, 42, 2), (64, 21, 1), (256, 85, 1)])
def test_block_partition(orc, D, blocks, tail):
    """Only the channels of the one block given a non-identity quaternion move;
    a 1-channel tail never moves."""
    assert blocks * 3 + tail == D
    x = _x(1, 3, D, 4)
    u, _ = _unit(x)
    ident = np.tile(np.array([1, 0, 0, 0], np.float32), (blocks + 1, 1))
    out, _ = _pre(orc, x, ident)
    assert np.allclose(out["pre"], u, atol=1e-7)
    for k in (0, blocks // 2, blocks - 1):
        q = ident.copy()
        q[k] = np.array([0.5, 0.5, 0.5, 0.5], np.float32)  # 120 degrees about (1,1,1): a cyclic shift
        out, _ = _pre(orc, x, q)
        moved = np.any(np.abs(out["pre"] - u) > 1e-6, axis=(0, 1, 2))
        assert set(np.nonzero(moved)[0]) <= set(range(3 * k, 3 * k + 3))
        assert np.allclose(out["pre"][..., 3 * k:3 * k + 3], u[..., [3 * k + 2, 3 * k, 3 * k + 1]], atol=1e-6)


@pytest.mark.parametrize("D", [128, 64])
def test_norm_preserved(orc, D):
    x = _x(2, 6, D, 6)
    out, _ = _pre(orc, x, W.iso3_tables(D, 7))
    u, _ = _unit(x)
    assert np.allclose(np.linalg.norm(out["pre"].astype(np.float64), axis=-1), np.linalg.norm(u, axis=-1),
                       atol=5e-6)


def test_codes_are_nearest_level(orc):
    """Each code is the codebook level nearest the fp64 rotation (ties and
    fp32 rounding aside: only values within 1e-5 of a midpoint may differ)."""
    D, bits = 128, 3
    x = _x(2, 9, D, 8)
    q = W.iso3_tables(D, 9)
    out, cb = _pre(orc, x, q, bits)
    u, _ = _unit(x)
    ref = np.empty_like(u)
    for k in range(D // 3):
        a, b, c, d = q[k].astype(np.float64)
        ref[..., 3 * k:3 * k + 3] = Rotation.from_quat([b, c, d, a]).apply(
            u[..., 3 * k:3 * k + 3].reshape(-1, 3)).reshape(u[..., 3 * k:3 * k + 3].shape)
    a, d = q[42, 0].astype(np.float64), q[42, 3].astype(np.float64)
    phi = 2 * math.atan2(d, a)
    ref[..., 126] = u[..., 126] * math.cos(phi) - u[..., 127] * math.sin(phi)
    ref[..., 127] = u[..., 126] * math.sin(phi) + u[..., 127] * math.cos(phi)
    near = np.argmin(np.abs(ref[..., None] - cb.astype(np.float64)), axis=-1)
    n = near.size
    codes = orc.unpack(out["codes"].reshape(-1), n, bits).reshape(near.shape)
    mid = 0.5 * (cb[1:].astype(np.float64) + cb[:-1].astype(np.float64))
    close = np.min(np.abs(ref[..., None] - mid), axis=-1) < 1e-5
    assert np.all((codes == near) | close)
    assert np.array_equal(out["norm"], _unit(x)[1][..., 0])


@pytest.mark.parametrize("D", [128, 64])
def test_decode_is_inverse_rotation(orc, D):
    """Decode of known codes: w = levels[codes] rotated back block by block
    (scipy's inverse rotation, the tail's planar rotation by -phi) and scaled
    by the stored norm."""
    rng = np.random.default_rng(12)
    q = W.iso3_tables(D, 13)
    cb = np.sort(rng.standard_normal(16)).astype(np.float32)
    codes = rng.integers(0, 16, size=(2, 1, 3, D)).astype(np.uint8)
    norm = rng.uniform(0.5, 4.0, size=(2, 1, 3)).astype(np.float32)
    packed = {"codes": orc.pack(codes.reshape(-1), 4).reshape(2, 1, 3, D // 2), "norm": norm}
    dec = orc.decode(packed, np.arange(3), (2, 1, 3, D), rot=orc.ROT_ISO3, quant=orc.Q_CODEBOOK, bits=4, qL=q,
                     cb=cb)
    w = cb[codes].astype(np.float64)
    back = np.empty_like(w)
    for k in range(D // 3):
        a, b, c, d = q[k].astype(np.float64)
        blk = w[..., 3 * k:3 * k + 3]
        back[..., 3 * k:3 * k + 3] = Rotation.from_quat([b, c, d, a]).inv().apply(blk.reshape(-1, 3)).reshape(
            blk.shape)
    if D % 3 == 2:
        a, d = q[D // 3, 0].astype(np.float64), q[D // 3, 3].astype(np.float64)
        phi = -2 * math.atan2(d, a)
        back[..., D - 2] = w[..., D - 2] * math.cos(phi) - w[..., D - 1] * math.sin(phi)
        back[..., D - 1] = w[..., D - 2] * math.sin(phi) + w[..., D - 1] * math.cos(phi)
    else:
        back[..., D - 1] = w[..., D - 1]
    # scipy normalises the fp32 table entry; the oracle takes it as unit: they agree to ~1e-7
    assert np.allclose(dec, back * norm[..., None].astype(np.float64), atol=1e-9, rtol=2e-6)
