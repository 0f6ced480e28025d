"""GPU parity of the dynamic IsoQuant codebooks ("KV缓存压缩技术：IsoQuant在大语言
模型中的应用", §4.2) against the oracle, through the C ABI.

Calibration: the GPU's per-channel scales equal the oracle's within a few
fp32 ulps (the rotated values differ by the matrix form of the sandwich, as
for the fixed codebook), and the outlier masks are equal. Encode: with the
GPU's tables given to both sides, codes (low bits and the outlier channels'
top bits) are compared with the codebook excuse rule; decode of the GPU's
codes within 1e-3 of the oracle's fp64 decode."""
import numpy as np
import pytest

import workloads as W
from parity import EXCUSE_FRAC, EXCUSE_REL, RECON_ABS, CodeReport, _record, unpack_all

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_rotation_b200 as K
    return K


CASES = [
    # name, rot, B, H, T, D, t0, bits, n_sink, outliers
    ("so4_b3_d128", "iso", 2, 2, 300, 128, 0, 3, 0, ("pairs", 0.03, 10.0, 50.0)),
    ("so4_b2_d64_t0_sinks", "iso", 3, 1, 257, 64, 5, 2, 4, ("pairs", 0.05, 5.0, 20.0)),
    ("so4_b4_student", "iso", 1, 4, 130, 128, 0, 4, 2, None),
    ("so3_b3_d128", "iso3", 2, 2, 200, 128, 0, 3, 0, ("pairs", 0.03, 10.0, 50.0)),
    ("so3_b2_d64", "iso3", 2, 2, 99, 64, 1, 2, 1, ("pairs", 0.05, 10.0, 30.0)),
    ("many_chunks", "iso", 2, 1, 2500, 128, 0, 3, 0, ("pairs", 0.03, 10.0, 50.0)),
]


def _inputs(name, B, H, T, D, outliers):
    if outliers is None:
        w = W.Workload(name, B=B, H=H, T=T, D=D, dist="student_t", seed=len(name))
    else:
        w = W.Workload(name, B=B, H=H, T=T, D=D, outliers=outliers, seed=len(name))
    return W.kv_tensor(w, "k")


def _full_codes(codes, ext, D, bits, wide):
    """[B][H][T][D] codes: the low bits plus each outlier channel's top bit."""
    c = unpack_all(codes, D, bits).astype(np.int32)
    for h in range(c.shape[1]):
        wch = [j for j in range(D) if (int(wide[h][j // 32]) >> (j % 32)) & 1]
        for i, j in enumerate(wch[:16]):
            c[:, h, :, j] |= ((ext[:, h].astype(np.int32) >> i) & 1) << bits
    return c


def _compare(cg, co, pre, sigma, wide, cb, cbw, D):
    diff = cg != co
    n_mis = int(diff.sum())
    exc = 0
    if n_mis:
        for b, h, t, j in zip(*np.nonzero(diff)):
            lv = cbw if (int(wide[h][j // 32]) >> (j % 32)) & 1 else cb
            L = (np.float32(sigma[h, j]) * lv).astype(np.float32).astype(np.float64)
            k = min(cg[b, h, t, j], co[b, h, t, j])
            if abs(int(cg[b, h, t, j]) - int(co[b, h, t, j])) != 1 or k + 1 >= L.size:
                continue
            beta = 0.5 * (L[k] + L[k + 1])
            v = float(pre[b, h, t, j])
            if abs(v - beta) <= EXCUSE_REL * max(abs(v), float(sigma[h, j])):
                exc += 1
    return _record(CodeReport(cg.size, n_mis, exc, n_mis - exc, 0))


def _run(K, orc, case):
    from kv_cache_rotation_b200 import torch_api as TA
    name, rot, B, H, T, D, t0, bits, n_sink, outliers = case
    x = _inputs(name, B, H, T, D, outliers)
    t_cap = t0 + T + 2
    qL, qR = (W.iso3_tables(D, 3), None) if rot == "iso3" else (W.unit_quaternions(D // 4, 3, 30),
                                                                  W.unit_quaternions(D // 4, 3, 31))
    d = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, t0=t0, t_cap=t_cap, bits=bits, n_sink=n_sink, rot=rot,
                     quant="codebook_dyn")
    cb, cbw = TA.lloyd_max_codebook(bits, 1), TA.lloyd_max_codebook(bits + 1, 1)
    tb = TA.make_tables(qL=torch.from_numpy(qL).cuda(), qR=torch.from_numpy(qR).cuda() if qR is not None else None,
                        codebook=cb, codebook_wide=cbw)
    xg = torch.from_numpy(x).cuda()
    tb.ch_scale, tb.ch_wide = TA.calibrate_codebook(d, xg, tb)
    assert K.kvq_check(0) == K.KVQ_OK
    pos = np.arange(t0, t0 + T)
    r = orc.ROT_ISO3 if rot == "iso3" else orc.ROT_ISO
    ocb, ocbw = orc.codebook(bits, 1), orc.codebook(bits + 1, 1)
    assert np.array_equal(ocb, cb.cpu().numpy()) and np.array_equal(ocbw, cbw.cpu().numpy())
    _, osig, owide = orc.dyn_calibrate(x.view(np.uint16), pos, rot=r, qL=qL, qR=qR, n_sink=n_sink)
    gsig = tb.ch_scale.cpu().numpy()
    gwide = tb.ch_wide.cpu().numpy().view(np.uint32)
    np.testing.assert_allclose(gsig, osig, rtol=1e-6, atol=0)
    assert np.array_equal(gwide, owide)
    # encode with the GPU's tables on both sides
    pk = TA.alloc_packed(d)
    TA.encode(d, xg, tb, pk)
    assert K.kvq_check(0) == K.KVQ_OK
    ref = orc.dyn_encode(x.view(np.uint16), pos, rot=r, bits=bits, qL=qL, qR=qR, cb=ocb, cbw=ocbw, sigma=gsig,
                         wide=gwide, n_sink=n_sink, want_pre=True)
    gc = pk.codes[:, :, t0:t0 + T].cpu().numpy()
    ge = pk.ext[:, :, t0:t0 + T].cpu().numpy().view(np.uint16)
    cg = _full_codes(gc, ge, D, bits, gwide)
    co = _full_codes(ref["codes"], ref["ext"], D, bits, gwide)
    rep = _compare(cg, co, ref["pre"], gsig, gwide, ocb, ocbw, D)
    assert rep.ok, rep
    gn = pk.norm[:, :, t0:t0 + T].cpu().numpy()
    assert np.array_equal(gn.view(np.uint32), ref["norm"].view(np.uint32))
    if n_sink:
        live = [m for m in pos if m < n_sink]
        assert np.array_equal(pk.sink.cpu().numpy().view(np.uint16)[:, :, live], ref["sink"][:, :, live])
    out32 = torch.empty((B, H, T, D), dtype=torch.float32, device="cuda")
    out16 = torch.empty((B, H, T, D), dtype=torch.float16, device="cuda")
    TA.decode(d, pk, tb, out32)
    TA.decode(d, pk, tb, out16)
    assert K.kvq_check(0) == K.KVQ_OK
    packed = {"codes": gc, "ext": ge, "norm": gn,
              "sink": pk.sink.cpu().numpy().view(np.uint16) if n_sink else None}
    dec = orc.dyn_decode(packed, pos, x.shape, rot=r, bits=bits, qL=qL, qR=qR, cb=ocb, cbw=ocbw, sigma=gsig,
                         wide=gwide, n_sink=n_sink)
    o32 = out32.cpu().numpy()
    assert np.max(np.abs(o32 - dec)) <= RECON_ABS
    assert np.array_equal(out16.cpu().numpy().view(np.uint16), o32.astype(np.float16).view(np.uint16))
    return rep, gwide


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_dyn_parity(K, orc, case):
    rep, wide = _run(K, orc, case)
    if case[-1] is not None:  # channel outliers are found
        assert any(int(v) for v in wide.ravel())


def test_dyn_calibrate_with_sink_list(K, orc):
    from kv_cache_rotation_b200 import torch_api as TA
    B, H, T, D = 2, 2, 150, 128
    x = _inputs("sl", B, H, T, D, ("pairs", 0.03, 10.0, 50.0))
    W.plant_massive(x, 3, 4)
    sp = np.array([[0, 40, -1], [0, 7, 99]], np.int32)
    qL, qR = W.unit_quaternions(D // 4, 3, 30), W.unit_quaternions(D // 4, 3, 31)
    d = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, bits=3, n_sink=3, rot="iso", quant="codebook_dyn")
    tb = TA.make_tables(qL=torch.from_numpy(qL).cuda(), qR=torch.from_numpy(qR).cuda(),
                        sink_pos=torch.from_numpy(sp).cuda())
    sc, wd = TA.calibrate_codebook(d, torch.from_numpy(x).cuda(), tb)
    _, osig, owide = orc.dyn_calibrate(x.view(np.uint16), np.arange(T), rot=orc.ROT_ISO, qL=qL, qR=qR, n_sink=3,
                                       sink_pos=sp)
    np.testing.assert_allclose(sc.cpu().numpy(), osig, rtol=1e-6)
    assert np.array_equal(wd.cpu().numpy().view(np.uint32), owide)


def test_dyn_calibrate_no_tokens(K):
    """No position counts (every token a sink): sigma = fp32(1/sqrt(D)), no outliers."""
    from kv_cache_rotation_b200 import torch_api as TA
    B, H, T, D = 1, 2, 4, 64
    x = torch.randn((B, H, T, D), device="cuda").half()
    d = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, bits=2, n_sink=4, rot="iso", quant="codebook_dyn")
    qL, qR = W.unit_quaternions(D // 4, 3, 30), W.unit_quaternions(D // 4, 3, 31)
    tb = TA.make_tables(qL=torch.from_numpy(qL).cuda(), qR=torch.from_numpy(qR).cuda())
    sc, wd = TA.calibrate_codebook(d, x, tb)
    assert torch.all(sc == np.float32(1.0 / np.sqrt(D))).item()
    assert not wd.any().item()


def test_dyn_full_size_sampled(K, orc):
    """The dynamic IsoQuant batch at full size (8192 x 2048 vectors of 128,
    3-bit, keys with outlier channels): GPU calibration and encode; sampled
    vectors re-encoded by the oracle with the GPU's tables."""
    from kv_cache_rotation_b200 import torch_api as TA
    w = W.WORKLOADS["isoquant_dyn_batch"]
    B, H, T, D = w.B, w.H, w.T, w.D
    x = W.kv_tensor_device(w, "k", "cuda")
    qL, qR = W.iso_tables(w)
    d = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, bits=w.bits, rot="iso", quant="codebook_dyn")
    cb, cbw = TA.lloyd_max_codebook(w.bits, 1), TA.lloyd_max_codebook(w.bits + 1, 1)
    tb = TA.make_tables(qL=torch.from_numpy(qL).cuda(), qR=torch.from_numpy(qR).cuda(), codebook=cb,
                        codebook_wide=cbw)
    tb.ch_scale, tb.ch_wide = TA.calibrate_codebook(d, x, tb)
    pk = TA.alloc_packed(d)
    TA.encode(d, x, tb, pk)
    assert K.kvq_check(0) == K.KVQ_OK
    gsig = tb.ch_scale.cpu().numpy()
    gwide = tb.ch_wide.cpu().numpy().view(np.uint32)
    assert any(int(v) for v in gwide.ravel())
    rng = np.random.default_rng(0)
    bs = np.sort(rng.choice(B, size=6, replace=False))
    xs = x[torch.from_numpy(bs).cuda()].cpu().numpy()
    ref = orc.dyn_encode(xs.view(np.uint16), np.arange(T), rot=orc.ROT_ISO, bits=w.bits, qL=qL, qR=qR,
                         cb=cb.cpu().numpy(), cbw=cbw.cpu().numpy(), sigma=gsig, wide=gwide, want_pre=True)
    gc = pk.codes[torch.from_numpy(bs).cuda()].cpu().numpy()
    ge = pk.ext[torch.from_numpy(bs).cuda()].cpu().numpy().view(np.uint16)
    cg = _full_codes(gc, ge, D, w.bits, gwide)
    co = _full_codes(ref["codes"], ref["ext"], D, w.bits, gwide)
    rep = _compare(cg, co, ref["pre"], gsig, gwide, cb.cpu().numpy(), cbw.cpu().numpy(), D)
    assert rep.ok, rep
    assert rep.excused <= EXCUSE_FRAC * rep.n
