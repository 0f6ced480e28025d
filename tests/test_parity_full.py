"""GPU parity at the full workload sizes, in the launch configuration the
benchmark uses: the whole tensors go through the kernels; the oracle then
recomputes a sample of token positions (every batch and head of each
sampled token) one by one, and those must match bit for bit (codes,
scale/zero, norms, sinks) or within tolerance (decode, scores)."""
import math

import numpy as np
import pytest

import workloads as W
from parity import SCORE_REL, compare_codebook, compare_minmax, recon_tolerance

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_rotation_b200 as K
    return K


def _sample(T, n, seed, always=()):
    rng = np.random.default_rng(seed)
    s = set(int(v) for v in rng.choice(T, size=min(n, T), replace=False))
    s.update(v for v in always if 0 <= v < T)
    return np.array(sorted(s))


def _check_minmax_sample(orc, x_np, gpu_pk, tok, okw, D, bits, group, n_sink):
    ref = orc.encode(np.ascontiguousarray(x_np[:, :, tok]).view(np.uint16), tok, want_pre=True, **okw)
    gc = gpu_pk.codes[:, :, tok].cpu().numpy()
    gs = gpu_pk.scale_zero[:, :, tok].cpu().numpy()
    rep = compare_minmax(gc, ref["codes"], gs, ref["sz"].view(np.int16), ref["pre"], D, bits, group)
    assert rep.ok and rep.mismatched == 0, rep
    if n_sink:
        live = [int(m) for m in tok if m < n_sink]
        if live:
            assert np.array_equal(gpu_pk.sink.cpu().numpy().view(np.uint16)[:, :, live], ref["sink"][:, :, live])
    return gc, gs


@pytest.mark.parametrize("which", ["k", "v"])
def test_full_llama3_8b_gqa(K, orc, which):
    from kv_cache_rotation_b200 import torch_api as TA
    w = W.WORKLOADS["llama3_8b_gqa"]
    rope = 1 if which == "k" else 0
    x = W.kv_tensor(w, which)
    d = TA.make_desc(batch=w.B, heads=w.H, head_dim=w.D, tokens=w.T, bits=w.bits, group=w.group,
                     group_heads=w.group_heads, rope=rope, rot="fwht_group")
    tb = TA.make_tables(rope_cs=TA.rope_table(w.T, w.D) if rope else None)
    pk = TA.alloc_packed(d)
    xg = torch.from_numpy(x).cuda()
    TA.encode(d, xg, tb, pk)
    out = torch.empty_like(xg)
    TA.decode(d, pk, tb, out)
    assert K.kvq_check(0) == K.KVQ_OK
    tok = _sample(w.T, 40, 3, always=(0, 1, 15, 16, w.T - 1))
    okw = dict(rot=orc.ROT_FWHT_GROUP, bits=w.bits, group=w.group, group_heads=w.group_heads, rope=rope)
    gc, gs = _check_minmax_sample(orc, x, pk, tok, okw, w.D, w.bits, w.group, 0)
    dec = orc.decode({"codes": gc, "sz": gs.view(np.uint16)}, tok, (w.B, w.H, tok.size, w.D), **okw)
    got = out[:, :, tok].float().cpu().numpy().astype(np.float64)
    # fp16 output: the fp32 result within 1e-3, then one fp16 rounding
    assert np.all(np.abs(got - dec) <= 1e-3 + np.abs(dec) * 2.0 ** -11), np.abs(got - dec).max()


@pytest.mark.parametrize("which", ["k", "v"])
def test_full_llama2_7b_mha(K, orc, which):
    """The Llama-2-7B MHA layer (8 x 32 x 4096 x 128) with its own channel
    permutation: kvq_calibrate_perm on the tensor itself (abs-max per channel,
    RoPE'd for the keys, sinks excluded), equal to the oracle's calibration,
    then encode / decode with it; 2-bit groups of 64, 4 fp16 sinks."""
    from kv_cache_rotation_b200 import torch_api as TA
    w = W.WORKLOADS["llama2_7b_mha"]
    rope = 1 if which == "k" else 0
    x = W.kv_tensor(w, which)
    d = TA.make_desc(batch=w.B, heads=w.H, head_dim=w.D, tokens=w.T, bits=w.bits, group=w.group, rope=rope,
                     n_sink=w.n_sink, rot="fwht_head")
    xg = torch.from_numpy(x).cuda()
    cs = TA.rope_table(w.T, w.D) if rope else None
    perm_g = TA.calibrate_perm(d, xg, TA.make_tables(rope_cs=cs))
    perm = perm_g.cpu().numpy()
    want = orc.calibrate_perm(x.view(np.uint16), W.positions(0, w.T), rope=rope, n_sink=w.n_sink)
    assert np.array_equal(perm, want)
    tb = TA.make_tables(perm=perm_g, rope_cs=cs)
    pk = TA.alloc_packed(d)
    TA.encode(d, xg, tb, pk)
    out = torch.empty(xg.shape, dtype=torch.float32, device="cuda")
    TA.decode(d, pk, tb, out)
    assert K.kvq_check(0) == K.KVQ_OK
    tok = _sample(w.T, 24, 5 + rope, always=(0, 1, 2, 3, 4, w.T - 1))
    okw = dict(rot=orc.ROT_FWHT_HEAD, bits=w.bits, group=w.group, rope=rope, n_sink=w.n_sink, perm=perm)
    gc, gs = _check_minmax_sample(orc, x, pk, tok, okw, w.D, w.bits, w.group, w.n_sink)
    dec = orc.decode({"codes": gc, "sz": gs.view(np.uint16), "sink": pk.sink.cpu().numpy().view(np.uint16)},
                     tok, (w.B, w.H, tok.size, w.D), **okw)
    err = np.abs(out[:, :, tok].cpu().numpy().astype(np.float64) - dec)
    assert np.all(err <= recon_tolerance(dec)), err.max()


@pytest.mark.parametrize("name", ["isoquant_batch", "isoquant_so3_batch"])
def test_full_isoquant_batch(K, orc, name):
    from kv_cache_rotation_b200 import torch_api as TA
    w = W.WORKLOADS[name]
    so3 = w.rot == "iso3"
    xg = W.kv_tensor_device(w, "k", "cuda")
    qL, qR = (W.iso3_tables(w.D, w.seed), None) if so3 else W.iso_tables(w)
    d = TA.make_desc(batch=w.B, heads=w.H, head_dim=w.D, tokens=w.T, bits=w.bits, rope=0, rot=w.rot,
                     quant="codebook")
    cb = TA.lloyd_max_codebook(w.bits, w.D)
    tb = TA.make_tables(qL=torch.from_numpy(qL).cuda(), qR=torch.from_numpy(qR).cuda() if qR is not None else None,
                        codebook=cb)
    pk = TA.alloc_packed(d)
    TA.encode(d, xg, tb, pk)
    out = torch.empty_like(xg)
    TA.decode(d, pk, tb, out)
    assert K.kvq_check(0) == K.KVQ_OK
    rng = np.random.default_rng(8)
    bs = np.sort(rng.choice(w.B, 48, replace=False))
    tok = _sample(w.T, 16, 9, always=(0, w.T - 1))
    x = xg[bs][:, :, tok].cpu().numpy()  # [48, 1, n, 128]
    ocb = orc.codebook(w.bits, w.D)
    okw = dict(rot=orc.ROT_ISO3 if so3 else orc.ROT_ISO, quant=orc.Q_CODEBOOK, bits=w.bits, qL=qL, qR=qR, cb=ocb)
    ref = orc.encode(x.view(np.uint16), tok, want_pre=True, **okw)
    gc = pk.codes[bs][:, :, tok].cpu().numpy()
    rep = compare_codebook(gc, ref["codes"], ref["pre"], ocb, w.D, w.bits)
    assert rep.ok, rep
    gn = pk.norm[bs][:, :, tok].cpu().numpy()
    assert np.array_equal(gn.view(np.uint32), ref["norm"].view(np.uint32))
    dec = orc.decode({"codes": gc, "norm": gn}, tok, x.shape, **okw)
    got = out[bs][:, :, tok].float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - dec) <= 1e-3 + np.abs(dec) * 2.0 ** -11), np.abs(got - dec).max()


def _score_full(K, orc, w, perm, n_tok_sample, seed, literal=False):
    from kv_cache_rotation_b200 import torch_api as TA
    D = w.D
    t_cap = w.T + w.append
    kw = dict(batch=w.B, heads=w.H, head_dim=D, t_cap=t_cap, bits=w.bits, group=w.group, rope=1, n_sink=w.n_sink,
              rot="fwht_head")
    tb = TA.make_tables(perm=torch.from_numpy(perm).cuda() if perm is not None else None,
                        rope_cs=TA.rope_table(t_cap, D))
    d_pre = TA.make_desc(tokens=w.T, t0=0, **kw)
    pk = TA.alloc_packed(d_pre)
    TA.encode(d_pre, torch.from_numpy(W.kv_tensor(w, "k")).cuda(), tb, pk)
    d_app = TA.make_desc(tokens=w.append, t0=w.T, **kw)
    TA.encode(d_app, torch.from_numpy(W.kv_tensor(w, "k_append", T=w.append)).cuda(), tb, pk)
    q = W.queries(w)
    scale = 1.0 / math.sqrt(D)
    out = torch.empty((w.B, w.Hq, t_cap), dtype=torch.float32, device="cuda")
    (TA.score_literal if literal else TA.score)(d_pre, torch.from_numpy(q).cuda(), pk, tb, t_cap, scale, out)
    assert K.kvq_check(0) == K.KVQ_OK
    assert torch.isfinite(out).all()
    tok = _sample(t_cap, n_tok_sample, seed, always=(0, 1, 2, 3, 4, t_cap - 2, t_cap - 1))
    rng = np.random.default_rng(seed)
    bs = np.sort(rng.choice(w.B, min(w.B, 6), replace=False))
    cache = {"codes": pk.codes[bs].cpu().numpy(), "sz": pk.scale_zero[bs].cpu().numpy().view(np.uint16),
             "sink": pk.sink[bs].cpu().numpy().view(np.uint16)}
    okw = dict(rot=orc.ROT_FWHT_HEAD, bits=w.bits, group=w.group, rope=1, n_sink=w.n_sink, perm=perm)
    ref = orc.score(q[bs].view(np.uint16), cache, tok, H=w.H, t_cap=t_cap, scale=scale, **okw)
    # L1 magnitude of each dot product from the oracle's attention-space keys
    codes_s = {"codes": cache["codes"][:, :, tok], "sz": cache["sz"][:, :, tok], "sink": cache["sink"]}
    khat = orc.decode(codes_s, tok, (bs.size, w.H, tok.size, D), **okw)
    got = out[bs][:, :, tok].cpu().numpy()
    gq = w.Hq // w.H
    for i in range(bs.size):
        for qh in range(w.Hq):
            kk = np.stack([orc.rope_f64(khat[i, qh // gq, j], n) for j, n in enumerate(tok)])
            bound = SCORE_REL * scale * (np.abs(kk) @ np.abs(q[bs[i], qh].astype(np.float64)))
            assert np.all(np.abs(got[i, qh] - ref[i, qh]) <= bound), (i, qh)


def test_full_decode_score(K, orc):
    w = W.WORKLOADS["decode_score"]
    _score_full(K, orc, w, W.random_perm(w.H, w.D, 23), 24, 11)


def test_full_llama3_8b_gqa_score(K, orc):
    w = W.WORKLOADS["llama3_8b_gqa_score"]
    _score_full(K, orc, w, None, 32, 12)


def test_full_decode_score_literal(K, orc):
    w = W.WORKLOADS["decode_score"]
    _score_full(K, orc, w, W.random_perm(w.H, w.D, 23), 24, 13, literal=True)


def test_full_llama3_8b_gqa_score_literal(K, orc):
    w = W.WORKLOADS["llama3_8b_gqa_score"]
    _score_full(K, orc, w, None, 32, 14, literal=True)
