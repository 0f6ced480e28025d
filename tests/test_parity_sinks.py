"""GPU parity of attention-sink detection (kvq_detect_sinks) and of the list
form of the sink set (kvq_tables.sink_pos) against the oracle, through the C
ABI ("RotateKV: Accurate and Robust 2-Bit KV Cache Quantization for LLMs via
Outlier-Aware Adaptive Rotations", abstract (iii) and 关键设计: sinks found
from their massive activations and kept at high precision).

Detection is integer work: the lists and counts must be equal. The list form
is checked on every rotation (head FWHT, none, grouped FWHT, IsoQuant SO(4)
and 3-D) for encode and decode, on the head and grouped scores, on the
calibration, and end to end (GPU detection feeding the GPU encode against the
oracle's detection feeding the oracle's encode)."""
import numpy as np
import pytest

import workloads as W
from parity import compare_codebook, compare_minmax, recon_tolerance, score_tolerance

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_rotation_b200 as K
    return K


def _x(B, H, T, D, seed, planted=3):
    w = W.Workload("sinks", B=B, H=H, T=T, D=D, seed=seed)
    x = W.kv_tensor(w, "k")
    if planted:
        W.plant_massive(x, planted, seed)
    return x


def _detect_gpu(K, x, t0, tau, max_sinks):
    from kv_cache_rotation_b200 import torch_api as TA
    B, H, T, D = x.shape
    d = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, t0=t0, t_cap=t0 + T, bits=2, group=64, rope=0)
    sp, cnt = TA.detect_sinks(d, torch.from_numpy(x).cuda(), tau=tau, max_sinks=max_sinks)
    assert K.kvq_check(0) == K.KVQ_OK
    return sp.cpu().numpy(), cnt.cpu().numpy()


DETECT = [
    # name, B, H, T, D, t0, tau, max_sinks, planted
    ("planted_d128", 2, 4, 37, 128, 0, 8.0, 4, 3),
    ("planted_d64_offset", 3, 8, 1025, 64, 17, 8.0, 6, 4),
    ("cap_below_planted", 2, 8, 700, 128, 0, 8.0, 2, 5),
    ("many_chunks", 2, 8, 5000, 128, 3, 8.0, 64, 40),
    ("low_tau_cap", 1, 4, 3000, 128, 0, 1.0, 64, 0),
    ("one_token", 1, 4, 1, 128, 5, 1.0, 2, 1),
    ("two_tokens", 1, 2, 2, 64, 0, 0.5, 4, 1),
    ("heads_not_multiple_of_4", 2, 3, 100, 128, 0, 8.0, 8, 3),
    # more keys than the selection stages in shared memory (49152): read from global memory
    ("long_unstaged", 2, 1, 50000, 64, 7, 3.0, 16, 6),
    ("long_unstaged_capped", 1, 2, 60000, 64, 0, 1.0, 12, 0),
]


@pytest.mark.parametrize("case", DETECT, ids=[c[0] for c in DETECT])
def test_detect_parity(K, orc, case):
    name, B, H, T, D, t0, tau, M, planted = case
    x = _x(B, H, T, D, seed=len(name), planted=planted)
    sp, cnt = _detect_gpu(K, x, t0, tau, M)
    osp, ocnt = orc.detect_sinks(x.view(np.uint16), np.arange(t0, t0 + T), tau=tau, max_sinks=M)
    assert np.array_equal(cnt, ocnt) and np.array_equal(sp, osp), (sp, osp)


def test_detect_ties_cap_and_strict_threshold(K, orc):
    """Equal magnitudes above the cut (the earlier tokens win), the largest
    taken first, a token exactly at tau * median (not a sink) and one fp16
    step above it; a sequence whose median is zero."""
    T = 2100
    x = np.zeros((3, 2, T, 64), np.float16)
    x[0, 0, :, 0] = np.float16(1.0)
    for t in (3, 900, 1500, 2000, 2099):
        x[0, 1, t, 5] = np.float16(64.0)
    x[0, 0, 1700, 9] = np.float16(-128.0)
    x[1, 0, :, 3] = np.float16(1.0)
    x[1, 1, 11, 0] = np.float16(4.0)  # exactly tau * median
    x[1, 1, 1234, 0] = np.float16(4.00390625)
    x[2, 1, 600, 1] = np.float16(1e-3)  # median zero: every nonzero token clears it
    x[2, 0, 7, 2] = np.float16(-2.0)
    for tau in (4.0, 10.0):
        sp, cnt = _detect_gpu(K, x, 0, tau, 3)
        osp, ocnt = orc.detect_sinks(x.view(np.uint16), np.arange(T), tau=tau, max_sinks=3)
        assert np.array_equal(sp, osp) and np.array_equal(cnt, ocnt), (tau, sp, osp)
    assert sp[0].tolist() == [3, 900, 1700] and sp[2].tolist() == [7, 600, -1]


def test_detect_full_size(K, orc):
    """The Llama-2-7B prefill shape (8 sequences x 32 heads x 4096 tokens x 128)
    with planted massive tokens: the GPU list equals the oracle's."""
    w = W.WORKLOADS["llama2_7b_mha"]
    x = W.kv_tensor(w, "k")
    planted = W.plant_massive(x, 4, 11)
    sp, cnt = _detect_gpu(K, x, 0, 8.0, 8)
    osp, ocnt = orc.detect_sinks(x.view(np.uint16), np.arange(w.T), tau=8.0, max_sinks=8)
    assert np.array_equal(sp, osp) and np.array_equal(cnt, ocnt)
    for b in range(w.B):  # the planted tokens are found
        assert set(planted[b]) <= set(sp[b].tolist())


def test_detect_rejects(K):
    from kv_cache_rotation_b200 import torch_api as TA
    x = torch.zeros((1, 2, 8, 64), dtype=torch.float16, device="cuda")
    d = TA.make_desc(batch=1, heads=2, head_dim=64, tokens=8, t_cap=8, bits=2, group=64)
    sp = torch.empty((1, 4), dtype=torch.int32, device="cuda")
    ws = TA.detect_sinks_workspace(d)
    assert K.kvq_detect_sinks(d, x.data_ptr(), float("inf"), 4, sp.data_ptr(), 0, ws.data_ptr(), ws.numel(),
                              0) == K.KVQ_ERR_INVALID
    assert K.kvq_detect_sinks(d, x.data_ptr(), 2.0, 0, sp.data_ptr(), 0, ws.data_ptr(), ws.numel(),
                              0) == K.KVQ_ERR_INVALID
    assert K.kvq_detect_sinks(d, x.data_ptr(), 2.0, 4, sp.data_ptr(), 0, ws.data_ptr(), 15, 0) == K.KVQ_ERR_INVALID
    d0 = TA.make_desc(batch=1, heads=2, head_dim=64, tokens=0, t_cap=8, bits=2, group=64)
    assert K.kvq_detect_sinks(d0, x.data_ptr(), 2.0, 4, sp.data_ptr(), 0, ws.data_ptr(), ws.numel(),
                              0) == K.KVQ_ERR_INVALID
    assert K.kvq_detect_sinks(d, x.data_ptr() + 2, 2.0, 4, sp.data_ptr(), 0, ws.data_ptr(), ws.numel(),
                              0) == K.KVQ_ERR_ALIGN


# ------------------------------------------------------------------ list form
LIST = [
    # name, rot, B, H, T, D, t0, bits, group, hg, rope, perm
    ("head_rope", "fwht_head", 2, 4, 37, 128, 0, 2, 64, 1, 1, True),
    ("head_half_split_t0", "fwht_head", 2, 4, 30, 128, 9, 3, 32, 1, 2, False),
    ("head_d64", "fwht_head", 1, 8, 40, 64, 2, 4, 32, 1, 1, True),
    ("none_values", "none", 2, 4, 33, 128, 0, 4, 128, 1, 0, False),
    ("group_hg8", "fwht_group", 1, 8, 40, 128, 0, 2, 128, 8, 1, True),
    ("group_hg2_half_t0", "fwht_group", 2, 4, 25, 128, 5, 3, 64, 2, 2, False),
    ("iso_so4", "iso", 2, 2, 30, 128, 0, 3, 0, 1, 0, False),
    ("iso_so3_d64", "iso3", 2, 2, 30, 64, 4, 2, 0, 1, 0, False),
]
ORC_ROT = {"none": 0, "fwht_head": 1, "fwht_group": 2, "iso": 3, "iso3": 4}


def _orope(orc, rope):
    return {0: 0, 1: orc.ROPE_STD, 2: orc.ROPE_STD + orc.ROPE_HALF}[rope]


def _lists(B, n_sink, lo, hi, seed):
    """[B][n_sink] distinct positions in [lo, hi) and some -1 entries (and one
    position outside this call's range for the t0 > 0 cases)."""
    rng = np.random.default_rng(seed)
    sp = np.full((B, n_sink), -1, np.int32)
    for b in range(B):
        k = min(n_sink - b % 2, hi - lo)
        sp[b, :k] = np.sort(rng.choice(np.arange(lo, hi), size=k, replace=False))
    return sp


@pytest.mark.parametrize("case", LIST, ids=[c[0] for c in LIST])
def test_list_encode_decode(K, orc, case):
    from kv_cache_rotation_b200 import torch_api as TA
    name, rot, B, H, T, D, t0, bits, group, hg, rope, use_perm = case
    iso = rot in ("iso", "iso3")
    w = W.Workload(name, B=B, H=H, T=T, D=D, seed=len(name), dist="student_t" if iso else "normal_outliers")
    x = W.kv_tensor(w, "k")
    n_sink = 4
    sp = _lists(B, n_sink, max(0, t0 - 2), t0 + T, 5)  # t0 > 0: some entries lie before this call
    t_cap = t0 + T + 3
    perm = W.random_perm(H, D, 3) if use_perm else None
    d = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, t0=t0, t_cap=t_cap, bits=bits, group=group or 128,
                     group_heads=hg, rope=rope, n_sink=n_sink, rot=rot, quant="codebook" if iso else "minmax")
    okw = dict(rot=ORC_ROT[rot], bits=bits, n_sink=n_sink, rope=_orope(orc, rope))
    tkw = dict(sink_pos=torch.from_numpy(sp).cuda())
    if iso:
        qL, qR = (W.iso3_tables(D, 61), None) if rot == "iso3" else W.iso_tables(w)
        cb = TA.lloyd_max_codebook(bits, D)
        tkw.update(qL=torch.from_numpy(qL).cuda(), qR=torch.from_numpy(qR).cuda() if qR is not None else None,
                   codebook=cb)
        okw.update(quant=orc.Q_CODEBOOK, qL=qL, qR=qR, cb=cb.cpu().numpy())
    else:
        okw.update(group=group, group_heads=hg, perm=perm)
        if perm is not None:
            tkw["perm"] = torch.from_numpy(perm).cuda()
        if rope:
            tkw["rope_cs"] = TA.rope_table(t_cap, D)
    tb = TA.make_tables(**tkw)
    pk = TA.alloc_packed(d)
    TA.encode(d, torch.from_numpy(x).cuda(), tb, pk)
    assert K.kvq_check(0) == K.KVQ_OK
    pos = np.arange(t0, t0 + T)
    ref = orc.encode(x.view(np.uint16), pos, want_pre=True, sink_pos=sp, **okw)
    gc = pk.codes[:, :, t0:t0 + T].cpu().numpy()
    if iso:
        rep = compare_codebook(gc, ref["codes"], ref["pre"], okw["cb"], D, bits)
        gn = pk.norm[:, :, t0:t0 + T].cpu().numpy()
        assert np.array_equal(gn.view(np.uint32), ref["norm"].view(np.uint32))
        packed_np = {"codes": gc, "norm": gn}
    else:
        gs = pk.scale_zero[:, :, t0:t0 + T].cpu().numpy()
        rep = compare_minmax(gc, ref["codes"], gs, ref["sz"].view(np.int16), ref["pre"], D, bits, group)
        packed_np = {"codes": gc, "sz": gs.view(np.uint16)}
    assert rep.ok and rep.mismatched == 0, rep
    gsink = pk.sink.cpu().numpy().view(np.uint16)
    for b in range(B):
        for k, m in enumerate(sp[b]):
            if t0 <= m < t0 + T:  # rows of this call's sinks, verbatim
                assert np.array_equal(gsink[b, :, k], ref["sink"][b, :, k])
                assert np.array_equal(gsink[b, :, k], x[b, :, m - t0].view(np.uint16))
    packed_np["sink"] = gsink
    out32 = torch.empty((B, H, T, D), dtype=torch.float32, device="cuda")
    out16 = torch.empty((B, H, T, D), dtype=torch.float16, device="cuda")
    TA.decode(d, pk, tb, out32)
    TA.decode(d, pk, tb, out16)
    assert K.kvq_check(0) == K.KVQ_OK
    dec = orc.decode(packed_np, pos, x.shape, sink_pos=sp, **okw)
    o32 = out32.cpu().numpy()
    err = np.abs(o32.astype(np.float64) - dec)
    assert np.all(err <= recon_tolerance(dec)), err.max()
    assert np.array_equal(out16.cpu().numpy().view(np.uint16), o32.astype(np.float16).view(np.uint16))


def test_list_of_prefix_equals_prefix_form(K):
    """The list 0 .. n_sink-1 gives the prefix form's bytes and decode."""
    from kv_cache_rotation_b200 import torch_api as TA
    B, H, T, D, S = 2, 8, 50, 128, 4
    x = torch.from_numpy(_x(B, H, T, D, 9, planted=0)).cuda()
    d = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, t_cap=T, bits=2, group=64, rope=1, n_sink=S)
    cs = TA.rope_table(T, D)
    a, b = TA.alloc_packed(d), TA.alloc_packed(d)
    ta = TA.make_tables(rope_cs=cs)
    tl = TA.make_tables(rope_cs=cs, sink_pos=torch.arange(S, dtype=torch.int32, device="cuda").repeat(B, 1))
    TA.encode(d, x, ta, a)
    TA.encode(d, x, tl, b)
    for f in ("codes", "scale_zero", "sink"):
        assert torch.equal(getattr(a, f), getattr(b, f))
    oa = torch.empty((B, H, T, D), dtype=torch.float32, device="cuda")
    ob = torch.empty_like(oa)
    TA.decode(d, a, ta, oa)
    TA.decode(d, b, tl, ob)
    assert torch.equal(oa, ob)
    q = torch.randn((B, 2 * H, D), device="cuda").half()
    sa = torch.empty((B, 2 * H, T), dtype=torch.float32, device="cuda")
    sb = torch.empty_like(sa)
    TA.score(d, q, a, ta, T, 0.1, sa)
    TA.score(d, q, b, tl, T, 0.1, sb)
    assert K.kvq_check(0) == K.KVQ_OK
    # coded slots: the same kernel and arithmetic; sink slots: the same fp32
    # dot product summed in another order
    assert torch.equal(sa[:, :, S:], sb[:, :, S:])
    torch.testing.assert_close(sa[:, :, :S], sb[:, :, :S], rtol=1e-5, atol=1e-4)


SCORE = [
    # name, rot, B, H, GQ, T, rope, hg, group
    ("head_gq4", "fwht_head", 2, 4, 4, 300, 1, 1, 128),
    ("head_half_split_g64", "fwht_head", 1, 8, 2, 150, 2, 1, 64),
    ("none_norope", "none", 2, 2, 1, 90, 0, 1, 128),
    ("group_hg8_gq4", "fwht_group", 1, 8, 4, 200, 1, 8, 128),
    ("group_hg2_half", "fwht_group", 2, 4, 2, 120, 2, 2, 128),
]


LITERAL = [(c, True) for c in SCORE if c[1] != "fwht_group"]


@pytest.mark.parametrize("case,literal", [(c, False) for c in SCORE] + LITERAL,
                         ids=[c[0] for c in SCORE] + [c[0] + "_literal" for c, _ in LITERAL])
def test_list_score(K, orc, case, literal):
    from kv_cache_rotation_b200 import torch_api as TA
    name, rot, B, H, GQ, T, rope, hg, group = case
    D, bits, n_sink, scale = 128, 2, 4, 0.0884
    # the tokens with massive activations are the sinks (the method keeps them
    # in fp16), plus one more listed position in even sequences
    x = _x(B, H, T, D, len(name), planted=0)
    planted = W.plant_massive(x, 3, len(name))
    rng = np.random.default_rng(7)
    sp = np.full((B, n_sink), -1, np.int32)
    for b in range(B):
        extra = [] if b % 2 else [int(rng.choice([t for t in range(T) if t not in planted[b]]))]
        lst = sorted(planted[b] + extra)
        sp[b, :len(lst)] = lst
    d = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, t_cap=T, bits=bits, group=group, group_heads=hg,
                     rope=rope, n_sink=n_sink, rot=rot)
    tb = TA.make_tables(rope_cs=TA.rope_table(T, D) if rope else None, sink_pos=torch.from_numpy(sp).cuda())
    pk = TA.alloc_packed(d)
    TA.encode(d, torch.from_numpy(x).cuda(), tb, pk)
    q = np.random.default_rng(3).standard_normal((B, H * GQ, D)).astype(np.float16)
    out = torch.empty((B, H * GQ, T), dtype=torch.float32, device="cuda")
    (TA.score_literal if literal else TA.score)(d, torch.from_numpy(q).cuda(), pk, tb, T, scale, out)
    assert K.kvq_check(0) == K.KVQ_OK
    okw = dict(rot=ORC_ROT[rot], bits=bits, group=group, group_heads=hg, rope=_orope(orc, rope), n_sink=n_sink)
    cache = {"codes": pk.codes.cpu().numpy(), "sz": pk.scale_zero.cpu().numpy().view(np.uint16),
             "sink": pk.sink.cpu().numpy().view(np.uint16)}
    toks = np.arange(T)
    ref = orc.score(q.view(np.uint16), cache, toks, H=H, t_cap=T, scale=scale, sink_pos=sp, **okw)
    # keys in attention space (fp64) for the L1 bound
    khat = orc.decode(cache, toks, (B, H, T, D), sink_pos=sp, **okw)
    g = out.cpu().numpy()
    for b in range(B):
        for qh in range(H * GQ):
            h = qh // GQ
            kk = np.stack([orc.rope_f64(khat[b, h, n], n, mode=okw["rope"]) for n in toks]) if rope else khat[b, h]
            tol = score_tolerance(q[b, qh], kk.T, scale)
            assert np.all(np.abs(g[b, qh] - ref[b, qh]) <= tol), (b, qh)


def test_list_calibrate(K, orc):
    from kv_cache_rotation_b200 import torch_api as TA
    B, H, T, D, S = 2, 4, 300, 128, 3
    x = _x(B, H, T, D, 21, planted=3)
    sp = _lists(B, S, 0, T, 9)
    for rope in (0, 1, 2):
        d = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, t_cap=T, bits=2, group=64, rope=rope, n_sink=S)
        tb = TA.make_tables(rope_cs=TA.rope_table(T, D) if rope else None, sink_pos=torch.from_numpy(sp).cuda())
        perm = TA.calibrate_perm(d, torch.from_numpy(x).cuda(), tb).cpu().numpy()
        ref = orc.calibrate_perm(x.view(np.uint16), np.arange(T), rope=_orope(orc, rope), n_sink=S, sink_pos=sp)
        assert np.array_equal(perm, ref), rope


def test_list_attend_needs_both_tables(K):
    """A sink list goes with both caches; naming it for the keys only is an error."""
    from kv_cache_rotation_b200 import torch_api as TA
    B, H, T, D = 1, 2, 16, 128
    dk = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, t_cap=T, bits=2, group=128, rope=1, n_sink=2)
    dv = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, t_cap=T, bits=2, group=128, rope=0, n_sink=2)
    sp = torch.tensor([[3, 7]], dtype=torch.int32, device="cuda")
    tk = TA.make_tables(rope_cs=TA.rope_table(T, D), sink_pos=sp)
    tv = TA.make_tables()
    kp, vp = TA.alloc_packed(dk), TA.alloc_packed(dv)
    q = torch.zeros((B, H, D), dtype=torch.float16, device="cuda")
    out = torch.empty((B, H, D), dtype=torch.float32, device="cuda")
    ws = TA.attend_workspace(dk, dv, H, T)
    with pytest.raises(K.KvqError) as e:
        TA.attend(dk, dv, q, kp, tk, vp, tv, T, 0.1, out, ws)
    assert e.value.status == K.KVQ_ERR_INVALID
    with pytest.raises(K.KvqError) as e:
        TA.attend_noalloc(dk, dv, q, kp, tk, vp, tv, T, 0.1, out)
    assert e.value.status == K.KVQ_ERR_INVALID
    tr = TA.make_tables(rope_cs=TA.rope_table(8, D), sink_pos=sp)  # RoPE rows must reach n_tokens
    with pytest.raises(K.KvqError) as e:
        TA.attend(dk, dv, q, kp, tr, vp, TA.make_tables(sink_pos=sp), T, 0.1, out, ws)
    assert e.value.status == K.KVQ_ERR_INVALID


def test_detect_then_encode_end_to_end(K, orc):
    """Prefill with detected sinks: the GPU's detected list drives the GPU's
    encode; the oracle's list drives the oracle's; lists and bytes agree."""
    from kv_cache_rotation_b200 import torch_api as TA
    B, H, T, D, S = 2, 8, 500, 128, 4
    x = _x(B, H, T, D, 33, planted=3)
    xg = torch.from_numpy(x).cuda()
    d = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, t_cap=T, bits=2, group=64, rope=1, n_sink=S)
    spg, _ = TA.detect_sinks(d, xg, tau=8.0, max_sinks=S)
    tb = TA.make_tables(rope_cs=TA.rope_table(T, D), sink_pos=spg)
    pk = TA.alloc_packed(d)
    TA.encode(d, xg, tb, pk)
    assert K.kvq_check(0) == K.KVQ_OK
    osp, _ = orc.detect_sinks(x.view(np.uint16), np.arange(T), tau=8.0, max_sinks=S)
    assert np.array_equal(spg.cpu().numpy(), osp)
    ref = orc.encode(x.view(np.uint16), np.arange(T), want_pre=True, rot=1, bits=2, group=64, rope=orc.ROPE_STD,
                     n_sink=S, sink_pos=osp)
    rep = compare_minmax(pk.codes.cpu().numpy(), ref["codes"], pk.scale_zero.cpu().numpy(),
                         ref["sz"].view(np.int16), ref["pre"], D, 2, 64)
    assert rep.ok and rep.mismatched == 0, rep
    assert np.array_equal(pk.sink.cpu().numpy().view(np.uint16), ref["sink"])
