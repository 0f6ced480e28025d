"""Race check by repetition: every kernel family run twice on the same inputs
must produce the same bytes. The kernels are deterministic by construction
(no floating-point atomics; the integer and max atomics of the calibration
and pair-energy reductions are order-independent), so a difference would
point at a read-before-write race on shared or global memory."""
import numpy as np
import pytest

import workloads as W

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def TA():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from kv_cache_rotation_b200 import torch_api as TA
    return TA


def _twice(f):
    a = f()
    b = f()
    torch.cuda.synchronize()
    return a, b


def test_grouped_encode_decode_repeat(TA):
    w = W.Workload("det_group", B=1, H=8, T=300, D=128, rot="fwht_group", group_heads=8, bits=2, group=128)
    x = torch.from_numpy(W.kv_tensor(w, "k")).cuda()
    d = TA.make_desc(batch=1, heads=8, head_dim=128, tokens=300, bits=2, group=128, group_heads=8, rope=1,
                     rot="fwht_group")
    tb = TA.make_tables(rope_cs=TA.rope_table(300, 128))

    def enc():
        pk = TA.alloc_packed(d)
        TA.encode(d, x, tb, pk)
        out = torch.empty((1, 8, 300, 128), dtype=torch.float16, device="cuda")
        TA.decode(d, pk, tb, out)
        return pk.codes.clone(), pk.scale_zero.clone(), out
    (c1, s1, o1), (c2, s2, o2) = _twice(enc)
    assert torch.equal(c1, c2) and torch.equal(s1, s2) and torch.equal(o1, o2)


def test_score_and_attention_repeat(TA):
    B, H, Hq, T, D = 2, 2, 8, 700, 128
    w = W.Workload("det_attend", B=B, H=H, Hq=Hq, T=T, D=D, bits=2, group=128, n_sink=4, seed=3)
    common = dict(batch=B, heads=H, head_dim=D, tokens=T, t_cap=T, bits=2, group=128, n_sink=4, rot="fwht_head")
    dk, dv = TA.make_desc(rope=1, **common), TA.make_desc(rope=0, **common)
    tk = TA.make_tables(rope_cs=TA.rope_table(T, D))
    tv = TA.make_tables()
    pk, pv = TA.alloc_packed(dk), TA.alloc_packed(dv)
    TA.encode(dk, torch.from_numpy(W.kv_tensor(w, "k")).cuda(), tk, pk)
    TA.encode(dv, torch.from_numpy(W.kv_tensor(w, "v")).cuda(), tv, pv)
    q = torch.from_numpy(W.queries(w)).cuda()
    ws = TA.attend_workspace(dk, dv, Hq, T)

    def run():
        s = torch.empty((B, Hq, T), dtype=torch.float32, device="cuda")
        TA.score(dk, q, pk, tk, T, 0.088, s)
        o = torch.empty((B, Hq, D), dtype=torch.float32, device="cuda")
        TA.attend(dk, dv, q, pk, tk, pv, tv, T, 0.088, o, ws)
        return s, o
    (s1, o1), (s2, o2) = _twice(run)
    assert torch.equal(s1, s2) and torch.equal(o1, o2)


def test_calibration_and_energy_repeat(TA):
    w = W.Workload("det_cal", B=2, H=4, T=3000, D=128, outliers=("pairs", 0.02, 10.0, 50.0))
    x = torch.from_numpy(W.kv_tensor(w, "k")).cuda()
    d = TA.make_desc(batch=2, heads=4, head_dim=128, tokens=3000, bits=2, group=128, rope=1, n_sink=4)
    tb = TA.make_tables(rope_cs=TA.rope_table(3000, 128))
    (p1, p2) = _twice(lambda: TA.calibrate_perm(d, x, tb).clone())
    assert torch.equal(p1, p2)
    (e1, e2) = _twice(lambda: tuple(t.cpu() for t in TA.pair_energy(d, x)))
    assert np.array_equal(e1[0].numpy(), e2[0].numpy()) and torch.equal(e1[1], e2[1])


def test_sink_detection_and_dynamic_tables_repeat(TA):
    w = W.Workload("det_sinks", B=3, H=4, T=2500, D=128, outliers=("pairs", 0.03, 10.0, 50.0))
    xn = W.kv_tensor(w, "k")
    W.plant_massive(xn, 5, 2)
    x = torch.from_numpy(xn).cuda()
    d = TA.make_desc(batch=3, heads=4, head_dim=128, tokens=2500, bits=3, rot="iso", quant="codebook_dyn")
    (s1, s2) = _twice(lambda: tuple(t.clone() for t in TA.detect_sinks(d, x, tau=4.0, max_sinks=16)))
    assert torch.equal(s1[0], s2[0]) and torch.equal(s1[1], s2[1])
    qL, qR = W.unit_quaternions(32, 1, 30), W.unit_quaternions(32, 1, 31)
    tb = TA.make_tables(qL=torch.from_numpy(qL).cuda(), qR=torch.from_numpy(qR).cuda())
    (c1, c2) = _twice(lambda: tuple(t.clone() for t in TA.calibrate_codebook(d, x, tb)))
    assert torch.equal(c1[0], c2[0]) and torch.equal(c1[1], c2[1])


def test_isoquant_repeat(TA):
    """Fixed (SO(4), 3-D) and dynamic codebooks: encode and decode twice, same bytes."""
    B, H, T, D, bits = 2, 2, 300, 128, 3
    w = W.Workload("det_iso", B=B, H=H, T=T, D=D, dist="student_t", seed=3)
    x = torch.from_numpy(W.kv_tensor(w, "k")).cuda()
    qL4, qR4 = W.unit_quaternions(D // 4, 3, 30), W.unit_quaternions(D // 4, 3, 31)
    for rot, quant in (("iso", "codebook"), ("iso3", "codebook"), ("iso", "codebook_dyn")):
        d = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, bits=bits, rot=rot, quant=quant)
        qL = W.iso3_tables(D, 5) if rot == "iso3" else qL4
        tb = TA.make_tables(qL=torch.from_numpy(qL).cuda(),
                            qR=torch.from_numpy(qR4).cuda() if rot == "iso" else None)
        if quant == "codebook_dyn":
            tb.codebook = TA.lloyd_max_codebook(bits, 1)
            tb.codebook_wide = TA.lloyd_max_codebook(bits + 1, 1)
            tb.ch_scale, tb.ch_wide = TA.calibrate_codebook(d, x, tb)
        else:
            tb.codebook = TA.lloyd_max_codebook(bits, D)

        def run():
            pk = TA.alloc_packed(d, zero=False)
            TA.encode(d, x, tb, pk)
            out = torch.empty((B, H, T, D), dtype=torch.float32, device="cuda")
            TA.decode(d, pk, tb, out)
            return pk, out
        (p1, o1), (p2, o2) = _twice(run)
        assert torch.equal(p1.codes, p2.codes) and torch.equal(p1.norm, p2.norm) and torch.equal(o1, o2)
        if quant == "codebook_dyn":
            assert torch.equal(p1.ext, p2.ext)
