"""GPU parity of the decode-step score kernel: the cache is written by the
GPU encoder (prefill + one appended token), and the GPU scores are compared
with the oracle's fp64 scores computed from that same cache, within
|s_gpu - s_orc| <= 1e-3 * scale * sum_j |q_j khat_j|."""
import math

import numpy as np
import pytest

import workloads as W
from parity import SCORE_REL

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_rotation_b200 as K
    return K


def build_cache(K, w, x, x_app, perm, rot="fwht_head", rope=1):
    from kv_cache_rotation_b200 import torch_api as TA
    B, H, T, D = x.shape
    t_cap = T + x_app.shape[2]
    kw = dict(batch=B, heads=H, head_dim=D, t_cap=t_cap, bits=w.bits, group=w.group, rope=rope, n_sink=w.n_sink,
              rot=rot, group_heads=w.group_heads)
    tb = TA.make_tables(perm=torch.from_numpy(perm).cuda() if perm is not None else None,
                        rope_cs=TA.rope_table(t_cap, D))
    d_pre = TA.make_desc(tokens=T, t0=0, **kw)
    pk = TA.alloc_packed(d_pre)
    TA.encode(d_pre, torch.from_numpy(x).cuda(), tb, pk)
    d_app = TA.make_desc(tokens=x_app.shape[2], t0=T, **kw)
    TA.encode(d_app, torch.from_numpy(x_app).cuda(), tb, pk)
    assert K.kvq_check(0) == K.KVQ_OK
    return d_pre, tb, pk


def run_score_case(K, orc, w, perm, rot="fwht_head", tokens=None, rope=1, literal=False):
    from kv_cache_rotation_b200 import torch_api as TA
    x = W.kv_tensor(w, "k")
    x_app = W.kv_tensor(w, "k_append", T=w.append)
    d, tb, pk = build_cache(K, w, x, x_app, perm, rot, rope)
    orope = 0 if rope == 0 else orc.ROPE_STD + (orc.ROPE_HALF if rope == 2 else 0)
    q = W.queries(w)
    n_tok = d.t_cap
    scale = 1.0 / math.sqrt(w.D)
    out = torch.full((w.B, w.Hq, n_tok), float("nan"), dtype=torch.float32, device="cuda")
    (TA.score_literal if literal else TA.score)(d, torch.from_numpy(q).cuda(), pk, tb, n_tok, scale, out)
    assert K.kvq_check(0) == K.KVQ_OK
    tok = np.arange(n_tok) if tokens is None else np.asarray(tokens)
    cache = {"codes": pk.codes.cpu().numpy(), "sz": pk.scale_zero.cpu().numpy().view(np.uint16),
             "sink": pk.sink.cpu().numpy().view(np.uint16) if w.n_sink else None}
    okw = dict(rot={"none": 0, "fwht_head": 1, "fwht_group": 2}[rot], bits=w.bits, group=w.group,
               group_heads=w.group_heads, rope=orope, n_sink=w.n_sink, perm=perm)
    ref = orc.score(q.view(np.uint16), cache, tok, H=w.H, t_cap=n_tok, scale=scale, **okw)
    # attention-space keys (fp64) for the L1 bound
    khat = orc.decode(cache, np.arange(n_tok), (w.B, w.H, n_tok, w.D), **okw)
    got = out.cpu().numpy()[:, :, tok]
    gq = w.Hq // w.H
    worst = 0.0
    for b in range(w.B):
        for qh in range(w.Hq):
            h = qh // gq
            kk = np.stack([orc.rope_f64(khat[b, h, n], n, mode=orope) for n in tok]) if rope else khat[b, h, tok]
            bound = SCORE_REL * scale * (np.abs(kk) @ np.abs(q[b, qh].astype(np.float64)))
            err = np.abs(got[b, qh] - ref[b, qh])
            assert np.all(err <= bound), (b, qh, np.max(err / bound))
            worst = max(worst, float(np.max(err / bound)))
    assert np.isfinite(out.cpu().numpy()).all()
    return worst


def test_score_mha_perm_sinks(K, orc):
    w = W.scaled(W.WORKLOADS["decode_score"], B=2, H=4, Hq=4, T=300)
    run_score_case(K, orc, w, W.random_perm(w.H, w.D, 11))


def test_score_gqa(K, orc):
    w = W.scaled(W.WORKLOADS["llama3_8b_gqa_score"], B=2, H=2, Hq=8, T=257)
    run_score_case(K, orc, w, None)


@pytest.mark.parametrize("bits,group", [(3, 32), (4, 128), (3, 64)])
def test_score_bits(K, orc, bits, group):
    w = W.scaled(W.WORKLOADS["decode_score"], B=1, H=2, Hq=4, T=130, bits=bits, group=group, n_sink=1)
    run_score_case(K, orc, w, W.random_perm(w.H, w.D, 2))


@pytest.mark.parametrize("bits,group,gq", [(2, 32, 2), (4, 32, 1), (4, 64, 8), (2, 64, 4)])
def test_score_mma_groups(K, orc, bits, group, gq):
    """The tensor-core score with 2 and 4 quantization groups per record (head_dim 128)."""
    w = W.scaled(W.WORKLOADS["decode_score"], B=2, H=2, Hq=2 * gq, T=161, bits=bits, group=group, n_sink=3)
    run_score_case(K, orc, w, W.random_perm(w.H, w.D, 9))


def test_score_no_rotation(K, orc):
    w = W.scaled(W.WORKLOADS["decode_score"], B=1, H=2, Hq=2, T=70, n_sink=0)
    run_score_case(K, orc, w, None, rot="none")


def test_score_d64(K, orc):
    w = W.scaled(W.WORKLOADS["decode_score"], B=2, H=2, Hq=2, T=64, D=64, group=32)
    run_score_case(K, orc, w, W.random_perm(2, 64, 5))


@pytest.mark.parametrize("hg,gq,bits,group,n_sink,T", [(8, 4, 2, 128, 0, 300), (8, 1, 4, 128, 2, 97),
                                                       (4, 2, 2, 128, 3, 150), (8, 8, 2, 64, 0, 61)])
def test_score_grouped_cache(K, orc, hg, gq, bits, group, n_sink, T):
    """A grouped-head cache (FWHT over hg heads x 128 before RoPE): every slot is
    decoded, turned by RoPE_n and dotted with the query heads of its KV head."""
    w = W.Workload("score_group", B=2, H=hg, T=T, rot="fwht_group", group_heads=hg, bits=bits, group=group,
                   n_sink=n_sink, Hq=hg * gq, append=1, seed=70 + hg + gq)
    run_score_case(K, orc, w, None, rot="fwht_group")


@pytest.mark.parametrize("rot,bits,group,D", [("fwht_head", 2, 128, 128), ("fwht_head", 3, 64, 128),
                                              ("fwht_head", 2, 32, 64)])
def test_score_half_split_sinks(K, orc, rot, bits, group, D):
    """Keys with half-split RoPE pairs: the fp16 sinks are turned on (i, i + D/2)
    (tensor-core and CUDA-core score kernels)."""
    w = W.scaled(W.WORKLOADS["decode_score"], B=2, H=2, Hq=4, T=150, D=D, bits=bits, group=group, n_sink=4)
    run_score_case(K, orc, w, W.random_perm(w.H, D, 12), rot=rot, rope=2)


def test_score_grouped_cache_half_split(K, orc):
    w = W.Workload("score_group_half", B=1, H=8, T=120, rot="fwht_group", group_heads=8, bits=2, group=128,
                   n_sink=3, Hq=16, append=1, seed=91)
    run_score_case(K, orc, w, None, rot="fwht_group", rope=2)


LITERAL = [
    # name, workload, overrides, perm seed (None: no permutation), rot, rope
    ("mha_perm_sinks_g64", "decode_score", dict(B=2, H=4, Hq=4, T=300), 11, "fwht_head", 1),
    ("gqa4_g128", "llama3_8b_gqa_score", dict(B=2, H=2, Hq=8, T=257), None, "fwht_head", 1),
    ("gq2_b3_g32", "decode_score", dict(B=1, H=2, Hq=4, T=130, bits=3, group=32, n_sink=1), 2, "fwht_head", 1),
    ("gq8_b4_g128", "decode_score", dict(B=1, H=2, Hq=16, T=97, bits=4, group=128, n_sink=2), 5, "fwht_head", 1),
    ("b3_g64_half_split", "decode_score", dict(B=2, H=2, Hq=4, T=150, bits=3, group=64, n_sink=4), 12,
     "fwht_head", 2),
    ("no_rotation", "decode_score", dict(B=1, H=2, Hq=2, T=70, n_sink=0), None, "none", 1),
    ("no_rope_b4_g32", "decode_score", dict(B=2, H=2, Hq=2, T=45, bits=4, group=32, n_sink=3), 8, "fwht_head", 0),
    ("only_sinks", "llama3_8b_gqa_score", dict(B=1, H=2, Hq=8, T=2, n_sink=4), None, "fwht_head", 1),
]


def test_score_only_sinks(K, orc):
    """Fewer cached slots than sinks: every score is a sink's exact dot."""
    w = W.scaled(W.WORKLOADS["llama3_8b_gqa_score"], B=1, H=2, Hq=8, T=2, n_sink=4)
    run_score_case(K, orc, w, None)


@pytest.mark.parametrize("case", LITERAL, ids=[c[0] for c in LITERAL])
def test_score_literal(K, orc, case):
    """The literal per-token form (every key unpacked, dequantized and inverse-
    transformed before the dot) against the same oracle scores."""
    name, wl, over, pseed, rot, rope = case
    w = W.scaled(W.WORKLOADS[wl], **over)
    perm = W.random_perm(w.H, w.D, pseed) if pseed is not None else None
    worst = run_score_case(K, orc, w, perm, rot=rot, rope=rope, literal=True)
    print(f"{name}: worst |err| / S2 bound = {worst:.3g}")


def test_score_literal_matches_query_rotation(K):
    """Both score forms over one cache: equal within the S2 bound's scale (the
    query-rotation kernel rounds the rotated query to 16-bit digits)."""
    from kv_cache_rotation_b200 import torch_api as TA
    w = W.scaled(W.WORKLOADS["llama3_8b_gqa_score"], B=2, H=2, Hq=8, T=513)
    d, tb, pk = build_cache(K, w, W.kv_tensor(w, "k"), W.kv_tensor(w, "k_append", T=w.append), None)
    q = torch.from_numpy(W.queries(w)).cuda()
    n = d.t_cap
    a = torch.empty((w.B, w.Hq, n), dtype=torch.float32, device="cuda")
    b = torch.empty_like(a)
    TA.score(d, q, pk, tb, n, 0.0884, a)
    TA.score_literal(d, q, pk, tb, n, 0.0884, b)
    assert K.kvq_check(0) == K.KVQ_OK
    assert torch.equal(a[:, :, :w.n_sink], b[:, :, :w.n_sink])  # the sinks take the same fp32 path
    torch.testing.assert_close(a, b, rtol=0, atol=1e-3 * float(b.abs().max()))


def test_score_literal_rejects(K):
    from kv_cache_rotation_b200 import torch_api as TA
    w = W.scaled(W.WORKLOADS["decode_score"], B=1, H=2, Hq=2, T=32, D=64, group=32)
    d, tb, pk = build_cache(K, w, W.kv_tensor(w, "k"), W.kv_tensor(w, "k_append", T=w.append), None)
    q = torch.zeros((1, 2, 64), dtype=torch.float16, device="cuda")
    out = torch.empty((1, 2, d.t_cap), dtype=torch.float32, device="cuda")
    assert K.kvq_score_literal(d, q.data_ptr(), 2, pk.struct(), tb.struct(), d.t_cap, 1.0, out.data_ptr(), 0) == \
        K.KVQ_ERR_UNSUPPORTED  # head_dim 64
