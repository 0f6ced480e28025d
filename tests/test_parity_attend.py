"""GPU parity of the decode-step attention (kvq_attend: "EliteKV -
RoPE频率选择与低秩投影" §2.2 scores, §7.1 softmax-weighted values). K and V
caches are written by the GPU encoder; the oracle reads those same caches.

Two checks per case:
  * tight: given the scores the GPU computes (kvq_score, same inputs), the
    softmax, the value accumulation in the rotated basis, the inverse rotation
    and the sink rows must match fp64 within 2e-5 * max|vhat| (fp32
    accumulation over at most a few thousand tokens);
  * end to end, against the oracle's scores: softmax weights move by at most
    a factor e^(2 * max|ds|), so |out - out_orc| <= (e^(2*ds_max) - 1) * max|vhat|
    + the tight bound, with ds_max the score contract's bound
    1e-3 * scale * sum_j |q_j khat_j|."""
import math

import numpy as np
import pytest

import workloads as W
from parity import SCORE_REL

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CASES = [
    # name, B, H, Hq, t_cap, n_tok, bits, group, n_sink, perm, rot
    ("gqa4_bits2_g128_sinks", 2, 2, 8, 300, 300, 2, 128, 4, False, "fwht_head"),
    ("mha_perm_g64_ragged", 1, 4, 4, 260, 257, 2, 64, 4, True, "fwht_head"),
    ("gqa2_bits3_g32", 1, 2, 4, 140, 130, 3, 32, 0, True, "fwht_head"),
    ("gqa8_bits4", 1, 1, 8, 129, 129, 4, 64, 2, False, "fwht_head"),
    ("no_rotation", 1, 2, 2, 64, 64, 2, 64, 2, True, "none"),
    ("single_token", 2, 2, 8, 16, 1, 2, 128, 0, False, "fwht_head"),
    ("sinks_only", 1, 2, 4, 16, 3, 2, 64, 4, True, "fwht_head"),
    ("gqa4_bits4_g32", 1, 2, 8, 100, 97, 4, 32, 2, True, "fwht_head"),
    ("gqa1_bits2_g32", 2, 2, 2, 150, 150, 2, 32, 0, False, "fwht_head"),
    # one group per record, 2 or 4 bits: the fused single-pass kernel
    ("fused_gqa4_perm_40_chunks", 1, 1, 4, 5000, 4999, 2, 128, 4, True, "fwht_head"),
    ("fused_gqa2_9_tiles_per_chunk", 2, 16, 32, 10000, 9990, 2, 128, 4, False, "fwht_head"),
    ("fused_gqa8_bits4_perm", 1, 2, 16, 700, 650, 4, 128, 4, True, "fwht_head"),
    ("fused_gqa1_no_rotation", 2, 2, 2, 300, 290, 2, 128, 0, False, "none"),
    ("fused_gqa2_bits4_ragged", 1, 2, 4, 200, 131, 4, 128, 2, False, "fwht_head"),
    ("fused_sinks_only", 1, 2, 8, 16, 3, 2, 128, 4, True, "fwht_head"),
    ("fused_single_token_no_sinks", 1, 1, 1, 8, 1, 4, 128, 0, False, "fwht_head"),
    # keys with half-split RoPE pairs (the fp16 sinks are turned on (i, i + 64))
    ("half_split_fused_sinks", 2, 2, 8, 300, 300, 2, 128, 4, True, "fwht_head"),
    ("half_split_three_kernel_sinks", 1, 2, 4, 260, 257, 2, 64, 4, True, "fwht_head"),
]
E2E_PAIRS = 8  # (batch, query head) pairs checked end to end on the larger cases


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_rotation_b200 as K
    return K


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_attend_parity(K, orc, case):
    from kv_cache_rotation_b200 import torch_api as TA
    name, B, H, Hq, t_cap, n_tok, bits, group, n_sink, use_perm, rot = case
    D = 128
    w = W.Workload(name, B=B, H=H, Hq=Hq, T=t_cap, D=D, bits=bits, group=group, n_sink=n_sink,
                   outliers=("pairs", 0.02, 10.0, 50.0))
    k, v, q = W.kv_tensor(w, "k"), W.kv_tensor(w, "v"), W.queries(w)
    kp = W.random_perm(H, D, 5) if use_perm else None
    vp = W.random_perm(H, D, 6) if use_perm else None
    common = dict(batch=B, heads=H, head_dim=D, tokens=t_cap, t_cap=t_cap, bits=bits, group=group,
                  n_sink=n_sink, rot=rot)
    krope = 2 if name.startswith("half_split") else 1  # 2: half-split RoPE pairs on the keys
    okrope = orc.ROPE_STD + (orc.ROPE_HALF if krope == 2 else 0)
    dk, dv = TA.make_desc(rope=krope, **common), TA.make_desc(rope=0, **common)
    tk = TA.make_tables(perm=torch.from_numpy(kp).cuda() if use_perm else None, rope_cs=TA.rope_table(t_cap, D))
    tv = TA.make_tables(perm=torch.from_numpy(vp).cuda() if use_perm else None)
    pk, pv = TA.alloc_packed(dk), TA.alloc_packed(dv)
    TA.encode(dk, torch.from_numpy(k).cuda(), tk, pk)
    TA.encode(dv, torch.from_numpy(v).cuda(), tv, pv)
    scale = 1.0 / math.sqrt(D)
    qg = torch.from_numpy(q).cuda()
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
    ws = TA.attend_workspace(dk, dv, Hq, n_tok)
    TA.attend(dk, dv, qg, pk, tk, pv, tv, n_tok, scale, out, ws)
    s_gpu = torch.empty((B, Hq, n_tok), dtype=torch.float32, device="cuda")
    TA.score(dk, qg, pk, tk, n_tok, scale, s_gpu)
    assert K.kvq_check(0) == K.KVQ_OK
    got, s_gpu = out.cpu().numpy().astype(np.float64), s_gpu.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got))

    rotv = {"none": 0, "fwht_head": 1}[rot]
    okw = dict(rot=rotv, bits=bits, group=group, n_sink=n_sink)
    kc = {"codes": pk.codes.cpu().numpy(), "sz": pk.scale_zero.cpu().numpy().view(np.uint16),
          "sink": pk.sink.cpu().numpy().view(np.uint16) if n_sink else None}
    vc = {"codes": pv.codes.cpu().numpy(), "sz": pv.scale_zero.cpu().numpy().view(np.uint16),
          "sink": pv.sink.cpu().numpy().view(np.uint16) if n_sink else None}
    pos = np.arange(t_cap)
    vhat = orc.decode(vc, pos, (B, H, t_cap, D), rope=0, perm=vp, **okw)[:, :, :n_tok]
    khat = orc.decode(kc, pos, (B, H, t_cap, D), rope=okrope, perm=kp, **okw)
    ref = orc.attend(q.view(np.uint16), kc, vc, n_tok, H=H, t_cap=t_cap, scale=scale, kperm=kp, vperm=vp,
                     krope=okrope, vrope=0, **okw)
    gq = Hq // H
    pairs = [(b, qh) for b in range(B) for qh in range(Hq)]
    e2e = set(pairs if len(pairs) <= E2E_PAIRS else
              [pairs[i] for i in np.random.default_rng(3).choice(len(pairs), E2E_PAIRS, replace=False)])
    krot = {}
    for b, qh in pairs:
        h = qh // gq
        vmax = np.abs(vhat[b, h]).max()
        # tight: the GPU's own scores through fp64 softmax and values
        sv = s_gpu[b, qh]
        p = np.exp(sv - sv.max())
        p /= p.sum()
        want = p @ vhat[b, h]
        tight = 2e-5 * vmax
        assert np.all(np.abs(got[b, qh] - want) <= tight), (b, qh, np.abs(got[b, qh] - want).max() / vmax)
        if (b, qh) not in e2e:
            continue
        # end to end against the oracle
        if (b, h) not in krot:
            krot[b, h] = np.stack([orc.rope_f64(khat[b, h, n], n, mode=okrope) for n in range(n_tok)])
        ds = SCORE_REL * scale * (np.abs(krot[b, h]) @ np.abs(q[b, qh].astype(np.float64)))
        bound = (math.exp(2 * ds.max()) - 1) * vmax + tight
        assert np.all(np.abs(got[b, qh] - ref[b, qh]) <= bound), (b, qh, np.abs(got[b, qh] - ref[b, qh]).max())


LISTED = [
    # name, B, H, Hq, t_cap, n_tok, bits, group, n_sink, perm, krope, noalloc
    ("fused_gqa4_list", 2, 2, 8, 600, 590, 2, 128, 4, True, 1, False),
    ("fused_bits4_half_split_list", 1, 2, 4, 300, 300, 4, 128, 3, False, 2, False),
    ("three_kernel_g64_list", 2, 2, 4, 400, 397, 2, 64, 4, True, 1, False),
    ("fused_list_noalloc", 1, 2, 8, 500, 500, 2, 128, 4, False, 1, True),
    ("fused_only_listed_tokens", 1, 1, 4, 16, 3, 2, 128, 4, False, 1, False),
    ("list_of_40_takes_three_kernels", 1, 2, 4, 300, 300, 2, 128, 40, False, 1, False),
]


def _sink_list(B, n_sink, n_tok, seed):
    """n_sink distinct positions per sequence, drawn below max(n_tok, n_sink) (so a
    list longer than the call names positions past n_tok), ascending."""
    rng = np.random.default_rng(seed)
    sp = np.full((B, n_sink), -1, np.int32)
    for b in range(B):
        n = n_sink
        cand = rng.choice(max(n_tok, n), size=min(n, max(n_tok, n)), replace=False)
        lst = sorted(int(c) for c in cand)
        sp[b, :len(lst)] = lst
    return sp


@pytest.mark.parametrize("case", LISTED, ids=[c[0] for c in LISTED])
def test_attend_listed_sinks(K, orc, case):
    """Caches whose sinks are a list of positions (both caches encoded with it):
    the listed slots enter with their exact fp16 scores and values."""
    from kv_cache_rotation_b200 import torch_api as TA
    name, B, H, Hq, t_cap, n_tok, bits, group, n_sink, use_perm, krope, noalloc = case
    D, rot = 128, "fwht_head"
    w = W.Workload(name, B=B, H=H, Hq=Hq, T=t_cap, D=D, bits=bits, group=group, n_sink=n_sink,
                   outliers=("pairs", 0.02, 10.0, 50.0))
    k, v, q = W.kv_tensor(w, "k"), W.kv_tensor(w, "v"), W.queries(w)
    planted = W.plant_massive(k, min(2, n_sink), len(name))  # tokens with massive keys, listed below
    sp = _sink_list(B, n_sink, n_tok, len(name))
    for b in range(B):  # every planted token is listed; drawn positions fill the rest (odd b: one -1 pad)
        rest = [int(x) for x in sp[b] if x >= 0 and int(x) not in planted[b]]
        lst = sorted(planted[b] + rest[:max(0, n_sink - len(planted[b]) - b % 2)])
        sp[b] = -1
        sp[b, :len(lst)] = lst
    kp = W.random_perm(H, D, 5) if use_perm else None
    vp = W.random_perm(H, D, 6) if use_perm else None
    common = dict(batch=B, heads=H, head_dim=D, tokens=t_cap, t_cap=t_cap, bits=bits, group=group,
                  n_sink=n_sink, rot=rot)
    okrope = orc.ROPE_STD + (orc.ROPE_HALF if krope == 2 else 0)
    dk, dv = TA.make_desc(rope=krope, **common), TA.make_desc(rope=0, **common)
    spg = torch.from_numpy(sp).cuda()
    tk = TA.make_tables(perm=torch.from_numpy(kp).cuda() if use_perm else None, rope_cs=TA.rope_table(t_cap, D),
                        sink_pos=spg)
    tv = TA.make_tables(perm=torch.from_numpy(vp).cuda() if use_perm else None, sink_pos=spg)
    pk, pv = TA.alloc_packed(dk), TA.alloc_packed(dv)
    TA.encode(dk, torch.from_numpy(k).cuda(), tk, pk)
    TA.encode(dv, torch.from_numpy(v).cuda(), tv, pv)
    scale = 1.0 / math.sqrt(D)
    qg = torch.from_numpy(q).cuda()
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
    if noalloc:
        TA.attend_noalloc(dk, dv, qg, pk, tk, pv, tv, n_tok, scale, out)
    else:
        TA.attend(dk, dv, qg, pk, tk, pv, tv, n_tok, scale, out, TA.attend_workspace(dk, dv, Hq, n_tok))
    s_gpu = torch.empty((B, Hq, n_tok), dtype=torch.float32, device="cuda")
    TA.score(dk, qg, pk, tk, n_tok, scale, s_gpu)
    assert K.kvq_check(0) == K.KVQ_OK
    got, s_gpu = out.cpu().numpy().astype(np.float64), s_gpu.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got))

    okw = dict(rot=1, bits=bits, group=group, n_sink=n_sink, sink_pos=sp)
    kc = {"codes": pk.codes.cpu().numpy(), "sz": pk.scale_zero.cpu().numpy().view(np.uint16),
          "sink": pk.sink.cpu().numpy().view(np.uint16)}
    vc = {"codes": pv.codes.cpu().numpy(), "sz": pv.scale_zero.cpu().numpy().view(np.uint16),
          "sink": pv.sink.cpu().numpy().view(np.uint16)}
    pos = np.arange(t_cap)
    vhat = orc.decode(vc, pos, (B, H, t_cap, D), rope=0, perm=vp, **okw)[:, :, :n_tok]
    khat = orc.decode(kc, pos, (B, H, t_cap, D), rope=okrope, perm=kp, **okw)
    ref = orc.attend(q.view(np.uint16), kc, vc, n_tok, H=H, t_cap=t_cap, scale=scale, kperm=kp, vperm=vp,
                     krope=okrope, vrope=0, **okw)
    gq = Hq // H
    for b in range(B):
        for qh in range(Hq):
            h = qh // gq
            vmax = np.abs(vhat[b, h]).max()
            sv = s_gpu[b, qh]
            p = np.exp(sv - sv.max())
            p /= p.sum()
            tight = 2e-5 * vmax
            assert np.all(np.abs(got[b, qh] - p @ vhat[b, h]) <= tight), (b, qh)
            krot = np.stack([orc.rope_f64(khat[b, h, n], n, mode=okrope) for n in range(n_tok)])
            ds = SCORE_REL * scale * (np.abs(krot) @ np.abs(q[b, qh].astype(np.float64)))
            bound = (math.exp(2 * ds.max()) - 1) * vmax + tight
            assert np.all(np.abs(got[b, qh] - ref[b, qh]) <= bound), (b, qh)
