"""Pins of the oracle's decode-step attention ("EliteKV - RoPE频率选择与低秩投影"
§2.2 scores, §7.1 softmax-weighted values) by closed forms that do not
repeat its arithmetic: one cached token gives that token's value exactly; a
zero scale gives the plain mean of the values; every output lies in the
values' convex hull; a large scale selects the value of the top-scoring key."""
import numpy as np
import pytest

import workloads as W

B, H, HQ, T, D = 2, 2, 8, 24, 128


@pytest.fixture(scope="module")
def caches(orc):
    w = W.Workload("attn_pin", B=B, H=H, Hq=HQ, T=T, D=D, bits=2, group=64, n_sink=3, perm=True)
    k = W.kv_tensor(w, "k").view(np.uint16)
    v = W.kv_tensor(w, "v").view(np.uint16)
    pos = np.arange(T)
    kp, vp = W.random_perm(H, D, 3), W.random_perm(H, D, 4)
    common = dict(rot=orc.ROT_FWHT_HEAD, bits=2, group=64, n_sink=3)
    kc = orc.encode(k, pos, rope=1, perm=kp, **common)
    vc = orc.encode(v, pos, rope=0, perm=vp, **common)
    vhat = orc.decode(vc, pos, (B, H, T, D), rope=0, perm=vp, **common)
    q = W.queries(w).view(np.uint16)
    return dict(kc=kc, vc=vc, vhat=vhat, q=q, kp=kp, vp=vp, common=common)


def _attend(orc, c, n_tok, scale):
    return orc.attend(c["q"], c["kc"], c["vc"], n_tok, H=H, t_cap=T, scale=scale, kperm=c["kp"], vperm=c["vp"],
                      **c["common"])


def test_single_token_is_its_value(orc, caches):
    out = _attend(orc, caches, 1, 0.3)
    for qh in range(HQ):
        assert np.array_equal(out[:, qh], caches["vhat"][:, qh // (HQ // H), 0])


def test_zero_scale_is_the_mean(orc, caches):
    out = _attend(orc, caches, T, 0.0)
    mean = caches["vhat"].mean(axis=2)
    for qh in range(HQ):
        np.testing.assert_allclose(out[:, qh], mean[:, qh // (HQ // H)], rtol=0, atol=1e-12)


def test_inside_convex_hull(orc, caches):
    out = _attend(orc, caches, T, 1.0 / np.sqrt(D))
    v = caches["vhat"]
    for qh in range(HQ):
        h = qh // (HQ // H)
        assert np.all(out[:, qh] <= v[:, h].max(axis=1) + 1e-12)
        assert np.all(out[:, qh] >= v[:, h].min(axis=1) - 1e-12)


def test_large_scale_selects_the_top_key(orc, caches):
    s = orc.score(caches["q"], caches["kc"], np.arange(T), H=H, t_cap=T, scale=1.0, rope=1, perm=caches["kp"],
                  **caches["common"])
    out = _attend(orc, caches, T, 1e4)
    for b in range(B):
        for qh in range(HQ):
            top = int(np.argmax(s[b, qh]))
            gap = np.sort(s[b, qh])[-1] - np.sort(s[b, qh])[-2]
            assert gap * 1e4 > 50  # the runner-up's weight is below e^-50
            np.testing.assert_allclose(out[b, qh], caches["vhat"][b, qh // (HQ // H), top], rtol=0, atol=1e-9)


def test_sinks_are_verbatim_values(orc, caches):
    # with three cached tokens, all sinks, the output is a convex mix of the fp16 sink rows themselves
    out = _attend(orc, caches, 3, 1.0 / np.sqrt(D))
    sink_v = caches["vc"]["sink"].view(np.float16).astype(np.float64)  # [B][H][n_sink][D]
    for qh in range(HQ):
        h = qh // (HQ // H)
        lo, hi = sink_v[:, h].min(axis=1), sink_v[:, h].max(axis=1)
        assert np.all(out[:, qh] >= lo - 1e-12) and np.all(out[:, qh] <= hi + 1e-12)
    # and a single sink token returns its row exactly
    one = _attend(orc, caches, 1, 0.7)
    for qh in range(HQ):
        assert np.array_equal(one[:, qh], sink_v[:, qh // (HQ // H), 0])


def test_query_heads_share_their_kv_head(orc, caches):
    # two query heads of the same KV head with the same query give the same output; the GQA grouping is
    # contiguous (query head qh reads KV head qh // (HQ / H))
    q = caches["q"].copy()
    q[:, 1] = q[:, 0]          # same group (KV head 0)
    q[:, HQ // H] = q[:, 0]    # first query head of KV head 1
    out = orc.attend(q, caches["kc"], caches["vc"], T, H=H, t_cap=T, scale=0.2, kperm=caches["kp"],
                     vperm=caches["vp"], **caches["common"])
    assert np.array_equal(out[:, 1], out[:, 0])
    assert not np.allclose(out[:, HQ // H], out[:, 0])  # a different cache gives a different result


def test_listed_prefix_is_the_prefix_form(orc, caches):
    # a sink list naming positions 0 .. n_sink-1 is the prefix form
    sp = np.tile(np.arange(3, dtype=np.int32), (B, 1))
    a = _attend(orc, caches, T, 1.0 / np.sqrt(D))
    b = orc.attend(caches["q"], caches["kc"], caches["vc"], T, H=H, t_cap=T, scale=1.0 / np.sqrt(D),
                   kperm=caches["kp"], vperm=caches["vp"], sink_pos=sp, **caches["common"])
    assert np.array_equal(a, b)


def test_listed_sinks_zero_scale_mean(orc):
    # caches whose sinks are listed positions: with a zero scale the output is the plain mean over the
    # slots, each listed slot contributing its fp16 row and every other slot its decoded codes
    w = W.Workload("attn_list", B=B, H=H, Hq=HQ, T=T, D=D, bits=2, group=64, n_sink=3)
    k = W.kv_tensor(w, "k").view(np.uint16)
    v = W.kv_tensor(w, "v").view(np.uint16)
    pos = np.arange(T)
    sp = np.array([[4, 11, -1], [0, 17, 23]], np.int32)
    common = dict(rot=orc.ROT_FWHT_HEAD, bits=2, group=64, n_sink=3, sink_pos=sp)
    kc = orc.encode(k, pos, rope=1, **common)
    vc = orc.encode(v, pos, rope=0, **common)
    out = orc.attend(W.queries(w).view(np.uint16), kc, vc, T, H=H, t_cap=T, scale=0.0, **common)
    plain = orc.decode(vc, pos, (B, H, T, D), rope=0, rot=orc.ROT_FWHT_HEAD, bits=2, group=64)  # no sinks
    rows = v.view(np.float16).astype(np.float64)
    for b in range(B):
        vals = plain[b].copy()  # [H][T][D]
        for p in sp[b]:
            if p >= 0:
                vals[:, p] = rows[b, :, p]
        for qh in range(HQ):
            np.testing.assert_allclose(out[b, qh], vals[qh // (HQ // H)].mean(axis=0), rtol=0, atol=1e-12)
