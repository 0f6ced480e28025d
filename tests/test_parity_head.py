"""GPU parity of the head-variant path (RoPE -> permutation -> FWHT over
head_dim -> min-max 2/3/4-bit -> packing, sinks; and the inverse) against the
CPU oracle, through the C ABI. Shapes are small enough for the oracle to
finish in seconds but span several tiles, a ragged tail, a nonzero first slot
and every supported (head_dim, bits, group)."""
import zlib

import numpy as np
import pytest

import workloads as W
from parity import RECON_ROW_REL, compare_minmax, recon_tolerance

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CASES = [
    # name, B, H, T, D, t0, extra_cap, bits, group, rope, perm, n_sink, rot
    ("tiny_workload", 1, 8, 256, 128, 0, 0, 4, 128, 1, False, 0, "fwht_head"),
    ("perm_sink_g64", 2, 4, 37, 128, 0, 5, 2, 64, 1, True, 4, "fwht_head"),
    ("t0_offset", 2, 4, 37, 128, 9, 3, 2, 64, 1, True, 4, "fwht_head"),
    ("bits3_g32_norope", 1, 2, 19, 128, 0, 0, 3, 32, 0, True, 3, "fwht_head"),
    ("d64_bits2", 2, 16, 33, 64, 0, 0, 2, 64, 1, False, 0, "fwht_head"),
    ("d64_bits3_g32", 1, 8, 40, 64, 2, 1, 3, 32, 1, True, 1, "fwht_head"),
    ("d64_bits4_g32", 1, 4, 17, 64, 0, 0, 4, 32, 0, False, 0, "fwht_head"),
    ("no_rotation", 1, 8, 50, 128, 0, 0, 4, 128, 1, False, 2, "none"),
    ("odd_heads_ht1", 1, 3, 130, 128, 0, 0, 2, 128, 1, False, 0, "fwht_head"),
    ("heads6_ht2", 2, 6, 70, 128, 1, 0, 3, 64, 1, True, 0, "fwht_head"),
    ("append_one", 2, 8, 1, 128, 40, 0, 2, 64, 1, True, 4, "fwht_head"),
    ("bits4_g64", 1, 8, 64, 128, 0, 0, 4, 64, 1, True, 0, "fwht_head"),
    ("bits2_g32", 1, 8, 64, 128, 0, 0, 2, 32, 1, False, 0, "fwht_head"),
    ("bits3_g128", 1, 8, 64, 128, 0, 0, 3, 128, 0, False, 0, "fwht_head"),
    # rope 2: half-split pairs (i, i + D/2)
    ("half_split_perm_sink", 2, 4, 37, 128, 5, 2, 2, 64, 2, True, 4, "fwht_head"),
    ("half_split_d64", 1, 8, 40, 64, 2, 1, 3, 32, 2, True, 1, "fwht_head"),
    ("half_split_no_rotation", 1, 8, 50, 128, 0, 0, 4, 128, 2, False, 2, "none"),
    # sink positions inside the call (t0 < n_sink < t0 + T), and more sinks than tokens
    ("sinks_cross_t0", 1, 4, 20, 128, 2, 0, 2, 64, 1, True, 5, "fwht_head"),
    ("all_sinks", 1, 2, 3, 128, 0, 0, 2, 128, 1, False, 8, "fwht_head"),
]


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_rotation_b200 as K
    return K


def _inputs(name, B, H, T, D, seed):
    w = W.Workload(name, B=B, H=H, T=T, D=D, seed=seed, outliers=("pairs", 0.02, 10.0, 50.0))
    return W.kv_tensor(w, "k")


def run_head_case(K, orc, x, *, t0, t_cap, bits, group, rope, perm, n_sink, rot, row_rel=0.0, freq=0):
    from kv_cache_rotation_b200 import torch_api as TA
    B, H, T, D = x.shape
    d = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, t0=t0, t_cap=t_cap, bits=bits, group=group,
                     rope=rope, n_sink=n_sink, rot=rot)
    xg = torch.from_numpy(x).cuda()
    cs = TA.rope_table(t_cap + 3, D, freq=freq) if rope else None
    pg = torch.from_numpy(perm).cuda() if perm is not None else None
    tb = TA.make_tables(perm=pg, rope_cs=cs)
    pk = TA.alloc_packed(d)
    TA.encode(d, xg, tb, pk)
    assert K.kvq_check(0) == K.KVQ_OK
    pos = np.arange(t0, t0 + T)
    # the oracle's rope flag names its table (1 standard, 2 frequency-aware) plus
    # ROPE_HALF for the half-split pairs the descriptor's rope = 2 selects
    table = orc.ROPE_FREQ_AWARE if freq == K.KVQ_ROPE_FREQ_AWARE else orc.ROPE_STD
    orope = 0 if not rope else table + (orc.ROPE_HALF if rope == 2 else 0)
    okw = dict(rot={"none": 0, "fwht_head": 1}[rot], bits=bits, group=group, rope=orope, n_sink=n_sink, perm=perm)
    ref = orc.encode(x.view(np.uint16), pos, want_pre=True, **okw)
    gc = pk.codes[:, :, t0:t0 + T].cpu().numpy()
    gs = pk.scale_zero[:, :, t0:t0 + T].cpu().numpy()
    rep = compare_minmax(gc, ref["codes"], gs, ref["sz"].view(np.int16), ref["pre"], D, bits, group)
    assert rep.ok, rep
    assert rep.mismatched == 0, rep  # the fixed fp32 order makes codes bit-exact
    # untouched slots stay zero
    if t0 > 0:
        assert not pk.codes[:, :, :t0].any().item()
    if n_sink:
        gsink = pk.sink.cpu().numpy().view(np.uint16)
        live = [m for m in pos if m < n_sink]
        if live:
            assert np.array_equal(gsink[:, :, live], ref["sink"][:, :, live])
    # decode the GPU's codes on both sides
    out32 = torch.empty((B, H, T, D), dtype=torch.float32, device="cuda")
    out16 = torch.empty((B, H, T, D), dtype=torch.float16, device="cuda")
    TA.decode(d, pk, tb, out32)
    TA.decode(d, pk, tb, out16)
    assert K.kvq_check(0) == K.KVQ_OK
    packed_np = {"codes": gc, "sz": gs.view(np.uint16),
                 "sink": pk.sink.cpu().numpy().view(np.uint16) if n_sink else None}
    dec = orc.decode(packed_np, pos, x.shape, **okw)
    o32 = out32.cpu().numpy()
    err = np.abs(o32.astype(np.float64) - dec)
    assert np.all(err <= recon_tolerance(dec, row_rel)), err.max()
    assert np.array_equal(out16.cpu().numpy().view(np.uint16), o32.astype(np.float16).view(np.uint16))
    return rep, err.max()


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_head_parity(K, orc, case):
    name, B, H, T, D, t0, extra, bits, group, rope, use_perm, n_sink, rot = case
    x = _inputs(name, B, H, T, D, seed=zlib.crc32(name.encode()) % 1000)
    perm = W.random_perm(H, D, 7) if use_perm else None
    run_head_case(K, orc, x, t0=t0, t_cap=t0 + T + extra, bits=bits, group=group, rope=rope, perm=perm,
                  n_sink=n_sink, rot=rot)


@pytest.mark.parametrize("which", ["k", "v"])
def test_tiny_workload_own_inputs(K, orc, which):
    """The tiny configuration on its own input recipe (1 sequence x 8 heads x
    256 tokens, N(0,1) with 4 channels per head scaled by 20): RoPE on the
    keys, FWHT over head_dim, 4-bit min-max with groups of 128, K and V."""
    w = W.WORKLOADS["tiny"]
    x = W.kv_tensor(w, which)
    assert x.shape == (1, 8, 256, 128)
    rep, _ = run_head_case(K, orc, x, t0=0, t_cap=w.T, bits=w.bits, group=w.group,
                           rope=1 if which == "k" else 0, perm=None, n_sink=w.n_sink, rot=w.rot)
    assert rep.n == x.size


def test_head_edge_values(K, orc):
    """Zero vectors, constant vectors, fp16 extremes that stay in range after
    the rotation, subnormals, and a mix in one batch."""
    B, H, T, D = 1, 8, 32, 128
    rng = np.random.default_rng(0)
    x = rng.standard_normal((B, H, T, D)).astype(np.float16)
    x[0, 0] = 0  # zero vectors
    x[0, 1] = np.float16(3.5)  # constant vectors
    x[0, 2, :, :] = np.float16(6e-8)  # subnormal
    x[0, 3, :, ::2] = np.float16(-5000.0)  # large, still in range after the FWHT
    x[0, 4, :16] = np.float16(-0.0)
    x[0, 5, :, 7] = np.float16(60000.0)  # one huge channel: rotated values ~ 5300
    run_head_case(K, orc, x, t0=0, t_cap=T, bits=2, group=64, rope=1, perm=None, n_sink=0, rot="fwht_head",
                  row_rel=RECON_ROW_REL)
    run_head_case(K, orc, x, t0=0, t_cap=T, bits=4, group=128, rope=0, perm=None, n_sink=0, rot="fwht_head",
                  row_rel=RECON_ROW_REL)


def test_head_deterministic(K):
    """Two encodes of the same input produce the same bytes."""
    from kv_cache_rotation_b200 import torch_api as TA
    x = _inputs("det", 2, 8, 300, 128, 5)
    d = TA.make_desc(batch=2, heads=8, tokens=300, bits=2, group=64, rope=1, n_sink=4)
    xg = torch.from_numpy(x).cuda()
    tb = TA.make_tables(rope_cs=TA.rope_table(300, 128))
    a, b = TA.alloc_packed(d), TA.alloc_packed(d)
    TA.encode(d, xg, tb, a)
    TA.encode(d, xg, tb, b)
    assert torch.equal(a.codes, b.codes) and torch.equal(a.scale_zero, b.scale_zero)


@pytest.mark.parametrize("D,group,rope", [(128, 64, 1), (64, 32, 1), (128, 64, 2)])
def test_head_freq_aware_rope_table(K, orc, D, group, rope):
    """KV-Latent frequency-aware RoPE: the kernels take the table they are given;
    codes stay bit-exact against the oracle rotating with the same frequencies
    (on interleaved or half-split pairs)."""
    x = _inputs("freq_aware", 2, 4, 70, D, 21)
    run_head_case(K, orc, x, t0=3, t_cap=80, bits=2, group=group, rope=rope, perm=W.random_perm(4, D, 8), n_sink=4,
                  rot="fwht_head", freq=K.KVQ_ROPE_FREQ_AWARE)
