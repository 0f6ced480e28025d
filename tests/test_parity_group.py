"""GPU parity of the grouped-head path (permutation -> FWHT over group_heads x
128 channels -> RoPE per head slice -> min-max -> packing; and the inverse)
against the oracle, through the C ABI."""
import numpy as np
import pytest

import workloads as W
from parity import RECON_ROW_REL, compare_minmax, recon_tolerance

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CASES = [
    # name, B, H, T, hg, bits, group, rope, perm, n_sink, t0
    ("llama3_like", 2, 8, 70, 8, 2, 128, 1, False, 0, 0),
    ("hg8_g64_bits4_perm_sink", 1, 8, 33, 8, 4, 64, 1, True, 3, 0),
    ("hg8_bits3_two_groups", 1, 16, 20, 8, 3, 128, 1, False, 2, 0),
    ("hg4_t0", 2, 8, 40, 4, 3, 64, 0, False, 0, 5),
    ("hg4_bits2_rope", 1, 4, 90, 4, 2, 128, 1, True, 0, 0),
    ("hg2_ragged", 1, 4, 130, 2, 2, 128, 1, True, 0, 0),
    ("hg2_bits4_g64", 2, 2, 65, 2, 4, 64, 0, False, 1, 0),
    ("append_one", 2, 8, 1, 8, 2, 128, 1, False, 4, 77),
    # rope 2: half-split pairs (i, i + 64)
    ("half_split_hg8_sinks", 2, 8, 70, 8, 2, 128, 2, False, 2, 0),
    ("half_split_hg4_perm", 1, 4, 90, 4, 2, 128, 2, True, 0, 3),
    ("half_split_hg2_g64", 1, 4, 130, 2, 3, 64, 2, True, 0, 0),
    # sink positions inside the call (t0 < n_sink < t0 + T), and more sinks than tokens
    ("sinks_cross_t0", 1, 8, 21, 8, 2, 128, 1, False, 6, 3),
    ("all_sinks", 2, 8, 3, 8, 2, 128, 1, True, 5, 0),
]


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_rotation_b200 as K
    return K


def run_group_case(K, orc, x, *, t0, t_cap, hg, bits, group, rope, perm, n_sink, row_rel=0.0):
    from kv_cache_rotation_b200 import torch_api as TA
    B, H, T, D = x.shape
    d = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, t0=t0, t_cap=t_cap, bits=bits, group=group,
                     group_heads=hg, rope=rope, n_sink=n_sink, rot="fwht_group")
    tb = TA.make_tables(perm=torch.from_numpy(perm).cuda() if perm is not None else None,
                        rope_cs=TA.rope_table(t_cap + 2, D) if rope else None)
    pk = TA.alloc_packed(d)
    TA.encode(d, torch.from_numpy(x).cuda(), tb, pk)
    assert K.kvq_check(0) == K.KVQ_OK
    pos = np.arange(t0, t0 + T)
    orope = {0: 0, 1: orc.ROPE_STD, 2: orc.ROPE_STD + orc.ROPE_HALF}[rope]
    okw = dict(rot=orc.ROT_FWHT_GROUP, bits=bits, group=group, group_heads=hg, rope=orope, n_sink=n_sink, perm=perm)
    ref = orc.encode(x.view(np.uint16), pos, want_pre=True, **okw)
    gc = pk.codes[:, :, t0:t0 + T].cpu().numpy()
    gs = pk.scale_zero[:, :, t0:t0 + T].cpu().numpy()
    rep = compare_minmax(gc, ref["codes"], gs, ref["sz"].view(np.int16), ref["pre"], D, bits, group)
    assert rep.ok and rep.mismatched == 0, rep
    if n_sink:
        live = [m for m in pos if m < n_sink]
        if live:
            assert np.array_equal(pk.sink.cpu().numpy().view(np.uint16)[:, :, live], ref["sink"][:, :, live])
    out32 = torch.empty((B, H, T, D), dtype=torch.float32, device="cuda")
    out16 = torch.empty((B, H, T, D), dtype=torch.float16, device="cuda")
    TA.decode(d, pk, tb, out32)
    TA.decode(d, pk, tb, out16)
    assert K.kvq_check(0) == K.KVQ_OK
    dec = orc.decode({"codes": gc, "sz": gs.view(np.uint16),
                      "sink": pk.sink.cpu().numpy().view(np.uint16) if n_sink else None}, pos, x.shape, **okw)
    o32 = out32.cpu().numpy()
    err = np.abs(o32.astype(np.float64) - dec)
    assert np.all(err <= recon_tolerance(dec, row_rel)), err.max()
    assert np.array_equal(out16.cpu().numpy().view(np.uint16), o32.astype(np.float16).view(np.uint16))


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_group_parity(K, orc, case):
    name, B, H, T, hg, bits, group, rope, use_perm, n_sink, t0 = case
    w = W.Workload(name, B=B, H=H, T=T, seed=len(name), outliers=("pairs", 0.01, 10.0, 50.0))
    x = W.kv_tensor(w, "k")
    perm = W.random_perm(H, 128, 3) if use_perm else None
    run_group_case(K, orc, x, t0=t0, t_cap=t0 + T + 2, hg=hg, bits=bits, group=group, rope=rope, perm=perm,
                   n_sink=n_sink)


def test_group_edge_values(K, orc):
    rng = np.random.default_rng(1)
    x = rng.standard_normal((1, 8, 24, 128)).astype(np.float16)
    x[0, :, 0] = 0
    x[0, :, 1] = np.float16(2.0)
    x[0, 2, 2:] = np.float16(-0.0)
    x[0, :, 3, 5] = np.float16(20000.0)
    run_group_case(K, orc, x, t0=0, t_cap=24, hg=8, bits=2, group=128, rope=1, perm=None, n_sink=0,
                   row_rel=RECON_ROW_REL)
