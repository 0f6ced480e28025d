"""GPU parity of the channel-permutation calibration (kvq_calibrate_perm:
"RotateKV: Accurate and Robust 2-Bit KV Cache Quantization for LLMs via
Outlier-Aware Adaptive Rotations", channel reordering by outlier magnitude).
The permutation is integer output decided by fp32 comparisons of values both
sides compute with the same arithmetic (fp16 input, the encoder's fp32 RoPE
order), so it must match the oracle exactly, ties included."""
import numpy as np
import pytest

import workloads as W

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CASES = [
    # name, B, H, T, D, t0, rope, n_sink, rot, group_heads
    ("keys_rope_sinks", 2, 3, 300, 128, 0, 1, 4, "fwht_head", 1),
    ("values_no_rope", 2, 2, 257, 128, 0, 0, 4, "fwht_head", 1),
    ("d64_rope_offset_t0", 1, 4, 130, 64, 50, 1, 60, "none", 1),
    ("grouped_permutes_raw_input", 1, 8, 64, 128, 0, 1, 2, "fwht_group", 8),
    ("single_token", 3, 2, 1, 128, 7, 1, 0, "fwht_head", 1),
    ("all_positions_are_sinks", 1, 2, 3, 128, 0, 1, 4, "fwht_head", 1),
    ("many_chunks", 4, 2, 9000, 128, 0, 1, 4, "fwht_head", 1),
    # rope 2: keys turned on half-split pairs (i, i + D/2) before the abs-max
    ("keys_half_split", 2, 3, 300, 128, 0, 2, 4, "fwht_head", 1),
    ("keys_half_split_d64_ragged", 1, 4, 77, 64, 9, 2, 10, "none", 1),
]


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_rotation_b200 as K
    return K


def _run(x, B, H, T, D, t0, rope, n_sink, rot, gh):
    from kv_cache_rotation_b200 import torch_api as TA
    d = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, t0=t0, t_cap=t0 + T, bits=2, group=min(128, D),
                     group_heads=gh, rope=rope, n_sink=n_sink, rot=rot)
    tb = TA.make_tables(rope_cs=TA.rope_table(t0 + T, D) if rope else None)
    perm = TA.calibrate_perm(d, torch.from_numpy(x).cuda(), tb)
    torch.cuda.synchronize()
    return perm.cpu().numpy()


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_calibrate_parity(K, orc, case):
    name, B, H, T, D, t0, rope, n_sink, rot, gh = case
    w = W.Workload(name, B=B, H=H, T=T, D=D, outliers=("pairs", 0.02, 10.0, 50.0))
    x = W.kv_tensor(w, "k")
    got = _run(x, B, H, T, D, t0, rope, n_sink, rot, gh)
    # the permutation's input is RoPE'd only where RoPE precedes it (head-dim variants)
    orope = rope if rot in ("none", "fwht_head") else 0
    orope = {0: 0, 1: orc.ROPE_STD, 2: orc.ROPE_STD + orc.ROPE_HALF}[orope]
    want = orc.calibrate_perm(x.view(np.uint16), W.positions(t0, T), rope=orope, n_sink=n_sink)
    assert got.dtype == np.int16 and got.shape == (H, D)
    assert np.array_equal(got, want), (np.argwhere(got != want)[:5])
    if n_sink >= t0 + T:  # nothing but sinks: every a_j is 0 and ties keep channel order
        assert np.array_equal(got, np.tile(np.arange(D, dtype=np.int16), (H, 1)))


def test_calibrate_ties(K, orc):
    # few distinct magnitudes: most channels tie, the order among them is by channel index
    B, H, T, D = 1, 2, 6, 128
    rng = np.random.default_rng(4)
    x = rng.choice(np.array([0.5, -0.5, 1.0, -1.0, 2.0], np.float16), size=(B, H, T, D))
    got = _run(x, B, H, T, D, 0, 0, 0, "fwht_head", 1)
    want = orc.calibrate_perm(x.view(np.uint16), W.positions(0, T), rope=0, n_sink=0)
    assert np.array_equal(got, want)


def test_calibrate_full_size(K, orc):
    # the Llama-3-8B GQA keys: 4 sequences x 8 KV heads x 32768 tokens, RoPE, 4 sinks
    ws = W.WORKLOADS["llama3_8b_gqa_score"]
    x = W.kv_tensor(ws, "k")
    got = _run(x, ws.B, ws.H, ws.T, ws.D, 0, 1, ws.n_sink, "fwht_head", 1)
    want = orc.calibrate_perm(x.view(np.uint16), W.positions(0, ws.T), rope=1, n_sink=ws.n_sink)
    assert np.array_equal(got, want)
