"""GPU parity of the RoPE-pair energy (kvq_pair_energy: "EliteKV -
RoPE频率选择与低秩投影" §3.1 frequency energy analysis). Both sides count
exact multiples of 2^-48 in 128-bit integers, so energies and rankings must
match the oracle exactly."""
import numpy as np
import pytest

import workloads as W

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CASES = [
    # name, B, H, T, D
    ("keys_small", 2, 3, 300, 128),
    ("head_dim_64", 1, 4, 130, 64),
    ("single_token", 3, 2, 1, 128),
    ("many_chunks", 4, 2, 9000, 128),
]


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_rotation_b200 as K
    return K


def _run(x):
    from kv_cache_rotation_b200 import torch_api as TA
    B, H, T, D = x.shape
    d = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, bits=2, group=min(128, D))
    e, r = TA.pair_energy(d, torch.from_numpy(x.view(np.float16)).cuda())
    torch.cuda.synchronize()
    return e.cpu().numpy(), r.cpu().numpy()


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_energy_parity(K, orc, case):
    name, B, H, T, D = case
    w = W.Workload(name, B=B, H=H, T=T, D=D, outliers=("pairs", 0.02, 10.0, 50.0))
    x = W.kv_tensor(w, "k").view(np.uint16)
    e, r = _run(x)
    we, wr = orc.pair_energy(x)
    assert np.array_equal(e, we)
    assert np.array_equal(r, wr)


def test_energy_extremes_and_ties(K, orc):
    # subnormals, the largest half, infinities and NaNs (which add nothing), exact ties
    rng = np.random.default_rng(12)
    x = rng.choice(np.array([0x0001, 0x03FF, 0x7BFF, 0xFBFF, 0x7C00, 0x7E00, 0x3C00, 0xBC00, 0], np.uint16),
                   size=(2, 2, 40, 128))
    x[:, 0, :, 6:8] = x[:, 0, :, 20:22]  # pairs 3 and 10 of head 0 tie
    e, r = _run(x)
    we, wr = orc.pair_energy(x)
    assert np.array_equal(e, we) and np.array_equal(r, wr)
    assert np.any(e[:, :, 1] > 0)  # the largest halves carry into the high word


def test_energy_full_size(K, orc):
    ws = W.WORKLOADS["llama3_8b_gqa_score"]
    x = W.kv_tensor(ws, "k").view(np.uint16)
    e, r = _run(x)
    we, wr = orc.pair_energy(x)
    assert np.array_equal(e, we) and np.array_equal(r, wr)
