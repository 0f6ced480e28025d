"""kvq_attend_noalloc (the fixed-scratch variant of kvq_attend) against
kvq_attend on the same caches: two calls in a row, both equal to the
workspace version. Collected last so it also runs after every other test
has used the library in the same process."""
import math

import numpy as np
import pytest

import workloads as W

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_rotation_b200 as K
    return K


def test_noalloc_matches_workspace_version(K):
    from kv_cache_rotation_b200 import torch_api as TA
    B, H, Hq, t_cap, D = 2, 2, 8, 600, 128
    w = W.Workload("noalloc", B=B, H=H, Hq=Hq, T=t_cap, D=D, bits=2, group=128, n_sink=4, seed=11)
    common = dict(batch=B, heads=H, head_dim=D, tokens=t_cap, t_cap=t_cap, bits=2, group=128, n_sink=4,
                  rot="fwht_head")
    dk, dv = TA.make_desc(rope=1, **common), TA.make_desc(rope=0, **common)
    tk = TA.make_tables(perm=torch.from_numpy(W.random_perm(H, D, 1)).cuda(), rope_cs=TA.rope_table(t_cap, D))
    tv = TA.make_tables(perm=torch.from_numpy(W.random_perm(H, D, 2)).cuda())
    pk, pv = TA.alloc_packed(dk), TA.alloc_packed(dv)
    TA.encode(dk, torch.from_numpy(W.kv_tensor(w, "k")).cuda(), tk, pk)
    TA.encode(dv, torch.from_numpy(W.kv_tensor(w, "v")).cuda(), tv, pv)
    q = torch.from_numpy(W.queries(w)).cuda()
    scale = 1.0 / math.sqrt(D)
    n_tok = t_cap - 3
    ref = torch.empty((B, Hq, D), dtype=torch.float32, device="cuda")
    TA.attend(dk, dv, q, pk, tk, pv, tv, n_tok, scale, ref, TA.attend_workspace(dk, dv, Hq, n_tok))
    outs = []
    for _ in range(2):
        o = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
        TA.attend_noalloc(dk, dv, q, pk, tk, pv, tv, n_tok, scale, o)
        outs.append(o)
    assert K.kvq_check(0) == K.KVQ_OK
    r = ref.cpu().numpy()
    assert np.all(np.isfinite(r))
    for o in outs:
        # same kernels on the same inputs: equal up to a last-bit tolerance
        np.testing.assert_allclose(o.cpu().numpy(), r, rtol=1e-6, atol=1e-6)
