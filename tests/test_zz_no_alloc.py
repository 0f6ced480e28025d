"""kvq_attend_noalloc, the attention entry point for callers that cannot
allocate device memory when they call (its workspace is a fixed 40 MiB array
inside the library), against kvq_attend with a caller-owned workspace on the
same caches. Both run the same kernels on the same inputs, so the outputs must
be equal byte for byte, on two calls in a row.

Cases: the fused form (2-bit codes, one group per record), the three-kernel
form (2-bit, groups of 64: scores and chunk partials both live in the array),
a shape whose workspace just fits the 40 MiB (and one token more, which must
be refused), and a fresh process under lazy module loading in which
kvq_attend_noalloc is the first library call. Collected last, so it also runs
after every other test has used the library in the same process."""
import math
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SCRATCH_BYTES = 40 << 20


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_rotation_b200 as K
    return K


# Random but valid cache contents, drawn on the GPU (no library call): any
# codes, positive fp16 scales, N(0,1) zeros and sinks. The caller below is the
# same source text that runs in the fresh-process case.
CACHE_SRC = '''
def random_caches(B, H, t_cap, bits, group, n_sink, Hq, seed):
    import math
    import numpy as np
    import torch
    from kv_cache_rotation_b200 import torch_api as TA
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    D = 128
    common = dict(batch=B, heads=H, head_dim=D, tokens=t_cap, t_cap=t_cap, bits=bits, group=group,
                  n_sink=n_sink, rot="fwht_head")
    dk, dv = TA.make_desc(rope=1, **common), TA.make_desc(rope=0, **common)
    packs = []
    for d in (dk, dv):
        p = TA.alloc_packed(d)
        p.codes.copy_(torch.randint(0, 256, p.codes.shape, generator=g, device="cuda", dtype=torch.int32)
                      .to(torch.uint8))
        s = (torch.rand(p.scale_zero.shape[:-1], generator=g, device="cuda") * 0.2 + 0.01).half()
        z = torch.randn(p.scale_zero.shape[:-1], generator=g, device="cuda").half()
        p.scale_zero.copy_(torch.stack([s.view(torch.int16), z.view(torch.int16)], dim=-1))
        if n_sink:
            p.sink.copy_(torch.randn(p.sink.shape, generator=g, device="cuda").half())
        packs.append(p)
    # (cos, sin) of m * 10000^(-2i/D), built with numpy (used for the fp16 sinks only)
    m = np.arange(max(n_sink, 1), dtype=np.float64)[:, None]
    th = 10000.0 ** (-2.0 * np.arange(D // 2) / D)
    cs = np.stack([np.cos(m * th), np.sin(m * th)], axis=-1).astype(np.float32)
    tk = TA.make_tables(rope_cs=torch.from_numpy(cs).cuda())
    tv = TA.make_tables()
    perm = torch.stack([torch.randperm(D, generator=g, device="cuda") for _ in range(H)]).to(torch.int16)
    tv.perm = perm
    q = torch.randn((B, Hq, D), generator=g, device="cuda").half()
    return dk, dv, packs[0], tk, packs[1], tv, q, 1.0 / math.sqrt(D)
'''
exec(CACHE_SRC)


def _pair(K, dk, dv, pk, tk, pv, tv, q, scale, n_tok):
    """kvq_attend with a workspace, then kvq_attend_noalloc twice; raw bytes."""
    from kv_cache_rotation_b200 import torch_api as TA
    B, Hq, D = q.shape
    ref = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
    TA.attend(dk, dv, q, pk, tk, pv, tv, n_tok, scale, ref, TA.attend_workspace(dk, dv, Hq, n_tok))
    outs = []
    for _ in range(2):
        o = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
        TA.attend_noalloc(dk, dv, q, pk, tk, pv, tv, n_tok, scale, o)
        outs.append(o)
    assert K.kvq_check(0) == K.KVQ_OK
    r = ref.cpu().numpy()
    assert np.all(np.isfinite(r))
    return r.view(np.uint32), [o.cpu().numpy().view(np.uint32) for o in outs]


@pytest.mark.parametrize("bits,group,n_tok_off", [(2, 128, 3), (2, 64, 5)], ids=["fused", "three_kernel"])
def test_noalloc_matches_workspace_version(K, bits, group, n_tok_off):
    t_cap = 2600
    dk, dv, pk, tk, pv, tv, q, scale = random_caches(2, 2, t_cap, bits, group, 4, 8, seed=11 + group)
    n_tok = t_cap - n_tok_off
    ref, outs = _pair(K, dk, dv, pk, tk, pv, tv, q, scale, n_tok)
    for o in outs:
        assert np.array_equal(o, ref)


def test_noalloc_near_limit(K):
    """The largest token count whose workspace fits the 40 MiB array is served
    (three-kernel form: 4.5 bytes per query head and token); one more token is
    refused with KVQ_ERR_UNSUPPORTED and launches nothing."""
    from kv_cache_rotation_b200 import torch_api as TA
    B, H, Hq, bits, group = 4, 8, 32, 2, 64
    t_cap = 80000
    dk, dv, pk, tk, pv, tv, q, scale = random_caches(B, H, t_cap, bits, group, 4, Hq, seed=5)
    need = lambda n: K.kvq_attend_workspace_bytes(dk, dv, Hq, n)
    lo, hi = 1, t_cap
    while lo < hi:  # largest n with need(n) <= SCRATCH_BYTES
        mid = (lo + hi + 1) // 2
        if need(mid) <= SCRATCH_BYTES:
            lo = mid
        else:
            hi = mid - 1
    n_fit = lo
    assert n_fit < t_cap and need(n_fit + 1) > SCRATCH_BYTES
    assert need(n_fit) > SCRATCH_BYTES - (1 << 20)  # within 1 MiB of the limit
    ref, outs = _pair(K, dk, dv, pk, tk, pv, tv, q, scale, n_fit)
    for o in outs:
        assert np.array_equal(o, ref)
    out = torch.zeros((B, Hq, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(K.KvqError) as e:
        TA.attend_noalloc(dk, dv, q, pk, tk, pv, tv, n_fit + 1, scale, out)
    assert e.value.status == K.KVQ_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert not out.any().item()


def test_noalloc_first_call_in_fresh_process(K):
    """Under lazy module loading, with kvq_attend_noalloc as the process's first
    library call (the caches are written with torch, not by the library), the
    call sets up the array and matches kvq_attend."""
    script = CACHE_SRC + textwrap.dedent('''
        import sys
        import numpy as np
        import torch
        sys.path.insert(0, ROOT)
        import kv_cache_rotation_b200 as K
        from kv_cache_rotation_b200 import torch_api as TA
        dk, dv, pk, tk, pv, tv, q, scale = random_caches(2, 2, 1500, 2, 128, 4, 8, seed=3)
        B, Hq, D = q.shape
        n_tok = 1497
        outs = []
        for _ in range(2):
            o = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
            TA.attend_noalloc(dk, dv, q, pk, tk, pv, tv, n_tok, scale, o)
            outs.append(o)
        ref = torch.empty((B, Hq, D), dtype=torch.float32, device="cuda")
        TA.attend(dk, dv, q, pk, tk, pv, tv, n_tok, scale, ref, TA.attend_workspace(dk, dv, Hq, n_tok))
        assert K.kvq_check(0) == K.KVQ_OK
        r = ref.cpu().numpy()
        assert np.all(np.isfinite(r))
        for o in outs:
            assert np.array_equal(o.cpu().numpy().view(np.uint32), r.view(np.uint32))
        print("NOALLOC_FIRST_CALL_OK")
    ''')
    env = dict(os.environ, CUDA_MODULE_LOADING="LAZY")
    r = subprocess.run([sys.executable, "-c", f"ROOT = {ROOT!r}\n" + script], env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and "NOALLOC_FIRST_CALL_OK" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
