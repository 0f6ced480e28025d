"""GPU parity of the IsoQuant path (norm split -> per-block SO(4) rotation
qL v qR, or the 3-D sandwich q v q* on 3-channel blocks -> Lloyd-Max codes
-> packing; and the inverse) against the oracle.
The kernel applies each sandwich as its 4x4 (3x3) matrix and divides by the norm
through a reciprocal, so codes may differ by one level within 1e-5 of a
decision boundary (at most 1e-4 of the elements); norms are bit-exact."""
import numpy as np
import pytest

import workloads as W
from parity import compare_codebook, recon_tolerance

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_rotation_b200 as K
    return K


CASES = [
    # name, B, H, T, D, bits, n_sink, t0
    ("iso_bits3", 3, 1, 300, 128, 3, 0, 0),
    ("iso_bits2", 2, 2, 77, 128, 2, 0, 0),
    ("iso_bits4_sinks", 1, 3, 129, 128, 4, 4, 0),
    ("iso_d64_t0", 2, 1, 50, 64, 3, 0, 11),
]
# the 3-D sandwich: d = 128 (42 blocks + a 2-D tail), 64 and 256 (1-channel tails)
CASES3 = [
    ("so3_bits3", 3, 1, 300, 128, 3, 0, 0),
    ("so3_bits2_sinks", 2, 2, 77, 128, 2, 3, 0),
    ("so3_bits4", 1, 2, 129, 128, 4, 0, 5),
    ("so3_d64_t0", 2, 1, 50, 64, 3, 0, 11),
]


def run_iso_case(K, orc, case, so3):
    from kv_cache_rotation_b200 import torch_api as TA
    name, B, H, T, D, bits, n_sink, t0 = case
    w = W.Workload(name, B=B, H=H, T=T, D=D, rot="iso", quant="codebook", bits=bits, rope_k=False,
                   dist="student_t", seed=40 + bits)
    x = W.kv_tensor(w, "k")
    if so3:
        qL, qR = W.iso3_tables(D, 60 + bits), None
    else:
        qL, qR = W.iso_tables(w)
    t_cap = t0 + T + 1
    d = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, t0=t0, t_cap=t_cap, bits=bits, rope=0, n_sink=n_sink,
                     rot="iso3" if so3 else "iso", quant="codebook")
    cb = TA.lloyd_max_codebook(bits, D)
    tb = TA.make_tables(qL=torch.from_numpy(qL).cuda(), qR=torch.from_numpy(qR).cuda() if qR is not None else None,
                        codebook=cb)
    pk = TA.alloc_packed(d)
    TA.encode(d, torch.from_numpy(x).cuda(), tb, pk)
    assert K.kvq_check(0) == K.KVQ_OK
    pos = np.arange(t0, t0 + T)
    ocb = orc.codebook(bits, D)
    assert np.array_equal(ocb, cb.cpu().numpy())
    okw = dict(rot=orc.ROT_ISO3 if so3 else orc.ROT_ISO, quant=orc.Q_CODEBOOK, bits=bits, n_sink=n_sink, qL=qL,
               qR=qR, cb=ocb)
    ref = orc.encode(x.view(np.uint16), pos, want_pre=True, **okw)
    gc = pk.codes[:, :, t0:t0 + T].cpu().numpy()
    rep = compare_codebook(gc, ref["codes"], ref["pre"], ocb, D, bits)
    assert rep.ok, rep
    gn = pk.norm[:, :, t0:t0 + T].cpu().numpy()
    assert np.array_equal(gn.view(np.uint32), ref["norm"].view(np.uint32))
    if n_sink:
        live = [m for m in pos if m < n_sink]
        assert np.array_equal(pk.sink.cpu().numpy().view(np.uint16)[:, :, live], ref["sink"][:, :, live])
    out32 = torch.empty((B, H, T, D), dtype=torch.float32, device="cuda")
    out16 = torch.empty((B, H, T, D), dtype=torch.float16, device="cuda")
    TA.decode(d, pk, tb, out32)
    TA.decode(d, pk, tb, out16)
    assert K.kvq_check(0) == K.KVQ_OK
    dec = orc.decode({"codes": gc, "norm": gn, "sink": pk.sink.cpu().numpy().view(np.uint16) if n_sink else None},
                     pos, x.shape, **okw)
    o32 = out32.cpu().numpy()
    err = np.abs(o32.astype(np.float64) - dec)
    assert np.all(err <= recon_tolerance(dec)), err.max()
    assert np.array_equal(out16.cpu().numpy().view(np.uint16), o32.astype(np.float16).view(np.uint16))
    return rep


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_iso_parity(K, orc, case):
    run_iso_case(K, orc, case, so3=False)


@pytest.mark.parametrize("case", CASES3, ids=[c[0] for c in CASES3])
def test_iso3_parity(K, orc, case):
    run_iso_case(K, orc, case, so3=True)

