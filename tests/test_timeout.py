"""Bounded waits: a kernel whose copy never arrives gives up after its limit,
sets the device error word and returns; kvq_check reports KVQ_ERR_TIMEOUT and
the context stays usable. No GPU fault, trap or hang is involved."""
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def test_expired_wait_reports_timeout():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_rotation_b200 as K
    from kv_cache_rotation_b200 import torch_api as TA
    assert K.kvq_check(0) == K.KVQ_OK
    assert K.kvq_debug_expire_wait(2000, 0) == K.KVQ_OK  # 2 ms limit
    assert K.kvq_check(0) == K.KVQ_ERR_TIMEOUT
    assert K.kvq_check(0) == K.KVQ_OK  # the word is cleared
    # the context still works
    d = TA.make_desc(batch=1, heads=8, tokens=16, bits=2, group=128)
    pk = TA.alloc_packed(d)
    TA.encode(d, torch.randn(1, 8, 16, 128, device="cuda").half(), TA.make_tables(), pk)
    assert K.kvq_check(0) == K.KVQ_OK
    assert pk.scale_zero.abs().sum().item() > 0
    assert K.kvq_debug_expire_wait(0, 0) == K.KVQ_ERR_INVALID
