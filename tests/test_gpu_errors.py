"""Error paths of the ABI on a GPU.  Every failure is made on the host (bad
arguments, exhausted pools, wrong call order, a NaN planted in the input
queries) or is a bounded device wait that runs out by design; none faults,
traps or hangs the device."""
import ctypes

import numpy as np
import pytest
import torch

import decode_kv_cache_paged_b200 as kvc
from decode_kv_cache_paged_b200 import Context, ContextSpec, KvcError

pytestmark = pytest.mark.gpu


def small(num_pages=64, B=4, W=8):
    spec = ContextSpec(num_requests=2, num_layers=1, num_kv_heads=2, head_dim=64, max_seq_len=256,
                       num_pages=num_pages, num_q_heads=4, num_beacons=B, query_window=W)
    return Context(spec, dtype=torch.bfloat16)


def kv(n, T, H=2, d=64, Hq=4):
    g = torch.Generator(device="cuda").manual_seed(1)
    k = torch.randn((n, 1, T, H, d), generator=g, device="cuda").bfloat16()
    v = torch.randn((n, 1, T, H, d), generator=g, device="cuda").bfloat16()
    q = torch.randn((n, 1, T, Hq, d), generator=g, device="cuda").bfloat16()
    return k, v, q


def test_out_of_pages_and_max_len():
    ctx = small(num_pages=4)
    k, v, _ = kv(1, 80)
    with pytest.raises(KvcError) as e:
        ctx.append([0], k, v)
    assert e.value.status == kvc.KVC_ERR_OUT_OF_PAGES
    ctx2 = small()
    k, v, _ = kv(1, 257)
    with pytest.raises(KvcError) as e:
        ctx2.append([0], k, v)
    assert e.value.status == kvc.KVC_ERR_OUT_OF_PAGES
    # nothing was taken: a fitting append still works
    k, v, _ = kv(1, 64)
    ctx.append([0], k, v)
    assert ctx.lengths()[0][0] == 64
    ctx.close()
    ctx2.close()


def test_protect_after_generated_is_a_state_error():
    ctx = small()
    k, v, _ = kv(1, 8)
    ctx.append([0], k, v, protect=True)
    ctx.append([0], k, v, protect=False)
    with pytest.raises(KvcError) as e:
        ctx.append([0], k, v, protect=True)
    assert e.value.status == kvc.KVC_ERR_STATE
    ctx.close()


def test_bad_arguments():
    ctx = small()
    k, v, q = kv(1, 8)
    with pytest.raises(KvcError):
        ctx.append([5], k, v)  # request out of range
    k2, v2, _ = kv(2, 8)
    with pytest.raises(KvcError):
        ctx.append([1, 1], k2, v2)  # duplicate
    with pytest.raises(KvcError):
        ctx.compress("random", np.array([-1, 3], np.int32), 0)  # negative budget
    host = torch.zeros(4096, dtype=torch.uint8)  # pageable host memory
    st = kvc.kvc_append(ctx.handle, np.array([0], np.int32).ctypes.data_as(ctypes.c_void_p), 1, 1,
                        ctypes.c_void_p(host.data_ptr()), ctypes.c_void_p(host.data_ptr()), None, 0)
    assert st == kvc.KVC_ERR_INVALID_ARG
    with pytest.raises(KvcError):
        ctx.set_option(kvc.KVC_OPT_BEACON_SCORE_IMPL, 5)
    ctx.close()


def test_beacon_order_errors():
    ctx = small(B=4, W=8)
    k, v, q = kv(2, 8)
    ctx.append([0, 1], k, v, q)
    with pytest.raises(KvcError) as e:  # no beacons yet
        ctx.compress("beacon", np.array([4, 4], np.int32), 0)
    assert e.value.status == kvc.KVC_ERR_STATE
    ctx.close()
    ctx = small(B=4, W=8)
    k, v, q = kv(1, 1)  # 1 step x G=2 points < B=4
    ctx.append([0], k, v, q)
    with pytest.raises(KvcError) as e:
        ctx.update_beacons()
    assert e.value.status == kvc.KVC_ERR_STATE
    ctx.close()
    nob = Context(ContextSpec(num_requests=1, num_layers=1, num_kv_heads=1, head_dim=64, max_seq_len=64,
                              num_pages=8), dtype=torch.bfloat16)
    with pytest.raises(KvcError) as e:
        nob.update_beacons()
    assert e.value.status == kvc.KVC_ERR_STATE
    nob.close()


def test_nan_query_is_reported_not_faulted():
    ctx = small(B=4, W=8)
    k, v, q = kv(2, 8)
    q[0, 0, 3, 1, 5] = float("nan")
    ctx.append([0, 1], k, v, q)
    with pytest.raises(KvcError) as e:
        ctx.update_beacons()
        ctx.sync()
    assert e.value.status == kvc.KVC_ERR_NAN
    ctx.sync()  # the status word was cleared; the context is still usable
    ctx.compress("random", np.array([4, 4], np.int32), 0)
    ctx.sync()
    assert list(ctx.lengths()[0]) == [4, 4]
    ctx.close()


def test_host_pinned_append_matches_device_append():
    a, b = small(), small()
    k, v, q = kv(2, 40)
    a.append([0, 1], k, v, q)
    b.append([0, 1], k.cpu().pin_memory(), v.cpu().pin_memory(), q.cpu().pin_memory())
    a.sync()
    b.sync()
    ka, va, pa = a.gather_dense(0)
    kb, vb, pb = b.gather_dense(0)
    assert torch.equal(ka, kb) and torch.equal(va, vb) and torch.equal(pa, pb)
    assert torch.equal(a.state_tensors()["query_ring"], b.state_tensors()["query_ring"])
    a.close()
    b.close()


def test_bounded_wait_timeout_is_reported_and_the_context_survives():
    """A device wait that runs out (an mbarrier nothing arrives on, 50 ms bound)
    records a timeout; the host reports KVC_ERR_DEVICE_TIMEOUT and the context
    keeps working."""
    ctx = small()
    k, v, _ = kv(2, 40)
    ctx.append([0, 1], k, v)
    with pytest.raises(KvcError) as e:
        ctx.check_wait_timeout(50)
    assert e.value.status == kvc.KVC_ERR_DEVICE_TIMEOUT
    ctx.sync()  # the status word was cleared
    ctx.compress("random", np.array([20, 20], np.int32), 1)
    ctx.sync()
    assert list(ctx.lengths()[0]) == [20, 20]
    ctx.close()
