"""The device-side time-out path of the bounded waits (needs a B200).

A test-only build of the library (``libkvq_test_timeout.so``, same sources,
built by ``rotated_int4_kv_kvq_b200.build``) gives up every bounded wait
after 1 ms, and its forward kernel arms the mbarrier of input tile 0 without
issuing the copy for it.  The warp waiting on that tile therefore runs out of
time with no copy in flight: no fault and no hang.  The kernel records
KVQ_ERR_DEVICE_TIMEOUT in the device status word and returns; the host reads
and clears the word, and the context stays usable."""

import ctypes
import os

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

TIMEOUT = 8  # KVQ_ERR_DEVICE_TIMEOUT


@pytest.fixture(scope="module")
def kvq():
    from rotated_int4_kv_kvq_b200 import kvq as mod
    return mod


@pytest.fixture(scope="module")
def tlib():
    from rotated_int4_kv_kvq_b200 import build
    path = build.variant_path("timeout")
    if not os.path.exists(path):
        build.build_test_variant("timeout")
    lib = ctypes.CDLL(path)
    p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    lib.kvq_rot_quant_fwd.argtypes = [p, i64, i32, i32, p, i32, p, p, p]
    lib.kvq_rot_quant_fwd.restype = i32
    lib.kvq_device_status.argtypes = [i32]
    lib.kvq_device_status.restype = i32
    return lib


def test_timed_out_wait_is_recorded_and_cleared(tlib, kvq):
    from rotated_int4_kv_kvq_b200 import workloads as W
    d, g, n = 64, 64, 64  # two input tiles of 32 vectors; tile 0 never arrives
    torch.manual_seed(0)
    x = torch.randn((n, d), device="cuda").half()
    signs = torch.from_numpy(W.make_signs(d)).cuda()
    packed = torch.zeros((n, d // 2), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((n, d // g), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert tlib.kvq_device_status(1) == 0  # nothing recorded yet
    st = tlib.kvq_rot_quant_fwd(x.data_ptr(), n, d, g, signs.data_ptr(), 0, packed.data_ptr(),
                                scales.data_ptr(), stream)
    assert st == 0  # enqueued
    assert tlib.kvq_device_status(0) == TIMEOUT  # recorded, read without clearing
    assert tlib.kvq_device_status(1) == TIMEOUT  # read and cleared
    assert tlib.kvq_device_status(1) == 0
    # the warp that gave up wrote nothing for tile 0; the other tile is done
    assert not packed[:32].any() and not scales[:32].any()
    p_ref, s_ref = kvq.kvq_rot_quant_fwd(x, signs, 0, g)
    torch.cuda.synchronize()
    assert torch.equal(packed[32:], p_ref[32:]) and torch.equal(scales[32:], s_ref[32:])
    # the context is still usable: the product library runs and agrees with itself
    p2, s2 = kvq.kvq_rot_quant_fwd(x, signs, 0, g)
    assert kvq.kvq_device_status() == 0
    assert torch.equal(p2, p_ref) and torch.equal(s2, s_ref)
    assert np.isfinite(s2.cpu().numpy()).all()
