"""The C ABI of libkvq.so without a GPU: it loads, exports every function
include/kvq.h declares, and rejects bad arguments on the host before any
CUDA call (fake pointers below are never dereferenced)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvq.h")


@pytest.fixture(scope="module")
def kvq():
    from rotated_int4_kv_kvq_b200 import build
    build.build()
    from rotated_int4_kv_kvq_b200 import kvq as mod
    return mod


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for fn in ("kvq_rot_quant_fwd", "kvq_dequant_rot_inv", "kvq_decode_step",
               "kvq_status_string"):
        assert fn in names


def test_library_exports_every_declared_symbol(kvq):
    lib = ctypes.CDLL(kvq.LIB_PATH)
    for fn in declared_functions():
        assert hasattr(lib, fn), fn
    assert set(kvq.EXPORTS) == set(declared_functions())


def test_status_strings(kvq):
    for code in range(11):
        assert kvq.status_string(code)
    assert kvq.status_string(0) == "ok"
    assert kvq.status_string(12345) == "unknown status"
    assert kvq.kvq_version() >= 100


A = 0x10000  # 16-byte aligned fake device address (never dereferenced)


@pytest.mark.parametrize("d,g,rot,expect", [
    (32, 32, 0, 2), (96, 32, 0, 2), (512, 32, 0, 2),
    (64, 16, 0, 3), (64, 128, 0, 3), (128, 48, 1, 3), (256, 512, 1, 3),
    (64, 32, 2, 5), (64, 32, -1, 5),
])
def test_bad_shape_is_rejected(kvq, d, g, rot, expect):
    lib = kvq.lib
    assert lib.kvq_rot_quant_fwd(A, 10, d, g, A, rot, A, A, None) == expect
    assert lib.kvq_dequant_rot_inv(A, A, 10, d, g, A, rot, A, None) == expect
    assert lib.kvq_decode_step(A, A, A, 2, 8, 3, d, g, A, rot, A, None) == expect


def test_null_and_misaligned_pointers(kvq):
    lib = kvq.lib
    assert lib.kvq_rot_quant_fwd(None, 10, 64, 32, A, 0, A, A, None) == 1
    assert lib.kvq_rot_quant_fwd(A, 10, 64, 32, None, 0, A, A, None) == 1
    assert lib.kvq_rot_quant_fwd(A, 10, 64, 32, A, 0, A, None, None) == 1
    assert lib.kvq_dequant_rot_inv(A, A, 10, 64, 32, A, 0, None, None) == 1
    assert lib.kvq_decode_step(A, None, A, 2, 8, 3, 64, 32, A, 0, A, None) == 1
    for bad in (A + 2, A + 8):
        assert lib.kvq_rot_quant_fwd(bad, 10, 64, 32, A, 0, A, A, None) == 4
        assert lib.kvq_rot_quant_fwd(A, 10, 64, 32, A, 0, bad, A, None) == 4
        assert lib.kvq_rot_quant_fwd(A, 10, 64, 32, A, 0, A, bad, None) == 4
        assert lib.kvq_dequant_rot_inv(A, A, 10, 64, 32, A, 0, bad, None) == 4
        assert lib.kvq_decode_step(A, A, A, 2, 8, 3, 64, 32, A, 0, bad, None) == 4
    assert lib.kvq_decode_step(A, A, A + 2, 2, 8, 3, 64, 32, A, 0, A, None) == 4


def test_bad_sizes(kvq):
    lib = kvq.lib
    assert lib.kvq_rot_quant_fwd(A, -1, 64, 32, A, 0, A, A, None) == 7
    assert lib.kvq_rot_quant_fwd(A, 1 << 31, 64, 32, A, 0, A, A, None) == 7
    assert lib.kvq_dequant_rot_inv(A, A, -5, 64, 32, A, 0, A, None) == 7
    # decode: pos must be < cap, cap >= 1, n_heads >= 0
    assert lib.kvq_decode_step(A, A, A, 2, 8, 8, 64, 32, A, 0, A, None) == 7
    assert lib.kvq_decode_step(A, A, A, 2, 0, 0, 64, 32, A, 0, A, None) == 7
    assert lib.kvq_decode_step(A, A, A, -1, 8, 3, 64, 32, A, 0, A, None) == 7
    assert lib.kvq_decode_step(A, A, A, 2, 8, -1, 64, 32, A, 0, A, None) == 7


def test_empty_calls_are_noops(kvq):
    lib = kvq.lib
    assert lib.kvq_rot_quant_fwd(A, 0, 64, 32, A, 0, A, A, None) == 0
    assert lib.kvq_dequant_rot_inv(A, A, 0, 256, 256, A, 1, A, None) == 0
    assert lib.kvq_decode_step(A, A, A, 0, 8, 3, 128, 64, A, 0, A, None) == 0


def test_windowed_decode_host_checks(kvq):
    lib = kvq.lib
    win = lib.kvq_decode_step_windowed
    # (x_new, packed, scales, kv, n_heads, cap, pos, window, d, group, signs, rot, stream)
    assert win(A, A, A, A, 2, 8, 3, 16, 96, 32, A, 0, None) == 2
    assert win(A, A, A, A, 2, 8, 3, 16, 64, 16, A, 0, None) == 3
    assert win(A, A, A, A, 2, 8, 3, 16, 64, 32, A, 3, None) == 5
    assert win(A, A, A, None, 2, 8, 3, 16, 64, 32, A, 0, None) == 1
    assert win(None, A, A, A, 2, 8, 3, 16, 64, 32, A, 0, None) == 1
    assert win(A, A, A, A + 8, 2, 8, 3, 16, 64, 32, A, 0, None) == 4
    assert win(A, A, A + 2, A, 2, 8, 3, 16, 64, 32, A, 0, None) == 4
    for window in (0, -3, 4097):
        assert win(A, A, A, A, 2, 8, 3, window, 64, 32, A, 0, None) == 7
    assert win(A, A, A, A, 2, 8, 8, 16, 64, 32, A, 0, None) == 7  # pos == cap
    assert win(A, A, A, A, -1, 8, 3, 16, 64, 32, A, 0, None) == 7
    assert win(A, A, A, A, 0, 8, 3, 16, 64, 32, A, 0, None) == 0  # no heads: no-op


def test_lambda_host_checks(kvq):
    lib = kvq.lib
    fwd, inv = lib.kvq_rot_quant_fwd_lambda, lib.kvq_dequant_rot_inv_lambda
    # (x, n, d, g, signs, lambda, rot, packed, scales, stream)
    assert fwd(A, 10, 64, 32, A, None, 0, A, A, None) == 1
    assert inv(A, A, 10, 64, 32, A, None, 0, A, None) == 1
    assert fwd(A, 10, 64, 32, A, A + 4, 0, A, A, None) == 4
    assert inv(A, A, 10, 64, 32, A, A + 4, 0, A, None) == 4
    assert fwd(A, 10, 96, 32, A, A, 0, A, A, None) == 2
    assert inv(A, A, 10, 64, 16, A, A, 0, A, None) == 3
    assert fwd(A, 0, 64, 32, A, A, 0, A, A, None) == 0
    assert inv(A, A, 0, 64, 32, A, A, 1, A, None) == 0


def test_attend_host_checks(kvq):
    lib = kvq.lib
    att = lib.kvq_attend_decode
    # (q, kp, ks, vp, vs, n_kv, n_q, cap, len, d, g, signs, rot, sm_scale, out, stream)
    assert att(A, A, A, A, A, 2, 4, 16, 10, 96, 32, A, 0, 0.125, A, None) == 2
    assert att(A, A, A, A, A, 2, 4, 16, 10, 64, 16, A, 0, 0.125, A, None) == 3
    assert att(A, A, A, A, A, 2, 4, 16, 10, 64, 32, A, 7, 0.125, A, None) == 5
    assert att(A, A, A, A, A, 2, 0, 16, 10, 64, 32, A, 0, 0.125, A, None) == 7
    assert att(A, A, A, A, A, 2, 9, 16, 10, 64, 32, A, 0, 0.125, A, None) == 7
    assert att(A, A, A, A, A, 2, 4, 16, 0, 64, 32, A, 0, 0.125, A, None) == 7
    assert att(A, A, A, A, A, 2, 4, 16, 17, 64, 32, A, 0, 0.125, A, None) == 7
    assert att(A, A, A, A, A, 70000, 4, 16, 10, 64, 32, A, 0, 0.125, A, None) == 7
    assert att(A, A, A, A, A, 2, 4, 16, 10, 64, 32, A, 0, float("inf"), A, None) == 7
    assert att(A, None, A, A, A, 2, 4, 16, 10, 64, 32, A, 0, 0.125, A, None) == 1
    assert att(A, A, A, A, A, 2, 4, 16, 10, 64, 32, A, 0, 0.125, None, None) == 1
    assert att(A + 8, A, A, A, A, 2, 4, 16, 10, 64, 32, A, 0, 0.125, A, None) == 4
    assert att(A, A, A + 2, A, A, 2, 4, 16, 10, 64, 32, A, 0, 0.125, A, None) == 4
    assert att(A, A, A, A, A, 0, 4, 16, 10, 64, 32, A, 0, 0.125, A, None) == 0


def test_bits_host_checks(kvq):
    lib = kvq.lib
    fwd, inv = lib.kvq_rot_quant_fwd_bits, lib.kvq_dequant_rot_inv_bits
    # (x, n, d, g, bits, signs, rot, packed, scales, stream)
    for bits in (0, 1, 2, 5, 7, 9, 16):
        assert fwd(A, 10, 128, 32, bits, A, 0, A, A, None) == 10
        assert inv(A, A, 10, 128, 32, bits, A, 0, A, None) == 10
    assert fwd(A, 10, 64, 32, 3, A, 0, A, A, None) == 10  # 24-byte rows
    assert fwd(A, 10, 96, 32, 8, A, 0, A, A, None) == 2
    assert fwd(A, 0, 128, 32, 3, A, 0, A, A, None) == 0
    assert inv(A, A, 0, 64, 64, 6, A, 1, A, None) == 0


def test_operands_on_different_devices_are_rejected_before_launch(kvq):
    import torch
    a = torch.empty(4, device="cpu")
    b = torch.empty(4, device="meta")
    with pytest.raises(ValueError, match="one CUDA device"):
        kvq._device_of((a, b, None), None)
    assert kvq._device_of((a, None, a), None) == a.device


def test_non_cuda_tensors_are_rejected_before_launch(kvq):
    import torch
    x = torch.zeros((32, 64), dtype=torch.float16)
    signs = torch.ones(64, dtype=torch.int8)
    with pytest.raises(TypeError, match="CUDA tensor"):
        kvq.kvq_rot_quant_fwd(x, signs, kvq.SRFT, 64)


@pytest.mark.gpu
def test_calls_run_on_the_tensors_device(kvq):
    """Operands on one device other than the current one run there; operands
    split over two devices, or a stream of another device, raise before any
    launch."""
    import torch
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two CUDA devices")
    d, g = 64, 64
    x1 = torch.randn((64, d), device="cuda:1").half()
    s1 = torch.ones(d, dtype=torch.int8, device="cuda:1")
    with torch.cuda.device(0):
        p1, sc1 = kvq.kvq_rot_quant_fwd(x1, s1, kvq.SRFT, g)
        torch.cuda.synchronize(1)
    with torch.cuda.device(1):
        p_ref, sc_ref = kvq.kvq_rot_quant_fwd(x1, s1, kvq.SRFT, g)
        torch.cuda.synchronize(1)
    assert torch.equal(p1, p_ref) and torch.equal(sc1, sc_ref)
    s0 = s1.to("cuda:0")
    with pytest.raises(ValueError, match="one CUDA device"):
        kvq.kvq_rot_quant_fwd(x1, s0, kvq.SRFT, g)
    with pytest.raises(ValueError, match="stream"):
        kvq.kvq_rot_quant_fwd(x1, s1, kvq.SRFT, g, stream=torch.cuda.Stream(device=0))


def test_library_exports_only_the_declared_functions(kvq):
    """Built with hidden visibility: the dynamic symbol table holds the C API
    and nothing else (no inline or template statics that a second build of
    the library in the same process would share)."""
    import shutil
    import subprocess
    nm = shutil.which("nm")
    if nm is None:
        pytest.skip("nm not available")
    r = subprocess.run([nm, "-D", "--defined-only", kvq.LIB_PATH], capture_output=True,
                       text=True, check=True)
    names = {line.split()[-1] for line in r.stdout.splitlines() if line.strip()}
    assert names == set(declared_functions())
