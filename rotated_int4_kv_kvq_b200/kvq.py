"""Thin Python binding over the C ABI of libkvq.so (include/kvq.h).

Argument marshalling only: tensors are checked and turned into raw device
pointers; all work runs in the library's CUDA kernels.  PyTorch supplies the
device memory and the stream.  There is no CPU fallback: importing this
module fails if libkvq.so has not been built
(``python -m rotated_int4_kv_kvq_b200.build``).
"""

from __future__ import annotations

import contextlib
import ctypes
import os

import torch

SRFT = 0
SRHT = 1

KVQ_OK = 0
STATUS = {
    0: "KVQ_OK", 1: "KVQ_ERR_NULL", 2: "KVQ_ERR_BAD_DIM", 3: "KVQ_ERR_BAD_GROUP",
    4: "KVQ_ERR_MISALIGNED", 5: "KVQ_ERR_BAD_ROT", 6: "KVQ_ERR_CUDA",
    7: "KVQ_ERR_BAD_SIZE", 8: "KVQ_ERR_DEVICE_TIMEOUT", 9: "KVQ_ERR_UNSUPPORTED_DEVICE",
    10: "KVQ_ERR_BAD_BITS",
}

LIB_PATH = os.environ.get("KVQ_LIBRARY") or os.path.join(
    os.path.dirname(os.path.abspath(__file__)), "libkvq.so")

EXPORTS = ("kvq_rot_quant_fwd", "kvq_dequant_rot_inv", "kvq_rot_quant_fwd_lambda",
           "kvq_dequant_rot_inv_lambda", "kvq_rot_quant_fwd_bits", "kvq_dequant_rot_inv_bits",
           "kvq_decode_step", "kvq_decode_step_windowed",
           "kvq_attend_decode", "kvq_status_string", "kvq_device_status", "kvq_version")


class KVQError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {STATUS.get(status, status)} ({status_string(status)})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m rotated_int4_kv_kvq_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    lib.kvq_rot_quant_fwd.argtypes = [p, i64, i32, i32, p, i32, p, p, p]
    lib.kvq_rot_quant_fwd.restype = i32
    lib.kvq_dequant_rot_inv.argtypes = [p, p, i64, i32, i32, p, i32, p, p]
    lib.kvq_dequant_rot_inv.restype = i32
    lib.kvq_rot_quant_fwd_lambda.argtypes = [p, i64, i32, i32, p, p, i32, p, p, p]
    lib.kvq_rot_quant_fwd_lambda.restype = i32
    lib.kvq_dequant_rot_inv_lambda.argtypes = [p, p, i64, i32, i32, p, p, i32, p, p]
    lib.kvq_dequant_rot_inv_lambda.restype = i32
    lib.kvq_decode_step.argtypes = [p, p, p, i64, i64, i64, i32, i32, p, i32, p, p]
    lib.kvq_decode_step.restype = i32
    lib.kvq_decode_step_windowed.argtypes = [p, p, p, p, i64, i64, i64, i32, i32, i32, p, i32, p]
    lib.kvq_decode_step_windowed.restype = i32
    lib.kvq_rot_quant_fwd_bits.argtypes = [p, i64, i32, i32, i32, p, i32, p, p, p]
    lib.kvq_rot_quant_fwd_bits.restype = i32
    lib.kvq_dequant_rot_inv_bits.argtypes = [p, p, i64, i32, i32, i32, p, i32, p, p]
    lib.kvq_dequant_rot_inv_bits.restype = i32
    lib.kvq_attend_decode.argtypes = [p, p, p, p, p, i64, i32, i64, i64, i32, i32, p, i32,
                                      ctypes.c_float, p, p]
    lib.kvq_attend_decode.restype = i32
    lib.kvq_status_string.argtypes = [i32]
    lib.kvq_status_string.restype = ctypes.c_char_p
    lib.kvq_device_status.argtypes = [i32]
    lib.kvq_device_status.restype = i32
    lib.kvq_version.argtypes = []
    lib.kvq_version.restype = i32
    return lib


lib = _load()


def status_string(status: int) -> str:
    return lib.kvq_status_string(int(status)).decode()


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


# torch's query of a device's current raw stream handle; building a
# torch.cuda.Stream object per call costs ~2 us, the raw query ~0.1 us.
_raw_current_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream, dev: torch.device) -> int | None:
    """Raw handle of `stream`; None means the current stream of `dev`."""
    if stream is None:
        if _raw_current_stream is not None and dev.index is not None:
            return _raw_current_stream(dev.index)
        stream = torch.cuda.current_stream(dev)
    return stream.cuda_stream if isinstance(stream, torch.cuda.Stream) else int(stream)


def _device_of(tensors, stream) -> torch.device:
    """The one CUDA device that every tensor argument lives on.

    The library launches on the calling thread's current device and builds
    its copy descriptors over the pointers it is given, so all operands of a
    call must share one device; an explicit torch stream must belong to it
    too.  Raises ValueError before anything is launched otherwise.  (A raw
    integer stream handle cannot be checked here; it must belong to the same
    device.)"""
    devs = {t.device for t in tensors if t is not None}
    if len(devs) != 1:
        raise ValueError("all tensor arguments must be on one CUDA device, got "
                         + ", ".join(sorted(str(d) for d in devs)))
    dev = devs.pop()
    if isinstance(stream, torch.cuda.Stream) and stream.device != dev:
        raise ValueError(f"stream is on {stream.device}, tensors on {dev}")
    return dev


def _current(dev: torch.device):
    """Context that makes `dev` the current device for one library call."""
    if dev.index is None or dev.index == torch.cuda.current_device():
        return contextlib.nullcontext()
    return torch.cuda.device(dev)


def _check(t: torch.Tensor, name: str, dtype, shape):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.shape != tuple(shape):  # torch.Size compares as a tuple
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _raise(fn: str, st: int):
    if st != KVQ_OK:
        raise KVQError(fn, st)


def kvq_rot_quant_fwd(x: torch.Tensor, signs: torch.Tensor, rot: int, group: int,
                      packed: torch.Tensor | None = None,
                      scales: torch.Tensor | None = None, stream=None,
                      lam: torch.Tensor | None = None):
    """Forward step on x [n_vec, d] fp16 -> (packed [n_vec, d/2] u8,
    scales [n_vec, d/group] f32).  Outputs are allocated when not given.
    With ``lam`` ([d] f32), x is scaled channel-wise first
    (kvq_rot_quant_fwd_lambda)."""
    n, d = x.shape
    _check(x, "x", torch.float16, (n, d))
    _check(signs, "signs", torch.int8, (d,))
    if packed is None:
        packed = torch.empty((n, d // 2), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((n, d // group), dtype=torch.float32, device=x.device)
    _check(packed, "packed", torch.uint8, (n, d // 2))
    _check(scales, "scales", torch.float32, (n, d // group))
    if lam is not None:
        _check(lam, "lam", torch.float32, (d,))
    dev = _device_of((x, signs, packed, scales, lam), stream)
    with _current(dev):
        if lam is None:
            st = lib.kvq_rot_quant_fwd(_ptr(x), n, d, group, _ptr(signs), rot, _ptr(packed),
                                       _ptr(scales), _stream(stream, dev))
            _raise("kvq_rot_quant_fwd", st)
        else:
            st = lib.kvq_rot_quant_fwd_lambda(_ptr(x), n, d, group, _ptr(signs), _ptr(lam), rot,
                                              _ptr(packed), _ptr(scales), _stream(stream, dev))
            _raise("kvq_rot_quant_fwd_lambda", st)
    return packed, scales


def kvq_dequant_rot_inv(packed: torch.Tensor, scales: torch.Tensor, signs: torch.Tensor,
                        rot: int, group: int, out: torch.Tensor | None = None, stream=None,
                        lam: torch.Tensor | None = None):
    """Inverse step -> out [n_vec, d] fp16 (allocated when not given).  With
    ``lam`` ([d] f32) the result is divided channel-wise by it
    (kvq_dequant_rot_inv_lambda)."""
    n, half = packed.shape
    d = 2 * half
    _check(packed, "packed", torch.uint8, (n, half))
    _check(scales, "scales", torch.float32, (n, d // group))
    _check(signs, "signs", torch.int8, (d,))
    if out is None:
        out = torch.empty((n, d), dtype=torch.float16, device=packed.device)
    _check(out, "out", torch.float16, (n, d))
    if lam is not None:
        _check(lam, "lam", torch.float32, (d,))
    dev = _device_of((packed, scales, signs, out, lam), stream)
    with _current(dev):
        if lam is None:
            st = lib.kvq_dequant_rot_inv(_ptr(packed), _ptr(scales), n, d, group, _ptr(signs),
                                         rot, _ptr(out), _stream(stream, dev))
            _raise("kvq_dequant_rot_inv", st)
        else:
            st = lib.kvq_dequant_rot_inv_lambda(_ptr(packed), _ptr(scales), n, d, group,
                                                _ptr(signs), _ptr(lam), rot, _ptr(out),
                                                _stream(stream, dev))
            _raise("kvq_dequant_rot_inv_lambda", st)
    return out


def kvq_rot_quant_fwd_bits(x: torch.Tensor, signs: torch.Tensor, rot: int, group: int,
                           bits: int, packed: torch.Tensor | None = None,
                           scales: torch.Tensor | None = None, stream=None):
    """Forward step with b-bit codes: packed [n_vec, d*bits/8] u8 (little-endian
    bitstream per vector), scales [n_vec, d/group] f32."""
    n, d = x.shape
    qp = d * bits // 8
    _check(x, "x", torch.float16, (n, d))
    _check(signs, "signs", torch.int8, (d,))
    if packed is None:
        packed = torch.empty((n, qp), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((n, d // group), dtype=torch.float32, device=x.device)
    _check(packed, "packed", torch.uint8, (n, qp))
    _check(scales, "scales", torch.float32, (n, d // group))
    dev = _device_of((x, signs, packed, scales), stream)
    with _current(dev):
        st = lib.kvq_rot_quant_fwd_bits(_ptr(x), n, d, group, bits, _ptr(signs), rot,
                                        _ptr(packed), _ptr(scales), _stream(stream, dev))
    _raise("kvq_rot_quant_fwd_bits", st)
    return packed, scales


def kvq_dequant_rot_inv_bits(packed: torch.Tensor, scales: torch.Tensor, signs: torch.Tensor,
                             rot: int, group: int, bits: int, out: torch.Tensor | None = None,
                             stream=None):
    """Inverse step of kvq_rot_quant_fwd_bits -> out [n_vec, d] fp16."""
    n, qp = packed.shape
    d = qp * 8 // bits
    _check(packed, "packed", torch.uint8, (n, qp))
    _check(scales, "scales", torch.float32, (n, d // group))
    _check(signs, "signs", torch.int8, (d,))
    if out is None:
        out = torch.empty((n, d), dtype=torch.float16, device=packed.device)
    _check(out, "out", torch.float16, (n, d))
    dev = _device_of((packed, scales, signs, out), stream)
    with _current(dev):
        st = lib.kvq_dequant_rot_inv_bits(_ptr(packed), _ptr(scales), n, d, group, bits,
                                          _ptr(signs), rot, _ptr(out), _stream(stream, dev))
    _raise("kvq_dequant_rot_inv_bits", st)
    return out


def kvq_decode_step(x_new: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, pos: int,
                    signs: torch.Tensor, rot: int, group: int,
                    out: torch.Tensor | None = None, stream=None):
    """Decode step on a head-major cache: packed [H, cap, d/2] u8 and
    scales [H, cap, d/group] f32 get row ``pos``; returns out [H, pos+1, d]."""
    h, d = x_new.shape
    cap = packed.shape[1]
    _check(x_new, "x_new", torch.float16, (h, d))
    _check(packed, "packed", torch.uint8, (h, cap, d // 2))
    _check(scales, "scales", torch.float32, (h, cap, d // group))
    _check(signs, "signs", torch.int8, (d,))
    if out is None:
        out = torch.empty((h, pos + 1, d), dtype=torch.float16, device=x_new.device)
    _check(out, "out", torch.float16, (h, pos + 1, d))
    dev = _device_of((x_new, packed, scales, signs, out), stream)
    with _current(dev):
        st = lib.kvq_decode_step(_ptr(x_new), _ptr(packed), _ptr(scales), h, cap, pos, d, group,
                                 _ptr(signs), rot, _ptr(out), _stream(stream, dev))
    _raise("kvq_decode_step", st)
    return out


def kvq_decode_step_windowed(x_new: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor,
                             kv: torch.Tensor, pos: int, signs: torch.Tensor, rot: int, group: int,
                             window: int = 16, stream=None):
    """Decode step with a dequantized-prefix cache: kv [H, cap, d] fp16 is the
    persistent attention view (row ``pos`` gets x_new; a completed window of
    ``window`` rows is quantized into packed/scales and replaced by its
    dequantized values).  Returns kv."""
    h, d = x_new.shape
    cap = packed.shape[1]
    _check(x_new, "x_new", torch.float16, (h, d))
    _check(packed, "packed", torch.uint8, (h, cap, d // 2))
    _check(scales, "scales", torch.float32, (h, cap, d // group))
    _check(kv, "kv", torch.float16, (h, cap, d))
    _check(signs, "signs", torch.int8, (d,))
    dev = _device_of((x_new, packed, scales, kv, signs), stream)
    with _current(dev):
        st = lib.kvq_decode_step_windowed(_ptr(x_new), _ptr(packed), _ptr(scales), _ptr(kv), h,
                                          cap, pos, window, d, group, _ptr(signs), rot,
                                          _stream(stream, dev))
    _raise("kvq_decode_step_windowed", st)
    return kv


def kvq_attend_decode(q: torch.Tensor, k_packed: torch.Tensor, k_scales: torch.Tensor,
                      v_packed: torch.Tensor, v_scales: torch.Tensor, length: int,
                      signs: torch.Tensor, rot: int, group: int, sm_scale: float | None = None,
                      out: torch.Tensor | None = None, stream=None):
    """Decode attention over the int4 cache: q [H, nq, d] fp16 against
    rows [0, length) of the K/V caches [H, cap, d/2] (+ scales); returns
    out [H, nq, d] fp16.  sm_scale defaults to 1/sqrt(d)."""
    h, nq, d = q.shape
    cap = k_packed.shape[1]
    _check(q, "q", torch.float16, (h, nq, d))
    for name, t in (("k_packed", k_packed), ("v_packed", v_packed)):
        _check(t, name, torch.uint8, (h, cap, d // 2))
    for name, t in (("k_scales", k_scales), ("v_scales", v_scales)):
        _check(t, name, torch.float32, (h, cap, d // group))
    _check(signs, "signs", torch.int8, (d,))
    if out is None:
        out = torch.empty((h, nq, d), dtype=torch.float16, device=q.device)
    _check(out, "out", torch.float16, (h, nq, d))
    scale = float(sm_scale) if sm_scale is not None else d ** -0.5
    dev = _device_of((q, k_packed, k_scales, v_packed, v_scales, signs, out), stream)
    with _current(dev):
        st = lib.kvq_attend_decode(_ptr(q), _ptr(k_packed), _ptr(k_scales), _ptr(v_packed),
                                   _ptr(v_scales), h, nq, cap, length, d, group, _ptr(signs),
                                   rot, scale, _ptr(out), _stream(stream, dev))
    _raise("kvq_attend_decode", st)
    return out


def kvq_device_status(clear: bool = True) -> int:
    """Synchronize the device and return the kernels' device status code."""
    return int(lib.kvq_device_status(1 if clear else 0))


def kvq_version() -> int:
    return int(lib.kvq_version())
