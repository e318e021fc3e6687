"""CPU oracle for rotate-then-quantize int4 KV-cache compression.

TEST INFRASTRUCTURE ONLY.  This module is imported by ``tests/``, by
``__graft_entry__.smoke()`` and by the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py``.  The product path (``rotated_int4_kv_kvq_b200``) never
imports, calls or links it, and this module imports nothing from the product.

It is a plain, slow, obviously correct restatement of what the method
computes, in float64 (numpy), with direct d x d matrices instead of fast
transforms.  Every function cites the passage it follows.  Sources:

* [P1] "Quantization Speed Is Often a Kernel Problem"
  (jecision.com/en/blog/quantization-kernel-dispatch), a write-up of
  arXiv 2605.05699v1.  Section "First, the 17%": each K/V vector is
  multiplied by a fixed random +-1 pattern, rotated with an FFT (SRFT),
  compressed to int4, later dequantized and rotated back; the control is a
  sign-randomized Hadamard transform (SRHT).  Section "Fusing four steps into
  two kernels is not enough": per-group abs-max scales (one per 32 values).
* [P4] "Quantization & Serving" (gowda.ai/ml-refresh/quantization.html):
  symmetric absmax quantization, x_hat_i = s q_i, rounding error at most s/2
  before clipping.
* [P3] "Day 9 - Quantization: Shrink the Bytes Themselves"
  (guan404ming.com/blog/9), section "Decode into HBM, or Decode into
  Registers": the dequantization belongs inside the consuming kernel, so the
  decoded values live only in registers.
* [P5] "Chapter 25 - Quantization: The Hardware View"
  (karam-nus.github.io/chips/25_quantization_hardware_view.html), section
  "Kernels: Marlin, CUTLASS, and Why INT4 Packing Needs Special Code": two
  int4 values per byte, w0 in the low nibble, w1 in the high nibble; section
  "Python: Quantize, Simulate the Integer GEMM...": qmax = 2**(b-1)-1,
  scale = amax/qmax, q = clamp(round(x/scale), -qmax-1, qmax).

Readings where the pages are silent:

* R1 real packing of the rfft output into d reals (stated with the problem):
  y[0] = Re X_0/sqrt(d), y[1] = Re X_{d/2}/sqrt(d),
  y[2k] = sqrt(2) Re X_k/sqrt(d), y[2k+1] = sqrt(2) Im X_k/sqrt(d), 1<=k<d/2.
* R2 DFT sign convention X_k = sum_n u_n exp(-2 pi i k n / d) (numpy/torch
  ``rfft``; [P1] names rfft/irfft).
* R3 SRHT = Sylvester-ordered Walsh-Hadamard H_ij = (-1)^popcount(i&j),
  scaled by 1/sqrt(d), full d -> d, no subsampling.
* R4 scale divisor 7 (qmax = 2^(4-1)-1, [P5]); codes in [-8, 7]; ties round
  half to even.
* R5 the quantizer takes its decision in float32, the precision of the pages'
  own sample quantizer ([P5], torch default dtype) and of the fused kernel's
  reduction ([P1] "Before you celebrate..."): y is rounded to float32 once,
  m = max|y| over the group, s = fl32(m / 7), q = rint(fl32(y / s)).
  A group with m = 0 gets s = 0 and q = 0.
* R6 nibble encoding: two's complement ``q & 0xF``; element 2b in the low
  nibble of byte b, element 2b+1 in the high nibble ([P5] packing figure).
* R7 groups are runs of g consecutive coordinates of the rotated, packed y.
* R8 inverse: x_hat = D R^T y_hat with y_hat = s q in float64, rounded to
  float16 (round to nearest even) at the end.
* R16 other code widths b: qmax = 2^(b-1) - 1 ([P5] formula), codes in a
  little-endian bitstream per vector (code i at bits [b i, b i + b)); b = 4
  is the nibble layout of R6.

Parity pins for every function live in ``tests/test_oracle.py``.
"""

from __future__ import annotations

import numpy as np

SRFT = 0
SRHT = 1
QMAX = 7  # 2**(4-1) - 1, [P5] sample quantizer
QMIN = -8  # -qmax - 1, [P5] sample quantizer

__all__ = [
    "SRFT", "SRHT", "QMAX", "QMIN",
    "sign_flip", "srft_matrix", "srht_matrix", "rotation_matrix",
    "rotate", "inverse_rotate", "quantize_groups", "dequantize_groups",
    "pack_nibbles", "unpack_nibbles", "rot_quant_fwd", "dequant_rot_inv",
    "rotated_values", "near_tie_distance", "decode_step", "decode_step_windowed",
    "dequant_rotated_f64", "attend_decode", "pack_codes", "unpack_codes",
]


def sign_flip(x, signs):
    """u = D x with D = diag(signs), signs in {+1, -1}.

    [P1] "First, the 17%": multiply by a fixed random +-1 pattern first.
    D is its own inverse, so the same function undoes the flip.
    """
    x = np.asarray(x, dtype=np.float64)
    s = np.asarray(signs, dtype=np.float64)
    if x.shape[-1] != s.shape[-1]:
        raise ValueError("signs must have one entry per coordinate")
    return x * s


def srft_matrix(d: int) -> np.ndarray:
    """Orthonormal real-packed DFT matrix R (d x d, float64), y = R u.

    Direct O(d^2) definition: row 0 is Re X_0, row 1 is Re X_{d/2}, rows 2k and
    2k+1 are sqrt(2) Re X_k and sqrt(2) Im X_k with
    X_k = sum_n u_n exp(-2 pi i k n / d) (readings R1, R2), all over sqrt(d).
    Angles are reduced exactly as 2 pi ((k n) mod d) / d before cos/sin.
    """
    if d < 2 or d % 2:
        raise ValueError("SRFT needs an even d >= 2")
    n = np.arange(d)
    r = np.empty((d, d), dtype=np.float64)
    r[0] = 1.0
    r[1] = np.where(n % 2 == 0, 1.0, -1.0)  # cos(pi n)
    for k in range(1, d // 2):
        ang = 2.0 * np.pi * ((k * n) % d) / d
        r[2 * k] = np.sqrt(2.0) * np.cos(ang)
        r[2 * k + 1] = -np.sqrt(2.0) * np.sin(ang)  # Im of exp(-i ang)
    return r / np.sqrt(d)


def _popcount(a: np.ndarray) -> np.ndarray:
    a = a.astype(np.int64)
    c = np.zeros_like(a)
    while np.any(a):
        c += a & 1
        a >>= 1
    return c


def srht_matrix(d: int) -> np.ndarray:
    """Orthonormal Walsh-Hadamard matrix H/sqrt(d) in Sylvester (natural) order.

    H_ij = (-1)^popcount(i & j) (reading R3); the control rotation of
    [P1] "First, the 17%" (sign-randomized Hadamard transform).
    """
    if d < 1 or d & (d - 1):
        raise ValueError("SRHT needs a power-of-two d")
    i = np.arange(d)
    parity = _popcount(np.bitwise_and.outer(i, i)) & 1
    return np.where(parity == 0, 1.0, -1.0) / np.sqrt(d)


def rotation_matrix(d: int, rot: int) -> np.ndarray:
    if rot == SRFT:
        return srft_matrix(d)
    if rot == SRHT:
        return srht_matrix(d)
    raise ValueError(f"unknown rotation {rot}")


def rotate(u, rot: int) -> np.ndarray:
    """y = R u for every row u of a [n, d] array (float64)."""
    u = np.asarray(u, dtype=np.float64)
    r = rotation_matrix(u.shape[-1], rot)
    return u @ r.T


def inverse_rotate(y, rot: int) -> np.ndarray:
    """u = R^T y for every row y (R is orthonormal, so R^T = R^-1)."""
    y = np.asarray(y, dtype=np.float64)
    r = rotation_matrix(y.shape[-1], rot)
    return y @ r


def quantize_groups(y, group: int, bits: int = 4):
    """Per-group symmetric absmax quantization (readings R4, R5, R7).

    [P1] "Fusing four steps...": one abs-max per group of consecutive values.
    [P5] sample quantizer: scale = amax / qmax, q = clamp(round(y/scale),
    -qmax-1, qmax) with qmax = 2**(bits-1) - 1 (7 for int4; the pages' other
    widths, [P1] "6-bit and 8-bit are lossless; 3-bit is worse", use the same
    formula).  [P4]: the rounding error is at most s/2.

    Returns (q int8 [n, d], s float32 [n, d/group]).
    """
    qmax = 2 ** (bits - 1) - 1
    y32 = np.asarray(y, dtype=np.float64).astype(np.float32)
    n, d = y32.shape
    if group <= 0 or d % group:
        raise ValueError("group must divide d")
    yg = y32.reshape(n, d // group, group)
    m = np.abs(yg).max(axis=2)  # exact in float32
    s = (m / np.float32(qmax)).astype(np.float32)  # one IEEE fp32 division
    safe = np.where(s > 0, s, np.float32(1.0))
    t = (yg / safe[..., None]).astype(np.float32)  # IEEE fp32 division
    t = np.where(s[..., None] > 0, t, np.float32(0.0))
    q = np.clip(np.rint(t), -qmax - 1, qmax)  # rint: round half to even
    return q.astype(np.int8).reshape(n, d), s


def dequantize_groups(q, s, group: int) -> np.ndarray:
    """y_hat_i = s_j q_i in float64 ([P4]: x_hat_i = s q_i)."""
    q = np.asarray(q, dtype=np.float64)
    n, d = q.shape
    s64 = np.asarray(s, dtype=np.float32).astype(np.float64)
    return (q.reshape(n, d // group, group) * s64[..., None]).reshape(n, d)


def pack_nibbles(q) -> np.ndarray:
    """Two int4 codes per byte, element 2b low nibble, 2b+1 high (R6, [P5])."""
    q = np.asarray(q)
    if q.shape[-1] % 2:
        raise ValueError("need an even number of codes")
    if q.min(initial=0) < QMIN or q.max(initial=0) > QMAX:
        raise ValueError("codes outside [-8, 7]")
    nib = (q.astype(np.int16) & 0xF).astype(np.uint8)
    return (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)


def pack_codes(q, bits: int) -> np.ndarray:
    """b-bit two's complement codes as one little-endian bitstream per row:
    code i occupies bits [b i, b i + b) and byte k holds bits [8k, 8k + 8)
    (reading R16; for b = 4 this is exactly pack_nibbles' layout)."""
    q = np.asarray(q)
    n, d = q.shape
    if (d * bits) % 8:
        raise ValueError("row does not fill whole bytes")
    lo, hi = -(2 ** (bits - 1)), 2 ** (bits - 1) - 1
    if q.min(initial=0) < lo or q.max(initial=0) > hi:
        raise ValueError("codes out of range")
    u = (q.astype(np.int32) & ((1 << bits) - 1)).astype(np.uint32)
    bitpos = np.arange(bits, dtype=np.uint32)
    stream = ((u[..., None] >> bitpos) & 1).astype(np.uint8).reshape(n, d * bits)
    return np.packbits(stream, axis=1, bitorder="little")


def unpack_codes(packed, bits: int) -> np.ndarray:
    """Inverse of pack_codes: sign-extended int8 codes [n, 8 * bytes / b]."""
    p = np.asarray(packed, dtype=np.uint8)
    n, nb = p.shape
    d = nb * 8 // bits
    stream = np.unpackbits(p, axis=1, bitorder="little")[:, : d * bits].reshape(n, d, bits)
    u = (stream.astype(np.int32) << np.arange(bits, dtype=np.int32)).sum(axis=2)
    return np.where(u >= 2 ** (bits - 1), u - 2 ** bits, u).astype(np.int8)


def unpack_nibbles(packed) -> np.ndarray:
    """Inverse of pack_nibbles: sign-extend each 4-bit two's complement code."""
    p = np.asarray(packed, dtype=np.uint8)
    lo = (p & 0xF).astype(np.int16)
    hi = (p >> 4).astype(np.int16)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    q = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.int8)
    q[..., 0::2] = lo
    q[..., 1::2] = hi
    return q


def rotated_values(x_fp16, signs, rot: int, lam=None) -> np.ndarray:
    """y = R D (lam * x) in float64 for fp16 rows x (exactly widened); lam is
    an optional per-channel float32 factor (see rot_quant_fwd)."""
    x = np.asarray(x_fp16, dtype=np.float16).astype(np.float64)
    if lam is not None:
        x = x * np.asarray(lam, dtype=np.float32).astype(np.float64)
    return rotate(sign_flip(x, signs), rot)


def rot_quant_fwd(x_fp16, signs, rot: int, group: int, lam=None, bits: int = 4):
    """Forward step: sign flip -> rotation -> per-group absmax int4 -> pack.

    [P1] "First, the 17%" and "Fusing four steps...": the forward kernel does
    rotate plus quantize.  Returns (packed uint8 [n, d/2], scales f32 [n, d/g]).
    With `lam`, every channel i is first multiplied by lam[i]: [P1] "Before
    you celebrate...", first condition (per-channel lambda plus per-group
    abs-max inside the fused kernel).  The pages leave lambda undefined; it is
    an input here, applied before the sign flip and the rotation.
    """
    y = rotated_values(x_fp16, signs, rot, lam)
    q, s = quantize_groups(y, group, bits)
    return (pack_nibbles(q) if bits == 4 else pack_codes(q, bits)), s


def dequant_rot_inv(packed, scales, signs, rot: int, group: int, lam=None,
                    bits: int = 4) -> np.ndarray:
    """Inverse step: unpack -> y_hat = s q -> u = R^T y_hat -> x_hat = D u.

    [P1] "First, the 17%": dequantized and rotated back when attention reads
    it.  The float64 result is rounded to float16 once (reading R8).  With
    `lam`, channel i is divided by lam[i] before that rounding (the inverse of
    rot_quant_fwd's scaling).  `bits`: the code width of rot_quant_fwd.
    """
    q = unpack_nibbles(packed) if bits == 4 else unpack_codes(packed, bits)
    yh = dequantize_groups(q, scales, group)
    u = sign_flip(inverse_rotate(yh, rot), signs)
    if lam is not None:
        u = u / np.asarray(lam, dtype=np.float32).astype(np.float64)
    return u.astype(np.float16)


def near_tie_distance(y, s, group: int) -> np.ndarray:
    """|y/s - (n + 1/2)| for the nearest half-integer, in float64.

    Used to classify codes whose rounding may legitimately differ between two
    float32 evaluations of the same rotation.  Zero-scale groups get +inf.
    """
    y = np.asarray(y, dtype=np.float64)
    n, d = y.shape
    s64 = np.asarray(s, dtype=np.float32).astype(np.float64)
    sb = np.repeat(s64, group, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = y / sb
        dist = np.abs(t - (np.floor(t) + 0.5))
    return np.where(sb > 0, dist, np.inf)


def decode_step(x_new, packed_cache, scales_cache, pos: int, signs, rot: int,
                group: int):
    """Decode step for one head-major cache.

    Quantizes the new token of every head into row ``pos`` of the cache
    (forward step) and returns the dequantized, inverse-rotated rows
    [0, pos] of every head.  The new row's output comes from its fresh codes:
    attention reads the quantized cache ([P1] "First, the 17%").

    x_new: [H, d] fp16; packed_cache: [H, cap, d/2] uint8 (updated in place);
    scales_cache: [H, cap, d/g] float32 (updated in place).
    Returns out [H, pos+1, d] fp16.
    """
    x_new = np.asarray(x_new, dtype=np.float16)
    h, d = x_new.shape
    p_new, s_new = rot_quant_fwd(x_new, signs, rot, group)
    packed_cache[:, pos, :] = p_new
    scales_cache[:, pos, :] = s_new
    rows_p = packed_cache[:, : pos + 1, :].reshape(h * (pos + 1), d // 2)
    rows_s = scales_cache[:, : pos + 1, :].reshape(h * (pos + 1), d // group)
    out = dequant_rot_inv(rows_p, rows_s, signs, rot, group)
    return out.reshape(h, pos + 1, d)


def decode_step_windowed(x_new, packed_cache, scales_cache, kv, pos: int, signs,
                         rot: int, group: int, window: int = 16):
    """Decode step with a dequantized-prefix cache and an fp16 tail.

    [P1] "Before you celebrate...", second condition: the dequantized prefix
    is cached between steps instead of recomputed, the last tokens (16 on
    the pages) stay in fp16, and the cache is refreshed when that window
    fills.  Reading: the window is the run of `window` positions ending at a
    multiple of `window`; row pos of the view receives the new token as is;
    when pos closes a window, the window's rows are quantized into the int4
    cache and the view keeps their dequantized values.  Refreshing only the
    closed window gives the same view as recomputing the whole prefix,
    because rows of earlier windows keep their codes.

    x_new: [H, d] fp16; packed_cache [H, cap, d/2] uint8, scales_cache
    [H, cap, d/g] float32 and kv [H, cap, d] fp16 are updated in place.
    """
    x_new = np.asarray(x_new, dtype=np.float16)
    h, d = x_new.shape
    kv[:, pos, :] = x_new
    if (pos + 1) % window != 0:
        return kv
    first = pos + 1 - window
    rows = kv[:, first: pos + 1, :].reshape(h * window, d)
    p_w, s_w = rot_quant_fwd(rows, signs, rot, group)
    packed_cache[:, first: pos + 1, :] = p_w.reshape(h, window, d // 2)
    scales_cache[:, first: pos + 1, :] = s_w.reshape(h, window, d // group)
    kv[:, first: pos + 1, :] = dequant_rot_inv(p_w, s_w, signs, rot, group).reshape(
        h, window, d)
    return kv


def dequant_rotated_f64(packed, scales, signs, rot: int, group: int) -> np.ndarray:
    """x_hat = D R^T y_hat in float64, without dequant_rot_inv's final fp16
    rounding: the value attention consumes when the dequantization happens
    inside it ([P3] "Decode into HBM, or Decode into Registers")."""
    q = unpack_nibbles(packed)
    yh = dequantize_groups(q, scales, group)
    return sign_flip(inverse_rotate(yh, rot), signs)


def attend_decode(q, k_packed, k_scales, v_packed, v_scales, length: int, signs, rot: int,
                  group: int, sm_scale: float):
    """Decode attention over the int4 cache: one query step.

    [P1] "First, the 17%": K and V are dequantized and rotated back when
    attention reads them; [P3]: that decode belongs inside the attention
    kernel.  For every KV head h and each of its queries i, with
    K_t, V_t = dequant_rotated_f64 of rows t < length of that head:
        s_t = sm_scale <q_i, K_t>,  p = softmax(s),  o_i = sum_t p_t V_t,
    in float64, rounded to fp16 at the end.

    q: [H, nq, d] fp16; k_/v_packed [H, cap, d/2] uint8; k_/v_scales
    [H, cap, d/g] float32.  Returns [H, nq, d] fp16.
    """
    q = np.asarray(q, dtype=np.float16).astype(np.float64)
    h, nq, d = q.shape
    out = np.empty((h, nq, d), dtype=np.float64)
    for hh in range(h):
        k = dequant_rotated_f64(k_packed[hh, :length], k_scales[hh, :length], signs, rot, group)
        v = dequant_rotated_f64(v_packed[hh, :length], v_scales[hh, :length], signs, rot, group)
        s = sm_scale * (q[hh] @ k.T)  # [nq, length]
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[hh] = p @ v
    return out.astype(np.float16)
