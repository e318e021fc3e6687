"""Element-by-element comparison of the CUDA path with the CPU oracle.

Tolerances (the codec's stated parity bar):
* int4 codes: bit-exact, except codes whose oracle y/s lies within 1e-4 of a
  rounding tie; such mismatches are counted, must be off by exactly one step,
  and must stay below 1e-4 of all codes;
* scales: 1e-6 relative (exactly 0 where the oracle's scale is 0);
* x_hat: max-abs 2e-3 * max|x| (per vector), in fp32.  The inverse is checked
  against the oracle's inverse of the GPU's own codes and scales, and end to
  end against the oracle's x_hat for vectors with no near-tie code flip.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

import oracle.kvq_oracle as O

TIE_WINDOW = 1e-4
MAX_FLIP_FRACTION = 1e-4
SCALE_RTOL = 1e-6
XHAT_ATOL_REL = 2e-3


@dataclass
class Report:
    n_codes: int
    flips: int
    max_scale_rel: float
    max_inv_err: float
    max_e2e_err: float

    @property
    def flip_fraction(self) -> float:
        return self.flips / max(1, self.n_codes)


FP16_OVERFLOW = 65520.0  # the smallest magnitude that rounds to inf in fp16


def _exact_xhat(packed, scales, signs, rot, group, lam=None, bits=4):
    """x_hat = D R^T (s q) (/ lam) in float64, before the fp16 rounding."""
    q = O.unpack_nibbles(packed) if bits == 4 else O.unpack_codes(packed, bits)
    u = O.sign_flip(O.inverse_rotate(O.dequantize_groups(q, scales, group), rot), signs)
    if lam is not None:
        u = u / np.asarray(lam, dtype=np.float32).astype(np.float64)
    return u


def _sat(v, exact, tol):
    """fp16 overflow as the next power of two (65536), so that inf on one
    side and 65504 on the other compare as one ulp apart.  An inf is accepted
    only where the exact float64 x_hat lies within the tolerance of the fp16
    overflow threshold; anywhere else it is a failure."""
    v = np.asarray(v, dtype=np.float64)
    inf = np.isinf(v)
    near = np.abs(exact) + tol >= FP16_OVERFLOW
    assert not np.any(inf & ~near), "fp16 overflow where the exact x_hat is well inside range"
    return np.where(inf, np.sign(v) * 65536.0, v)


def check_fwd(x16, signs, rot, group, packed, scales, max_flip_fraction=MAX_FLIP_FRACTION,
              lam=None, bits=4):
    """Return (codes, scales, flips, max scale rel err, flipped-row mask).

    `max_flip_fraction` bounds near-tie flips on realistic data; structured
    inputs (e.g. +-c vectors, whose rotations hit exact ties) pass None.
    `lam`: per-channel factor of the lambda entry points; `bits`: code width."""
    x16 = np.asarray(x16, dtype=np.float16)
    y = O.rotated_values(x16, signs, rot, lam)
    q_ref, s_ref = O.quantize_groups(y, group, bits)
    s = np.asarray(scales, dtype=np.float32)
    pk = np.asarray(packed, dtype=np.uint8)
    q = O.unpack_nibbles(pk) if bits == 4 else O.unpack_codes(pk, bits)
    assert q.shape == q_ref.shape and s.shape == s_ref.shape

    # scales
    zero = s_ref == 0
    assert np.all(s[zero] == 0), "scale of an all-zero group must be 0"
    rel = np.abs(s.astype(np.float64) - s_ref) / np.where(zero, 1.0, s_ref)
    max_rel = float(rel[~zero].max(initial=0.0))
    assert max_rel <= SCALE_RTOL, f"scale rel err {max_rel:.3g}"

    # codes
    qmax = 2 ** (bits - 1) - 1
    assert q.min(initial=0) >= -qmax - 1 and q.max(initial=0) <= qmax
    diff = q.astype(np.int16) - q_ref.astype(np.int16)
    bad = diff != 0
    flips = int(bad.sum())
    if flips:
        dist = O.near_tie_distance(y, s_ref, group)
        assert np.all(np.abs(diff[bad]) == 1), "a code differs by more than one step"
        worst = float(dist[bad].max())
        assert worst < TIE_WINDOW, f"code mismatch away from a tie (distance {worst:.3g})"
        if max_flip_fraction is not None:
            assert flips < max_flip_fraction * q.size, f"{flips} near-tie flips of {q.size}"
    return q, s, flips, max_rel, bad.any(axis=1)


def check_inv(x16, signs, rot, group, packed, scales, out, flipped_rows=None, lam=None, bits=4):
    """x_hat of the GPU against the oracle inverse of the same codes/scales,
    and against the oracle's own x_hat on rows without a code flip.  With
    `lam` the tolerance follows the channel scaling: the error of lam * x_hat
    is bounded like that of an unscaled x_hat."""
    x = np.asarray(x16, dtype=np.float16).astype(np.float64)
    tol = XHAT_ATOL_REL * np.maximum(np.abs(x).max(axis=1, keepdims=True), 1e-30)
    if lam is not None:
        lam64 = np.asarray(lam, np.float32).astype(np.float64)
        tol = XHAT_ATOL_REL * np.maximum(np.abs(x * lam64).max(axis=1, keepdims=True),
                                         1e-30) / lam64 + np.float64(2.0 ** -24)
    exact = _exact_xhat(packed, scales, signs, rot, group, lam, bits)
    with np.errstate(over="ignore"):
        ref = _sat(O.dequant_rot_inv(packed, scales, signs, rot, group, lam, bits), exact, tol)
    got = _sat(np.asarray(out, dtype=np.float16), exact, tol)
    err = np.abs(got - ref)
    inv_err = float((err / tol).max(initial=0.0))
    assert np.all(err <= tol), f"inverse error {inv_err:.3g} x tolerance"
    e2e = 0.0
    p_ref, s_ref = O.rot_quant_fwd(np.asarray(x16, np.float16), signs, rot, group, lam, bits)
    exact_full = _exact_xhat(p_ref, s_ref, signs, rot, group, lam, bits)
    with np.errstate(over="ignore"):
        full = _sat(O.dequant_rot_inv(p_ref, s_ref, signs, rot, group, lam, bits), exact_full,
                    tol)
    rows = np.ones(x.shape[0], bool) if flipped_rows is None else ~flipped_rows
    if rows.any():
        e = np.abs(got[rows] - full[rows]) / tol[rows]
        e2e = float(e.max())
        assert e2e <= 1.0, f"end-to-end x_hat error {e2e:.3g} x tolerance"
    return inv_err, e2e


def full_check(x16, signs, rot, group, packed, scales, out,
               max_flip_fraction=MAX_FLIP_FRACTION) -> Report:
    q, s, flips, max_rel, flipped = check_fwd(x16, signs, rot, group, packed, scales,
                                              max_flip_fraction)
    inv_err, e2e = check_inv(x16, signs, rot, group, packed, scales, out, flipped)
    return Report(q.size, flips, max_rel, inv_err, e2e)
