"""Pins for the CPU oracle (CPU only).

Every check below ties the oracle to something other than itself: a library
routine that computes the same definition a different way (numpy's FFT,
scipy's Hadamard), closed forms written out by hand, exact rational
arithmetic, invariants the pages state (the s/2 error bound of
"Quantization & Serving"), or brute force on tiny inputs.  The mutation tests
at the end plant plausible mistakes in the oracle and check that a pin
catches each one.
"""

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg

import oracle.kvq_oracle as O
from rotated_int4_kv_kvq_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
SQ2 = math.sqrt(2.0)


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _ev(expr):
    return eval(expr, {"__builtins__": {}}, {"sqrt": math.sqrt})


# ----------------------------------------------------------------- checks ---
# Each check raises AssertionError when the oracle disagrees with its pin, so
# the mutation tests can reuse them.

def check_srft_vs_numpy_rfft(d, seed=0):
    """R u against numpy.fft.rfft packed by reading R1 (independent FFT)."""
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((16, d))
    y = O.rotate(u, O.SRFT)
    X = np.fft.rfft(u, axis=1)  # exp(-2 pi i k n / d), reading R2
    ref = np.empty_like(u)
    ref[:, 0] = X[:, 0].real
    ref[:, 1] = X[:, d // 2].real
    ref[:, 2::2] = SQ2 * X[:, 1:d // 2].real
    ref[:, 3::2] = SQ2 * X[:, 1:d // 2].imag
    ref /= math.sqrt(d)
    err = np.abs(y - ref).max()
    assert err <= 1e-12 * np.abs(u).sum(axis=1).max(), err


def check_srht_vs_scipy(d):
    h = O.srht_matrix(d) * math.sqrt(d)
    assert np.array_equal(h, scipy.linalg.hadamard(d).astype(np.float64))


def check_orthonormal(d, rot, seed=0):
    r = O.rotation_matrix(d, rot)
    assert np.abs(r.T @ r - np.eye(d)).max() <= 1e-12
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((1000, d)) * rng.uniform(0.01, 100, (1000, 1))
    y = O.rotate(x, rot)
    nx = np.linalg.norm(x, axis=1)
    assert np.abs(np.linalg.norm(y, axis=1) - nx).max() <= 1e-12 * nx.max()


def check_srft_d8_closed_form():
    """SRFT d = 8 written out by hand: sqrt(8) R, rows Re/Im of exp(-i 2 pi k n/8)."""
    s = SQ2
    rows = [
        [1, 1, 1, 1, 1, 1, 1, 1],
        [1, -1, 1, -1, 1, -1, 1, -1],
        [s, 1, 0, -1, -s, -1, 0, 1],          # sqrt2 cos(2 pi n/8)
        [0, -1, -s, -1, 0, 1, s, 1],          # -sqrt2 sin(2 pi n/8)
        [s, 0, -s, 0, s, 0, -s, 0],           # sqrt2 cos(pi n/2)
        [0, -s, 0, s, 0, -s, 0, s],           # -sqrt2 sin(pi n/2)
        [s, -1, 0, 1, -s, 1, 0, -1],          # sqrt2 cos(3 pi n/4)
        [0, -1, s, -1, 0, 1, -s, 1],          # -sqrt2 sin(3 pi n/4)
    ]
    ref = np.array(rows, dtype=np.float64) / math.sqrt(8)
    assert np.abs(O.srft_matrix(8) - ref).max() <= 1e-15


def check_d4_matrices():
    s = SQ2
    srft = np.array([[1, 1, 1, 1], [1, -1, 1, -1], [s, 0, -s, 0], [0, -s, 0, s]]) / 2
    srht = np.array([[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]]) / 2
    assert np.abs(O.srft_matrix(4) - srft).max() <= 1e-15
    assert np.array_equal(O.srht_matrix(4), srht)


def check_worked_example(rot_name):
    g = _load("worked_example_d4.json")
    case = g[rot_name]
    rot = O.SRFT if rot_name == "srft" else O.SRHT
    x = np.array(g["x"], dtype=np.float16)[None]
    signs = np.array(g["signs"], dtype=np.int8)
    y = O.rotated_values(x, signs, rot)[0]
    assert np.abs(y - np.array([_ev(e) for e in case["y"]])).max() <= 1e-14
    packed, s = O.rot_quant_fwd(x, signs, rot, g["group"])
    assert np.float32(s[0, 0]) == np.float32(_ev(case["s"]))
    assert O.unpack_nibbles(packed)[0].tolist() == case["q"]
    assert packed[0].tolist() == case["packed"]
    xh = O.dequant_rot_inv(packed, s, signs, rot, g["group"])[0]
    exact = np.array([_ev(e) for e in case["x_hat"]])
    # float16 rounding of the exact value, plus the float32 scale's error
    assert np.abs(xh.astype(np.float64) - exact).max() <= 2.0 ** -10 * 4


def check_exact_ties_d4():
    g = _load("exact_ties_d4.json")
    signs = np.array(g["signs"], dtype=np.int8)
    for c in g["cases"]:
        x = np.array(c["x"], dtype=np.float16)[None]
        y = O.rotated_values(x, signs, O.SRHT)[0]
        assert y.tolist() == c["y"]
        packed, s = O.rot_quant_fwd(x, signs, O.SRHT, g["group"])
        assert float(s[0, 0]) == c["s"]
        assert O.unpack_nibbles(packed)[0].tolist() == c["q"]
        assert packed[0].tolist() == c["packed"]
        xh = O.dequant_rot_inv(packed, s, signs, O.SRHT, g["group"])[0]
        assert xh.astype(np.float64).tolist() == c["x_hat"]


def tie_vector_srht(d, signs):
    """x with y = H D x / sqrt(d) exactly dyadic, max|y| = 7 (s = 1), and
    many exact .5 ties.  Returns (x fp16 [1, d], y float64 [d])."""
    cyc = [7, 2.5, 0.5, -1.5, -2.5, -0.5, 3.5, 1.5, -3.5, 4.5, -4.5, 5.5,
           -5.5, 6.5, -6.5, 0.0]
    y = np.array([cyc[i % len(cyc)] for i in range(d)], dtype=np.float64)
    h = scipy.linalg.hadamard(d).astype(np.float64)
    u = h @ y / math.sqrt(d)  # multiples of 1/16 for d = 64
    x = u * signs
    assert np.array_equal(x.astype(np.float16).astype(np.float64), x)
    return x.astype(np.float16)[None], y


def check_exact_ties_srht(d):
    signs = W.make_signs(d)
    x, y = tie_vector_srht(d, signs)
    yo = O.rotated_values(x, signs, O.SRHT)[0]
    assert np.array_equal(yo, y)
    packed, s = O.rot_quant_fwd(x, signs, O.SRHT, d)
    assert float(s[0, 0]) == 1.0
    expect = [int(round(v)) for v in y]  # Python's round() is half-to-even
    assert O.unpack_nibbles(packed)[0].tolist() == expect


def check_quantizer_bruteforce(seed=0, n=200, group=8):
    """Each code is the integer in [-8, 7] nearest to y/s in exact rational
    arithmetic (ties to even), and s is m/7 rounded to float32."""
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((n, group)) * rng.uniform(0.001, 50, (n, 1))
    y[0] = 0.0
    q, s = O.quantize_groups(y, group)
    y32 = y.astype(np.float32)
    for r in range(n):
        m = Fraction(float(np.abs(y32[r]).max()))
        sf = Fraction(float(s[r, 0]))
        if m == 0:
            assert sf == 0 and not q[r].any()
            continue
        ulp = Fraction(float(np.spacing(np.float32(s[r, 0]))))
        assert abs(sf - m / 7) <= ulp / 2
        for i in range(group):
            t = Fraction(float(y32[r, i])) / sf
            best = min(range(-8, 8), key=lambda c: (abs(t - c), c % 2))
            if abs(abs(t - math.floor(t)) - Fraction(1, 2)) < Fraction(1, 10 ** 6):
                continue  # float32 division may land either side of a tie
            assert q[r, i] == best, (r, i, float(t), q[r, i], best)


def check_error_bound(rot, group, seed=0):
    """|y_hat - y| <= s/2 elementwise ("Quantization & Serving")."""
    shape = W.scaled(W.config(3), layers=1, heads=2, tokens=64)
    x = W.make_kv(shape, seed=seed).numpy()
    d = x.shape[1]
    signs = W.make_signs(d)
    y = O.rotated_values(x, signs, rot)
    q, s = O.quantize_groups(y, group)
    yh = O.dequantize_groups(q, s, group)
    sb = np.repeat(s.astype(np.float64), group, axis=1)
    # y is rounded to float32 before the decision: allow that rounding
    assert np.all(np.abs(yh - y) <= sb / 2 * (1 + 1e-6) + np.abs(y) * 2.0 ** -23)
    assert q.max() <= 7 and q.min() >= -7
    nz = s > 0
    peak = np.abs(q.reshape(q.shape[0], -1, group)).max(axis=2)
    assert np.all(peak[nz] == 7)


def check_pack_layout():
    q = np.array([[a, b] for a in range(-8, 8) for b in range(-8, 8)], dtype=np.int8)
    p = O.pack_nibbles(q)
    for (a, b), byte in zip(q.tolist(), p[:, 0].tolist()):
        bits = format(byte, "08b")
        hi, lo = int(bits[:4], 2), int(bits[4:], 2)
        assert lo == (a + 16) % 16 and hi == (b + 16) % 16
    assert np.array_equal(O.unpack_nibbles(p), q)


def check_decode_step(rot=O.SRFT, d=64, group=32):
    rng = np.random.default_rng(5)
    H, cap, pos = 3, 10, 6
    signs = W.make_signs(d)
    hist = (rng.standard_normal((H, pos, d)) * 3).astype(np.float16)
    pc = np.zeros((H, cap, d // 2), np.uint8)
    sc = np.zeros((H, cap, d // group), np.float32)
    p, s = O.rot_quant_fwd(hist.reshape(-1, d), signs, rot, group)
    pc[:, :pos] = p.reshape(H, pos, -1)
    sc[:, :pos] = s.reshape(H, pos, -1)
    xn = (rng.standard_normal((H, d)) * 3).astype(np.float16)
    out = O.decode_step(xn, pc, sc, pos, signs, rot, group)
    allx = np.concatenate([hist, xn[:, None]], axis=1)
    p2, s2 = O.rot_quant_fwd(allx.reshape(-1, d), signs, rot, group)
    assert np.array_equal(pc[:, : pos + 1].reshape(-1, d // 2), p2)
    assert np.array_equal(sc[:, : pos + 1].reshape(-1, d // group), s2)
    ref = O.dequant_rot_inv(p2, s2, signs, rot, group).reshape(H, pos + 1, d)
    assert np.array_equal(out, ref)


def check_decode_windowed(rot=O.SRFT, d=64, group=32, window=4, steps=11):
    """The windowed step against the plain decode step on the same tokens:
    after every step the view's closed windows equal the plain step's
    output rows and the open window holds the tokens themselves; a step
    leaves rows before its window bit-identical; packed/scales rows of the
    open window stay untouched."""
    rng = np.random.default_rng(7)
    H, cap = 2, steps + 3
    signs = W.make_signs(d)
    pc = np.zeros((H, cap, d // 2), np.uint8)
    sc = np.zeros((H, cap, d // group), np.float32)
    kv = np.zeros((H, cap, d), np.float16)
    pc2 = np.zeros_like(pc)
    sc2 = np.zeros_like(sc)
    toks = (rng.standard_normal((steps, H, d)) * 3).astype(np.float16)
    for pos in range(steps):
        before = kv.copy()
        O.decode_step_windowed(toks[pos], pc, sc, kv, pos, signs, rot, group, window)
        out = O.decode_step(toks[pos], pc2, sc2, pos, signs, rot, group)
        closed = ((pos + 1) // window) * window
        assert np.array_equal(kv[:, :closed], out[:, :closed])
        assert np.array_equal(kv[:, closed: pos + 1], toks[closed: pos + 1].transpose(1, 0, 2))
        first = pos + 1 - window if (pos + 1) % window == 0 else pos
        assert np.array_equal(kv[:, :first], before[:, :first])
        assert not pc[:, closed:].any() and not sc[:, closed:].any()


def check_lambda(rot=O.SRFT, d=64, group=32):
    """The per-channel lambda hook against the plain steps: lambda = 1 is the
    plain step; a constant power of two scales only the scales; per-channel
    powers of two equal the plain step on the pre-scaled fp16 input (exact),
    and the inverse divides channel-wise."""
    rng = np.random.default_rng(11)
    signs = W.make_signs(d)
    x = (rng.standard_normal((9, d)) * 3).astype(np.float16)
    p0, s0 = O.rot_quant_fwd(x, signs, rot, group)
    p1, s1 = O.rot_quant_fwd(x, signs, rot, group, np.ones(d, np.float32))
    assert np.array_equal(p0, p1) and np.array_equal(s0, s1)
    p4, s4 = O.rot_quant_fwd(x, signs, rot, group, np.full(d, 4.0, np.float32))
    assert np.array_equal(p4, p0) and np.array_equal(s4, (4 * s0).astype(np.float32))
    assert np.array_equal(O.dequant_rot_inv(p4, s4, signs, rot, group, np.full(d, 4.0, np.float32)),
                          O.dequant_rot_inv(p0, s0, signs, rot, group))
    lam = (2.0 ** rng.integers(-1, 3, d)).astype(np.float32)
    xs = (x.astype(np.float64) * lam).astype(np.float16)
    assert np.array_equal(xs.astype(np.float64), x.astype(np.float64) * lam)  # exact
    pl, sl = O.rot_quant_fwd(x, signs, rot, group, lam)
    pr, sr = O.rot_quant_fwd(xs, signs, rot, group)
    assert np.array_equal(pl, pr) and np.array_equal(sl, sr)
    xi = O.dequant_rot_inv(pl, sl, signs, rot, group, lam).astype(np.float64)
    xr = O.dequant_rot_inv(pr, sr, signs, rot, group).astype(np.float64)
    assert np.array_equal(xi, xr / lam)


def _attn_case(rot, d=64, group=32, h=2, nq=3, n=9, seed=13):
    rng = np.random.default_rng(seed)
    signs = W.make_signs(d)
    kx = (rng.standard_normal((h * n, d)) * 2).astype(np.float16)
    vx = (rng.standard_normal((h * n, d)) * 2).astype(np.float16)
    kp, ks = O.rot_quant_fwd(kx, signs, rot, group)
    vp, vs = O.rot_quant_fwd(vx, signs, rot, group)
    q = (rng.standard_normal((h, nq, d))).astype(np.float16)
    return (signs, q, kp.reshape(h, n, -1), ks.reshape(h, n, -1), vp.reshape(h, n, -1),
            vs.reshape(h, n, -1))


def check_attention(rot=O.SRFT, d=64, group=32):
    """Decode attention over the int4 cache: one key gives its value; a zero
    softmax scale gives the mean value; a large scale with a unique best key
    gives that key's value; and the whole result equals the same attention
    computed in the rotated domain (scores <R D q, y_hat_K>, values
    D R^T sum_t p_t y_hat_V,t), a different route through R."""
    signs, q, kp, ks, vp, vs = _attn_case(rot, d, group)
    h, nq, _ = q.shape
    n = kp.shape[1]
    v64 = [O.dequant_rotated_f64(vp[i], vs[i], signs, rot, group) for i in range(h)]
    one = O.attend_decode(q, kp, ks, vp, vs, 1, signs, rot, group, 0.125)
    assert np.array_equal(one, np.repeat(np.stack([v[0] for v in v64])[:, None], nq, 1)
                          .astype(np.float16))
    flat = O.attend_decode(q, kp, ks, vp, vs, n, signs, rot, group, 0.0)
    assert np.array_equal(flat, np.repeat(np.stack([v.mean(0) for v in v64])[:, None], nq, 1)
                          .astype(np.float16))
    k64 = [O.dequant_rotated_f64(kp[i], ks[i], signs, rot, group) for i in range(h)]
    sc = np.stack([q[i].astype(np.float64) @ k64[i].T for i in range(h)])  # [h, nq, n]
    order = np.sort(sc, axis=2)
    if np.all(order[..., -1] - order[..., -2] > 1e-3):
        sharp = O.attend_decode(q, kp, ks, vp, vs, n, signs, rot, group, 1e7)
        best = sc.argmax(axis=2)
        ref = np.stack([[v64[i][best[i, j]] for j in range(nq)] for i in range(h)])
        assert np.array_equal(sharp, ref.astype(np.float16))
    got = O.attend_decode(q, kp, ks, vp, vs, n, signs, rot, group, 0.3)
    for i in range(h):
        qr = O.rotate(O.sign_flip(q[i].astype(np.float64), signs), rot)  # [nq, d]
        yk = O.dequantize_groups(O.unpack_nibbles(kp[i]), ks[i], group)
        yv = O.dequantize_groups(O.unpack_nibbles(vp[i]), vs[i], group)
        s_ = 0.3 * (qr @ yk.T)
        p_ = np.exp(s_ - s_.max(axis=1, keepdims=True))
        p_ /= p_.sum(axis=1, keepdims=True)
        o_ = O.sign_flip(O.inverse_rotate(p_ @ yv, rot), signs)
        assert np.array_equal(got[i], o_.astype(np.float16)) or \
            np.abs(got[i].astype(np.float64) - o_).max() <= 2.0 ** -10 * np.abs(o_).max()


def check_bitstream_golden():
    """Little-endian bitstream, written out by hand from the two's complement
    codes (R16): b = 3 codes 1,-1,3,-4,0,2,-2,1 are 001 111 011 100 000 010
    110 001 LSB-first -> bytes F9 08 39; b = 6 codes 5,-20,31,-32 are 000101
    101100 011111 100000 -> bytes 05 FB 81."""
    q3 = np.array([[1, -1, 3, -4, 0, 2, -2, 1]], np.int8)
    assert O.pack_codes(q3, 3).tolist() == [[0xF9, 0x08, 0x39]]
    q6 = np.array([[5, -20, 31, -32]], np.int8)
    assert O.pack_codes(q6, 6).tolist() == [[0x05, 0xFB, 0x81]]
    for q, b in ((q3, 3), (q6, 6)):
        assert np.array_equal(O.unpack_codes(O.pack_codes(q, b), b), q)
    rng = np.random.default_rng(3)
    q4 = rng.integers(-8, 8, (4, 64)).astype(np.int8)
    assert np.array_equal(O.pack_codes(q4, 4), O.pack_nibbles(q4))  # b = 4 is R6


def check_bits_quantizer(bits, d=64, group=32):
    """b-bit groups: s = fl32(max/qmax), |q| <= qmax with qmax reached in
    every non-zero group, error <= s/2 ([P4]), exact pack round trip."""
    qmax = 2 ** (bits - 1) - 1
    rng = np.random.default_rng(bits)
    y = rng.standard_normal((50, d)) * rng.uniform(0.1, 10, (50, 1))
    q, s = O.quantize_groups(y, group, bits)
    yg = np.asarray(y, np.float64).astype(np.float32).reshape(50, d // group, group)
    m = np.abs(yg).max(axis=2)
    assert np.array_equal(s, (m / np.float32(qmax)).astype(np.float32))
    qg = q.reshape(50, d // group, group).astype(np.int32)
    assert np.abs(qg).max() <= qmax and np.all(np.abs(qg).max(axis=2) == qmax)
    err = np.abs(qg * s[..., None].astype(np.float64) - yg.astype(np.float64))
    assert np.all(err <= s[..., None].astype(np.float64) * (0.5 + 1e-6))
    assert np.array_equal(O.unpack_codes(O.pack_codes(q, bits), bits), q)


# ------------------------------------------------------------------ tests ---

@pytest.mark.parametrize("d", [2, 4, 8, 64, 128, 256])
def test_srft_matches_numpy_rfft(d):
    check_srft_vs_numpy_rfft(d)


@pytest.mark.parametrize("d", [1, 2, 4, 8, 64, 128, 256])
def test_srht_matches_scipy_hadamard(d):
    check_srht_vs_scipy(d)


@pytest.mark.parametrize("d", [4, 8, 64, 128, 256])
@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
def test_orthonormal_and_norm_preserving(d, rot):
    check_orthonormal(d, rot)


def test_d4_and_d8_closed_forms():
    check_d4_matrices()
    check_srft_d8_closed_form()


@pytest.mark.parametrize("rot", ["srft", "srht"])
def test_worked_example_d4(rot):
    check_worked_example(rot)


def test_exact_ties_half_even():
    check_exact_ties_d4()
    for d in (64, 256):  # sqrt(d) must be a power of two for dyadic x
        check_exact_ties_srht(d)


def test_quantizer_matches_bruteforce():
    check_quantizer_bruteforce()


@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
@pytest.mark.parametrize("group", [32, 128])
def test_error_bound_and_qmax(rot, group):
    check_error_bound(rot, group)


def test_pack_layout_and_roundtrip():
    check_pack_layout()


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
def test_exact_inverse_without_quantization(d, rot):
    rng = np.random.default_rng(1)
    x = rng.standard_normal((50, d)) * 10
    signs = W.make_signs(d)
    u = O.sign_flip(O.inverse_rotate(O.rotate(O.sign_flip(x, signs), rot), rot), signs)
    assert np.abs(u - x).max() <= 1e-12 * np.abs(x).max()


@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
def test_zero_vectors_and_zero_groups(rot):
    d, g = 64, 16
    signs = W.make_signs(d)
    x = np.zeros((3, d), np.float16)
    p, s = O.rot_quant_fwd(x, signs, rot, g)
    assert not p.any() and not s.any()
    assert not O.dequant_rot_inv(p, s, signs, rot, g).any()
    if rot == O.SRHT:
        # y = c e_0 exactly: every group but the first has s = 0 and q = 0
        x1 = (signs.astype(np.float64) * 0.375).astype(np.float16)[None]
        p1, s1 = O.rot_quant_fwd(x1, signs, rot, g)
        assert s1[0, 0] == np.float32(3.0 / 7.0) and not s1[0, 1:].any()
        assert O.unpack_nibbles(p1)[0].tolist() == [7] + [0] * (d - 1)


def test_decode_step_is_fwd_then_inv():
    check_decode_step()


@pytest.mark.parametrize("window", [1, 4, 16])
@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
def test_decode_windowed_matches_plain_decode(rot, window):
    check_decode_windowed(rot, window=window, steps=2 * window + 3)


@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
@pytest.mark.parametrize("d,group", [(64, 32), (256, 256)])
def test_lambda_hook(rot, d, group):
    check_lambda(rot, d, group)


@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
@pytest.mark.parametrize("d,group", [(64, 32), (256, 256)])
def test_attention(rot, d, group):
    check_attention(rot, d, group)


def test_bitstream_golden():
    check_bitstream_golden()


@pytest.mark.parametrize("bits", [3, 4, 6, 8])
def test_bits_quantizer(bits):
    check_bits_quantizer(bits)


def test_bits_mse_falls_with_width():
    """More bits, smaller error ([P1]: 6 and 8 bits are lossless in the
    pages' test; 3 bits is worse than 4)."""
    x = W.make_kv(W.scaled(W.config(5, d=64, group=64), heads=1, tokens=256)).numpy()
    signs = W.make_signs(64)
    mse = []
    for b in (3, 4, 6, 8):
        p, s = O.rot_quant_fwd(x, signs, O.SRFT, 64, bits=b)
        xh = O.dequant_rot_inv(p, s, signs, O.SRFT, 64, bits=b).astype(np.float64)
        mse.append(((xh - x.astype(np.float64)) ** 2).mean())
    assert mse[0] > mse[1] > mse[2] > mse[3]


def test_granularity_monotone():
    """Per-group error falls as groups shrink ("Quantization & Serving")."""
    for d in (64, 128):
        shape = W.scaled(W.config(5, d=d), heads=4, tokens=256)
        x = W.make_kv(shape).numpy()
        signs = W.make_signs(d)
        for rot in (O.SRFT, O.SRHT):
            y = O.rotated_values(x, signs, rot)
            mse = {}
            for g in (32, d):
                q, s = O.quantize_groups(y, g)
                mse[g] = np.mean((O.dequantize_groups(q, s, g) - y) ** 2)
            assert mse[32] <= mse[d]


def test_rotation_spreads_outliers():
    """Rotating first cuts the int4 error on outlier-heavy K/V
    ("Before you celebrate, check the quality bill": rotation is not optional)."""
    shape = W.scaled(W.config(2), layers=1, heads=4, tokens=256)
    x = W.make_kv(shape).numpy().astype(np.float64)
    d = x.shape[1]
    signs = W.make_signs(d)
    q0, s0 = O.quantize_groups(x, d)
    e_plain = np.mean((O.dequantize_groups(q0, s0, d) - x) ** 2)
    for rot in (O.SRFT, O.SRHT):
        p, s = O.rot_quant_fwd(x.astype(np.float16), signs, rot, d)
        xh = O.dequant_rot_inv(p, s, signs, rot, d).astype(np.float64)
        assert np.mean((xh - x) ** 2) < 0.5 * e_plain


def test_near_tie_distance():
    y = np.array([[0.5, 1.25, -0.5, 0.0]])
    s = np.array([[1.0, 0.0]], np.float32)
    dist = O.near_tie_distance(y, s, 2)
    assert dist[0, 0] == 0.0 and dist[0, 1] == 0.25
    assert np.isinf(dist[0, 2:]).all()


# ------------------------------------------------------- planted mistakes ---

def _mut_srft_drop_sqrt2(d):
    n = np.arange(d)
    r = np.empty((d, d))
    r[0] = 1.0
    r[1] = np.where(n % 2 == 0, 1.0, -1.0)
    for k in range(1, d // 2):
        ang = 2 * np.pi * ((k * n) % d) / d
        r[2 * k] = np.cos(ang)  # missing sqrt(2)
        r[2 * k + 1] = -np.sin(ang)
    return r / np.sqrt(d)


def _mut_srft_wrong_sign(d):
    n = np.arange(d)
    r = np.empty((d, d))
    r[0] = 1.0
    r[1] = np.where(n % 2 == 0, 1.0, -1.0)
    for k in range(1, d // 2):
        ang = 2 * np.pi * ((k * n) % d) / d
        r[2 * k] = np.sqrt(2) * np.cos(ang)
        r[2 * k + 1] = np.sqrt(2) * np.sin(ang)  # exp(+i ...) convention
    return r / np.sqrt(d)


def _mut_srft_transposed(d):
    return _ORIG["srft_matrix"](d).T


def _mut_srht_bitreversed(d):
    h = _ORIG["srht_matrix"](d)
    bits = int(math.log2(d)) if d > 1 else 0
    perm = [int(format(i, f"0{bits}b")[::-1], 2) if bits else 0 for i in range(d)]
    return h[perm]


def _mut_quant_half_away(y, group, bits=4):
    y32 = np.asarray(y, np.float64).astype(np.float32)
    n, d = y32.shape
    yg = y32.reshape(n, d // group, group)
    s = (np.abs(yg).max(axis=2) / np.float32(7)).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1))
    t = yg / safe[..., None]
    q = np.clip(np.sign(t) * np.floor(np.abs(t) + 0.5), -8, 7)
    return q.astype(np.int8).reshape(n, d), s


def _mut_quant_div8(y, group, bits=4):
    y32 = np.asarray(y, np.float64).astype(np.float32)
    n, d = y32.shape
    yg = y32.reshape(n, d // group, group)
    s = (np.abs(yg).max(axis=2) / np.float32(8)).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1))
    q = np.clip(np.rint(yg / safe[..., None]), -8, 7)
    return q.astype(np.int8).reshape(n, d), s


def _mut_pack_swapped(q):
    nib = (np.asarray(q).astype(np.int16) & 0xF).astype(np.uint8)
    return (nib[..., 1::2] | (nib[..., 0::2] << 4)).astype(np.uint8)


def _mut_window_flush_early(x_new, packed_cache, scales_cache, kv, pos, signs, rot, group,
                            window=16):
    """Off by one: closes a window at pos % window == 0 instead of at its
    last position."""
    return _flush_if(pos > 0 and pos % window == 0, x_new, packed_cache, scales_cache, kv, pos,
                     signs, rot, group, window)


def _flush_if(cond, x_new, packed_cache, scales_cache, kv, pos, signs, rot, group, window):
    x_new = np.asarray(x_new, dtype=np.float16)
    h, d = x_new.shape
    kv[:, pos, :] = x_new
    if not cond:
        return kv
    first = max(0, pos + 1 - window)
    n = pos + 1 - first
    rows = kv[:, first: pos + 1, :].reshape(h * n, d)
    p_w, s_w = O.rot_quant_fwd(rows, signs, rot, group)
    packed_cache[:, first: pos + 1, :] = p_w.reshape(h, n, d // 2)
    scales_cache[:, first: pos + 1, :] = s_w.reshape(h, n, d // group)
    kv[:, first: pos + 1, :] = O.dequant_rot_inv(p_w, s_w, signs, rot, group).reshape(h, n, d)
    return kv


def _mut_lambda_after_rotation(x_fp16, signs, rot, lam=None):
    # lambda applied to y instead of x
    x = np.asarray(x_fp16, dtype=np.float16).astype(np.float64)
    y = O.rotate(O.sign_flip(x, signs), rot)
    if lam is not None:
        y = y * np.asarray(lam, np.float32).astype(np.float64)
    return y


def _mut_attn_fp16_keys(packed, scales, signs, rot, group):
    # keys and values rounded to fp16 first (a different definition)
    q = O.unpack_nibbles(packed)
    yh = O.dequantize_groups(q, scales, group)
    x = O.sign_flip(O.inverse_rotate(yh, rot), signs)
    return x.astype(np.float16).astype(np.float64) * (1 + 2.0 ** -9)


def _mut_pack_msb_first(q, bits):
    q = np.asarray(q)
    n, d = q.shape
    u = (q.astype(np.int32) & ((1 << bits) - 1)).astype(np.uint32)
    bitpos = np.arange(bits, dtype=np.uint32)
    stream = ((u[..., None] >> bitpos) & 1).astype(np.uint8).reshape(n, d * bits)
    return np.packbits(stream, axis=1, bitorder="big")


def _mut_inverse_no_transpose(y, rot):
    return np.asarray(y, np.float64) @ O.rotation_matrix(y.shape[-1], rot).T


_ORIG = {"srft_matrix": O.srft_matrix, "srht_matrix": O.srht_matrix}

MUTATIONS = [
    ("srft_matrix", _mut_srft_drop_sqrt2,
     [lambda: check_srft_vs_numpy_rfft(8), lambda: check_orthonormal(8, O.SRFT)]),
    ("srft_matrix", _mut_srft_wrong_sign,
     [lambda: check_srft_vs_numpy_rfft(8), check_srft_d8_closed_form,
      lambda: check_worked_example("srft")]),
    ("srft_matrix", _mut_srft_transposed,
     [lambda: check_srft_vs_numpy_rfft(8), check_srft_d8_closed_form]),
    ("srht_matrix", _mut_srht_bitreversed,
     [lambda: check_srht_vs_scipy(8), lambda: check_worked_example("srht")]),
    ("quantize_groups", _mut_quant_half_away,
     [check_exact_ties_d4, lambda: check_exact_ties_srht(64)]),
    ("quantize_groups", _mut_quant_div8,
     [lambda: check_worked_example("srft"), check_quantizer_bruteforce,
      lambda: check_error_bound(O.SRFT, 32)]),
    ("pack_nibbles", _mut_pack_swapped,
     [check_pack_layout, lambda: check_worked_example("srht")]),
    ("inverse_rotate", _mut_inverse_no_transpose,
     [lambda: check_worked_example("srft")]),
    ("decode_step_windowed", _mut_window_flush_early,
     [lambda: check_decode_windowed(window=4)]),
    ("rotated_values", _mut_lambda_after_rotation, [check_lambda]),
    ("dequant_rotated_f64", _mut_attn_fp16_keys, [check_attention]),
    ("pack_codes", _mut_pack_msb_first, [check_bitstream_golden]),
]


@pytest.mark.parametrize("name,mut,checks", MUTATIONS,
                         ids=[f"{m[0]}:{m[1].__name__}" for m in MUTATIONS])
def test_planted_mistake_is_caught(monkeypatch, name, mut, checks):
    monkeypatch.setattr(O, name, mut)
    for check in checks:
        with pytest.raises(AssertionError):
            check()
