"""The generated FFT codelets (kvq_rfft.cuh) without a GPU: the committed
header is what the generator writes today, the generator's own checks pass
(graph against numpy's FFT, emitted instruction list against the graph),
and the emitted programs compute the packed real DFT and its transpose."""

import importlib.util
import math
import os

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "rotated_int4_kv_kvq_b200", "csrc")


def load_gen():
    spec = importlib.util.spec_from_file_location("gen_rfft", os.path.join(CSRC, "gen_rfft.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_committed_header_is_current(tmp_path):
    gen = load_gen()
    out = gen.main(str(tmp_path / "kvq_rfft.cuh"))
    with open(out) as f, open(os.path.join(CSRC, "kvq_rfft.cuh")) as g:
        assert f.read() == g.read(), "kvq_rfft.cuh is stale: rerun gen_rfft.py"


def packed_rfft(x):
    """y[0] = X_0/sqrt2, y[1] = X_{n/2}/sqrt2, y[2k], y[2k+1] = Re, Im X_k."""
    n = len(x)
    X = np.fft.rfft(x)
    y = np.empty(n)
    y[0], y[1] = X[0].real / math.sqrt(2), X[n // 2].real / math.sqrt(2)
    y[2::2], y[3::2] = X[1:n // 2].real, X[1:n // 2].imag
    return y


def test_programs_are_the_packed_dft_and_its_transpose():
    gen = load_gen()
    rng = np.random.default_rng(11)
    for n in (32, 64):
        gf, of = gen.build_forward(n)
        gi, oi = gen.build_inverse(n)
        _, _, pf, progf = gen.emit_x2("f", gf, of, "x", "y", n)
        _, _, pi, progi = gen.emit_x2("i", gi, oi, "y", "x", n)
        # the packed DFT as a matrix, column by column
        A = np.stack([packed_rfft(e) for e in np.eye(n)], axis=1)
        for _ in range(3):
            x = rng.standard_normal(n)
            y = gen.run_x2(gf, *progf, {f"x[{i}]": x[i] for i in range(n)}) * np.array(pf)
            assert np.allclose(y, A @ x, rtol=0, atol=1e-5 * np.abs(A @ x).max())
            v = rng.standard_normal(n)
            z = gen.run_x2(gi, *progi, {f"y[{i}]": v[i] for i in range(n)}) * np.array(pi)
            assert np.allclose(z, A.T @ v, rtol=0, atol=1e-5 * np.abs(A.T @ v).max())
        # A^T A = (n/2) I: the transpose is the inverse up to that factor
        assert np.allclose(A.T @ A, (n / 2) * np.eye(n), atol=1e-9)


def test_operation_counts_do_not_grow():
    gen = load_gen()
    counts = {}
    for n in (32, 64):
        for fwd in (True, False):
            g, o = gen.build_forward(n) if fwd else gen.build_inverse(n)
            _, total, _, _ = gen.emit_x2("c", g, o, "x" if fwd else "y", "y" if fwd else "x", n)
            counts[(n, fwd)] = total
    # forward / inverse f32x2 instructions of the committed codelets
    assert counts[(32, True)] <= 167 and counts[(32, False)] <= 165
    assert counts[(64, True)] <= 416 and counts[(64, False)] <= 414
