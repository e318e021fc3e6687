"""The seeded input generators (CPU only)."""

import numpy as np
import torch

from rotated_int4_kv_kvq_b200 import workloads as W


def test_signs_are_pm1_and_seeded():
    for d in (4, 64, 128, 256):
        s = W.make_signs(d)
        assert s.dtype == np.int8 and s.shape == (d,)
        assert set(np.unique(s).tolist()) <= {-1, 1}
        assert np.array_equal(s, W.make_signs(d))
    assert not np.array_equal(W.make_signs(64, 1), W.make_signs(64, 2))
    # both signs occur in a 256-long draw
    assert (W.make_signs(256) == -1).sum() > 64


def test_config_shapes():
    assert W.config(1).n_vec == 2560
    assert W.config(2).n_vec == 6291456
    assert W.config(3).n_vec == 229376
    assert W.config(5, d=64).n_vec == 8388608
    assert W.config(4).d == 256 and W.config(4).group == 256


def test_make_kv_deterministic_with_outliers():
    shape = W.scaled(W.config(1), tokens=32)
    a = W.make_kv(shape)
    b = W.make_kv(shape)
    assert a.dtype == torch.float16 and a.shape == (shape.n_vec, 64)
    assert torch.equal(a, b)
    x = a.float().reshape(1, 2, shape.heads, shape.tokens, 64)
    # every head has channels whose rms is ~20x the rest
    rms = x.pow(2).mean(dim=3).sqrt()
    top = rms.topk(2, dim=-1).values.min(dim=-1).values
    med = rms.median(dim=-1).values
    assert torch.all(top > 8 * med)


def test_student_t_noise_is_heavy_tailed():
    shape = W.scaled(W.config(3), layers=1, heads=1, tokens=512)
    x = W.make_kv(shape).float().reshape(2, 512, 128)
    k, v = x[0], x[1]
    assert k.abs().max() > v.abs().max() * 0.5
    assert torch.isfinite(x).all()


def test_sample_rows():
    idx = W.sample_rows(1000, 50)
    assert idx[0] == 0 and idx[-1] == 999 and len(np.unique(idx)) == len(idx)
