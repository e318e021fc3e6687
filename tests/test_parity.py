"""CUDA path vs the CPU oracle, through the C ABI (needs a B200).

Small workloads are compared in full; the full-size caches (SmolLM2-1.7B,
the large-batch sweep) are run whole on the GPU in the launch configuration
the benchmark times, then compared on sampled rows, plus properties checked
on every output (code range, one |q| = 7 per non-zero group, finite x_hat).
"""

import numpy as np
import pytest
import torch

import oracle.kvq_oracle as O
from parity import full_check
from rotated_int4_kv_kvq_b200 import workloads as W

pytestmark = pytest.mark.gpu

ROTS = [O.SRFT, O.SRHT]


@pytest.fixture(scope="module")
def kvq():
    from rotated_int4_kv_kvq_b200 import kvq as mod
    return mod


def run(kvq, x_dev, d, rot, group, signs_np):
    signs = torch.from_numpy(signs_np).cuda()
    packed, scales = kvq.kvq_rot_quant_fwd(x_dev, signs, rot, group)
    out = kvq.kvq_dequant_rot_inv(packed, scales, signs, rot, group)
    torch.cuda.synchronize()
    assert kvq.kvq_device_status() == 0
    return packed, scales, out


def check_all(kvq, x16, rot, group, **kw):
    d = x16.shape[1]
    signs = W.make_signs(d)
    x_dev = torch.from_numpy(np.ascontiguousarray(x16)).cuda()
    p, s, o = run(kvq, x_dev, d, rot, group, signs)
    return full_check(x16, signs, rot, group, p.cpu().numpy(), s.cpu().numpy(),
                      o.cpu().numpy(), **kw)


@pytest.mark.parametrize("rot", ROTS)
@pytest.mark.parametrize("group", [64, 32])
def test_tiny_layer_full(kvq, rot, group):
    x = W.make_kv(W.config(1)).numpy()
    rep = check_all(kvq, x, rot, group)
    assert rep.n_codes == x.size


@pytest.mark.parametrize("rot", ROTS)
def test_qwen_gqa_cache_full(kvq, rot):
    x = W.make_kv(W.config(3)).numpy()
    rep = check_all(kvq, x, rot, 32)
    assert rep.flip_fraction < 1e-4


@pytest.mark.parametrize("d,group", [(64, 32), (64, 64), (128, 32), (128, 64), (128, 128),
                                     (256, 32), (256, 64), (256, 128), (256, 256)])
@pytest.mark.parametrize("rot", ROTS)
def test_every_shape_small(kvq, d, group, rot):
    # several warp tiles plus a ragged tail, fewer rows than one grid wave
    shape = W.scaled(W.config(5, d=d, group=group), heads=3, tokens=331)
    x = W.make_kv(shape).numpy()
    check_all(kvq, x, rot, group)


@pytest.mark.parametrize("n", [1, 2, 15, 17, 31, 33, 1000])
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("rot", ROTS)
def test_ragged_row_counts(kvq, n, d, rot):
    rng = np.random.default_rng(n * 7 + d)
    x = (rng.standard_normal((n, d)) * 4).astype(np.float16)
    check_all(kvq, x, rot, 32)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("rot", ROTS)
def test_zero_and_extreme_vectors(kvq, d, rot):
    rng = np.random.default_rng(d + rot)
    x = (rng.standard_normal((40, d)) * 3).astype(np.float16)
    x[0] = 0  # all groups zero: s = 0, q = 0, x_hat = 0
    x[5] = 60000.0  # largest magnitudes the generator emits
    x[6] = -60000.0
    x[7, ::3] = 65504.0  # fp16 max
    x[8] = np.float16(6e-8)  # fp16 subnormals
    x[9, 0] = 1.0  # one-hot
    # +-c vectors rotate onto exact ties, so near-tie flips are not capped;
    # x_hat of +-60000 rows may overflow fp16 on both sides
    rep = check_all(kvq, x, rot, 32, max_flip_fraction=None)
    signs = torch.from_numpy(W.make_signs(d)).cuda()
    p, s = kvq.kvq_rot_quant_fwd(torch.from_numpy(x).cuda(), signs, rot, 32)
    assert not s[0].any() and not p[0].any()
    assert rep.n_codes == x.size


@pytest.mark.parametrize("d", [64, 256])
def test_exact_ties_round_half_even(kvq, d):
    """SRHT inputs whose rotated values are exact .5 ties with s = 1."""
    import math
    import scipy.linalg
    signs = W.make_signs(d)
    cyc = [7, 2.5, 0.5, -1.5, -2.5, -0.5, 3.5, 1.5, -3.5, 4.5, -4.5, 5.5, -5.5, 6.5, -6.5, 0.0]
    y = np.array([cyc[i % 16] for i in range(d)])
    x = (scipy.linalg.hadamard(d) @ y / math.sqrt(d) * signs).astype(np.float16)[None]
    sg = torch.from_numpy(signs).cuda()
    p, s = kvq.kvq_rot_quant_fwd(torch.from_numpy(x).cuda(), sg, O.SRHT, d)
    assert float(s[0, 0]) == pytest.approx(1.0, rel=1e-7)
    q = O.unpack_nibbles(p.cpu().numpy())[0].tolist()
    assert q == [int(round(v)) for v in y]


@pytest.mark.parametrize("rot", ROTS)
def test_zero_groups_after_rotation(kvq, rot):
    """A vector whose rotated energy sits in the first group only (SRHT: exact)."""
    d, g = 64, 32
    signs = W.make_signs(d)
    x = (signs.astype(np.float64) * 0.375).astype(np.float16)[None]
    sg = torch.from_numpy(signs).cuda()
    p, s = kvq.kvq_rot_quant_fwd(torch.from_numpy(x).cuda(), sg, rot, g)
    q = O.unpack_nibbles(p.cpu().numpy())[0]
    assert q[0] == 7 and not q[1:].any()
    assert float(s[0, 1]) == 0.0


def _sampled_full_size(kvq, shape, rot, group, n_sample=1 << 15):
    d = shape.d
    x = W.make_kv(shape, device="cuda")
    signs_np = W.make_signs(d)
    p, s, o = run(kvq, x, d, rot, group, signs_np)
    # properties of every output row
    q_lo = (p & 0xF).to(torch.int16)
    q_hi = (p >> 4).to(torch.int16)
    assert not torch.any(q_lo == 8) and not torch.any(q_hi == 8)  # never -8
    q = torch.stack([torch.where(q_lo > 7, q_lo - 16, q_lo),
                     torch.where(q_hi > 7, q_hi - 16, q_hi)], dim=-1).reshape(x.shape[0], d)
    peak = q.abs().reshape(x.shape[0], d // group, group).amax(-1)
    assert torch.all((peak == 7) | (s == 0))
    assert torch.isfinite(o.float()).all()
    # sampled rows against the oracle
    idx = W.sample_rows(x.shape[0], n_sample)
    ti = torch.from_numpy(idx).cuda()
    return full_check(x[ti].cpu().numpy(), signs_np, rot, group, p[ti].cpu().numpy(),
                      s[ti].cpu().numpy(), o[ti].cpu().numpy())


@pytest.mark.parametrize("rot", ROTS)
def test_smollm2_full_cache_sampled(kvq, rot):
    rep = _sampled_full_size(kvq, W.config(2), rot, 64)
    assert rep.flip_fraction < 1e-4


@pytest.mark.parametrize("d,group", [(64, 32), (64, 64), (128, 32), (128, 128), (256, 32),
                                     (256, 256)])
@pytest.mark.parametrize("rot", ROTS)
def test_large_batch_sweep_sampled(kvq, d, group, rot):
    rep = _sampled_full_size(kvq, W.config(5, d=d, group=group), rot, group, 1 << 14)
    assert rep.flip_fraction < 1e-4
