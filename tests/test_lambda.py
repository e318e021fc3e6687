"""The per-channel lambda hook on the B200: kvq_rot_quant_fwd_lambda and
kvq_dequant_rot_inv_lambda against the oracle (codes, scales, x_hat), and
against the plain entry points where they must agree exactly."""

import numpy as np
import pytest
import torch

import oracle.kvq_oracle as O
from parity import check_fwd, check_inv
from rotated_int4_kv_kvq_b200 import workloads as W

pytestmark = pytest.mark.gpu

SHAPES = [(64, 32), (64, 64), (128, 32), (128, 128), (256, 64), (256, 256)]


@pytest.fixture(scope="module")
def kvq():
    from rotated_int4_kv_kvq_b200 import kvq as mod
    return mod


def make_lambda(d, seed):
    g = np.random.default_rng(seed)
    return np.exp(g.normal(0.0, 0.5, d)).astype(np.float32)  # log-normal around 1


@pytest.mark.parametrize("d,g", SHAPES)
@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
@pytest.mark.parametrize("n", [1, 33, 1000])
def test_lambda_parity(kvq, d, g, rot, n):
    shape = W.scaled(W.config(5, d=d, group=g), heads=1, tokens=max(n, 16))
    x = W.make_kv(shape, device="cuda")[:n].contiguous()
    signs_np = W.make_signs(d)
    signs = torch.from_numpy(signs_np).cuda()
    lam_np = make_lambda(d, d + n)
    lam = torch.from_numpy(lam_np).cuda()
    packed, scales = kvq.kvq_rot_quant_fwd(x, signs, rot, g, lam=lam)
    out = kvq.kvq_dequant_rot_inv(packed, scales, signs, rot, g, lam=lam)
    torch.cuda.synchronize()
    assert kvq.kvq_device_status() == 0
    xn = x.cpu().numpy()
    _, _, _, _, flipped = check_fwd(xn, signs_np, rot, g, packed.cpu().numpy(),
                                    scales.cpu().numpy(), max_flip_fraction=None, lam=lam_np)
    check_inv(xn, signs_np, rot, g, packed.cpu().numpy(), scales.cpu().numpy(),
              out.cpu().numpy(), flipped, lam=lam_np)


@pytest.mark.parametrize("d,g", [(64, 64), (128, 32), (256, 256)])
@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
def test_lambda_power_of_two_is_prescaling(kvq, d, g, rot):
    """Per-channel powers of two: the lambda forward equals the plain
    forward on the exactly pre-scaled input, bit for bit; the lambda inverse
    equals the plain inverse divided channel-wise (exact in fp16)."""
    n = 777
    shape = W.scaled(W.config(5, d=d, group=g), heads=1, tokens=n)
    x = W.make_kv(shape, device="cuda")[:n].contiguous()
    signs = torch.from_numpy(W.make_signs(d)).cuda()
    # factors 1, 2, 4: exact in fp16 for every value here (halving would
    # round subnormal inputs)
    e = torch.from_numpy(np.random.default_rng(d).integers(0, 3, d)).cuda()
    lam = torch.pow(2.0, e.float()).contiguous()
    xs = (x.float() * lam).half()
    assert torch.equal(xs.float(), x.float() * lam)
    p1, s1 = kvq.kvq_rot_quant_fwd(x, signs, rot, g, lam=lam)
    p2, s2 = kvq.kvq_rot_quant_fwd(xs, signs, rot, g)
    assert torch.equal(p1, p2) and torch.equal(s1, s2)
    o1 = kvq.kvq_dequant_rot_inv(p1, s1, signs, rot, g, lam=lam)
    o2 = kvq.kvq_dequant_rot_inv(p2, s2, signs, rot, g)
    ok = (o2.float() / lam).abs() >= 2.0 ** -14  # fp16 normal after the division
    assert torch.equal(o1.float()[ok], (o2.float() / lam)[ok])


def test_lambda_null_is_rejected(kvq):
    x = torch.zeros((4, 64), dtype=torch.float16, device="cuda")
    signs = torch.from_numpy(W.make_signs(64)).cuda()
    p = torch.empty((4, 32), dtype=torch.uint8, device="cuda")
    s = torch.empty((4, 1), dtype=torch.float32, device="cuda")
    st = kvq.lib.kvq_rot_quant_fwd_lambda(x.data_ptr(), 4, 64, 64, signs.data_ptr(), None, 0,
                                          p.data_ptr(), s.data_ptr(), None)
    assert st == 1
