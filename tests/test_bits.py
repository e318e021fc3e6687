"""Other code widths on the B200: kvq_rot_quant_fwd_bits and
kvq_dequant_rot_inv_bits (3, 6 and 8 bits) against the oracle's b-bit
quantizer and little-endian bitstream, with the same parity bar as int4."""

import numpy as np
import pytest
import torch

import oracle.kvq_oracle as O
from parity import check_fwd, check_inv
from rotated_int4_kv_kvq_b200 import workloads as W

pytestmark = pytest.mark.gpu

CASES = [(64, 32), (64, 64), (128, 32), (128, 128), (256, 64), (256, 256)]


@pytest.fixture(scope="module")
def kvq():
    from rotated_int4_kv_kvq_b200 import kvq as mod
    return mod


@pytest.mark.parametrize("d,g", CASES)
@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
@pytest.mark.parametrize("bits", [3, 6, 8])
@pytest.mark.parametrize("n", [1, 1000])
def test_bits_parity(kvq, d, g, rot, bits, n):
    if bits == 3 and d == 64:
        pytest.skip("3-bit rows of d = 64 are 24 bytes: rejected (see test below)")
    shape = W.scaled(W.config(5, d=d, group=g), heads=1, tokens=max(n, 16))
    x = W.make_kv(shape, device="cuda")[:n].contiguous()
    signs_np = W.make_signs(d)
    signs = torch.from_numpy(signs_np).cuda()
    packed, scales = kvq.kvq_rot_quant_fwd_bits(x, signs, rot, g, bits)
    out = kvq.kvq_dequant_rot_inv_bits(packed, scales, signs, rot, g, bits)
    torch.cuda.synchronize()
    assert kvq.kvq_device_status() == 0
    assert packed.shape == (n, d * bits // 8)
    xn = x.cpu().numpy()
    # the near-tie window scales with the code step, so flips are not capped
    _, _, _, _, flipped = check_fwd(xn, signs_np, rot, g, packed.cpu().numpy(),
                                    scales.cpu().numpy(), max_flip_fraction=None, bits=bits)
    check_inv(xn, signs_np, rot, g, packed.cpu().numpy(), scales.cpu().numpy(),
              out.cpu().numpy(), flipped, bits=bits)


@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
def test_four_bits_through_the_bits_entry_points(kvq, rot):
    """bits = 4 through the _bits calls is the plain int4 path, bit for bit."""
    shape = W.scaled(W.config(5, d=128, group=32), heads=1, tokens=333)
    x = W.make_kv(shape, device="cuda")
    signs = torch.from_numpy(W.make_signs(128)).cuda()
    p1, s1 = kvq.kvq_rot_quant_fwd_bits(x, signs, rot, 32, 4)
    p2, s2 = kvq.kvq_rot_quant_fwd(x, signs, rot, 32)
    assert torch.equal(p1, p2) and torch.equal(s1, s2)
    assert torch.equal(kvq.kvq_dequant_rot_inv_bits(p1, s1, signs, rot, 32, 4),
                       kvq.kvq_dequant_rot_inv(p2, s2, signs, rot, 32))


def test_bad_bits_rejected(kvq):
    """3 bits at d = 64 and widths other than 3/4/6/8: KVQ_ERR_BAD_BITS, nothing
    launched."""
    x = torch.zeros((4, 64), dtype=torch.float16, device="cuda")
    signs = torch.from_numpy(W.make_signs(64)).cuda()
    p = torch.zeros((4, 64), dtype=torch.uint8, device="cuda")
    s = torch.zeros((4, 1), dtype=torch.float32, device="cuda")
    for bits in (2, 3, 5, 16):
        st = kvq.lib.kvq_rot_quant_fwd_bits(x.data_ptr(), 4, 64, 64, bits, signs.data_ptr(), 0,
                                            p.data_ptr(), s.data_ptr(), None)
        assert st == 10
    torch.cuda.synchronize()
    assert not p.any()
