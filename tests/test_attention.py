"""Decode attention over the int4 cache (needs a B200): kvq_attend_decode
against the oracle's attend_decode (float64 softmax over the exactly
dequantized, inverse-rotated K and V).  The cache rows are written by the
library's own forward kernel; rows beyond `len` hold garbage that must not
leak into the result."""

import numpy as np
import pytest
import torch

import oracle.kvq_oracle as O
from rotated_int4_kv_kvq_b200 import workloads as W

pytestmark = pytest.mark.gpu

OUT_RTOL = 2e-3  # of the largest output element of the row (fp16 rounding: 2^-11)


@pytest.fixture(scope="module")
def kvq():
    from rotated_int4_kv_kvq_b200 import kvq as mod
    return mod


def make_cache(kvq, heads, cap, d, group, rot, signs, seed, ramp=0.0):
    """ramp > 0: K rows drift along the all-ones direction (by ramp at the
    last row) and the queries point along it, so the scores rise through
    the sequence and the running maximum moves many times."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    out = []
    for kv in range(2):  # K, V
        x = torch.randn((heads * cap, d), generator=g, device="cuda") * 2
        x[:, 7] *= 15  # an outlier channel
        if ramp and kv == 0:
            t = torch.arange(cap, device="cuda", dtype=torch.float32).repeat(heads) / cap
            x += ramp * t[:, None]
        x = x.half()
        p, s = kvq.kvq_rot_quant_fwd(x, signs, rot, group)
        out += [p.reshape(heads, cap, -1), s.reshape(heads, cap, -1)]
    q = (torch.randn((heads, 8, d), generator=g, device="cuda")).half()
    if ramp:
        q = (q.float() * 0.1 + 1.0).half()
    return out, q


def run_case(kvq, d, group, rot, heads, nq, length, sm_scale=None, seed=0, ramp=0.0):
    cap = length + 5
    signs_np = W.make_signs(d)
    signs = torch.from_numpy(signs_np).cuda()
    (kp, ks, vp, vs), qall = make_cache(kvq, heads, cap, d, group, rot, signs, seed, ramp)
    # garbage beyond len
    kp[:, length:] = 0x77
    vp[:, length:] = 0x17
    ks[:, length:] = 1e30
    vs[:, length:] = 1e30
    q = qall[:, :nq].contiguous()
    scale = d ** -0.5 if sm_scale is None else sm_scale
    out = kvq.kvq_attend_decode(q, kp, ks, vp, vs, length, signs, rot, group, scale)
    torch.cuda.synchronize()
    assert kvq.kvq_device_status() == 0
    ref = O.attend_decode(q.cpu().numpy(), kp.cpu().numpy(), ks.cpu().numpy(), vp.cpu().numpy(),
                          vs.cpu().numpy(), length, signs_np, rot, group, scale)
    got = out.cpu().numpy().astype(np.float64)
    r = ref.astype(np.float64)
    tol = OUT_RTOL * np.abs(r).max(axis=2, keepdims=True) + 1e-6
    err = np.abs(got - r)
    assert np.all(err <= tol), f"max err {(err / tol).max():.3g} x tol"
    return got


@pytest.mark.parametrize("d,group", [(64, 32), (64, 64), (128, 32), (128, 128), (256, 64),
                                     (256, 256)])
@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
@pytest.mark.parametrize("nq,length", [(1, 1), (4, 7), (1, 300), (2, 333), (4, 2500),
                                       (8, 1000), (6, 97)])
def test_attention_parity(kvq, d, group, rot, nq, length):
    run_case(kvq, d, group, rot, heads=2, nq=nq, length=length, seed=d + length + nq)


@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
def test_attention_sharp_and_flat(kvq, rot):
    """sm_scale 0: the mean of V; a large scale: close to one-hot weights."""
    run_case(kvq, 256, 256, rot, heads=1, nq=4, length=513, sm_scale=0.0, seed=3)
    run_case(kvq, 128, 32, rot, heads=3, nq=2, length=200, sm_scale=4.0, seed=4)


def test_attention_gemma_shape(kvq):
    """Gemma-3-1B-like layer: 1 KV head, 4 queries, d = g = 256, 4096 rows."""
    run_case(kvq, 256, 256, O.SRFT, heads=1, nq=4, length=4096, seed=9)


def test_attention_many_heads(kvq):
    """SmolLM2-1.7B-like layer: 32 KV heads, one query each, d = g = 64."""
    run_case(kvq, 64, 64, O.SRFT, heads=32, nq=1, length=1024, seed=10)


@pytest.mark.parametrize("group", [32, 64])
@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
@pytest.mark.parametrize("heads,length,scale", [(1, 4096, None), (3, 9001, None), (2, 2048, 0.0),
                                                (5, 1500, 3.0), (40, 777, None), (1, 1, None),
                                                (300, 2500, None)])
def test_attention_lane_pair_d64(kvq, group, rot, heads, length, scale):
    """d = 64 with one query per KV head (the lane-pair kernel): single blocks
    and clusters of several blocks, ragged token splits, flat and sharp
    softmax, a single row, and more heads than SMs (one block per head)."""
    run_case(kvq, 64, group, rot, heads=heads, nq=1, length=length, sm_scale=scale,
             seed=heads + length + group)


@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
@pytest.mark.parametrize("heads,nq,length,scale", [(1, 4, 1, None), (2, 3, 15, None), (1, 4, 16, None),
                                                   (3, 4, 17, 2.0), (1, 3, 4096, None), (2, 4, 5003, 0.0),
                                                   (64, 4, 700, None), (1, 4, 33, 6.0)])
def test_attention_tensor_core_d256(kvq, rot, heads, nq, length, scale):
    """d = g = 256 with 3 or 4 queries per KV head (the tensor-core kernel):
    single tokens, partial and whole 16-token chunks, several blocks per
    head, flat and sharp softmax, more heads than one block each."""
    run_case(kvq, 256, 256, rot, heads=heads, nq=nq, length=length, sm_scale=scale,
             seed=heads * 7 + nq + length)


@pytest.mark.parametrize("d,group,nq", [(256, 256, 4), (128, 128, 3), (64, 64, 2), (64, 64, 1),
                                        (256, 64, 4)])
@pytest.mark.parametrize("heads,length", [(1, 4096), (2, 777), (40, 1500)])
def test_attention_rising_scores(kvq, d, group, nq, heads, length):
    """Scores that rise through the sequence (by tens of log2 units): the
    running maximum of every warp moves many times, in steps below and
    above any slack the kernels allow it."""
    run_case(kvq, d, group, O.SRFT, heads=heads, nq=nq, length=length, sm_scale=0.5 / d ** 0.5,
             seed=heads + length + d, ramp=6.0)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
@pytest.mark.parametrize("heads,nq,length,scale", [(1, 5, 1, None), (2, 8, 17, None), (3, 6, 700, 2.0),
                                                   (1, 8, 4096, None), (40, 7, 333, None),
                                                   (2, 8, 1000, 0.0), (100, 8, 64, None)])
def test_attention_tensor_core_query_groups(kvq, d, rot, heads, nq, length, scale):
    """g = d with 5-8 queries per KV head: the tensor-core kernel in two
    groups of 4 queries per head (the second group partly padding for 5-7),
    single and many heads, ragged lengths, flat and sharp softmax."""
    run_case(kvq, d, d, rot, heads=heads, nq=nq, length=length, sm_scale=scale,
             seed=heads * 11 + nq + length + d)
