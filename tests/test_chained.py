"""Dependent decode-path calls launched back to back (needs a B200).

The decode-step, windowed-step and attention kernels may be scheduled
while the previous kernel of the stream drains, and wait for it before
their first global access.  These tests chain calls where each one reads
what the one before it wrote (cache row pos, the attention view, the K/V
rows a step just appended), replay the chain from a CUDA graph so that the
launches follow each other with no host gap, and require the result to be
bit-identical to the same calls run one at a time with a device
synchronize after each.
"""

import pytest
import torch

import oracle.kvq_oracle as O
from rotated_int4_kv_kvq_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvq():
    from rotated_int4_kv_kvq_b200 import kvq as mod
    return mod


def state(d, group, heads, cap, pre, seed, kvq, rot, signs):
    g = torch.Generator(device="cuda").manual_seed(seed)
    hist = (torch.randn((heads, cap, d), generator=g, device="cuda") * 2).half()
    packed = torch.zeros((heads, cap, d // 2), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((heads, cap, d // group), dtype=torch.float32, device="cuda")
    p, s = kvq.kvq_rot_quant_fwd(hist[:, :pre].reshape(-1, d).contiguous(), signs, rot, group)
    packed[:, :pre] = p.reshape(heads, pre, -1)
    scales[:, :pre] = s.reshape(heads, pre, -1)
    return hist, packed, scales


def run_eager_and_graph(chain, init, tensors):
    """chain() issues the calls; init() resets every tensor the chain
    writes; tensors() lists what is compared."""
    init()
    torch.cuda.synchronize()
    chain(sync=True)
    torch.cuda.synchronize()
    want = [t.clone() for t in tensors()]

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up outside the capture
        init()
        chain(sync=False)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        chain(sync=False)
    for _ in range(3):
        init()
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        got = tensors()
        for w, x in zip(want, got):
            assert torch.equal(w, x)
    del graph


@pytest.mark.parametrize("d,group,nq", [(64, 64, 4), (64, 64, 1), (256, 256, 4), (128, 32, 4)])
@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
def test_consecutive_decode_steps_and_attention(kvq, d, group, nq, rot):
    """Each position: decode step on the K heads, on the V heads (each
    appends row pos and decodes rows [0, pos]), then attention over
    pos + 1 rows that include the two rows just written (d = 64 with one
    query per head runs the lane-pair attention kernel)."""
    heads, cap, pre, steps = 2, 48, 20, 12
    signs = torch.from_numpy(W.make_signs(d)).cuda()
    k_hist, k0p, k0s = state(d, group, heads, cap, pre, 11 + d, kvq, rot, signs)
    v_hist, v0p, v0s = state(d, group, heads, cap, pre, 12 + d, kvq, rot, signs)
    kp, ks, vp, vs = k0p.clone(), k0s.clone(), v0p.clone(), v0s.clone()
    g = torch.Generator(device="cuda").manual_seed(13)
    q = (torch.randn((heads, nq, d), generator=g, device="cuda")).half()
    k_out = [torch.empty((heads, pos + 1, d), dtype=torch.float16, device="cuda")
             for pos in range(pre, pre + steps)]
    v_out = [torch.empty_like(o) for o in k_out]
    a_out = [torch.empty((heads, nq, d), dtype=torch.float16, device="cuda") for _ in k_out]
    xk = [k_hist[:, pos].contiguous() for pos in range(pre, pre + steps)]
    xv = [v_hist[:, pos].contiguous() for pos in range(pre, pre + steps)]

    def init():
        kp.copy_(k0p), ks.copy_(k0s), vp.copy_(v0p), vs.copy_(v0s)
        for o in k_out + v_out + a_out:
            o.zero_()

    def chain(sync):
        for i, pos in enumerate(range(pre, pre + steps)):
            kvq.kvq_decode_step(xk[i], kp, ks, pos, signs, rot, group, k_out[i])
            kvq.kvq_decode_step(xv[i], vp, vs, pos, signs, rot, group, v_out[i])
            kvq.kvq_attend_decode(q, kp, ks, vp, vs, pos + 1, signs, rot, group, out=a_out[i])
            if sync:
                torch.cuda.synchronize()

    run_eager_and_graph(chain, init, lambda: [kp, ks, vp, vs] + k_out + v_out + a_out)
    assert kvq.kvq_device_status() == 0


@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
def test_consecutive_windowed_steps(kvq, rot):
    """Windowed steps over three flushes: each step writes row pos of the
    attention view and every 16th step quantizes the window the previous
    steps filled (flushes at positions 31, 47 and 63)."""
    d, group, heads, cap, window = 256, 256, 2, 96, 16
    first, steps = 31, 36  # positions 31 .. 66
    signs = torch.from_numpy(W.make_signs(d)).cuda()
    g = torch.Generator(device="cuda").manual_seed(21)
    seq = (torch.randn((heads, cap, d), generator=g, device="cuda") * 2).half()
    p0 = torch.zeros((heads, cap, d // 2), dtype=torch.uint8, device="cuda")
    s0 = torch.zeros((heads, cap, d // group), dtype=torch.float32, device="cuda")
    kv0 = torch.zeros((heads, cap, d), dtype=torch.float16, device="cuda")
    packed, scales, kv = p0.clone(), s0.clone(), kv0.clone()
    xs = [seq[:, pos].contiguous() for pos in range(first, first + steps)]

    def init():
        packed.copy_(p0), scales.copy_(s0), kv.copy_(kv0)

    def chain(sync):
        for i, pos in enumerate(range(first, first + steps)):
            kvq.kvq_decode_step_windowed(xs[i], packed, scales, kv, pos, signs, rot, group,
                                         window)
            if sync:
                torch.cuda.synchronize()

    run_eager_and_graph(chain, init, lambda: [packed, scales, kv])
    assert kvq.kvq_device_status() == 0
