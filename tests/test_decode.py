"""The fused decode step (needs a B200): one launch quantizes the new token
of every head into cache row `pos` and dequantizes rows [0, pos] of every
head.  Checked bit-for-bit against the separate forward / inverse kernels
(themselves checked against the oracle) and against the oracle's decode step.
"""

import numpy as np
import pytest
import torch

import oracle.kvq_oracle as O
from parity import check_fwd, check_inv
from rotated_int4_kv_kvq_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvq():
    from rotated_int4_kv_kvq_b200 import kvq as mod
    return mod


def make_cache(kvq, heads, cap, pos, d, group, rot, signs, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    hist = (torch.randn((heads, cap, d), generator=g, device="cuda") * 3).half()
    hist[:, :, 5] *= 20  # an outlier channel
    packed = torch.zeros((heads, cap, d // 2), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((heads, cap, d // group), dtype=torch.float32, device="cuda")
    if pos > 0:
        p, s = kvq.kvq_rot_quant_fwd(hist[:, :pos].reshape(-1, d).contiguous(), signs, rot, group)
        packed[:, :pos] = p.reshape(heads, pos, -1)
        scales[:, :pos] = s.reshape(heads, pos, -1)
    # stale garbage beyond pos must not leak into the output
    packed[:, pos + 1:] = 0x77
    scales[:, pos + 1:] = 1e30
    x_new = (torch.randn((heads, d), generator=g, device="cuda") * 3).half()
    return packed, scales, x_new


WIDE_MAX_ROWS = 1 << 16  # calls with more rows run the tiled kernel


def run_and_check(kvq, d, group, rot, heads, cap, pos, seed):
    signs_np = W.make_signs(d)
    signs = torch.from_numpy(signs_np).cuda()
    packed, scales, x_new = make_cache(kvq, heads, cap, pos, d, group, rot, signs, seed)
    before_p, before_s = packed.clone(), scales.clone()
    out = kvq.kvq_decode_step(x_new, packed, scales, pos, signs, rot, group)
    torch.cuda.synchronize()
    assert kvq.kvq_device_status() == 0
    # untouched rows
    keep = torch.ones(cap, dtype=torch.bool)
    keep[pos] = False
    assert torch.equal(packed[:, keep], before_p[:, keep])
    assert torch.equal(scales[:, keep], before_s[:, keep])
    p_new, s_new = kvq.kvq_rot_quant_fwd(x_new, signs, rot, group)
    rows_p = packed[:, : pos + 1].reshape(-1, d // 2).contiguous()
    rows_s = scales[:, : pos + 1].reshape(-1, d // group).contiguous()
    ref = kvq.kvq_dequant_rot_inv(rows_p, rows_s, signs, rot, group).reshape(heads, pos + 1, d)
    xn = x_new.cpu().numpy()
    if heads * (pos + 1) > WIDE_MAX_ROWS:
        # tiled kernel: same arithmetic as the forward / inverse kernels
        assert torch.equal(packed[:, pos], p_new)
        assert torch.equal(scales[:, pos], s_new)
        assert torch.equal(out, ref)
    # new row against the oracle (codes, scales) and its output row
    check_fwd(xn, signs_np, rot, group, packed[:, pos].cpu().numpy(),
              scales[:, pos].cpu().numpy(), max_flip_fraction=None)
    o = out.cpu().numpy()
    check_inv(xn, signs_np, rot, group, packed[:, pos].cpu().numpy(),
              scales[:, pos].cpu().numpy(), o[:, pos], None)
    # every row against the oracle inverse of the stored codes and scales
    ref_o = O.dequant_rot_inv(rows_p.cpu().numpy(), rows_s.cpu().numpy(), signs_np, rot,
                              group).reshape(heads, pos + 1, d).astype(np.float64)
    tol = 2e-3 * np.abs(ref_o).max(axis=2, keepdims=True) + 1e-6
    assert np.all(np.abs(o.astype(np.float64) - ref_o) <= tol)
    # and against the inverse kernel on the same rows
    assert np.all(np.abs(o.astype(np.float64) - ref.cpu().numpy().astype(np.float64)) <= tol)


@pytest.mark.parametrize("d,group", [(64, 32), (64, 64), (128, 32), (128, 128), (256, 64),
                                     (256, 256), (256, 32), (128, 64)])
@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
@pytest.mark.parametrize("heads,cap,pos", [(1, 1, 0), (2, 40, 0), (2, 40, 17), (3, 64, 63),
                                           (5, 300, 257), (52, 70, 33)])
def test_decode_small_calls(kvq, d, group, rot, heads, cap, pos):
    run_and_check(kvq, d, group, rot, heads, cap, pos, seed=d + 7 * pos + heads)


@pytest.mark.parametrize("d,group", [(64, 64), (128, 32), (256, 256)])
@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
def test_decode_large_call_tiled(kvq, d, group, rot):
    """More than 2^16 rows: the tiled kernel, bit-identical to fwd / inv."""
    run_and_check(kvq, d, group, rot, heads=3, cap=23000, pos=22001, seed=d + rot)


def test_gemma_decode_steps(kvq):
    """Config-4 shape: 26 layers x (K, V) x d=256, g=256, one call per layer
    with K and V as two heads, several consecutive steps from a 256 prefix."""
    shape = W.scaled(W.config(4), tokens=264)
    seq = W.make_decode_sequence(shape, device="cuda")  # [52, 264, 256]
    d, group, cap, pre = 256, 256, 264, 256
    signs_np = W.make_signs(d)
    signs = torch.from_numpy(signs_np).cuda()
    for rot in (O.SRFT, O.SRHT):
        packed = torch.zeros((52, cap, d // 2), dtype=torch.uint8, device="cuda")
        scales = torch.zeros((52, cap, 1), dtype=torch.float32, device="cuda")
        p, s = kvq.kvq_rot_quant_fwd(seq[:, :pre].reshape(-1, d).contiguous(), signs, rot, group)
        packed[:, :pre] = p.reshape(52, pre, -1)
        scales[:, :pre] = s.reshape(52, pre, -1)
        for pos in range(pre, cap):
            for layer in range(26):
                hs = slice(2 * layer, 2 * layer + 2)
                kv_p = packed[hs]
                kv_s = scales[hs]
                # per-layer views are contiguous slices of the head-major cache
                out = kvq.kvq_decode_step(seq[hs, pos].contiguous(), kv_p, kv_s, pos, signs,
                                          rot, group)
                if layer == 25 and pos == cap - 1:
                    x_all = seq[hs, : pos + 1].reshape(-1, d).cpu().numpy()
                    p_all = kv_p[:, : pos + 1].reshape(-1, d // 2).cpu().numpy()
                    s_all = kv_s[:, : pos + 1].reshape(-1, 1).cpu().numpy()
                    _, _, flips, _, flipped = check_fwd(x_all, signs_np, rot, group, p_all, s_all)
                    check_inv(x_all, signs_np, rot, group, p_all, s_all,
                              out.reshape(-1, d).cpu().numpy(), flipped)
        torch.cuda.synchronize()
        assert kvq.kvq_device_status() == 0


@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
def test_decode_52_heads_just_past_the_wide_limit(kvq, rot):
    """52 heads in one call at pos 1260 (65,572 rows): the first position at
    which a 52-head call leaves the one-warp-per-vector kernel."""
    assert 52 * 1261 > WIDE_MAX_ROWS >= 52 * 1260
    run_and_check(kvq, 256, 256, rot, heads=52, cap=1262, pos=1260, seed=11 + rot)


@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
def test_gemma_decode_step_across_the_prefix_sweep(kvq, rot):
    """Config 4 at the prefix lengths the step is measured at (pos 1024,
    2048, 4095): the cache rows [0, pos) come from the forward call over the
    token stream, then one 26-call decode step (K and V of a layer as two
    heads) runs at pos.  Every layer's new row is checked against the oracle
    (codes, scales, x_hat), and every output row of every layer against the
    oracle inverse of the stored codes and scales."""
    shape = W.config(4)
    seq = W.make_decode_sequence(shape, device="cuda")  # [52, 4096, 256]
    d, group, cap = 256, 256, 4096
    signs_np = W.make_signs(d)
    signs = torch.from_numpy(signs_np).cuda()
    seq_np = seq.cpu().numpy()
    flips = codes = 0
    for pos in (1024, 2048, 4095):
        packed = torch.zeros((52, cap, d // 2), dtype=torch.uint8, device="cuda")
        scales = torch.zeros((52, cap, 1), dtype=torch.float32, device="cuda")
        p, s = kvq.kvq_rot_quant_fwd(seq[:, :pos].reshape(-1, d).contiguous(), signs, rot, group)
        packed[:, :pos] = p.reshape(52, pos, -1)
        scales[:, :pos] = s.reshape(52, pos, -1)
        outs = []
        for layer in range(26):
            hs = slice(2 * layer, 2 * layer + 2)
            outs.append(kvq.kvq_decode_step(seq[hs, pos].contiguous(), packed[hs], scales[hs],
                                            pos, signs, rot, group))
        torch.cuda.synchronize()
        assert kvq.kvq_device_status() == 0
        out = torch.cat(outs).cpu().numpy()  # [52, pos + 1, 256]
        # the new row of every head against the oracle
        x_new = seq_np[:, pos]
        p_new = packed[:, pos].cpu().numpy()
        s_new = scales[:, pos].cpu().numpy()
        q, _, nf, _, flipped = check_fwd(x_new, signs_np, rot, group, p_new, s_new,
                                         max_flip_fraction=None)
        flips += nf
        codes += q.size
        check_inv(x_new, signs_np, rot, group, p_new, s_new, out[:, pos], flipped)
        # every row of every head against the oracle inverse of the stored codes
        rows_p = packed[:, : pos + 1].reshape(-1, d // 2).cpu().numpy()
        rows_s = scales[:, : pos + 1].reshape(-1, 1).cpu().numpy()
        ref_o = O.dequant_rotated_f64(rows_p, rows_s, signs_np, rot, group)
        got = out.reshape(-1, d).astype(np.float64)
        tol = 2e-3 * np.abs(ref_o).max(axis=1, keepdims=True) + 1e-6
        assert np.all(np.abs(got - ref_o) <= tol)
        # the cached codes themselves against the oracle's forward step
        q, _, nf, _, _ = check_fwd(seq_np[:, :pos].reshape(-1, d), signs_np, rot, group,
                                   rows_p.reshape(52, pos + 1, -1)[:, :pos].reshape(-1, d // 2),
                                   rows_s.reshape(52, pos + 1, -1)[:, :pos].reshape(-1, 1),
                                   max_flip_fraction=None)
        flips += nf
        codes += q.size
        del packed, scales, outs
    assert flips < 1e-4 * codes, f"{flips} near-tie flips of {codes} codes"
