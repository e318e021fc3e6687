"""The windowed decode step (needs a B200): a dequantized-prefix cache with an
fp16 tail.  Every step is checked against the oracle's windowed step on the
same tokens, and against the plain decode step: closed windows of the view
must equal the plain step's output rows bit for bit (both run the same
one-warp-per-vector arithmetic)."""

import numpy as np
import pytest
import torch

import oracle.kvq_oracle as O
from parity import MAX_FLIP_FRACTION, TIE_WINDOW, check_fwd, check_inv
from rotated_int4_kv_kvq_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvq():
    from rotated_int4_kv_kvq_b200 import kvq as mod
    return mod


def run_steps(kvq, d, group, rot, heads, window, steps, seed):
    cap = steps + 2
    signs_np = W.make_signs(d)
    signs = torch.from_numpy(signs_np).cuda()
    g = torch.Generator(device="cuda").manual_seed(seed)
    toks = (torch.randn((steps, heads, d), generator=g, device="cuda") * 3).half()
    toks[:, :, 3] *= 25  # an outlier channel
    packed = torch.full((heads, cap, d // 2), 0x77, dtype=torch.uint8, device="cuda")
    scales = torch.full((heads, cap, d // group), 1e30, dtype=torch.float32, device="cuda")
    kv = torch.zeros((heads, cap, d), dtype=torch.float16, device="cuda")
    # the plain decode step on its own cache, for the bit-identity check
    packed2 = torch.zeros_like(packed)
    scales2 = torch.zeros_like(scales)
    toks_np = toks.cpu().numpy()
    closed = 0
    flips = codes = 0
    for pos in range(steps):
        kv_before = kv.clone()
        p_before, s_before = packed.clone(), scales.clone()
        kvq.kvq_decode_step_windowed(toks[pos], packed, scales, kv, pos, signs, rot, group,
                                     window)
        out = kvq.kvq_decode_step(toks[pos], packed2, scales2, pos, signs, rot, group)
        flush = (pos + 1) % window == 0
        first = pos + 1 - window if flush else pos
        # rows before this step's window are untouched
        assert torch.equal(kv[:, :first], kv_before[:, :first])
        assert torch.equal(packed[:, :first], p_before[:, :first])
        assert torch.equal(scales[:, :first], s_before[:, :first])
        if flush:
            closed = pos + 1
            wp = packed[:, first: pos + 1].reshape(-1, d // 2).cpu().numpy()
            ws = scales[:, first: pos + 1].reshape(-1, d // group).cpu().numpy()
            x_w = toks_np[first: pos + 1].transpose(1, 0, 2).reshape(-1, d)
            q, _, nf, _, flipped = check_fwd(x_w, signs_np, rot, group, wp, ws,
                                             max_flip_fraction=None)
            flips += nf
            codes += q.size
            check_inv(x_w, signs_np, rot, group, wp, ws,
                      kv[:, first: pos + 1].reshape(-1, d).cpu().numpy(), flipped)
        else:
            # the open window's codes and scales are not written
            assert torch.equal(packed[:, pos], p_before[:, pos])
            assert torch.equal(scales[:, pos], s_before[:, pos])
        # open window: the tokens themselves
        assert torch.equal(kv[:, closed: pos + 1], toks[closed: pos + 1].transpose(0, 1))
        # closed windows: identical to the plain decode step's rows
        assert torch.equal(kv[:, :closed], out[:, :closed])
        assert torch.equal(packed[:, :closed], packed2[:, :closed])
        assert torch.equal(scales[:, :closed], scales2[:, :closed])
    torch.cuda.synchronize()
    assert kvq.kvq_device_status() == 0
    # near-tie flips against the oracle, over every closed window of the run
    assert flips < MAX_FLIP_FRACTION * max(codes, 1), f"{flips} near-tie flips of {codes} codes"
    return kv, packed, scales, toks_np, signs_np


@pytest.mark.parametrize("d,group", [(64, 32), (64, 64), (128, 32), (128, 128), (256, 64),
                                     (256, 256)])
@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
@pytest.mark.parametrize("heads,window,steps", [(1, 1, 3), (2, 4, 11), (3, 16, 35)])
def test_windowed_steps(kvq, d, group, rot, heads, window, steps):
    run_steps(kvq, d, group, rot, heads, window, steps, seed=d + 13 * window + rot)


@pytest.mark.parametrize("rot", [O.SRFT, O.SRHT])
def test_windowed_against_oracle_view(kvq, rot):
    """The whole view after 2 windows and a partial one, against the oracle
    run of the windowed step on the same tokens (GPU codes replace the
    oracle's at near-tie flips, so the view is compared on rows whose codes
    agree, and through the oracle inverse of the GPU codes elsewhere)."""
    d, group, heads, window, steps = 256, 256, 2, 16, 37
    kv, packed, scales, toks, signs_np = run_steps(kvq, d, group, rot, heads, window, steps, 5)
    cap = steps + 2
    pc = np.zeros((heads, cap, d // 2), np.uint8)
    sc = np.zeros((heads, cap, d // group), np.float32)
    kvo = np.zeros((heads, cap, d), np.float16)
    for pos in range(steps):
        O.decode_step_windowed(toks[pos], pc, sc, kvo, pos, signs_np, rot, group, window)
    closed = (steps // window) * window
    kv_np = kv.cpu().numpy()
    assert np.array_equal(kv_np[:, closed:steps], kvo[:, closed:steps])
    gp = packed[:, :closed].cpu().numpy()
    gs = scales[:, :closed].cpu().numpy()
    rel = np.abs(gs - sc[:, :closed]) / np.where(sc[:, :closed] > 0, sc[:, :closed], 1)
    assert rel.max() <= 1e-6
    # codes: identical except near-tie flips, fewer than 1e-4 of all codes
    qg = O.unpack_nibbles(gp.reshape(-1, d // 2))
    qo = O.unpack_nibbles(pc[:, :closed].reshape(-1, d // 2))
    bad = qg != qo
    if bad.any():
        x_c = toks[:closed].transpose(1, 0, 2).reshape(-1, d)
        y = O.rotated_values(x_c, signs_np, rot)
        dist = O.near_tie_distance(y, sc[:, :closed].reshape(-1, d // group), group)
        assert dist[bad].max() < TIE_WINDOW
    assert bad.sum() < MAX_FLIP_FRACTION * qg.size
    same = (gp == pc[:, :closed]).all(axis=2)
    tol = 2e-3 * np.abs(kvo[:, :closed].astype(np.float64)).max(axis=2, keepdims=True) + 1e-6
    err = np.abs(kv_np[:, :closed].astype(np.float64) - kvo[:, :closed].astype(np.float64))
    assert np.all(err[same] <= tol.repeat(d, axis=2)[same])


def test_windowed_never_flushes_before_window(kvq):
    """window larger than the sequence: the view is the tokens, exactly."""
    kv, packed, _, toks, _ = run_steps(kvq, 128, 64, O.SRFT, 2, 64, 10, 3)
    assert np.array_equal(kv[:, :10].cpu().numpy(), toks.transpose(1, 0, 2))
    assert (packed[:, :10] == 0x77).all()
