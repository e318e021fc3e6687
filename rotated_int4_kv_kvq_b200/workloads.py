"""Seeded synthetic K/V workloads and sign vectors.

This module only draws random inputs.  It holds none of the codec's
arithmetic, so both the CUDA path (bench, tests) and the CPU oracle (tests)
can be fed from it without sharing any of the method.

The shapes follow the KV caches of the models measured on the pages
("Quantization Speed Is Often a Kernel Problem", sections "Fusing four steps
into two kernels is not enough" and "A scene": SmolLM2-360M/1.7B,
Qwen2.5-1.5B, Gemma-3 1B).  No weights or datasets are used; the values are
N(0, 1) with a few fixed large "outlier" channels per head, the structure the
rotation is meant to spread ("First, the 17%").

Vectors are laid out row-major as [layer][K|V][head][token][d], so one
contiguous [n_vec, d] fp16 tensor holds a whole cache.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

_MASK64 = (1 << 64) - 1


def splitmix64(seed: int, count: int) -> list[int]:
    """``count`` outputs of Vigna's SplitMix64 generator started at ``seed``."""
    state = seed & _MASK64
    out = []
    for _ in range(count):
        state = (state + 0x9E3779B97F4A7C15) & _MASK64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
        out.append(z ^ (z >> 31))
    return out


def make_signs(d: int, seed: int | None = None) -> np.ndarray:
    """The fixed +-1 sign vector D: -1 where the top bit of the i-th
    SplitMix64 output is set.  Default seed is 1000 + d."""
    if seed is None:
        seed = 1000 + d
    return np.array([-1 if (z >> 63) else 1 for z in splitmix64(seed, d)],
                    dtype=np.int8)


@dataclass(frozen=True)
class KVShape:
    """One synthetic KV workload."""

    name: str
    layers: int
    heads: int
    tokens: int
    d: int
    group: int
    n_outlier: int  # outlier channels per (layer, K|V, head)
    outlier_lo: float  # outlier factor ~ U(lo, hi); lo == hi means fixed
    outlier_hi: float
    k_bias_var: float = 0.0  # K gets a per-(head, channel) bias ~ N(0, var)
    k_student_t: bool = False  # K gets additive Student-t(3) noise
    seed: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def n_vec(self) -> int:
        return self.layers * 2 * self.heads * self.tokens


def config(i: int, d: int | None = None, group: int | None = None) -> KVShape:
    """The five workloads, numbered 1..5 (seed i-1)."""
    if i == 1:  # SmolLM2-360M-like single layer
        return KVShape("tiny-smollm2-360m-layer", 1, 5, 256, 64, 64, 2, 20.0,
                       20.0, k_bias_var=2.0, seed=0)
    if i == 2:  # SmolLM2-1.7B-like full cache
        return KVShape("smollm2-1.7b-cache", 24, 32, 4096, 64, 64, 4, 10.0,
                       30.0, seed=1)
    if i == 3:  # Qwen2.5-1.5B-like GQA cache
        return KVShape("qwen2.5-1.5b-gqa-cache", 28, 2, 2048, 128, 32, 3, 25.0,
                       25.0, k_student_t=True, seed=2)
    if i == 4:  # Gemma-3-1B-like decode, full token sequence up to 4096
        return KVShape("gemma3-1b-decode", 26, 1, 4096, 256, 256, 2, 20.0,
                       20.0, seed=3, extra={"prefix": 256})
    if i == 5:  # large-batch sweep: 64 sequences x 8 heads folded into heads
        dd = 128 if d is None else d
        gg = 32 if group is None else group
        return KVShape(f"sweep-d{dd}-g{gg}", 1, 64 * 8, 8192, dd, gg, 4, 20.0,
                       20.0, seed=4)
    raise ValueError(f"no workload {i}")


def scaled(shape: KVShape, **changes) -> KVShape:
    """A copy of ``shape`` with fewer layers/heads/tokens (same recipe)."""
    fields = dict(shape.__dict__)
    fields.update(changes)
    return KVShape(**fields)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_kv(shape: KVShape, device="cpu", seed: int | None = None,
            chunk_heads: int = 64) -> torch.Tensor:
    """Draw the [n_vec, d] fp16 cache of ``shape`` on ``device``.

    Per (layer, K|V, head): ``n_outlier`` distinct channels are scaled by a
    factor ~ U(lo, hi) for every token.  K additionally gets a per-channel
    bias ~ N(0, k_bias_var) and/or additive Student-t(3) noise.  Values are
    clamped to +-60000 before the fp16 cast.
    """
    seed = shape.seed if seed is None else seed
    g = _gen(device, seed)
    L, H, T, d = shape.layers, shape.heads, shape.tokens, shape.d
    out = torch.empty((L, 2, H, T, d), dtype=torch.float16, device=device)
    for layer in range(L):
        for kv in range(2):
            for h0 in range(0, H, chunk_heads):
                h1 = min(H, h0 + chunk_heads)
                nh = h1 - h0
                v = torch.randn((nh, T, d), generator=g, device=device)
                order = torch.rand((nh, d), generator=g, device=device)
                ch = order.argsort(dim=1)[:, : shape.n_outlier]
                fac = shape.outlier_lo + (shape.outlier_hi - shape.outlier_lo) * \
                    torch.rand((nh, shape.n_outlier), generator=g, device=device)
                scale = torch.ones((nh, d), device=device)
                scale.scatter_(1, ch, fac)
                v *= scale[:, None, :]
                if kv == 0 and shape.k_bias_var > 0:
                    bias = torch.randn((nh, d), generator=g, device=device)
                    v += (shape.k_bias_var ** 0.5) * bias[:, None, :]
                if kv == 0 and shape.k_student_t:
                    z = torch.randn((nh, T, d), generator=g, device=device)
                    c = torch.randn((3, nh, T, d), generator=g, device=device)
                    v += z / torch.sqrt((c * c).sum(0) / 3.0)
                out[layer, kv, h0:h1] = v.clamp_(-60000.0, 60000.0).half()
    return out.reshape(shape.n_vec, d)


def make_decode_sequence(shape: KVShape, device="cpu", seed: int | None = None):
    """Config-4 style token stream: [layers*2 heads, tokens, d] fp16 where the
    K and V of every layer are consecutive heads (head = 2*layer + kv)."""
    kv = make_kv(shape, device=device, seed=seed)
    L, H, T, d = shape.layers, shape.heads, shape.tokens, shape.d
    return kv.reshape(L * 2 * H, T, d)


def sample_rows(n_vec: int, count: int, seed: int = 12345) -> np.ndarray:
    """Sorted distinct row indices for sampled parity checks (always includes
    the first and the last row)."""
    rng = np.random.default_rng(seed)
    count = min(count, n_vec)
    idx = rng.choice(n_vec, size=count, replace=False)
    idx[0] = 0
    if count > 1:
        idx[1] = n_vec - 1
    return np.unique(idx)
