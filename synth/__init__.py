"""Seeded synthetic inputs for the Jano hot path.

This module is shared by the GPU library's tests and benchmark and by the
CPU oracle's tests.  It holds none of the method's arithmetic: no block
score, no level classification, no schedule, no scatter and no attention.
It only draws random numbers and shapes them into latents, per-token fields
and BF16 activations with the structure of the workloads the Jano pages
describe (Flux-1-dev images and Wan2.1 videos, whose weights and prompts are
not used).  All randomness comes from ``numpy.random.default_rng(seed)`` or a seeded
``torch.Generator``.

Recipe (one line per input kind):

* latent history  x_k = n + s_k * G,  k = 0..K, s_k = (k/K)^2, with
  n ~ N(0,1) drawn once (shape [C,F,H,W]) and G a sum of 3D Gaussian blobs
  (amplitude uniform in [1,3], sigma in latent pixels) shared by all channels;
  stored fp32 as [K+1][C][F][H][W], w fastest.
* per-token field  a sum of Gaussian blobs over the token grid
  [TF][TH][TW]; in video grids each blob centre drifts by at most one token
  per frame, so the structure persists across frames; stored fp32, token id
  t = (f*TH + h)*TW + w.
* activations  Q/K/V ~ N(0,1) rounded to BF16 (round to nearest even),
  layout [tokens][heads][d]; small ones as uint16 bit patterns from numpy,
  large ones as torch BF16 tensors from a seeded torch CPU generator.
* stale cache  K_cache = K + N(0, 0.05) rounded to BF16.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "rng", "gaussian_blobs", "latent_history",
    "token_field", "bf16_bits", "bf16_normal", "bf16_perturb", "bf16_to_f32",
    "normal_bf16", "perturb_bf16", "bits_of", "tensor_of", "step_rows",
]


def rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def gaussian_blobs(shape, n_blobs, sigma, gen, amp=(1.0, 3.0), drift=0.0):
    """Sum of isotropic Gaussian blobs on a (F, H, W) grid, fp64.

    Each blob has a random centre, amplitude uniform in ``amp`` and a random
    per-frame velocity in [-drift, drift]^2 (h, w); ``drift=0`` gives blobs
    that are static across frames.
    """
    F, H, W = shape
    f = np.arange(F, dtype=np.float64)[:, None, None]
    h = np.arange(H, dtype=np.float64)[None, :, None]
    w = np.arange(W, dtype=np.float64)[None, None, :]
    out = np.zeros((F, H, W), dtype=np.float64)
    for _ in range(n_blobs):
        ch = gen.uniform(0, H)
        cw = gen.uniform(0, W)
        cf = gen.uniform(0, F)
        a = gen.uniform(*amp)
        vh, vw = gen.uniform(-drift, drift, size=2) if drift > 0 else (0.0, 0.0)
        hh = h - (ch + vh * f)
        ww = w - (cw + vw * f)
        r2 = hh * hh + ww * ww
        if drift == 0.0 and F > 1:
            # static 3D blob: Gaussian in f as well (sigma in frames = sigma/2)
            r2 = r2 + ((f - cf) * 2.0) ** 2
        out += a * np.exp(-r2 / (2.0 * sigma * sigma))
    return out


def latent_history(K, C, F, H, W, seed, n_blobs=3, sigma=4.0):
    """Latent snapshots x_0..x_K, fp32, shape [K+1, C, F, H, W]."""
    g = rng(seed)
    n = g.standard_normal((C, F, H, W))
    G = gaussian_blobs((F, H, W), n_blobs, sigma, g)
    x = np.empty((K + 1, C, F, H, W), dtype=np.float32)
    for k in range(K + 1):
        s = (k / K) ** 2
        x[k] = (n + s * G[None]).astype(np.float32)
    return x


def token_field(TF, TH, TW, seed, n_blobs=6, sigma=6.0, drift=1.0):
    """Smooth seeded per-token field, fp32, flat [TF*TH*TW] in token order."""
    g = rng(seed)
    fld = gaussian_blobs((TF, TH, TW), n_blobs, sigma, g,
                         drift=drift if TF > 1 else 0.0)
    # a small seeded ripple keeps the field free of exact ties
    fld += 1e-3 * g.standard_normal(fld.shape)
    return fld.reshape(-1).astype(np.float32)


def bf16_bits(x_f32: np.ndarray) -> np.ndarray:
    """Round fp32 to BF16 (nearest even) and return the uint16 bit patterns."""
    x = np.ascontiguousarray(x_f32, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    nan = np.isnan(x)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    r[nan] = 0x7FC0
    return r


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_normal(shape, gen) -> np.ndarray:
    return bf16_bits(gen.standard_normal(shape).astype(np.float32))


def bf16_perturb(bits, sigma, gen) -> np.ndarray:
    x = bf16_to_f32(bits).astype(np.float64)
    return bf16_bits((x + sigma * gen.standard_normal(x.shape)).astype(np.float32))


def normal_bf16(shape, seed):
    """N(0,1) rounded to BF16 as a torch CPU tensor (seeded torch generator;
    used for the large activation tensors, where it is ~5x faster than numpy)."""
    import torch
    g = torch.Generator().manual_seed(int(seed))
    return torch.randn(tuple(shape), generator=g, dtype=torch.float32).to(torch.bfloat16)


def linear_weight_bf16(n_out, n_in, seed):
    """Random linear-layer weight [n_out][n_in]: N(0, 1/n_in) rounded to BF16
    (torch CPU tensor, seeded), so x @ w^T keeps unit-scale activations."""
    import torch
    g = torch.Generator().manual_seed(int(seed))
    w = torch.randn((n_out, n_in), generator=g, dtype=torch.float32) * (n_in ** -0.5)
    return w.to(torch.bfloat16)


def perturb_bf16(x, sigma, seed):
    """BF16(x + N(0, sigma^2)) for a BF16 torch CPU tensor x (a stale cache)."""
    import torch
    g = torch.Generator().manual_seed(int(seed))
    out = torch.empty_like(x)
    flat_x, flat_o = x.view(-1), out.view(-1)
    step = 1 << 26
    for i in range(0, flat_x.numel(), step):
        n = torch.randn(min(step, flat_x.numel() - i), generator=g, dtype=torch.float32)
        flat_o[i:i + step] = (flat_x[i:i + step].float() + sigma * n).to(torch.bfloat16)
    return out


def bits_of(t) -> np.ndarray:
    """uint16 bit patterns (numpy view) of a contiguous BF16 torch CPU tensor."""
    import torch
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def tensor_of(bits: np.ndarray):
    """BF16 torch CPU tensor sharing memory with uint16 bit patterns."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def step_rows(tokens: np.ndarray, step: int, n_rows: int, shift: int = 7) -> np.ndarray:
    """Pool rows that supply token ids `tokens` with fresh activations at
    sampling step `step`: row (t + shift*step) mod n_rows.  A pure indexing
    rule, so a few seeded pools stand in for new activations at every step."""
    return (np.asarray(tokens, dtype=np.int64) + shift * step) % n_rows


@dataclass(frozen=True)
class Workload:
    """One configuration of the hot path (sizes from the Jano pages' models)."""
    name: str
    seed: int
    K: int              # latent snapshots are x_0..x_K
    C: int
    F: int
    H: int
    W: int
    block: tuple        # (bf, bh, bw) analyzer block, latent elements
    patch: tuple        # (pf, ph, pw) token patch, latent elements
    heads: int
    d: int
    frac_active: float
    frac_static: float
    T: int = 50
    warmup: int = 5
    cooldown: int = 5
    period_moderate: int = 2
    period_static: int = 4
    field_sigma: float = 6.0
    extra: dict = field(default_factory=dict)

    @property
    def grid(self):
        pf, ph, pw = self.patch
        return (self.F // pf, self.H // ph, self.W // pw)

    @property
    def n_tokens(self):
        a, b, c = self.grid
        return a * b * c

    @property
    def n_blocks(self):
        bf, bh, bw = self.block
        return (-(-self.F // bf)) * (-(-self.H // bh)) * (-(-self.W // bw))

    @property
    def latent_shape(self):
        return (self.K + 1, self.C, self.F, self.H, self.W)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 5, 16, 4, 32, 32, (1, 4, 4), (1, 2, 2), 4, 64,
                     0.30, 0.70, field_sigma=3.0),
    "image": Workload("image", 2, 5, 16, 1, 128, 128, (1, 2, 2), (1, 2, 2), 24, 128,
                      0.30, 0.40),
    "small": Workload("small", 3, 5, 16, 21, 60, 104, (1, 4, 4), (1, 2, 2), 12, 128,
                      0.35, 0.65),
    "large": Workload("large", 4, 5, 16, 21, 90, 160, (1, 4, 4), (1, 2, 2), 40, 128,
                      0.25, 0.45),
    "schedule50": Workload("schedule50", 5, 5, 16, 21, 60, 104, (1, 2, 2), (1, 2, 2), 12, 128,
                           0.30, 0.40),
}
