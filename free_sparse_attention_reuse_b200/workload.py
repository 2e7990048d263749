"""Seeded synthetic DiT-shaped attention inputs (no attention arithmetic lives here).

The method is evaluated on video models (Minimax-H3-Base, HunyuanVideo, Wan2.1) and a 3D
asset model ("MC-Sparse가 확산 트랜스포머 희소 어텐션의 품질 격차를 좁힌다", section 전제와 한계);
none of those weights or datasets are available, so these tensors stand in for one attention
layer's Q, K and V:

* tokens are the cells of a (t, h, w) or (x, y, z) grid, flattened row-major;
* each token gets 3 axes x 16 frequencies x (sin, cos) = 96 positional features, with
  angular frequency pi * (1 / L_axis) ** (f / 15), f = 0..15;
* each head draws one projection W (96 x d, entries N(0, 1/96)), shared by Q, K and V, so
  that nearby tokens have large logits (the locality a DiT's attention shows);
* each tensor adds its own N(0, 0.5^2) noise and is rounded to bf16;
* a denoising step perturbs the fp32 state by N(0, 0.05^2) and re-rounds to bf16.

The random numbers come from torch's CPU generator (mt19937, ``torch.Generator``), seeded
with ``1000 + config_index`` for the base tensors and ``seed * 1000 + step`` for step noise.
Both the oracle tests and the CUDA path receive exactly these tensors.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from fractions import Fraction

import torch

N_FREQ = 16
N_FEAT = 3 * N_FREQ * 2  # 96
NOISE_STD = 0.5
STEP_STD = 0.05


@dataclass(frozen=True)
class Workload:
    """One synthetic attention layer shape."""

    name: str
    index: int  # seeds derive from it
    B: int
    H: int
    d: int
    grid: tuple
    C: int
    densities: tuple = field(default=(0.15,))

    @property
    def N(self) -> int:
        return self.grid[0] * self.grid[1] * self.grid[2]

    @property
    def G(self) -> int:
        return self.N // self.C

    def k(self, density: float) -> int:
        """k = floor(s * N), computed in exact rational arithmetic from the decimal s."""
        return int(math.floor(Fraction(str(density)) * self.N))

    @property
    def seed(self) -> int:
        return 1000 + self.index


WORKLOADS = {
    "tiny": Workload("tiny", 0, 1, 2, 64, (4, 16, 16), 64, (0.25,)),
    "480p": Workload("480p", 1, 1, 24, 128, (21, 32, 48), 128, (0.15, 0.25)),
    "720p": Workload("720p", 2, 1, 40, 128, (21, 48, 80), 128, (0.15,)),
    "3d": Workload("3d", 3, 1, 16, 64, (32, 32, 32), 128, (0.15,)),
    "sweep": Workload("sweep", 4, 1, 24, 128, (21, 32, 48), 128, (0.05, 0.10, 0.15, 0.25, 0.50)),
}


def custom(name: str, B: int, H: int, d: int, grid: tuple, C: int, densities=(0.25,), index: int = 9):
    """A workload of arbitrary size built by the same recipe (used by small tests)."""
    return Workload(name, index, B, H, d, tuple(grid), C, tuple(densities))


def positional_features(grid) -> torch.Tensor:
    """[N, 96] float64 sinusoidal features of the flattened grid cells."""
    axes = []
    for L in grid:
        pos = torch.arange(L, dtype=torch.float64)
        f = torch.arange(N_FREQ, dtype=torch.float64)
        omega = math.pi * (1.0 / L) ** (f / (N_FREQ - 1))
        ang = pos[:, None] * omega[None, :]
        axes.append(torch.cat([torch.sin(ang), torch.cos(ang)], dim=1))  # [L, 32]
    a0, a1, a2 = axes
    n0, n1, n2 = (x.shape[0] for x in axes)
    f0 = a0[:, None, None, :].expand(n0, n1, n2, -1)
    f1 = a1[None, :, None, :].expand(n0, n1, n2, -1)
    f2 = a2[None, None, :, :].expand(n0, n1, n2, -1)
    return torch.cat([f0, f1, f2], dim=-1).reshape(n0 * n1 * n2, N_FEAT)


class Generator:
    """Produces the anchor-step tensors and the perturbed tensors of later steps.

    ``state`` holds the fp32 random-walk state of Q, K and V ([B, H, N, d] each); ``step(s)``
    returns bf16 tensors for step s (s = 0 is the unperturbed start).
    """

    def __init__(self, wl: Workload, device: str = "cpu"):
        """``device="cuda"`` draws the same recipe with the device's generator (a different
        random stream from the CPU one, used for full-size benchmark inputs)."""
        self.wl = wl
        self.device = torch.device(device)
        g = torch.Generator(device=self.device).manual_seed(wl.seed)
        phi = positional_features(wl.grid).to(torch.float32).to(self.device)  # [N, F]
        W = torch.randn(wl.B, wl.H, N_FEAT, wl.d, generator=g, device=self.device) / math.sqrt(N_FEAT)
        base = torch.matmul(phi, W)  # [B, H, N, d]
        self.state = []
        for _ in range(3):
            self.state.append(base + NOISE_STD * torch.randn(base.shape, generator=g, device=self.device))
        self._step = 0

    def current(self):
        return tuple(x.to(torch.bfloat16) for x in self.state)

    def advance(self):
        """Apply one denoising-step perturbation (seed * 1000 + step) and return bf16 Q, K, V."""
        self._step += 1
        g = torch.Generator(device=self.device).manual_seed(self.wl.seed * 1000 + self._step)
        for x in self.state:
            x.add_(STEP_STD * torch.randn(x.shape, generator=g, device=self.device))
        return self.current()


def make_qkv(wl: Workload, step: int = 0):
    """Q, K, V (bf16, [B, H, N, d], CPU) of ``wl`` after ``step`` perturbations."""
    gen = Generator(wl)
    out = gen.current()
    for _ in range(step):
        out = gen.advance()
    return out


def lattice_qkv(B: int, H: int, N: int, d: int, seed: int, lo: int = -2, hi: int = 2):
    """Small-integer bf16 tensors: with d = 64 the scale 1/8 is exact, so every logit is an
    exact multiple of 1/8 in any fp32 accumulation order."""
    g = torch.Generator().manual_seed(seed)
    t = [torch.randint(lo, hi + 1, (B, H, N, d), generator=g).to(torch.bfloat16) for _ in range(3)]
    return tuple(t)
