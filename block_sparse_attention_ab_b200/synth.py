"""Seeded synthetic inputs shaped like video-DiT attention (Q, K, V in BHND layout).

This module only draws inputs. It holds none of the method's arithmetic, so both the
CUDA path and the CPU oracle can be fed from it.

The AB-Attention news page ("AB-Attention ускорил генерацию видео до 2,23× и
пропускает 92% внимания", section «Как мерили и что вышло») measures on Wan2.1 and
HunyuanVideo latents at 720p with the Penguin Video prompts. Neither the models nor the
prompts are available, so these generators stand in for them: they keep the token
count (frames x height x width latent grid, frame-major), the head count and head
dimension, and give attention a positional, block-local structure through a low-rank
smooth 3-D feature shared by Q and K.

Recipe (all draws on the CPU from ``torch.Generator().manual_seed(seed)``, fp32, then
rounded to bf16 with round-to-nearest-even):
  * grid (T_f, Y, X); token n = t*Y*X + y*X + x;
  * F[n, r] = cos(2*pi*(a_r t/T_f + b_r y/Y + c_r x/X) + phi_r), r < 16, a_r, b_r, c_r
    uniform on {0, 1, 2}, phi_r ~ U[0, 2*pi); columns standardised over the N tokens;
  * per head A_h ~ N(0, 1/16) of shape [16, d]; P_h = F A_h;
  * Q = alpha P_h + beta Z_q, K = alpha P_h + beta Z_k, V ~ N(0, 1), with
    (alpha, beta) = (0.7, 0.3) (tiny: (1, 1));
  * optional per-head temperature tau_h ~ U[0.5, 2]: Q <- tau_h Q;
  * optional heavy-tailed key-block gains: per head ln g_j = 1.5 z_j + 5.28 [j hot],
    hot = a seeded 2% of the key blocks; unit vector u_h; Q += u_h and
    K_t += sqrt(d) ln g_j u_h for t in block j, so block j's logits shift by ln g_j;
  * rows t >= N (padding up to a multiple of 128) are zero.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

BLOCK = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    grid: tuple  # (T_f, Y, X)
    d: int
    budgets: tuple  # fractions of key blocks
    data_seed: int
    alpha: float = 0.7
    beta: float = 0.3
    temperature: bool = False
    hot_gains: bool = False
    fp32_source: bool = False  # values drawn in fp32 (rounded to bf16 before the GPU call)
    topk_budget: Optional[float] = None
    iters: int = 5
    n_clusters: int = 8
    sip_seed: int = 0

    @property
    def N(self) -> int:
        t, y, x = self.grid
        return t * y * x

    @property
    def N_pad(self) -> int:
        return (self.N + BLOCK - 1) // BLOCK * BLOCK

    @property
    def n_blocks(self) -> int:
        return self.N_pad // BLOCK

    def budget_blocks(self, frac: float) -> int:
        """Integer block budget: round-half-up of frac * n_blocks, at least 1."""
        return max(1, int(math.floor(frac * self.n_blocks + 0.5)))


WORKLOADS = {
    # 8 x 8 blocks of 128, head_dim 64, full-strength positional term, 3 of 8 blocks.
    "tiny": Workload("tiny", 1, 2, (4, 16, 16), 64, (3 / 8,), data_seed=0,
                     alpha=1.0, beta=1.0, fp32_source=True, topk_budget=3 / 8),
    # Wan2.1-1.3B shaped 480p clip: 21 x 30 x 52 = 32760 tokens, padded to 32768.
    "wan13b": Workload("wan13b", 1, 12, (21, 30, 52), 128, (0.10,), data_seed=1,
                       topk_budget=0.10),
    # Wan2.1-14B shaped: 40 heads, per-head temperature; 32768 tokens (grid 32 x 32 x 32
    # gives exactly 32768, no padding).
    "wan14b": Workload("wan14b", 1, 40, (32, 32, 32), 128, (0.08, 0.11, 0.20), data_seed=2,
                       temperature=True, topk_budget=0.11),
    # HunyuanVideo shaped 720p: 33 x 45 x 80 = 118800 tokens, padded to 118912.
    "hunyuan720": Workload("hunyuan720", 1, 24, (33, 45, 80), 128, (0.10,), data_seed=3,
                           topk_budget=0.10),
    # Long-context stress: 64^3 = 262144 tokens, mass concentrated on 2% of key blocks.
    "long": Workload("long", 1, 24, (64, 64, 64), 128,
                     (0.05, 0.10, 0.15, 0.20, 0.25, 0.30), data_seed=4, hot_gains=True,
                     topk_budget=0.10),
}


def positional_features(grid, gen: torch.Generator, rank: int = 16) -> torch.Tensor:
    """Rank-`rank` smooth 3-D cosine features F [N, rank], columns standardised."""
    T_f, Y, X = grid
    coef = torch.randint(0, 3, (3, rank), generator=gen).to(torch.float64)
    phase = torch.rand(rank, generator=gen, dtype=torch.float64) * (2 * math.pi)
    t = torch.arange(T_f, dtype=torch.float64).view(T_f, 1, 1) / T_f
    y = torch.arange(Y, dtype=torch.float64).view(1, Y, 1) / Y
    x = torch.arange(X, dtype=torch.float64).view(1, 1, X) / X
    F = torch.empty(T_f * Y * X, rank, dtype=torch.float64)
    for r in range(rank):
        arg = 2 * math.pi * (coef[0, r] * t + coef[1, r] * y + coef[2, r] * x) + phase[r]
        F[:, r] = torch.cos(arg).reshape(-1)
    F = F - F.mean(dim=0, keepdim=True)
    std = F.std(dim=0, keepdim=True)
    # A constant column (all coefficients 0) has zero spread; keep it at zero.
    F = torch.where(std > 0, F / std.clamp_min(1e-30), torch.zeros_like(F))
    return F.to(torch.float32)


def make_qkv(w: Workload, heads: Optional[list] = None, dtype=torch.bfloat16):
    """Draw Q, K, V [B, H, N_pad, d] for workload `w` (host tensors, `dtype`).

    `heads` restricts generation to a subset of head indices (the draws of every head
    are still keyed by the head index, so a subset equals the same heads of the full
    tensor). The returned tensors then have len(heads) heads.
    """
    B, H, N, N_pad, d = w.B, w.H, w.N, w.N_pad, w.d
    heads = list(range(H)) if heads is None else list(heads)
    base = torch.Generator().manual_seed(w.data_seed)
    F = positional_features(w.grid, base)
    nb = w.n_blocks
    q = torch.zeros(B, len(heads), N_pad, d, dtype=dtype)
    k = torch.zeros_like(q)
    v = torch.zeros_like(q)
    for b in range(B):
        for hi, h in enumerate(heads):
            g = torch.Generator().manual_seed(w.data_seed * 1_000_003 + b * 10_007 + h + 1)
            A = torch.randn(16, d, generator=g) / 4.0
            P = F @ A
            Zq = torch.randn(N, d, generator=g)
            Zk = torch.randn(N, d, generator=g)
            V = torch.randn(N, d, generator=g)
            Q = w.alpha * P + w.beta * Zq
            K = w.alpha * P + w.beta * Zk
            if w.temperature:
                tau = 0.5 + 1.5 * torch.rand(1, generator=g).item()
                Q = tau * Q
            if w.hot_gains:
                z = torch.randn(nb, generator=g)
                n_hot = max(1, int(round(0.02 * nb)))
                hot = torch.randperm(nb, generator=g)[:n_hot]
                lng = 1.5 * z
                lng[hot] += 5.28
                u = torch.randn(d, generator=g)
                u = u / u.norm()
                Q = Q + u.view(1, d)
                shift = (math.sqrt(d) * lng).repeat_interleave(BLOCK)[:N]
                K = K + shift.view(N, 1) * u.view(1, d)
            q[b, hi, :N] = Q.to(dtype)
            k[b, hi, :N] = K.to(dtype)
            v[b, hi, :N] = V.to(dtype)
    return q, k, v


def bf16_bits(t: torch.Tensor) -> torch.Tensor:
    """Raw bf16 bit patterns of a bf16 tensor, as int16 (same memory)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16)
