"""Seeded synthetic Q/K/V shaped like video-DiT attention inputs.

This module holds only input generation. It contains none of the attention
method's arithmetic, so both the CUDA path and the CPU oracle may consume what it
produces.

Recipe (one head at a time, every draw from its own seeded stream):

* Token n of an (T, Hg, Wg) latent grid is flattened frame-major:
  n = t*Hg*Wg + h*Wg + w.
* A smooth per-head field G(pos) in R^d is the sum of 16 random sinusoids over
  (t, h, w), each sin(2*pi*(f . pos/extent) + phase) with frequencies f drawn
  from U[0, 0.5] cycles per grid-axis extent (pos/extent = (t/T, h/Hg, w/Wg))
  and phases from U[0, 2*pi),
  projected to d channels by a Gaussian matrix of variance 1/8, so that every
  channel of G has unit variance.
* Q = s*(G + 0.5*eps_q), K = s*(G + 0.5*eps_k) with independent eps ~ N(0, 1)
  and the same G for Q and K of a head, so that nearby tokens attend to each
  other; s sets how peaked attention is.
* V ~ N(0, 1).
* Everything is rounded to bfloat16 with round-to-nearest-even.

The video workloads these shapes come from (480p and 720p Wan2.1 generations,
SpargeAttention2 article "Tsinghua invents an AI attention-slimming technique",
section 5) are not available here; these tensors stand in for their attention
inputs.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence, Tuple

import numpy as np
import torch

_N_SINUSOIDS = 16

# Stream ids keep every tensor of every head reproducible on its own, so a
# subset of heads can be regenerated without drawing the others.
_STREAM_FIELD, _STREAM_EPS_Q, _STREAM_EPS_K, _STREAM_V, _STREAM_ALPHA = 1, 2, 3, 4, 5
_STREAM_ROUTER_BASE, _STREAM_ROUTER_Q, _STREAM_ROUTER_K = 6, 7, 8
_STREAM_DOUT = 9


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention workload: shape, block sizes, mask knobs and generator knobs."""

    name: str
    B: int
    H: int
    N: int
    d: int
    grid: Tuple[int, int, int]
    bq: int
    bk: int
    topk: float
    topp: float
    s: float
    sla2: bool  # alpha drawn from U[0.6, 1.0] per head when True, else alpha = 1
    seed: int = 0

    @property
    def nqb(self) -> int:
        return -(-self.N // self.bq)

    @property
    def nkb(self) -> int:
        return -(-self.N // self.bk)


# The five workload families. The sizes follow the latent grids of 480p and 720p
# Wan2.1 video generation (SpargeAttention2 article, section 5); head counts,
# grids, scales and mask knobs are this build's choices.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 4096, 64, (4, 32, 32), 64, 64, 0.10, 0.9, 1.5, False),
    "480p": Workload("480p", 1, 12, 32760, 128, (21, 30, 52), 128, 64, 0.05, 0.9, 2.0, False),
    "sweep_flat": Workload("sweep_flat", 1, 16, 32768, 128, (16, 32, 64), 128, 64, 0.05, 0.9, 0.3, False),
    "sweep_peaked": Workload("sweep_peaked", 1, 16, 32768, 128, (16, 32, 64), 128, 64, 0.05, 0.9, 3.0, False),
    "sla2_480p": Workload("sla2_480p", 2, 12, 32760, 128, (21, 30, 52), 128, 64, 0.03, 0.9, 2.0, True),
    "720p": Workload("720p", 1, 40, 75600, 128, (21, 45, 80), 128, 64, 0.03, 0.9, 2.5, True),
}

# Mask-regime sweep of the 32768-token workload: top-k x top-p, for each of the
# flat and peaked distributions, and the Top-k-only / Top-p-only / hybrid modes.
SWEEP_TOPK = (0.03, 0.05, 0.10, 0.20)
SWEEP_TOPP = (0.8, 0.9, 0.95)


def _rng(seed: int, b: int, h: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, b, h, stream])))


def _grid_positions(N: int, grid: Optional[Sequence[int]]) -> np.ndarray:
    """(N, 3) float64 array of (t, h, w) coordinates, frame-major order."""
    if grid is None:
        grid = (1, 1, N)
    T, Hg, Wg = grid
    if T * Hg * Wg < N:
        raise ValueError(f"grid {grid} holds fewer than N={N} tokens")
    n = np.arange(N, dtype=np.int64)
    t = n // (Hg * Wg)
    h = (n // Wg) % Hg
    w = n % Wg
    return np.stack([t, h, w], axis=1).astype(np.float64)


def _to_bf16(x: np.ndarray) -> torch.Tensor:
    # torch's float32 -> bfloat16 conversion rounds to nearest even.
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def smooth_field(N: int, d: int, grid, seed: int, b: int, h: int) -> np.ndarray:
    """The per-head smooth field G, float32 (N, d)."""
    rng = _rng(seed, b, h, _STREAM_FIELD)
    freqs = rng.uniform(0.0, 0.5, size=(_N_SINUSOIDS, 3))
    phases = rng.uniform(0.0, 2.0 * math.pi, size=_N_SINUSOIDS)
    proj = rng.normal(0.0, math.sqrt(1.0 / 8.0), size=(_N_SINUSOIDS, d))
    pos = _grid_positions(N, grid) / np.asarray(grid if grid is not None else (1, 1, N), np.float64)
    feats = np.sin(2.0 * math.pi * (pos @ freqs.T) + phases)  # (N, 16)
    return (feats @ proj).astype(np.float32)


def make_qkv(
    B: int,
    H: int,
    N: int,
    d: int,
    grid=None,
    s: float = 1.0,
    seed: int = 0,
    heads: Optional[Sequence[Tuple[int, int]]] = None,
):
    """Seeded bf16 Q, K, V of shape [B, H, N, d] (CPU, contiguous).

    heads: optional list of (b, h) pairs to generate; the result then has shape
    [1, len(heads), N, d] and holds exactly the values those heads have in the
    full tensor.
    """
    pairs = list(heads) if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    nh = len(pairs)
    out_shape = (B, H, N, d) if heads is None else (1, nh, N, d)
    Q = torch.empty(out_shape, dtype=torch.bfloat16)
    K = torch.empty(out_shape, dtype=torch.bfloat16)
    V = torch.empty(out_shape, dtype=torch.bfloat16)
    q2 = Q.view(nh, N, d)
    k2 = K.view(nh, N, d)
    v2 = V.view(nh, N, d)
    for i, (b, h) in enumerate(pairs):
        G = smooth_field(N, d, grid, seed, b, h)
        eq = _rng(seed, b, h, _STREAM_EPS_Q).standard_normal((N, d), dtype=np.float32)
        ek = _rng(seed, b, h, _STREAM_EPS_K).standard_normal((N, d), dtype=np.float32)
        q2[i] = _to_bf16(np.float32(s) * (G + np.float32(0.5) * eq))
        k2[i] = _to_bf16(np.float32(s) * (G + np.float32(0.5) * ek))
        v2[i] = _to_bf16(_rng(seed, b, h, _STREAM_V).standard_normal((N, d), dtype=np.float32))
    return Q, K, V


def make_alpha(H: int, seed: int = 0, sla2: bool = True) -> torch.Tensor:
    """Per-head mixing ratio, float32 [H]: U[0.6, 1.0] when sla2, else all ones."""
    if not sla2:
        return torch.ones(H, dtype=torch.float32)
    rng = _rng(seed, 0, 0, _STREAM_ALPHA)
    return torch.from_numpy(rng.uniform(0.6, 1.0, size=H).astype(np.float32))


def make_router(H: int, d: int, dr: int, seed: int = 0) -> Tuple[torch.Tensor, torch.Tensor]:
    """Router projections Wq, Wk, float32 [H, d, dr], standing in for trained ones.

    Per head: a random partial isometry (QR of a seeded Gaussian matrix:
    orthonormal columns when dr <= d, orthonormal rows when dr > d), times
    (max(d, dr) / min(d, dr))^(1/4) so that the projected dot products over
    sqrt(dr) keep, on average, the scale of the pooled ones over sqrt(d),
    plus independent N(0, 0.1^2/d) perturbations for Wq and Wk, so the two
    differ."""
    Wq = np.zeros((H, d, dr), np.float32)
    Wk = np.zeros((H, d, dr), np.float32)
    gain = (max(d, dr) / min(d, dr)) ** 0.25
    for h in range(H):
        g = _rng(seed, 0, h, _STREAM_ROUTER_BASE)
        if dr <= d:
            base = np.linalg.qr(g.standard_normal((d, dr)))[0]
        else:
            base = np.linalg.qr(g.standard_normal((dr, d)))[0].T
        eq = _rng(seed, 0, h, _STREAM_ROUTER_Q).standard_normal((d, dr)) * (0.1 / math.sqrt(d))
        ek = _rng(seed, 0, h, _STREAM_ROUTER_K).standard_normal((d, dr)) * (0.1 / math.sqrt(d))
        Wq[h] = base * gain + eq
        Wk[h] = base * gain + ek
    return torch.from_numpy(Wq), torch.from_numpy(Wk)


def make_dout(B: int, H: int, N: int, d: int, seed: int = 0, heads=None) -> torch.Tensor:
    """Output gradient dL/dO for the backward, bf16 [B,H,N,d]: N(0, 1) per
    element, one seeded stream per (b, h); `heads` as in make_qkv."""
    pairs = list(heads) if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    out = torch.empty((B, H, N, d) if heads is None else (1, len(pairs), N, d), dtype=torch.bfloat16)
    o2 = out.view(len(pairs), N, d)
    for i, (b, h) in enumerate(pairs):
        o2[i] = _to_bf16(_rng(seed, b, h, _STREAM_DOUT).standard_normal((N, d), dtype=np.float32))
    return out


def make_workload(w: Workload, heads=None):
    """Q, K, V, alpha for a named workload."""
    Q, K, V = make_qkv(w.B, w.H, w.N, w.d, w.grid, w.s, w.seed, heads=heads)
    alpha = make_alpha(w.H, w.seed, w.sla2)
    return Q, K, V, alpha


def random_mask(B: int, H: int, nqb: int, nkb: int, max_keep: int, seed: int = 0):
    """Seeded arbitrary block masks for kernel tests: kv_idx [B,H,nqb,nkb] int32
    holding ascending kept-block lists and kv_cnt [B,H,nqb] int32, with kept
    counts drawn from [0, max_keep] (0 included on purpose)."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 99])))
    kv_idx = np.zeros((B, H, nqb, nkb), dtype=np.int32)
    kv_cnt = np.zeros((B, H, nqb), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(nqb):
                c = int(rng.integers(0, max_keep + 1))
                sel = np.sort(rng.choice(nkb, size=c, replace=False)).astype(np.int32)
                kv_idx[b, h, i, :c] = sel
                kv_cnt[b, h, i] = c
    return torch.from_numpy(kv_idx), torch.from_numpy(kv_cnt)
