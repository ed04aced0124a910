"""Seeded synthetic workloads for the tile-sparse attention hot path.

This module only draws inputs; it holds none of the method's arithmetic.  Both
the CUDA path and the oracle receive the same tensors from it.

The shapes follow the workloads the Veda project page describes ("Scaling Law
in Practice": per-layer latency as the token count grows up to 245K; the 480P
and 720P Waver/Wan latents of "Inference Latency"; 90% and 95% sparsity).  The
pages give no data, so the values are synthetic:

* V ~ N(0, 1).
* Q = Z_q + alpha * Phi(pos) U_h and K = Z_k + alpha * Phi(pos) U_h with
  Z ~ N(0, 1), alpha = d ** 0.25, Phi a rank-8 smooth basis of the 3-D position
  (cos and sin of 2*pi*(a t/T + b y/Hs + c x/Ws) for four frequency triples
  (a, b, c) in {1,2,3}^3 drawn by seed) and U_h in R^{8 x d} with unit-norm
  Gaussian rows, per head and shared by Q and K.  q.k then gains a translation
  invariant term sum cos(omega . dpos) that peaks at dpos = 0 (about +4 nats
  after the 1/sqrt(d) scale), so attention is local-heavy.
* W_q, W_k ~ N(0, 1/d), fp32, per head.
* Head tile shapes (head-aware configs) drawn by seed from
  {(1,8,16), (2,8,8), (4,4,8)}.

Values are drawn with torch's generator on the requested device (CPU draws and
CUDA draws differ; every run feeds one set of tensors to both sides).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Sequence, Tuple

import numpy as np
import torch

HEAD_SHAPES = [(1, 8, 16), (2, 8, 8), (4, 4, 8)]


def sparsity_to_k(nT: int, sparsity_pct: int) -> int:
    """Tiles kept per query-tile row at a given sparsity, rounded to nearest."""
    return max(1, (nT * (100 - sparsity_pct) + 50) // 100)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    T: int
    Hs: int
    Ws: int
    tile_shapes: Tuple[Tuple[int, int, int], ...]  # one per head
    k: int
    sparsity: int
    seed: int = 0

    @property
    def N(self) -> int:
        return self.T * self.Hs * self.Ws

    @property
    def grid(self) -> Tuple[int, int, int]:
        return (self.T, self.Hs, self.Ws)

    @property
    def Bt(self) -> int:
        pt, ph, pw = self.tile_shapes[0]
        return pt * ph * pw

    @property
    def nT(self) -> int:
        return self.N // self.Bt

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def shapes_array(self) -> np.ndarray:
        return np.asarray(self.tile_shapes, dtype=np.int32).reshape(self.H, 3)

    def sparse_flops(self) -> float:
        """FLOPs of the selected tile pairs: QK^T and PV, 2 flops per MAC."""
        return 4.0 * self.B * self.H * self.nT * self.k * self.Bt * self.Bt * self.d

    def dense_flops(self) -> float:
        return 4.0 * self.B * self.H * self.nT * self.nT * self.Bt * self.Bt * self.d

    def describe(self) -> dict:
        return dict(workload=self.name, B=self.B, H=self.H, d=self.d,
                    grid=f"{self.T}x{self.Hs}x{self.Ws}", tokens=self.N, tile_tokens=self.Bt,
                    tiles=self.nT, k=self.k, sparsity_pct=self.sparsity, seed=self.seed,
                    head_shapes=sorted({tuple(s) for s in self.tile_shapes}))


def head_aware_shapes(H: int, seed: int) -> Tuple[Tuple[int, int, int], ...]:
    pick = np.random.default_rng(seed).integers(0, 3, H)
    return tuple(HEAD_SHAPES[int(p)] for p in pick)


def _make(name, B, H, d, grid, shapes, sparsity, seed=0) -> Workload:
    T, Hs, Ws = grid
    if isinstance(shapes, str):
        shapes = head_aware_shapes(H, seed)
    elif len(shapes) == 1:
        shapes = tuple(shapes) * H
    pt, ph, pw = shapes[0]
    nT = (T * Hs * Ws) // (pt * ph * pw)
    return Workload(name, B, H, d, T, Hs, Ws, tuple(tuple(s) for s in shapes),
                    sparsity_to_k(nT, sparsity), sparsity, seed)


def tiny(seed: int = 0) -> Workload:
    """B=1, H=2, d=64, grid 4x8x16 = 512 tokens, tile (1,8,8), 8 tiles, k=2."""
    return _make("tiny", 1, 2, 64, (4, 8, 16), [(1, 8, 8)], 75, seed)


def p480(seed: int = 0) -> Workload:
    """480P-like: B=1, H=12, d=128, grid 20x32x48 = 30,720, tile (2,8,8), k=24."""
    return _make("480p", 1, 12, 128, (20, 32, 48), [(2, 8, 8)], 90, seed)


def p720(seed: int = 0) -> Workload:
    """720P-like head-aware: B=1, H=40, d=128, grid 20x48x80 = 76,800, k=30."""
    return _make("720p", 1, 40, 128, (20, 48, 80), "head-aware", 95, seed)


def long_video(seed: int = 0, H: int = 32) -> Workload:
    """Long video: B=1, H=32, d=128, grid 60x64x64 = 245,760, 1,920 tiles, k=96.
    A smaller H gives the same problem with fewer heads (the first H heads'
    tile shapes, the same k; its own seeded data), a case that fits the
    few-GB rule of counter captures."""
    name = "long_video_245k" if H == 32 else f"long_video_245k_h{H}"
    return _make(name, 1, H, 128, (60, 64, 64), "head-aware", 95, seed)


SWEEP_T = (4, 8, 20, 32, 64)
SWEEP_SPARSITY = (0, 50, 80, 90, 95, 98)


def sweep(T: int, sparsity: int, seed: int = 0) -> Workload:
    """Sweep point: H=24, d=128, latent plane 48x80, T frames, head-aware tiles."""
    return _make(f"sweep_T{T}_s{sparsity}", 1, 24, 128, (T, 48, 80), "head-aware", sparsity,
                 seed)


def sweep_points(seed: int = 0) -> List[Workload]:
    return [sweep(T, s, seed) for T in SWEEP_T for s in SWEEP_SPARSITY]


def custom(name, B, H, d, grid, shapes: Sequence, k: int, seed: int = 0) -> Workload:
    """A workload with explicit per-head tile shapes and k (tests, edge cases)."""
    if len(shapes) == 1:
        shapes = list(shapes) * H
    return Workload(name, B, H, d, *grid, tuple(tuple(int(v) for v in s) for s in shapes), int(k),
                    -1, seed)


CONFIGS = {"tiny": tiny, "480p": p480, "720p": p720, "long_video": long_video}


def _generator(device, seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + stream * 7919) % (2 ** 63))
    return g


def position_basis(w: Workload, device="cpu") -> torch.Tensor:
    """Phi: [N, 8] fp32, cos/sin of four seeded frequency triples (a, b, c)."""
    rng = np.random.default_rng([w.seed, 17])
    freqs = rng.integers(1, 4, size=(4, 3))
    t = torch.arange(w.T, device=device, dtype=torch.float64).view(-1, 1, 1) / w.T
    y = torch.arange(w.Hs, device=device, dtype=torch.float64).view(1, -1, 1) / w.Hs
    x = torch.arange(w.Ws, device=device, dtype=torch.float64).view(1, 1, -1) / w.Ws
    feats = []
    for a, b, c in freqs:
        theta = 2.0 * math.pi * (int(a) * t + int(b) * y + int(c) * x)
        feats.append(torch.cos(theta).reshape(-1))
        feats.append(torch.sin(theta).reshape(-1))
    return torch.stack(feats, dim=1).to(torch.float32)


def generate(w: Workload, device="cpu", with_v: bool = True):
    """Draw Q, K, V (bf16 [B,H,N,d]) and W_q, W_k (fp32 [H,d,d]) on ``device``.

    Generated head by head to bound the fp32 temporaries.
    """
    B, H, N, d = w.B, w.H, w.N, w.d
    alpha = d ** 0.25
    phi = position_basis(w, device)
    gu = _generator(device, w.seed, 1)
    U = torch.randn((H, 8, d), generator=gu, device=device, dtype=torch.float32)
    U = U / U.norm(dim=-1, keepdim=True)
    out = {}
    for name, stream in (("Q", 2), ("K", 3), ("V", 4)):
        if name == "V" and not with_v:
            continue
        g = _generator(device, w.seed, stream)
        t = torch.empty((B, H, N, d), device=device, dtype=torch.bfloat16)
        for b in range(B):
            for h in range(H):
                z = torch.randn((N, d), generator=g, device=device, dtype=torch.float32)
                if name != "V":
                    z.addmm_(phi, U[h], alpha=alpha)
                t[b, h].copy_(z)
                del z
        out[name] = t
    gw = _generator(device, w.seed, 5)
    out["Wq"] = torch.randn((H, d, d), generator=gw, device=device) / math.sqrt(d)
    out["Wk"] = torch.randn((H, d, d), generator=gw, device=device) / math.sqrt(d)
    return out


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """A bf16 tensor's bit patterns as a host uint16 numpy array."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def sample_units(w: Workload, per_head: int, seed: int = 0) -> np.ndarray:
    """Seeded (b, h, i) query-tile sample per head, always with tiles 0 and nT-1."""
    rng = np.random.default_rng([seed, 99])
    units = []
    for b in range(w.B):
        for h in range(w.H):
            pick = {0, w.nT - 1}
            extra = rng.choice(w.nT, size=min(per_head, w.nT), replace=False)
            for i in extra:
                if len(pick) >= per_head:
                    break
                pick.add(int(i))
            units.extend((b, h, i) for i in sorted(pick))
    return np.asarray(units, dtype=np.int64)
