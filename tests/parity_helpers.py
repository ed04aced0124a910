"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs, and compare by the parity rules.

Parity rules (tolerances derived from the arithmetic):
* TripPool max/min: bit-exact (a max of bf16 values is exact in fp32);
  avg: |gpu - oracle| <= (Bt - 1) * 2^-24 * mean|x| + 2^-24 * |avg|, the error
  bound of an fp32 sum of Bt terms followed by an exact division by 2^m.
* scores: |gpu - oracle| <= 9e-5 * (|stats_q| |W_q|) . (|stats_k| |W_k|)^T: each
  of the two projections is a three-term TF32 product with fp32 accumulation
  of d terms (d * 2^-24 + 3 * 2^-21 relative to the absolute terms), the score
  a three-term TF32 product (3 * 2^-21) accumulated over 9d terms in fp32:
  (2d + 9d + 4) * 2^-24 + 9 * 2^-21 = 8.84e-5 at d = 128, worst case on the
  absolute terms.
* mask rows: bit-exact wherever the oracle's k-th and (k+1)-th scores differ
  by more than 1e-3 relative; in other rows the GPU row must hold exactly k
  tiles and every tile whose oracle score clears s_(k) by that margin.
* attention output: max-abs <= 2e-2 and mean-abs <= 5e-3 against the fp64
  oracle on the same index list (bf16 inputs, fp32 accumulation, bf16 P);
  lse: abs error <= 2e-3.
"""
from __future__ import annotations

import numpy as np
import torch

import workloads
from oracle import Oracle

O_MAX_ABS = 2e-2
O_MEAN_ABS = 5e-3
LSE_ABS = 2e-3
SCORE_GAMMA = 9e-5
GAP_REL = 1e-3


def to_host_bits(t: torch.Tensor) -> np.ndarray:
    return workloads.bf16_bits(t)


def slice_heads(bits: np.ndarray, heads) -> np.ndarray:
    return np.ascontiguousarray(bits[:, heads])


def gpu_mask_prep(vb, prob, Q, K, Wq, Wk):
    """Runs the three mask-prep entry points; returns dict of torch tensors."""
    B, H, nT, d = prob.B, prob.H, prob.nT, prob.d
    dev = Q.device
    statsQ = torch.empty((B, H, nT, 3, d), dtype=torch.float32, device=dev)
    statsK = torch.empty_like(statsQ)
    vb.veda_tripool(prob, Q, K, statsQ, statsK)
    S = torch.empty((B, H, nT, nT), dtype=torch.float32, device=dev)
    ws = vb.alloc_workspace(prob, dev)
    vb.veda_tile_score(prob, statsQ, statsK, Wq, Wk, S, ws)
    mask = torch.empty((B, H, nT, nT), dtype=torch.uint8, device=dev)
    idx = torch.empty((B, H, nT, prob.k), dtype=torch.int32, device=dev)
    vb.veda_topk_mask(prob, S, mask, idx)
    torch.cuda.synchronize()
    assert vb.veda_get_status(ws) == 0
    return dict(statsQ=statsQ, statsK=statsK, S=S, mask=mask, idx=idx)


def check_stats(gpu_stats: np.ndarray, ora_stats: np.ndarray, Bt: int, X_f64_abs_mean=None):
    g = gpu_stats.astype(np.float64)
    np.testing.assert_array_equal(g[..., 1:, :], ora_stats[..., 1:, :])
    u = 2.0 ** -24
    # mean |x| over the tile is at most max(|max|, |min|)
    mag = np.maximum(np.abs(ora_stats[..., 1, :]), np.abs(ora_stats[..., 2, :]))
    bound = (Bt - 1) * u * mag + u * np.abs(ora_stats[..., 0, :]) + 1e-30
    err = np.abs(g[..., 0, :] - ora_stats[..., 0, :])
    assert np.all(err <= bound), f"avg error {err.max()} above bound"


def score_bound(ora, Wq, Wk):
    """Per-element fp32 error bound of the score from the oracle's stats."""
    aq = np.einsum("bhjsc,hce->bhjse", np.abs(ora["statsQ"]), np.abs(Wq.astype(np.float64)))
    ak = np.einsum("bhjsc,hce->bhjse", np.abs(ora["statsK"]), np.abs(Wk.astype(np.float64)))
    return SCORE_GAMMA * np.einsum("bhise,bhjse->bhij", aq, ak)


def exempt_rows(S_ora: np.ndarray, k: int) -> np.ndarray:
    """Rows where the k-th and (k+1)-th oracle scores are within 1e-3 relative."""
    nT = S_ora.shape[-1]
    flat = S_ora.reshape(-1, nT)
    if k >= nT:
        return np.zeros(flat.shape[0], dtype=bool).reshape(S_ora.shape[:-1])
    part = -np.sort(-flat, axis=1)
    sk, sk1 = part[:, k - 1], part[:, k]
    gap = sk - sk1
    return (gap <= GAP_REL * np.maximum(np.abs(sk), np.abs(sk1))).reshape(S_ora.shape[:-1])


# One line per mask comparison of the session: (label, rows, exempt rows,
# rows identical to the oracle's).  tests/conftest.py prints it at the end.
MASK_REPORT = []

# Ceilings and floors, measured on the seeded inputs (CPU draws) with a margin.
# The 1e-3 gap rule exempts many rows, because neighbouring tiles have close
# scores: 23-29% at 480P / 720P, 59% at long video, 2-84% across the sweep (the
# most at T = 64, s <= 80%).  What bounds the claim instead is the floor on rows
# identical to the oracle's, exempt or not: an fp32 score agrees with the fp64
# one on >= 99.86% of the rows at every size (the GPU's three-term TF32 score is
# as accurate as fp32), so at least 99% must be identical.
MAX_EXEMPT_FRAC = 0.9
MIN_EXACT_FRAC = 0.99


def check_masks(mask_gpu: np.ndarray, idx_gpu: np.ndarray, S_ora: np.ndarray, mask_ora, idx_ora,
                k: int, label: str = "", max_exempt_frac: float = MAX_EXEMPT_FRAC,
                min_exact_frac: float = MIN_EXACT_FRAC):
    """Bit-exact on non-exempt rows; exempt rows: k ones and every clear winner kept.

    Also bounds how much the gap rule exempts (at most ``max_exempt_frac`` of
    the rows) and how many rows, exempt or not, must equal the oracle's row
    exactly (at least ``min_exact_frac``); returns the exempt-row count."""
    ex = exempt_rows(S_ora, k)
    nT = S_ora.shape[-1]
    assert np.all(mask_gpu.sum(-1) == k)
    assert np.all(np.diff(idx_gpu, axis=-1) > 0)
    ok = ~ex
    np.testing.assert_array_equal(mask_gpu[ok], mask_ora[ok])
    np.testing.assert_array_equal(idx_gpu[ok], idx_ora[ok])
    flat_S = S_ora.reshape(-1, nT)
    flat_m = mask_gpu.reshape(-1, nT)
    for r in np.nonzero(ex.reshape(-1))[0]:
        sk = -np.sort(-flat_S[r])[k - 1]
        clear = flat_S[r] > sk + GAP_REL * abs(sk)
        assert np.all(flat_m[r][clear] == 1)
    rows = int(ex.size)
    n_ex = int(ex.sum())
    n_exact = int(np.all(mask_gpu.reshape(-1, nT) == np.asarray(mask_ora).reshape(-1, nT),
                         axis=1).sum())
    MASK_REPORT.append((label or f"nT={nT} k={k}", rows, n_ex, n_exact))
    assert n_ex <= max_exempt_frac * rows, f"{label}: {n_ex} of {rows} rows exempt"
    assert n_exact >= min_exact_frac * rows, f"{label}: only {n_exact} of {rows} rows exact"
    return n_ex


def check_attention(O_gpu_bits: np.ndarray, lse_gpu: np.ndarray, units, O_ora, lse_ora, toks):
    """O_gpu_bits [B,H,N,d] uint16; units rows (b,h,i); O_ora [nu,Bt,d]."""
    errs = []
    lerr = []
    for u, (b, h, i) in enumerate(units):
        g = (O_gpu_bits[b, h][toks[u]].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        errs.append(np.abs(g - O_ora[u]))
        if lse_gpu is not None:
            lerr.append(np.abs(lse_gpu[b, h][toks[u]].astype(np.float64) - lse_ora[u]))
    e = np.concatenate([x.ravel() for x in errs])
    assert e.max() <= O_MAX_ABS, f"O max-abs error {e.max()}"
    assert e.mean() <= O_MEAN_ABS, f"O mean-abs error {e.mean()}"
    if lerr:
        le = np.concatenate(lerr)
        assert le.max() <= LSE_ABS, f"lse max-abs error {le.max()}"
    return float(e.max()), float(e.mean())


def oracle_mask_prep_heads(oracle: Oracle, w, Qb, Kb, Wq, Wk, heads):
    """Oracle mask prep restricted to a subset of heads (heads are independent)."""
    shapes = [w.tile_shapes[h] for h in heads]
    return oracle.mask_prep(slice_heads(Qb, heads), slice_heads(Kb, heads), Wq[heads], Wk[heads],
                            w.grid, shapes, w.k)
