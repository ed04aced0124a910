"""Independent numpy brute force for the Veda hot path (pins the C oracle).

Written separately from the C oracle and in a different style: tiles come from
reshaping the token grid, attention uses an explicit N x N token mask, Top-k is
a full stable sort.  Tiny inputs only.

Source: "Veda: Scalable Video Diffusion via Distilled Sparse Attention"
(project page) -- "Attention Structure Distillation" (Teacher, Estimator,
Execution), "Principle 01 Full-Attention Structure Distillation",
"Principle 02 Head-Conditioned Tile Geometry", "Theoretical Rationale" 1
(Softmax Geometry), 2 (Tile Statistics) and 4 (Distillation Objective).
"""
from __future__ import annotations

import numpy as np


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def tile_view(X: np.ndarray, grid, shape) -> np.ndarray:
    """[N, ...] token-major array -> [nT, Bt, ...] by splitting the T x Hs x Ws grid."""
    T, Hs, Ws = grid
    pt, ph, pw = shape
    rest = X.shape[1:]
    Y = X.reshape((T // pt, pt, Hs // ph, ph, Ws // pw, pw) + rest)
    nd = len(rest)
    Y = Y.transpose((0, 2, 4, 1, 3, 5) + tuple(range(6, 6 + nd)))
    return Y.reshape((-1, pt * ph * pw) + rest)


def token_of_tile_row(grid, shape) -> np.ndarray:
    T, Hs, Ws = grid
    return tile_view(np.arange(T * Hs * Ws), grid, shape)


def tripool(X: np.ndarray, grid, shapes) -> np.ndarray:
    """X [B,H,N,d] fp64 -> stats [B,H,nT,3,d] (avg, max, min)."""
    B, H, N, d = X.shape
    out = []
    for b in range(B):
        per_h = []
        for h in range(H):
            tiles = tile_view(X[b, h], grid, shapes[h])
            per_h.append(np.stack([tiles.mean(1), tiles.max(1), tiles.min(1)], axis=1))
        out.append(np.stack(per_h))
    return np.stack(out)


def scores(statsQ, statsK, Wq, Wk) -> np.ndarray:
    qt = np.einsum("bhjsc,hce->bhjse", statsQ, Wq.astype(np.float64))
    kt = np.einsum("bhjsc,hce->bhjse", statsK, Wk.astype(np.float64))
    return np.einsum("bhise,bhjse->bhij", qt, kt)


def topk(S: np.ndarray, k: int):
    nT = S.shape[-1]
    flat = S.reshape(-1, nT)
    idx = np.empty((flat.shape[0], k), dtype=np.int32)
    mask = np.zeros(flat.shape, dtype=np.uint8)
    js = np.arange(nT)
    for r, row in enumerate(flat):
        order = np.lexsort((js, -row))  # primary: -score, secondary: index
        keep = np.sort(order[:k])
        idx[r] = keep
        mask[r, keep] = 1
    return mask.reshape(S.shape), idx.reshape(S.shape[:-1] + (k,))


def token_mask(tile_mask: np.ndarray, grid, shape) -> np.ndarray:
    """[nT, nT] tile mask -> [N, N] token mask for one head."""
    tok = token_of_tile_row(grid, shape)
    N = tok.size
    tile_of = np.empty(N, dtype=np.int64)
    for j, row in enumerate(tok):
        tile_of[row] = j
    return tile_mask[np.ix_(tile_of, tile_of)].astype(bool)


def masked_attention(Q, K, V, allowed, scale):
    """Q,K,V [N,d] fp64, allowed [N,N] bool -> O [N,d], lse [N]."""
    logits = scale * Q @ K.T
    logits = np.where(allowed, logits, -np.inf)
    m = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - m)
    z = e.sum(axis=1, keepdims=True)
    return (e / z) @ V, (m + np.log(z))[:, 0]


def sparse_attention(Q, K, V, tile_mask, grid, shapes, scale):
    B, H, N, d = Q.shape
    O = np.empty_like(Q)
    lse = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            allowed = token_mask(tile_mask[b, h], grid, shapes[h])
            O[b, h], lse[b, h] = masked_attention(Q[b, h], K[b, h], V[b, h], allowed, scale)
    return O, lse


def dense_probs(Q, K, scale):
    logits = scale * Q @ K.T
    m = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - m)
    return e / e.sum(axis=1, keepdims=True)


def teacher(Q, K, grid, shapes, scale):
    """Tile-wise max of the dense probability matrix, [B,H,nT,nT]."""
    B, H, N, d = Q.shape
    out = []
    for b in range(B):
        per_h = []
        for h in range(H):
            P = dense_probs(Q[b, h], K[b, h], scale)
            tok = token_of_tile_row(grid, shapes[h])
            per_h.append(P[tok[:, :, None, None], tok[None, None, :, :]].max(axis=(1, 3)))
        out.append(np.stack(per_h))
    return np.stack(out)


def distill_kl(statsQ, statsK, Wq, Wk, teacher, tau) -> float:
    """Distillation loss from its definition ("Theoretical Rationale" 4).

    Per query-tile row: the target distribution is the teacher row divided by
    its sum, the estimator distribution is softmax(S / tau) over the key tiles,
    and the row's term is KL(target || estimator) = sum_j t_j log(t_j / p_j),
    evaluated by scipy's relative entropy (0 where t_j = 0).  The loss is the
    mean of the row terms over all B*H*nT rows.
    """
    from scipy.special import rel_entr, softmax

    S = scores(statsQ, statsK, Wq, Wk)
    nT = S.shape[-1]
    pred = softmax(S.reshape(-1, nT) / tau, axis=1)
    tgt = teacher.reshape(-1, nT) / teacher.reshape(-1, nT).sum(axis=1, keepdims=True)
    rows = rel_entr(tgt, pred).sum(axis=1)
    return float(rows.mean())
