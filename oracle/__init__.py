"""fp64 CPU oracle for Veda's inference hot path (ctypes wrapper over veda_oracle.c).

TEST INFRASTRUCTURE ONLY: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  It shares
no code with the CUDA path (``tile_sparse_attention_b200``) and imports nothing
from it.

Source: "Veda: Scalable Video Diffusion via Distilled Sparse Attention" (project
page), sections "Attention Structure Distillation" (Teacher / Estimator /
Execution), "Principle 02 Head-Conditioned Tile Geometry" and "Theoretical
Rationale" 1-2.  Each C function cites the passage it follows.

Every function is pinned by ``tests/test_oracle_pins.py`` (brute force on tiny
grids, closed forms, invariants and a mutation check); none is "parity
unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "veda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libveda_oracle.so")

_lib = None


def build(src: str = _SRC, out: str = _LIB_PATH, extra_flags=()) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, strict IEEE: no -ffast-math)."""
    if os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src) and not extra_flags:
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
           "-ffp-contract=off", *extra_flags, src, "-o", out + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


_I64 = ctypes.c_int64
_P = ctypes.c_void_p


def _bind(lib):
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
    lib.oracle_tile_tokens.argtypes = [_I64, _I64, _I64, ctypes.c_int32, ctypes.c_int32,
                                       ctypes.c_int32, _P]
    lib.oracle_tripool.argtypes = [_I64] * 6 + [_P, _P, _P]
    lib.oracle_project.argtypes = [_I64] * 4 + [_P, _P, _P]
    lib.oracle_score.argtypes = [_I64] * 4 + [_P, _P, _P]
    lib.oracle_topk.argtypes = [_I64, _I64, _I64, _P, _P, _P]
    lib.oracle_sparse_attention.argtypes = ([_I64] * 6 + [_P, _I64, ctypes.c_double]
                                            + [_P] * 4 + [_I64, _P, _P, _P])
    lib.oracle_teacher.argtypes = [_I64] * 6 + [_P, ctypes.c_double, _P, _P, _P, _P]
    lib.oracle_tile_recall.argtypes = [_I64, _I64, _P, _P, _P]
    lib.oracle_tile_recall.restype = ctypes.c_double
    lib.oracle_distill_kl.argtypes = [_I64] * 4 + [_P] * 5 + [ctypes.c_double, _P, _P]
    lib.oracle_distill_kl.restype = ctypes.c_double
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_int32]
    lib.oracle_e4m3_decode.restype = ctypes.c_double
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
    lib.oracle_e4m3_encode.restype = ctypes.c_int32
    lib.oracle_quantize_e4m3.argtypes = [_I64, _I64, _P, _P, _P]
    lib.oracle_dequantize_e4m3.argtypes = [_I64, _I64, _P, _P, _P]
    return lib


def load(path: str | None = None):
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _bf16_bits(x) -> np.ndarray:
    """Accept a uint16 array of bf16 bit patterns (or a torch bf16 tensor)."""
    if hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        x = x.contiguous().view(__import__("torch").int16).numpy().view(np.uint16)
    a = np.ascontiguousarray(x)
    if a.dtype != np.uint16:
        raise TypeError("bf16 inputs are passed as uint16 bit patterns")
    return a


def _shapes(tile_shapes) -> np.ndarray:
    s = np.ascontiguousarray(np.asarray(tile_shapes, dtype=np.int32).reshape(-1, 3))
    return s


class Oracle:
    """Thin numpy-facing wrapper; ``lib`` may be a mutant build (tests only)."""

    def __init__(self, lib=None):
        self.lib = lib if lib is not None else load()

    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())

    def set_num_threads(self, n: int) -> None:
        self.lib.oracle_set_num_threads(int(n))

    def tile_tokens(self, grid, shape) -> np.ndarray:
        T, Hs, Ws = grid
        pt, ph, pw = (int(v) for v in shape)
        nT = (T // pt) * (Hs // ph) * (Ws // pw)
        out = np.empty((nT, pt * ph * pw), dtype=np.int64)
        self.lib.oracle_tile_tokens(T, Hs, Ws, pt, ph, pw, _ptr(out))
        return out

    def tripool(self, X, grid, tile_shapes) -> np.ndarray:
        X = _bf16_bits(X)
        B, H, N, d = X.shape
        T, Hs, Ws = grid
        s = _shapes(tile_shapes)
        Bt = int(np.prod(s[0]))
        nT = N // Bt
        out = np.empty((B, H, nT, 3, d), dtype=np.float64)
        self.lib.oracle_tripool(B, H, d, T, Hs, Ws, _ptr(s), _ptr(X), _ptr(out))
        return out

    def project(self, stats: np.ndarray, W) -> np.ndarray:
        stats = np.ascontiguousarray(stats, dtype=np.float64)
        W = np.ascontiguousarray(W, dtype=np.float32)
        B, H, nT, _, d = stats.shape
        out = np.empty_like(stats)
        self.lib.oracle_project(B, H, nT, d, _ptr(stats), _ptr(W), _ptr(out))
        return out

    def score(self, qt: np.ndarray, kt: np.ndarray) -> np.ndarray:
        qt = np.ascontiguousarray(qt, dtype=np.float64)
        kt = np.ascontiguousarray(kt, dtype=np.float64)
        B, H, nT, _, d = qt.shape
        S = np.empty((B, H, nT, nT), dtype=np.float64)
        self.lib.oracle_score(B, H, nT, d, _ptr(qt), _ptr(kt), _ptr(S))
        return S

    def topk(self, S: np.ndarray, k: int):
        S = np.ascontiguousarray(S, dtype=np.float64)
        nT = S.shape[-1]
        rows = S.size // nT
        mask = np.empty(S.shape, dtype=np.uint8)
        idx = np.empty(S.shape[:-1] + (k,), dtype=np.int32)
        self.lib.oracle_topk(rows, nT, k, _ptr(S), _ptr(mask), _ptr(idx))
        return mask, idx

    def mask_prep(self, Q, K, Wq, Wk, grid, tile_shapes, k):
        """TripPool -> projection -> score -> Top-k; returns a dict of every stage."""
        sq = self.tripool(Q, grid, tile_shapes)
        sk = self.tripool(K, grid, tile_shapes)
        qt = self.project(sq, Wq)
        kt = self.project(sk, Wk)
        S = self.score(qt, kt)
        mask, idx = self.topk(S, k)
        return dict(statsQ=sq, statsK=sk, qt=qt, kt=kt, S=S, mask=mask, idx=idx)

    def sparse_attention(self, Q, K, V, idx, grid, tile_shapes, scale, units=None):
        """Attention over the selected tiles for the given (b, h, i) units.

        Returns (O [nunits, Bt, d], lse [nunits, Bt], tokens [nunits, Bt]).
        ``units`` defaults to every (b, h, i).
        """
        Q, K, V = _bf16_bits(Q), _bf16_bits(K), _bf16_bits(V)
        B, H, N, d = Q.shape
        T, Hs, Ws = grid
        s = _shapes(tile_shapes)
        Bt = int(np.prod(s[0]))
        nT = N // Bt
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        k = idx.shape[-1]
        if units is None:
            units = np.array([(b, h, i) for b in range(B) for h in range(H) for i in range(nT)],
                             dtype=np.int64)
        units = np.ascontiguousarray(np.asarray(units, dtype=np.int64).reshape(-1, 3))
        nu = units.shape[0]
        O = np.empty((nu, Bt, d), dtype=np.float64)
        lse = np.empty((nu, Bt), dtype=np.float64)
        self.lib.oracle_sparse_attention(B, H, d, T, Hs, Ws, _ptr(s), k, float(scale),
                                         _ptr(Q), _ptr(K), _ptr(V), _ptr(idx), nu,
                                         _ptr(units), _ptr(O), _ptr(lse))
        toks = np.stack([self.tile_tokens(grid, s[int(h)])[int(i)] for (_, h, i) in units]) \
            if nu else np.empty((0, Bt), dtype=np.int64)
        return O, lse, toks

    def teacher(self, Q, K, grid, tile_shapes, scale):
        """Max-pooled dense attention teacher [B,H,nT,nT] and dense lse [B,H,N]."""
        Q, K = _bf16_bits(Q), _bf16_bits(K)
        B, H, N, d = Q.shape
        T, Hs, Ws = grid
        s = _shapes(tile_shapes)
        Bt = int(np.prod(s[0]))
        nT = N // Bt
        teacher = np.empty((B, H, nT, nT), dtype=np.float64)
        lse = np.empty((B, H, N), dtype=np.float64)
        self.lib.oracle_teacher(B, H, d, T, Hs, Ws, _ptr(s), float(scale), _ptr(Q), _ptr(K),
                                _ptr(teacher), _ptr(lse))
        return teacher, lse

    def tile_recall(self, idx_pred, idx_ref):
        """Per-row recall of idx_ref by idx_pred (same shape [..., k]) and the mean."""
        a = np.ascontiguousarray(idx_pred, dtype=np.int32)
        b = np.ascontiguousarray(idx_ref, dtype=np.int32)
        k = a.shape[-1]
        rows = a.size // k
        per = np.empty(a.shape[:-1], dtype=np.float64)
        mean = self.lib.oracle_tile_recall(rows, k, _ptr(a), _ptr(b), _ptr(per))
        return per, float(mean)

    def distill_kl(self, statsQ, statsK, Wq, Wk, teacher, tau, grads=True):
        """KL distillation loss (mean over rows) and, optionally, dL/dWq, dL/dWk."""
        sq = np.ascontiguousarray(statsQ, dtype=np.float64)
        sk = np.ascontiguousarray(statsK, dtype=np.float64)
        Wq = np.ascontiguousarray(Wq, dtype=np.float32)
        Wk = np.ascontiguousarray(Wk, dtype=np.float32)
        T = np.ascontiguousarray(teacher, dtype=np.float64)
        B, H, nT, _, d = sq.shape
        dWq = np.empty((H, d, d), dtype=np.float64) if grads else None
        dWk = np.empty((H, d, d), dtype=np.float64) if grads else None
        loss = self.lib.oracle_distill_kl(B, H, nT, d, _ptr(sq), _ptr(sk), _ptr(Wq), _ptr(Wk),
                                          _ptr(T), float(tau),
                                          _ptr(dWq) if grads else None,
                                          _ptr(dWk) if grads else None)
        return (float(loss), dWq, dWk) if grads else float(loss)

    def e4m3_decode(self, code: int) -> float:
        """Value of an fp8 E4M3 code (NaN for 0x7F / 0xFF)."""
        return float(self.lib.oracle_e4m3_decode(int(code)))

    def e4m3_encode(self, x: float) -> int:
        """Nearest E4M3 code of an fp32 value (ties to the even code, saturating)."""
        return int(self.lib.oracle_e4m3_encode(float(np.float32(x))))

    def quantize_e4m3(self, W):
        """Per-head fp8 E4M3 weights: codes uint8 [H, ...] and fp32 scale [H]."""
        W = np.ascontiguousarray(W, dtype=np.float32)
        H = W.shape[0]
        n = W.size // H
        codes = np.empty(W.shape, dtype=np.uint8)
        scale = np.empty((H,), dtype=np.float32)
        self.lib.oracle_quantize_e4m3(H, n, _ptr(W), _ptr(codes), _ptr(scale))
        return codes, scale

    def dequantize_e4m3(self, codes, scale):
        """fp32 weights e4m3(code) * scale[h]."""
        codes = np.ascontiguousarray(codes, dtype=np.uint8)
        scale = np.ascontiguousarray(scale, dtype=np.float32)
        H = codes.shape[0]
        n = codes.size // H
        W = np.empty(codes.shape, dtype=np.float32)
        self.lib.oracle_dequantize_e4m3(H, n, _ptr(codes), _ptr(scale), _ptr(W))
        return W

    def full_attention(self, Q, K, V, grid, tile_shapes, scale):
        """Dense softmax attention for every token: O [B,H,N,d] fp64, lse [B,H,N]."""
        Qb = _bf16_bits(Q)
        B, H, N, d = Qb.shape
        s = _shapes(tile_shapes)
        nT = N // int(np.prod(s[0]))
        idx = np.broadcast_to(np.arange(nT, dtype=np.int32), (B, H, nT, nT)).copy()
        O, lse, toks = self.sparse_attention(Q, K, V, idx, grid, tile_shapes, scale)
        return self._scatter(O, lse, toks, B, H, N, d, nT)

    @staticmethod
    def _scatter(O, lse, toks, B, H, N, d, nT):
        Of = np.empty((B, H, N, d))
        lf = np.empty((B, H, N))
        u = 0
        for b in range(B):
            for h in range(H):
                for i in range(nT):
                    Of[b, h, toks[u]] = O[u]
                    lf[b, h, toks[u]] = lse[u]
                    u += 1
        return Of, lf

    def tile_search(self, Q, K, V, Wq, Wk, grid, candidates, k, scale):
        """Head-aware tile search ("Head-Aware Tile Search"): for each candidate
        tiling (applied to every head) the squared Frobenius distance between
        full attention and the sparse layer output, per (candidate, b, h), and
        per head the candidate with the smallest distance summed over b."""
        Qb = _bf16_bits(Q)
        B, H, N, d = Qb.shape
        O_full, _ = self.full_attention(Q, K, V, grid, [candidates[0]] * H, scale)
        err = np.empty((len(candidates), B, H))
        for c, shape in enumerate(candidates):
            shapes = [tuple(shape)] * H
            r = self.mask_prep(Q, K, Wq, Wk, grid, shapes, k)
            nT = r["idx"].shape[2]
            O, lse, toks = self.sparse_attention(Q, K, V, r["idx"], grid, shapes, scale)
            Oc, _ = self._scatter(O, lse, toks, B, H, N, d, nT)
            err[c] = ((O_full - Oc) ** 2).sum(axis=(2, 3))
        best = np.argmin(err.sum(axis=1), axis=0).astype(np.int32)  # first index on ties
        return err, best, O_full
