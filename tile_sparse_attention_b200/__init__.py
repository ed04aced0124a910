"""Python binding of the B200 tile-sparse attention library (``libveda.so``).

Argument marshalling only: every step of the hot path runs in the library's
CUDA kernels.  PyTorch provides device memory and the current CUDA stream.
The functions mirror the C ABI in ``include/veda.h`` one to one and take
caller-allocated torch tensors.  There is no CPU fallback: if the library is
missing, every call raises.

Method: "Veda: Scalable Video Diffusion via Distilled Sparse Attention"
(project page), "Attention Structure Distillation" (Estimator: TripPool and
head-specific projections; Execution: head-aware Top-k and the tile-skipping
kernel).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libveda.so")

VEDA_STATUS_BYTES = 256
STATUS_NAMES = {0: "VEDA_OK", 1: "VEDA_ERR_INVALID_ARG", 2: "VEDA_ERR_SHAPE",
                3: "VEDA_ERR_UNSUPPORTED", 4: "VEDA_ERR_ALIGN", 5: "VEDA_ERR_CUDA",
                6: "VEDA_ERR_TIMEOUT", 7: "VEDA_ERR_BAD_INDEX"}


class VedaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


class veda_problem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("H", ctypes.c_int64), ("d", ctypes.c_int64),
                ("T", ctypes.c_int64), ("Hs", ctypes.c_int64), ("Ws", ctypes.c_int64),
                ("tile_shapes", ctypes.POINTER(ctypes.c_int32)), ("k", ctypes.c_int64),
                ("scale", ctypes.c_float)]


_lib = None
_P = ctypes.c_void_p


def load_library(path: str = LIB_PATH):
    """Load ``libveda.so`` (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libveda.so not found at {path}: build it with "
                           "`python -m tile_sparse_attention_b200.build`")
    lib = ctypes.CDLL(path)
    st = ctypes.c_int
    lib.veda_version.restype = ctypes.c_int
    lib.veda_last_error.restype = ctypes.c_char_p
    lib.veda_workspace_size.argtypes = [ctypes.POINTER(veda_problem), ctypes.POINTER(ctypes.c_size_t)]
    lib.veda_workspace_size.restype = st
    lib.veda_tripool.argtypes = [ctypes.POINTER(veda_problem), _P, _P, _P, _P, _P]
    lib.veda_tripool.restype = st
    lib.veda_tile_score.argtypes = [ctypes.POINTER(veda_problem)] + [_P] * 7
    lib.veda_tile_score.restype = st
    lib.veda_topk_mask.argtypes = [ctypes.POINTER(veda_problem), _P, _P, _P, _P]
    lib.veda_topk_mask.restype = st
    lib.veda_forward_host.argtypes = ([ctypes.POINTER(veda_problem)] + [_P] * 15
                                      + [ctypes.c_int32, _P])
    lib.veda_forward_host.restype = st
    lib.veda_quantize_fp8.argtypes = [_P, ctypes.c_int64, ctypes.c_int64, _P, _P, _P]
    lib.veda_quantize_fp8.restype = st
    lib.veda_dequantize_fp8.argtypes = [_P, _P, ctypes.c_int64, ctypes.c_int64, _P, _P]
    lib.veda_dequantize_fp8.restype = st
    lib.veda_mask_fused.argtypes = [ctypes.POINTER(veda_problem)] + [_P] * 8
    lib.veda_mask_fused.restype = st
    lib.veda_sparse_attn.argtypes = [ctypes.POINTER(veda_problem)] + [_P] * 8
    lib.veda_sparse_attn.restype = st
    lib.veda_forward.argtypes = [ctypes.POINTER(veda_problem)] + [_P] * 11
    lib.veda_forward.restype = st
    lib.veda_get_status.argtypes = [_P, _P, ctypes.POINTER(ctypes.c_int32)]
    lib.veda_get_status.restype = st
    lib.veda_teacher.argtypes = [ctypes.POINTER(veda_problem)] + [_P] * 8
    lib.veda_teacher.restype = st
    lib.veda_tile_recall.argtypes = [ctypes.POINTER(veda_problem)] + [_P] * 6
    lib.veda_tile_recall.restype = st
    lib.veda_distill_workspace_size.argtypes = [ctypes.POINTER(veda_problem),
                                                ctypes.POINTER(ctypes.c_size_t)]
    lib.veda_distill_workspace_size.restype = st
    lib.veda_distill_kl.argtypes = ([ctypes.POINTER(veda_problem)] + [_P] * 6 + [ctypes.c_float]
                                    + [_P] * 4 + [_P])
    lib.veda_distill_kl.restype = st
    lib.veda_tile_search.argtypes = ([ctypes.POINTER(veda_problem), _P, ctypes.c_int32]
                                     + [_P] * 11)
    lib.veda_tile_search.restype = st
    lib.veda_noalloc_scratch_bytes.restype = ctypes.c_size_t
    lib.veda_tile_score_noalloc.argtypes = [ctypes.POINTER(veda_problem)] + [_P] * 6
    lib.veda_tile_score_noalloc.restype = st
    lib.veda_noalloc_get_status.argtypes = [_P, ctypes.POINTER(ctypes.c_int32)]
    lib.veda_noalloc_get_status.restype = st
    _lib = lib
    return lib


class Problem:
    """Owns a ``veda_problem`` and its host tile-shape table."""

    def __init__(self, B: int, H: int, d: int, grid: Sequence[int], tile_shapes, k: int,
                 scale: float = 0.0):
        T, Hs, Ws = (int(v) for v in grid)
        shapes = [tuple(int(v) for v in s) for s in tile_shapes]
        if len(shapes) == 1 and H > 1:
            shapes = shapes * H
        flat = [v for s in shapes for v in s]
        self._shapes = (ctypes.c_int32 * len(flat))(*flat)
        self.c = veda_problem(int(B), int(H), int(d), T, Hs, Ws,
                              ctypes.cast(self._shapes, ctypes.POINTER(ctypes.c_int32)), int(k),
                              float(scale))
        self.B, self.H, self.d, self.grid, self.k = int(B), int(H), int(d), (T, Hs, Ws), int(k)
        self.N = T * Hs * Ws
        self.Bt = shapes[0][0] * shapes[0][1] * shapes[0][2] if shapes else 0
        self.nT = self.N // self.Bt if self.Bt else 0

    @classmethod
    def from_workload(cls, w, k: Optional[int] = None, scale: float = 0.0):
        return cls(w.B, w.H, w.d, w.grid, w.tile_shapes, w.k if k is None else k, scale)


def _check(code: int):
    if code != 0:
        raise VedaError(code, load_library().veda_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to the library must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _expect(t, dtype, name):
    if t is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def version() -> int:
    return int(load_library().veda_version())


def veda_workspace_size(problem: Problem) -> int:
    n = ctypes.c_size_t(0)
    _check(load_library().veda_workspace_size(ctypes.byref(problem.c), ctypes.byref(n)))
    return int(n.value)


def veda_tripool(problem: Problem, Q, K, statsQ, statsK, stream=None) -> None:
    for t, n in ((Q, "Q"), (K, "K")):
        _expect(t, torch.bfloat16, n)
    for t, n in ((statsQ, "statsQ"), (statsK, "statsK")):
        _expect(t, torch.float32, n)
    _check(load_library().veda_tripool(ctypes.byref(problem.c), _ptr(Q), _ptr(K), _ptr(statsQ),
                                       _ptr(statsK), _stream(stream)))


def veda_tile_score(problem: Problem, statsQ, statsK, Wq, Wk, S, ws, stream=None) -> None:
    for t, n in ((statsQ, "statsQ"), (statsK, "statsK"), (Wq, "Wq"), (Wk, "Wk"), (S, "S")):
        _expect(t, torch.float32, n)
    _check(load_library().veda_tile_score(ctypes.byref(problem.c), _ptr(statsQ), _ptr(statsK),
                                          _ptr(Wq), _ptr(Wk), _ptr(S), _ptr(ws), _stream(stream)))


def veda_topk_mask(problem: Problem, S, mask, idx, stream=None) -> None:
    _expect(S, torch.float32, "S")
    _expect(mask, torch.uint8, "mask")
    _expect(idx, torch.int32, "idx")
    _check(load_library().veda_topk_mask(ctypes.byref(problem.c), _ptr(S), _ptr(mask), _ptr(idx),
                                         _stream(stream)))


def _host_ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if t.is_cuda:
        raise ValueError("host buffers must live in host memory")
    if not t.is_contiguous():
        raise ValueError("host buffers must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def veda_forward_host(problem: Problem, hQ, hK, hV, hWq, hWk, hO, hlse, dQ, dK, dV, dWq, dWk, dO,
                      dlse, ws, head_chunk: int = 0, stream=None) -> None:
    """The layer from host buffers (pinned for overlap), pipelined over head chunks."""
    for t, n in ((hQ, "hQ"), (hK, "hK"), (hV, "hV"), (hO, "hO"), (dQ, "dQ"), (dK, "dK"),
                 (dV, "dV"), (dO, "dO")):
        _expect(t, torch.bfloat16, n)
    for t, n in ((hWq, "hWq"), (hWk, "hWk"), (dWq, "dWq"), (dWk, "dWk")):
        _expect(t, torch.float32, n)
    _check(load_library().veda_forward_host(
        ctypes.byref(problem.c), _host_ptr(hQ), _host_ptr(hK), _host_ptr(hV), _host_ptr(hWq),
        _host_ptr(hWk), _host_ptr(hO), _host_ptr(hlse), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dWq),
        _ptr(dWk), _ptr(dO), _ptr(dlse), _ptr(ws), int(head_chunk), _stream(stream)))


def veda_quantize_fp8(W, W8, scale, stream=None) -> None:
    """W fp32 [H, d, d] -> W8 uint8 [H, d, d] (E4M3 codes), scale fp32 [H]."""
    _expect(W, torch.float32, "W")
    _expect(W8, torch.uint8, "W8")
    _expect(scale, torch.float32, "scale")
    H, d = W.shape[0], W.shape[-1]
    _check(load_library().veda_quantize_fp8(_ptr(W), H, d, _ptr(W8), _ptr(scale), _stream(stream)))


def veda_dequantize_fp8(W8, scale, W, stream=None) -> None:
    """W8 uint8 [H, d, d], scale fp32 [H] -> W fp32 [H, d, d]."""
    _expect(W8, torch.uint8, "W8")
    _expect(scale, torch.float32, "scale")
    _expect(W, torch.float32, "W")
    H, d = W8.shape[0], W8.shape[-1]
    _check(load_library().veda_dequantize_fp8(_ptr(W8), _ptr(scale), H, d, _ptr(W),
                                              _stream(stream)))


def veda_mask_fused(problem: Problem, statsQ, statsK, Wq, Wk, mask, idx, ws, stream=None) -> None:
    for t, n in ((statsQ, "statsQ"), (statsK, "statsK"), (Wq, "Wq"), (Wk, "Wk")):
        _expect(t, torch.float32, n)
    _expect(idx, torch.int32, "idx")
    if mask is not None:
        _expect(mask, torch.uint8, "mask")
    _check(load_library().veda_mask_fused(ctypes.byref(problem.c), _ptr(statsQ), _ptr(statsK),
                                          _ptr(Wq), _ptr(Wk), _ptr(mask), _ptr(idx), _ptr(ws),
                                          _stream(stream)))


def veda_sparse_attn(problem: Problem, Q, K, V, idx, O, lse, ws, stream=None) -> None:
    for t, n in ((Q, "Q"), (K, "K"), (V, "V"), (O, "O")):
        _expect(t, torch.bfloat16, n)
    _expect(idx, torch.int32, "idx")
    _expect(lse, torch.float32, "lse")
    _check(load_library().veda_sparse_attn(ctypes.byref(problem.c), _ptr(Q), _ptr(K), _ptr(V),
                                           _ptr(idx), _ptr(O), _ptr(lse), _ptr(ws),
                                           _stream(stream)))


def veda_forward(problem: Problem, Q, K, V, Wq, Wk, O, lse, idx_out, mask_out, ws,
                 stream=None) -> None:
    for t, n in ((Q, "Q"), (K, "K"), (V, "V"), (O, "O")):
        _expect(t, torch.bfloat16, n)
    for t, n in ((Wq, "Wq"), (Wk, "Wk"), (lse, "lse")):
        _expect(t, torch.float32, n)
    _expect(idx_out, torch.int32, "idx_out")
    _expect(mask_out, torch.uint8, "mask_out")
    _check(load_library().veda_forward(ctypes.byref(problem.c), _ptr(Q), _ptr(K), _ptr(V),
                                       _ptr(Wq), _ptr(Wk), _ptr(O), _ptr(lse), _ptr(idx_out),
                                       _ptr(mask_out), _ptr(ws), _stream(stream)))


def veda_teacher(problem: Problem, Q, K, V, O_dense, lse_dense, teacher, ws, stream=None) -> None:
    for t, n in ((Q, "Q"), (K, "K"), (V, "V"), (O_dense, "O_dense")):
        _expect(t, torch.bfloat16, n)
    for t, n in ((lse_dense, "lse_dense"), (teacher, "teacher")):
        _expect(t, torch.float32, n)
    _check(load_library().veda_teacher(ctypes.byref(problem.c), _ptr(Q), _ptr(K), _ptr(V),
                                       _ptr(O_dense), _ptr(lse_dense), _ptr(teacher), _ptr(ws),
                                       _stream(stream)))


def veda_tile_recall(problem: Problem, idx_pred, idx_ref, recall_rows, recall_mean, ws,
                     stream=None) -> None:
    _expect(idx_pred, torch.int32, "idx_pred")
    _expect(idx_ref, torch.int32, "idx_ref")
    _expect(recall_rows, torch.float32, "recall_rows")
    _expect(recall_mean, torch.float64, "recall_mean")
    _check(load_library().veda_tile_recall(ctypes.byref(problem.c), _ptr(idx_pred), _ptr(idx_ref),
                                           _ptr(recall_rows), _ptr(recall_mean), _ptr(ws),
                                           _stream(stream)))


def veda_distill_workspace_size(problem: Problem) -> int:
    n = ctypes.c_size_t(0)
    _check(load_library().veda_distill_workspace_size(ctypes.byref(problem.c), ctypes.byref(n)))
    return int(n.value)


def veda_distill_kl(problem: Problem, statsQ, statsK, Wq, Wk, S, teacher, tau, loss, dWq, dWk,
                    ws, stream=None) -> None:
    for t, n in ((statsQ, "statsQ"), (statsK, "statsK"), (Wq, "Wq"), (Wk, "Wk"), (S, "S"),
                 (teacher, "teacher"), (dWq, "dWq"), (dWk, "dWk")):
        _expect(t, torch.float32, n)
    _expect(loss, torch.float64, "loss")
    _check(load_library().veda_distill_kl(ctypes.byref(problem.c), _ptr(statsQ), _ptr(statsK),
                                          _ptr(Wq), _ptr(Wk), _ptr(S), _ptr(teacher),
                                          ctypes.c_float(tau), _ptr(loss), _ptr(dWq), _ptr(dWk),
                                          _ptr(ws), _stream(stream)))


def veda_tile_search(problem: Problem, candidates, Q, K, V, Wq, Wk, O_dense, O_cand, err, best,
                     ws, stream=None) -> None:
    for t, n in ((Q, "Q"), (K, "K"), (V, "V"), (O_dense, "O_dense"), (O_cand, "O_cand")):
        _expect(t, torch.bfloat16, n)
    _expect(err, torch.float64, "err")
    _expect(best, torch.int32, "best")
    flat = [int(v) for c in candidates for v in c]
    arr = (ctypes.c_int32 * len(flat))(*flat)
    _check(load_library().veda_tile_search(ctypes.byref(problem.c), ctypes.cast(arr, _P),
                                           len(candidates), _ptr(Q), _ptr(K), _ptr(V), _ptr(Wq),
                                           _ptr(Wk), _ptr(O_dense), _ptr(O_cand), _ptr(err),
                                           _ptr(best), _ptr(ws), _stream(stream)))


def veda_get_status(ws, stream=None) -> int:
    out = ctypes.c_int32(0)
    _check(load_library().veda_get_status(_ptr(ws), _stream(stream), ctypes.byref(out)))
    return int(out.value)


def veda_tile_score_noalloc(problem: Problem, statsQ, statsK, Wq, Wk, S, stream=None) -> None:
    """veda_tile_score without a workspace, for callers that cannot allocate device
    memory: the library's fixed scratch array (veda_noalloc_scratch_bytes()) is
    used instead.  Calls that overlap on the GPU race on that array."""
    for t, n in ((statsQ, "statsQ"), (statsK, "statsK"), (Wq, "Wq"), (Wk, "Wk"), (S, "S")):
        _expect(t, torch.float32, n)
    _check(load_library().veda_tile_score_noalloc(ctypes.byref(problem.c), _ptr(statsQ),
                                                  _ptr(statsK), _ptr(Wq), _ptr(Wk), _ptr(S),
                                                  _stream(stream)))


def veda_noalloc_scratch_bytes() -> int:
    return int(load_library().veda_noalloc_scratch_bytes())


def veda_noalloc_get_status(stream=None) -> int:
    """Device status word of the last veda_tile_score_noalloc call on the current
    device (0, or VEDA_ERR_TIMEOUT when a bounded wait gave up); waits for the
    stream first."""
    out = ctypes.c_int32(0)
    _check(load_library().veda_noalloc_get_status(_stream(stream), ctypes.byref(out)))
    return int(out.value)


def alloc_workspace(problem: Problem, device="cuda") -> torch.Tensor:
    """A device workspace of veda_workspace_size() bytes (torch-owned memory)."""
    return torch.empty(veda_workspace_size(problem), dtype=torch.uint8, device=device)
