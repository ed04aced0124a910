"""veda_tile_score_noalloc: the tile score for callers that cannot allocate
device memory (they only receive device pointers for inputs and outputs, or may
not call cudaMalloc on their hot path).  It must give what veda_tile_score
gives, call after call, while its scratch lives in a fixed array inside the
library that every call reuses.

This file is collected last on purpose: it shares the library's one scratch
array, and it must pass both alone in a fresh process and after every other
test."""
import ctypes

import numpy as np
import pytest
import torch

import workloads


def _problem(vb, w):
    return vb.Problem.from_workload(w)


def test_noalloc_rejects_problems_beyond_its_scratch():
    from tile_sparse_attention_b200 import build as b
    import tile_sparse_attention_b200 as vb
    b.build()
    lib = vb.load_library()
    limit = vb.veda_noalloc_scratch_bytes()
    assert limit == 64 << 20
    w = workloads.p720()  # 256 + 2*40*600*384*4 bytes > 64 MiB
    prob = _problem(vb, w)
    p = ctypes.c_void_p(0x10000)
    code = lib.veda_tile_score_noalloc(ctypes.byref(prob.c), p, p, p, p, p, None)
    assert code == 3  # VEDA_ERR_UNSUPPORTED, nothing launched
    assert b"scratch" in lib.veda_last_error()


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tile_sparse_attention_b200 as vb
    vb.load_library()
    w = workloads.p480()
    t = {n: v.cuda() for n, v in workloads.generate(w, device="cpu").items()}
    prob = _problem(vb, w)
    B, H, nT, d = w.B, w.H, w.nT, w.d
    statsQ = torch.empty((B, H, nT, 3, d), dtype=torch.float32, device="cuda")
    statsK = torch.empty_like(statsQ)
    vb.veda_tripool(prob, t["Q"], t["K"], statsQ, statsK)
    ref = torch.empty((B, H, nT, nT), dtype=torch.float32, device="cuda")
    ws = vb.alloc_workspace(prob)
    vb.veda_tile_score(prob, statsQ, statsK, t["Wq"], t["Wk"], ref, ws)
    # a second problem in between leaves different contents in the shared scratch
    w2 = workloads.custom("other", 1, 2, 128, (4, 16, 32), [(2, 8, 8)], 4, seed=5)
    t2 = {n: v.cuda() for n, v in workloads.generate(w2, device="cpu").items()}
    p2 = _problem(vb, w2)
    s2q = torch.empty((1, 2, w2.nT, 3, 128), dtype=torch.float32, device="cuda")
    s2k = torch.empty_like(s2q)
    vb.veda_tripool(p2, t2["Q"], t2["K"], s2q, s2k)
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        vb.veda_tile_score_noalloc(prob, statsQ, statsK, t["Wq"], t["Wk"], out)
        torch.cuda.synchronize()
        # same kernels, same order of operations: the scores agree exactly, well
        # inside the fp32 score tolerance of the parity tests
        assert torch.equal(out, ref), f"call {call}: max diff {(out - ref).abs().max().item()}"
        other = torch.empty((1, 2, w2.nT, w2.nT), dtype=torch.float32, device="cuda")
        vb.veda_tile_score_noalloc(p2, s2q, s2k, t2["Wq"], t2["Wk"], other)
        torch.cuda.synchronize()
        other_ref = torch.empty_like(other)
        ws2 = vb.alloc_workspace(p2)
        vb.veda_tile_score(p2, s2q, s2k, t2["Wq"], t2["Wk"], other_ref, ws2)
        torch.cuda.synchronize()
        assert torch.equal(other, other_ref)
    assert np.isfinite(ref.cpu().numpy()).all()
