"""veda_tile_score_noalloc: the tile score for callers that cannot allocate
device memory (they only receive device pointers for inputs and outputs, or may
not call cudaMalloc on their hot path).  It must give what veda_tile_score
gives, call after call, while its scratch lives in a fixed array inside the
library that every call reuses; veda_noalloc_get_status reads that array's
status word.

This file is collected last on purpose: it shares the library's one scratch
array, and it must pass both alone in a fresh process and after every other
test."""
import ctypes
import os

import numpy as np
import pytest
import torch

import workloads

# Scratch a problem needs: the status word (256 bytes) plus q^ and k^, each
# B*H*nT rows of 9*d fp32 (three statistics, each as the hi/hi/lo TF32 split).
STATUS_BYTES = 256


def _need(w):
    return STATUS_BYTES + 2 * w.B * w.H * w.nT * 9 * w.d * 4


def _problem(vb, w):
    return vb.Problem.from_workload(w)


# just under the 64 MiB limit: 7 heads x 1,040 tiles x d = 128 -> 67,092,736 bytes
JUST_UNDER = workloads.custom("noalloc_under", 1, 7, 128, (13, 64, 160), [(1, 8, 16)], 8)
# just over: 2 heads x 3,641 tiles -> 67,111,168 bytes
JUST_OVER = workloads.custom("noalloc_over", 1, 2, 128, (11, 8, 5296), [(1, 8, 16)], 8)


def test_noalloc_rejects_problems_beyond_its_scratch():
    from tile_sparse_attention_b200 import build as b
    import tile_sparse_attention_b200 as vb
    b.build()
    lib = vb.load_library()
    limit = vb.veda_noalloc_scratch_bytes()
    assert limit == 64 << 20
    assert _need(JUST_UNDER) <= limit < _need(JUST_OVER)
    p = ctypes.c_void_p(0x10000)
    for w in (workloads.p720(), JUST_OVER):
        assert _need(w) > limit
        prob = _problem(vb, w)
        code = lib.veda_tile_score_noalloc(ctypes.byref(prob.c), p, p, p, p, p, None)
        assert code == 3  # VEDA_ERR_UNSUPPORTED, nothing launched
        assert b"scratch" in lib.veda_last_error()


def _score_both(vb, w, t, calls=2):
    """veda_tile_score with a workspace, then `calls` no-allocation calls; every
    no-allocation result must equal the workspace one."""
    prob = _problem(vb, w)
    B, H, nT, d = w.B, w.H, w.nT, w.d
    statsQ = torch.empty((B, H, nT, 3, d), dtype=torch.float32, device="cuda")
    statsK = torch.empty_like(statsQ)
    vb.veda_tripool(prob, t["Q"], t["K"], statsQ, statsK)
    ref = torch.empty((B, H, nT, nT), dtype=torch.float32, device="cuda")
    ws = vb.alloc_workspace(prob)
    vb.veda_tile_score(prob, statsQ, statsK, t["Wq"], t["Wk"], ref, ws)
    assert vb.veda_get_status(ws) == 0
    outs = []
    for _ in range(calls):
        out = torch.full_like(ref, float("nan"))
        vb.veda_tile_score_noalloc(prob, statsQ, statsK, t["Wq"], t["Wk"], out)
        assert vb.veda_noalloc_get_status() == 0
        outs.append(out)
    return prob, statsQ, statsK, ref, outs


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
        assert vb.veda_noalloc_get_status() == 0
        # same kernels, same order of operations: the scores agree exactly, well
        # inside the fp32 score tolerance of the parity tests
        assert torch.equal(out, ref), f"call {call}: max diff {(out - ref).abs().max().item()}"
        other = torch.empty((1, 2, w2.nT, w2.nT), dtype=torch.float32, device="cuda")
        vb.veda_tile_score_noalloc(p2, s2q, s2k, t2["Wq"], t2["Wk"], other)
        assert vb.veda_noalloc_get_status() == 0
        other_ref = torch.empty_like(other)
        ws2 = vb.alloc_workspace(p2)
        vb.veda_tile_score(p2, s2q, s2k, t2["Wq"], t2["Wk"], other_ref, ws2)
        torch.cuda.synchronize()
        assert torch.equal(other, other_ref)
    assert np.isfinite(ref.cpu().numpy()).all()


@pytest.mark.gpu
def test_noalloc_just_under_its_limit():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tile_sparse_attention_b200 as vb
    vb.load_library()
    w = JUST_UNDER
    t = workloads.generate(w, device="cuda")
    _, _, _, ref, outs = _score_both(vb, w, t, calls=2)
    for out in outs:
        assert torch.equal(out, ref)


@pytest.mark.gpu
def test_noalloc_timeout_is_readable():
    """A bounded wait of the score kernel that runs out (the test hook withholds
    the first operand load) is reported through veda_noalloc_get_status, and the
    next call on the same context succeeds and clears it."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tile_sparse_attention_b200 as vb
    vb.load_library()
    w = workloads.p480()
    t = {n: v.cuda() for n, v in workloads.generate(w, device="cpu").items()}
    prob, statsQ, statsK, ref, _ = _score_both(vb, w, t, calls=1)
    out = torch.zeros_like(ref)
    os.environ["VEDA_WAIT_LIMIT_MS"] = "300"
    os.environ["VEDA_TEST_WITHHOLD_ARRIVE"] = "1"
    try:
        vb.veda_tile_score_noalloc(prob, statsQ, statsK, t["Wq"], t["Wk"], out)
        status = vb.veda_noalloc_get_status()
    finally:
        del os.environ["VEDA_TEST_WITHHOLD_ARRIVE"]
        del os.environ["VEDA_WAIT_LIMIT_MS"]
    assert status == 6  # VEDA_ERR_TIMEOUT
    assert torch.count_nonzero(out).item() == 0  # CTAs that gave up write no scores
    vb.veda_tile_score_noalloc(prob, statsQ, statsK, t["Wq"], t["Wk"], out)
    assert vb.veda_noalloc_get_status() == 0
    assert torch.equal(out, ref)
