"""GPU parity of the fused score + Top-k (veda_mask_fused).

The fused kernel computes every score with the same tensor-core products, in
the same order, as veda_tile_score, so its index lists and masks must equal
the two-call path bit for bit; against the fp64 oracle the usual mask rule
applies (bit-exact rows away from near-ties).  Exact ties are made by giving
several key tiles identical statistics; the expected selection is then the
oracle's Top-k run on the GPU's own fp32 scores (the decision is taken on the
same values on both sides).
"""
import numpy as np
import pytest
import torch

import parity_helpers as ph
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tile_sparse_attention_b200 as m
    m.load_library()
    return m


def _stats(vb, prob, t):
    B, H, nT, d = prob.B, prob.H, prob.nT, prob.d
    sq = torch.empty((B, H, nT, 3, d), dtype=torch.float32, device="cuda")
    sk = torch.empty_like(sq)
    vb.veda_tripool(prob, t["Q"], t["K"], sq, sk)
    return sq, sk


def _both_paths(vb, prob, sq, sk, Wq, Wk):
    B, H, nT, k = prob.B, prob.H, prob.nT, prob.k
    ws = vb.alloc_workspace(prob)
    S = torch.empty((B, H, nT, nT), dtype=torch.float32, device="cuda")
    vb.veda_tile_score(prob, sq, sk, Wq, Wk, S, ws)
    m2 = torch.empty((B, H, nT, nT), dtype=torch.uint8, device="cuda")
    i2 = torch.empty((B, H, nT, k), dtype=torch.int32, device="cuda")
    vb.veda_topk_mask(prob, S, m2, i2)
    mf = torch.full((B, H, nT, nT), 7, dtype=torch.uint8, device="cuda")
    i_f = torch.full((B, H, nT, k), -1, dtype=torch.int32, device="cuda")
    vb.veda_mask_fused(prob, sq, sk, Wq, Wk, mf, i_f, ws)
    torch.cuda.synchronize()
    assert vb.veda_get_status(ws) == 0
    return S, (m2, i2), (mf, i_f)


CASES = [
    ("tiny", workloads.tiny),
    ("480p", workloads.p480),
    ("720p", workloads.p720),
    ("long_video", workloads.long_video),
    ("d64_ragged_b2", lambda: workloads.custom("r", 2, 3, 64, (3, 16, 40), [(1, 8, 8)], 7)),
    ("k1", lambda: workloads.custom("k1", 1, 2, 128, (4, 16, 32), [(2, 8, 8)], 1)),
    ("k_all", lambda: workloads.custom("kall", 1, 2, 128, (4, 16, 32), [(2, 8, 8)], 16)),
    ("k128", lambda: workloads.custom("k128", 1, 2, 128, (20, 32, 48), [(2, 8, 8)], 128)),
    ("nT_129", lambda: workloads.custom("n129", 1, 2, 64, (1, 8, 129 * 8), [(1, 8, 8)], 9)),
]


@pytest.mark.parametrize("name,make", CASES)
def test_fused_equals_two_call_path(vb, name, make):
    w = make()
    t = {n: v.cuda() for n, v in workloads.generate(w, device="cpu").items()}
    prob = vb.Problem.from_workload(w)
    sq, sk = _stats(vb, prob, t)
    _, (m2, i2), (mf, i_f) = _both_paths(vb, prob, sq, sk, t["Wq"], t["Wk"])
    assert torch.equal(i_f, i2), f"{name}: index lists differ"
    assert torch.equal(mf, m2), f"{name}: masks differ"


@pytest.mark.parametrize("make,heads", [(workloads.tiny, None), (workloads.p480, None),
                                        (workloads.p720, [0, 13, 39])])
def test_fused_against_oracle(vb, oracle, make, heads):
    w = make()
    t = {n: v.cuda() for n, v in workloads.generate(w, device="cpu").items()}
    prob = vb.Problem.from_workload(w)
    sq, sk = _stats(vb, prob, t)
    B, H, nT = w.B, w.H, w.nT
    ws = vb.alloc_workspace(prob)
    mf = torch.empty((B, H, nT, nT), dtype=torch.uint8, device="cuda")
    i_f = torch.empty((B, H, nT, w.k), dtype=torch.int32, device="cuda")
    vb.veda_mask_fused(prob, sq, sk, t["Wq"], t["Wk"], mf, i_f, ws)
    torch.cuda.synchronize()
    assert vb.veda_get_status(ws) == 0
    heads = list(range(H)) if heads is None else heads
    Qb, Kb = ph.to_host_bits(t["Q"]), ph.to_host_bits(t["K"])
    Wq, Wk = t["Wq"].cpu().numpy(), t["Wk"].cpu().numpy()
    ora = ph.oracle_mask_prep_heads(oracle, w, Qb, Kb, Wq, Wk, heads)
    ph.check_masks(mf[:, heads].cpu().numpy(), i_f[:, heads].cpu().numpy(), ora["S"],
                   ora["mask"], ora["idx"], w.k, label=f"fused {w.name}")


def test_fused_exact_ties_and_zero_scores(vb, oracle):
    """Key tiles with identical statistics give bit-identical score columns."""
    w = workloads.custom("ties", 1, 3, 128, (20, 32, 48), [(2, 8, 8)], 24)
    t = {n: v.cuda() for n, v in workloads.generate(w, device="cpu").items()}
    prob = vb.Problem.from_workload(w)
    sq, sk = _stats(vb, prob, t)
    sk[:, :, 10] = sk[:, :, 3]
    sk[:, :, 200] = sk[:, :, 3]
    sk[:, :, 131] = sk[:, :, 7]
    sk[:, 1, 40:60] = sk[:, 1, 39:40]     # twenty equal columns in head 1
    sk[:, 2, 5] = 0.0                     # a zero score column
    sk[:, 2, 130] = 0.0
    S, (m2, i2), (mf, i_f) = _both_paths(vb, prob, sq, sk, t["Wq"], t["Wk"])
    m_o, i_o = oracle.topk(S.cpu().numpy().astype(np.float64), w.k)
    np.testing.assert_array_equal(i_f.cpu().numpy(), i_o)
    np.testing.assert_array_equal(mf.cpu().numpy(), m_o)
    assert torch.equal(i_f, i2)


def test_fused_mask_may_be_null(vb):
    w = workloads.p480()
    t = {n: v.cuda() for n, v in workloads.generate(w, device="cpu").items()}
    prob = vb.Problem.from_workload(w)
    sq, sk = _stats(vb, prob, t)
    _, (_, i2), _ = _both_paths(vb, prob, sq, sk, t["Wq"], t["Wk"])
    ws = vb.alloc_workspace(prob)
    i_f = torch.empty_like(i2)
    vb.veda_mask_fused(prob, sq, sk, t["Wq"], t["Wk"], None, i_f, ws)
    torch.cuda.synchronize()
    assert torch.equal(i_f, i2)


def test_fused_limits_are_reported(vb):
    z = torch.zeros((64,), dtype=torch.float32, device="cuda")
    zi = torch.zeros((64,), dtype=torch.int32, device="cuda")
    ws = torch.zeros((4096,), dtype=torch.uint8, device="cuda")
    big_k = vb.Problem.from_workload(workloads.custom("bk", 1, 1, 128, (20, 32, 48), [(2, 8, 8)], 129))
    with pytest.raises(vb.VedaError):
        vb.veda_mask_fused(big_k, z, z, z, z, None, zi, ws)
    big_n = vb.Problem.from_workload(workloads.custom("bn", 1, 1, 64, (1, 8, 6152 * 8), [(1, 8, 8)], 4))
    with pytest.raises(vb.VedaError):
        vb.veda_mask_fused(big_n, z, z, z, z, None, zi, ws)
