"""GPU parity of the KL structure distillation (loss and dL/dWq, dL/dWk).

Project page, "Principle 01 Full-Attention Structure Distillation" and
"Theoretical Rationale" 4 (Distillation Objective).

The GPU gets its own statistics, scores and teacher from the CUDA path; the
oracle computes everything in fp64 from the same Q, K, W.  The tolerance is a
first-order bound propagated from the per-stage bounds of the other tests
(scores: 8e-5 of the absolute products; teacher: relative error
scale * d * 2^-24 * max sum|q||k| + rounding; TripPool avg: Bt * 2^-24) through
p = softmax(S / tau), t = T / sum T, G = (p - t) / (tau R), dq~ = G k~,
dW = stats^T dq~, plus fp32 rounding of every product, times 2.
"""
import numpy as np
import pytest
import torch

import parity_helpers as ph
import workloads

pytestmark = pytest.mark.gpu
U = 2.0 ** -24


@pytest.fixture(scope="module")
def vb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tile_sparse_attention_b200 as m
    m.load_library()
    return m


def _bits_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _bounds(w, Q, K, sq, sk, Wq, Wk, T_o, tau, oracle):
    aWq, aWk = np.abs(Wq.astype(np.float64)), np.abs(Wk.astype(np.float64))
    qt = oracle.project(sq, Wq)
    kt = oracle.project(sk, Wk)
    S = oracle.score(qt, kt)
    R = S.size // S.shape[-1]
    x = S / tau
    p = np.exp(x - x.max(-1, keepdims=True))
    p /= p.sum(-1, keepdims=True)
    t = T_o / T_o.sum(-1, keepdims=True)
    G = (p - t) / (tau * R)
    dS = ph.score_bound(dict(statsQ=sq, statsK=sk), Wq, Wk)
    row_dS = dS.max(-1, keepdims=True)
    # teacher: relative error from the fp32 dot products and the dense lse
    eT = 0.0
    for b in range(w.B):
        for h in range(w.H):
            m = np.abs(Q[b, h]) @ np.abs(K[b, h]).T
            eT = max(eT, w.scale * w.d * U * m.max())
    eT += 16 * U
    logratio = np.where(t > 0, np.abs(np.log(np.maximum(t, 1e-300)) - np.log(np.maximum(p, 1e-300))), 0)
    dL = np.mean(2 * eT * (t * logratio).sum(-1) + 2 * eT + 2 * row_dS[..., 0] / tau)
    dL += 8 * w.nT * U * (1 + np.mean((t * logratio).sum(-1)))
    dG = (p * 2 * row_dS / tau + t * 2 * eT) / (tau * R) + 4 * U * (p + t) / (tau * R)
    # TripPool avg rounding: stats error <= Bt * u * max(|max|, |min|) per channel
    def dstats(st):
        mag = np.maximum(np.abs(st[..., 1, :]), np.abs(st[..., 2, :]))
        e = np.zeros_like(st)
        e[..., 0, :] = w.Bt * U * mag
        return e
    eq, ek = dstats(sq), dstats(sk)
    aq = np.einsum("bhjsc,hce->bhjse", np.abs(sq), aWq).reshape(qt.shape[:3] + (-1,))
    ak = np.einsum("bhjsc,hce->bhjse", np.abs(sk), aWk).reshape(kt.shape[:3] + (-1,))
    dqt = (np.einsum("bhjsc,hce->bhjse", eq, aWq).reshape(aq.shape) + w.d * U * aq)
    dkt = (np.einsum("bhjsc,hce->bhjse", ek, aWk).reshape(ak.shape) + w.d * U * ak)
    aG = np.abs(G)
    qf, kf = qt.reshape(aq.shape), kt.reshape(ak.shape)
    dq = np.einsum("bhij,bhjc->bhic", G, kf)
    dk = np.einsum("bhji,bhjc->bhic", G, qf)
    e_dq = (np.einsum("bhij,bhjc->bhic", dG, np.abs(kf)) + np.einsum("bhij,bhjc->bhic", aG, dkt)
            + w.nT * U * np.einsum("bhij,bhjc->bhic", aG, np.abs(kf)))
    e_dk = (np.einsum("bhji,bhjc->bhic", dG, np.abs(qf)) + np.einsum("bhji,bhjc->bhic", aG, dqt)
            + w.nT * U * np.einsum("bhji,bhjc->bhic", aG, np.abs(qf)))
    sh = sq.shape
    def dW_bound(st, est, dgrad, e_grad):
        sflat = np.abs(st).reshape(sh[0], sh[1], -1, sh[-1])
        eflat = est.reshape(sflat.shape)
        g = np.abs(dgrad).reshape(sh[0], sh[1], -1, sh[-1])
        eg = e_grad.reshape(g.shape)
        return (np.einsum("bhrc,bhre->hce", eflat, g) + np.einsum("bhrc,bhre->hce", sflat, eg)
                + 3 * w.nT * U * np.einsum("bhrc,bhre->hce", sflat, g))
    return 2 * dL, 2 * dW_bound(sq, eq, dq, e_dq), 2 * dW_bound(sk, ek, dk, e_dk)


CASES = [
    ("tiny", lambda: workloads.tiny(), 1.0),
    ("mixed_b2", lambda: workloads.custom("mixed", 2, 3, 128, (4, 16, 32),
                                          [(1, 8, 16), (2, 8, 8), (4, 4, 8)], 3), 0.5),
    ("d64", lambda: workloads.custom("d64", 1, 2, 64, (4, 16, 32), [(2, 8, 8)], 4), 4.0),
]


@pytest.mark.parametrize("name,make,tau", CASES)
def test_distill_loss_and_gradients(vb, oracle, name, make, tau):
    w = make()
    t = {n: v.cuda() for n, v in workloads.generate(w, device="cpu").items()}
    prob = vb.Problem.from_workload(w)
    B, H, nT, d = w.B, w.H, w.nT, w.d
    statsQ = torch.empty((B, H, nT, 3, d), dtype=torch.float32, device="cuda")
    statsK = torch.empty_like(statsQ)
    vb.veda_tripool(prob, t["Q"], t["K"], statsQ, statsK)
    S = torch.empty((B, H, nT, nT), dtype=torch.float32, device="cuda")
    ws = vb.alloc_workspace(prob)
    vb.veda_tile_score(prob, statsQ, statsK, t["Wq"], t["Wk"], S, ws)
    O = torch.empty_like(t["Q"])
    lse = torch.empty((B, H, w.N), dtype=torch.float32, device="cuda")
    T = torch.empty((B, H, nT, nT), dtype=torch.float32, device="cuda")
    vb.veda_teacher(prob, t["Q"], t["K"], t["V"], O, lse, T, ws)
    loss = torch.empty((1,), dtype=torch.float64, device="cuda")
    dWq = torch.empty_like(t["Wq"])
    dWk = torch.empty_like(t["Wk"])
    dws = torch.empty(vb.veda_distill_workspace_size(prob), dtype=torch.uint8, device="cuda")
    vb.veda_distill_kl(prob, statsQ, statsK, t["Wq"], t["Wk"], S, T, tau, loss, dWq, dWk, dws)
    assert vb.veda_get_status(dws) == 0

    Qb, Kb = ph.to_host_bits(t["Q"]), ph.to_host_bits(t["K"])
    Wq, Wk = t["Wq"].cpu().numpy(), t["Wk"].cpu().numpy()
    sq = oracle.tripool(Qb, w.grid, w.tile_shapes)
    sk = oracle.tripool(Kb, w.grid, w.tile_shapes)
    T_o, _ = oracle.teacher(Qb, Kb, w.grid, w.tile_shapes, w.scale)
    L_o, dWq_o, dWk_o = oracle.distill_kl(sq, sk, Wq, Wk, T_o, tau)
    bL, bq, bk = _bounds(w, _bits_f64(Qb), _bits_f64(Kb), sq, sk, Wq, Wk, T_o, tau, oracle)
    assert abs(loss.item() - L_o) <= bL, (loss.item(), L_o, bL)
    eq = np.abs(dWq.cpu().numpy().astype(np.float64) - dWq_o)
    ek = np.abs(dWk.cpu().numpy().astype(np.float64) - dWk_o)
    assert np.all(eq <= bq), f"dWq error {eq.max()} vs bound {bq[np.argmax(eq - bq)] if eq.size else 0}"
    assert np.all(ek <= bk), f"dWk error {ek.max()}"
    assert L_o > 0


def test_distill_rejects_ragged_tile_count(vb):
    w = workloads.custom("odd", 1, 1, 128, (3, 8, 16), [(1, 8, 16)], 1)
    prob = vb.Problem.from_workload(w)
    z = torch.zeros((1,), dtype=torch.float32, device="cuda")
    loss = torch.zeros((1,), dtype=torch.float64, device="cuda")
    dws = torch.empty(vb.veda_distill_workspace_size(prob), dtype=torch.uint8, device="cuda")
    with pytest.raises(vb.VedaError):
        vb.veda_distill_kl(prob, z, z, z, z, z, z, 1.0, loss, z, z, dws)
