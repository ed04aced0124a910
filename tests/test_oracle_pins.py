"""Pins for the fp64 oracle: it is checked against things other than itself.

* a hand-worked example (tests/golden/hand_example.json);
* an independent numpy brute force on tiny grids (tests/brute_force.py);
* closed forms and special cases: k = all tiles is dense softmax attention,
  the (1,1,Bt) tile shape is textbook 1-D block-sparse attention, constant
  tiles give avg = max = min, W = I gives the raw statistics, average pooling;
* invariants: min <= avg <= max, the Bhatia-Davis variance bound, exactly k
  ones per mask row, ascending unique index lists, renormalisation of the kept
  probabilities by Z / Z_hat >= 1, the teacher as tile-max of dense P.

Source: "Veda: Scalable Video Diffusion via Distilled Sparse Attention"
(project page): "Attention Structure Distillation" (Teacher, Estimator,
Execution), "Theoretical Rationale" 1 (Softmax Geometry: kept keys are
renormalised by Z/Z_hat) and 2 (Tile Statistics: avg/max/min, Bhatia-Davis).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import brute_force as bf
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32_to_bf16_bits(a) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    bits = a.view(np.uint32)
    assert np.all(bits & 0xFFFF == 0), "values must be exact in bf16"
    return (bits >> 16).astype(np.uint16)


def draw(grid, shapes, d, B=1, H=None, k=1, seed=0):
    H = H if H is not None else len(shapes)
    w = workloads.custom("pin", B, H, d, grid, shapes, k, seed)
    t = workloads.generate(w)
    return w, {n: workloads.bf16_bits(t[n]) for n in ("Q", "K", "V")}, t["Wq"].numpy(), \
        t["Wk"].numpy()


SMALL_CASES = [
    # grid, per-head shapes, d
    ((2, 4, 8), [(1, 2, 4), (2, 2, 2)], 8),
    ((4, 4, 4), [(2, 2, 2), (1, 2, 4), (4, 2, 1)], 4),
    ((1, 6, 6), [(1, 3, 3)], 5),
]


# ---------------------------------------------------------------- hand example
def test_hand_example(oracle):
    g = json.load(open(os.path.join(GOLDEN, "hand_example.json")))
    grid, shape = tuple(g["grid"]), tuple(g["tile_shape"])
    d = g["d"]
    Q = f32_to_bf16_bits(g["Q"]).reshape(1, 1, -1, d)
    K = f32_to_bf16_bits(g["K"]).reshape(1, 1, -1, d)
    V = f32_to_bf16_bits(g["V"]).reshape(1, 1, -1, d)
    Wq = np.asarray(g["Wq"], np.float32)[None]
    Wk = np.asarray(g["Wk"], np.float32)[None]
    assert oracle.tile_tokens(grid, shape).tolist() == g["tokens_of_tiles"]
    r = oracle.mask_prep(Q, K, Wq, Wk, grid, [shape], g["k"])
    np.testing.assert_array_equal(r["statsQ"][0, 0], np.asarray(g["statsQ"], float))
    np.testing.assert_array_equal(r["statsK"][0, 0], np.asarray(g["statsK"], float))
    np.testing.assert_array_equal(r["S"][0, 0], np.asarray(g["S"], float))
    np.testing.assert_array_equal(r["idx"][0, 0], np.asarray(g["idx"]))
    O, lse, toks = oracle.sparse_attention(Q, K, V, r["idx"], grid, [shape], g["scale"])
    env = {"exp": math.exp, "log": math.log, "e": math.e}
    for u in range(O.shape[0]):
        for row in range(O.shape[1]):
            t = str(int(toks[u, row]))
            want = [eval(s, env) for s in g["O_by_token"][t]]
            np.testing.assert_allclose(O[u, row], want, rtol=0, atol=1e-14)
            assert abs(lse[u, row] - eval(g["lse_by_token"][t], env)) < 1e-14


# ---------------------------------------------------------------- tile geometry
@pytest.mark.parametrize("grid,shape", [((4, 8, 16), (1, 8, 8)), ((20, 48, 80), (4, 4, 8)),
                                        ((20, 48, 80), (1, 8, 16)), ((2, 6, 6), (2, 3, 2))])
def test_tiles_partition_grid_into_boxes(oracle, grid, shape):
    tok = oracle.tile_tokens(grid, shape)
    T, Hs, Ws = grid
    assert np.array_equal(np.sort(tok.ravel()), np.arange(T * Hs * Ws))
    t, y, x = tok // (Hs * Ws), (tok // Ws) % Hs, tok % Ws
    for coord, p in ((t, shape[0]), (y, shape[1]), (x, shape[2])):
        assert np.all(coord.max(1) - coord.min(1) == p - 1)
        assert np.all(coord.min(1) % p == 0)
    np.testing.assert_array_equal(tok, bf.token_of_tile_row(grid, shape))


def test_1d_tile_shape_is_contiguous_blocks(oracle):
    tok = oracle.tile_tokens((3, 2, 64), (1, 1, 64))
    np.testing.assert_array_equal(tok, np.arange(3 * 2 * 64).reshape(6, 64))


# ---------------------------------------------------------------- TripPool
@pytest.mark.parametrize("grid,shapes,d", SMALL_CASES)
def test_tripool_brute_force(oracle, grid, shapes, d):
    w, x, _, _ = draw(grid, shapes, d, B=2)
    got = oracle.tripool(x["Q"], grid, shapes)
    want = bf.tripool(bf.bits_to_f64(x["Q"]), grid, shapes)
    np.testing.assert_array_equal(got[:, :, :, 1:], want[:, :, :, 1:])  # max, min exact
    np.testing.assert_allclose(got[:, :, :, 0], want[:, :, :, 0], rtol=0, atol=1e-13)


def test_tripool_invariants(oracle):
    w, x, _, _ = draw((4, 8, 16), [(1, 8, 8), (2, 4, 8)], 16)
    st = oracle.tripool(x["K"], w.grid, w.tile_shapes)
    avg, mx, mn = st[:, :, :, 0], st[:, :, :, 1], st[:, :, :, 2]
    assert np.all(mn <= avg) and np.all(avg <= mx)
    tiles_var = np.stack([bf.tile_view(bf.bits_to_f64(x["K"])[0, h], w.grid, w.tile_shapes[h])
                          .var(axis=1) for h in range(w.H)])[None]
    assert np.all(tiles_var <= (mx - avg) * (avg - mn) + 1e-12)  # Bhatia-Davis


def test_tripool_constant_tiles(oracle):
    grid, shape = (2, 4, 4), (1, 2, 2)
    tok = oracle.tile_tokens(grid, shape)
    X = np.zeros((1, 1, 32, 3), np.float32)
    for j, row in enumerate(tok):
        X[0, 0, row] = [j, -2.0 * j, 0.5]
    st = oracle.tripool(f32_to_bf16_bits(X), grid, [shape])
    for j in range(tok.shape[0]):
        for s in range(3):
            np.testing.assert_array_equal(st[0, 0, j, s], [j, -2.0 * j, 0.5])


# ---------------------------------------------------------------- projection + score
def test_projection_identity_and_linearity(oracle):
    w, x, _, _ = draw((2, 4, 8), [(1, 2, 4)], 6)
    st = oracle.tripool(x["Q"], w.grid, w.tile_shapes)
    I = np.eye(6, dtype=np.float32)[None]
    np.testing.assert_array_equal(oracle.project(st, I), st)
    rng = np.random.default_rng(3)
    W = rng.standard_normal((1, 6, 6)).astype(np.float32)
    proj = oracle.project(st, W)
    # mean commutes with a linear map: avg(X) W == avg(X W)
    XW = bf.bits_to_f64(x["Q"])[0, 0] @ W[0].astype(np.float64)
    np.testing.assert_allclose(proj[0, 0, :, 0], bf.tile_view(XW, w.grid, (1, 2, 4)).mean(1),
                               rtol=1e-12, atol=1e-12)
    # a negative diagonal map swaps max and min
    D = -np.diag(rng.uniform(0.5, 2, 6)).astype(np.float32)[None]
    pd = oracle.project(st, D)
    XD = bf.bits_to_f64(x["Q"])[0, 0] @ D[0].astype(np.float64)
    tiles_XD = bf.tile_view(XD, w.grid, (1, 2, 4))
    np.testing.assert_allclose(pd[0, 0, :, 1], tiles_XD.min(1), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(pd[0, 0, :, 2], tiles_XD.max(1), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("grid,shapes,d", SMALL_CASES)
def test_score_brute_force(oracle, grid, shapes, d):
    w, x, Wq, Wk = draw(grid, shapes, d, B=2)
    r = oracle.mask_prep(x["Q"], x["K"], Wq, Wk, grid, shapes, 2)
    sq = bf.tripool(bf.bits_to_f64(x["Q"]), grid, shapes)
    sk = bf.tripool(bf.bits_to_f64(x["K"]), grid, shapes)
    np.testing.assert_allclose(r["S"], bf.scores(sq, sk, Wq, Wk), rtol=1e-11, atol=1e-11)


def test_score_reduces_to_average_pooling(oracle):
    """Constant tiles + W = I: S = 3 * <mean-pooled q, mean-pooled k>."""
    grid, shape = (2, 4, 4), (2, 2, 2)
    tok = oracle.tile_tokens(grid, shape)
    rng = np.random.default_rng(5)
    d = 4
    Q = np.zeros((1, 1, 32, d), np.float32)
    K = np.zeros((1, 1, 32, d), np.float32)
    for j, row in enumerate(tok):
        Q[0, 0, row] = rng.integers(-4, 5, d)
        K[0, 0, row] = rng.integers(-4, 5, d)
    I = np.eye(d, dtype=np.float32)[None]
    r = oracle.mask_prep(f32_to_bf16_bits(Q), f32_to_bf16_bits(K), I, I, grid, [shape], 1)
    qbar = Q[0, 0][tok].mean(1).astype(np.float64)
    kbar = K[0, 0][tok].mean(1).astype(np.float64)
    np.testing.assert_array_equal(r["S"][0, 0], 3.0 * qbar @ kbar.T)


# ---------------------------------------------------------------- Top-k
def test_topk_matches_stable_sort_and_counts(oracle):
    rng = np.random.default_rng(11)
    for nT, k in ((8, 2), (17, 5), (40, 40), (33, 1)):
        S = rng.standard_normal((3, nT))
        S[:, ::3] = S[:, :1]  # many exact ties
        S[0, 1] = -0.0
        S[0, 2] = 0.0
        mask, idx = oracle.topk(S, k)
        m2, i2 = bf.topk(S, k)
        np.testing.assert_array_equal(mask, m2)
        np.testing.assert_array_equal(idx, i2)
        assert np.all(mask.sum(-1) == k)
        assert np.all(np.diff(idx, axis=-1) > 0)


def test_topk_tie_goes_to_lower_index(oracle):
    S = np.array([[1.0, 2.0, 2.0, 2.0, 0.5, 2.0], [-0.0, 0.0, -0.0, 0.0, -1, -1]])
    _, idx = oracle.topk(S, 2)
    assert idx.tolist() == [[1, 2], [0, 1]]


# ---------------------------------------------------------------- attention
@pytest.mark.parametrize("grid,shapes,d", SMALL_CASES)
def test_attention_brute_force_token_mask(oracle, grid, shapes, d):
    w, x, Wq, Wk = draw(grid, shapes, d, B=2)
    nT = w.nT
    k = max(1, nT // 3)
    r = oracle.mask_prep(x["Q"], x["K"], Wq, Wk, grid, shapes, k)
    scale = 1 / math.sqrt(d)
    O, lse, toks = oracle.sparse_attention(x["Q"], x["K"], x["V"], r["idx"], grid, shapes, scale)
    Qf, Kf, Vf = (bf.bits_to_f64(x[n]) for n in "QKV")
    Ob, lseb = bf.sparse_attention(Qf, Kf, Vf, r["mask"], grid, shapes, scale)
    units = [(b, h, i) for b in range(w.B) for h in range(w.H) for i in range(nT)]
    for u, (b, h, i) in enumerate(units):
        np.testing.assert_allclose(O[u], Ob[b, h][toks[u]], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(lse[u], lseb[b, h][toks[u]], rtol=1e-12, atol=1e-12)


def test_attention_all_tiles_is_dense_softmax(oracle):
    grid, shapes, d = (2, 4, 8), [(1, 2, 4), (2, 2, 2)], 8
    w, x, _, _ = draw(grid, shapes, d)
    nT = w.nT
    idx = np.broadcast_to(np.arange(nT, dtype=np.int32), (1, w.H, nT, nT)).copy()
    scale = 0.3
    O, lse, toks = oracle.sparse_attention(x["Q"], x["K"], x["V"], idx, grid, shapes, scale)
    Qf, Kf, Vf = (bf.bits_to_f64(x[n]) for n in "QKV")
    for u in range(O.shape[0]):
        h = u // nT
        logits = scale * Qf[0, h] @ Kf[0, h].T
        P = np.exp(logits - logits.max(1, keepdims=True))
        P /= P.sum(1, keepdims=True)
        np.testing.assert_allclose(O[u], (P @ Vf[0, h])[toks[u]], rtol=1e-11, atol=1e-12)
        lse_d = np.log(np.exp(logits).sum(1))
        np.testing.assert_allclose(lse[u], lse_d[toks[u]], rtol=1e-12)


def test_attention_1d_tiles_is_block_sparse(oracle):
    """Tile shape (1,1,Bt) on a grid with Ws = Bt is plain 1-D block-sparse attention."""
    Bt, d = 4, 8
    grid = (1, 5, Bt)
    w, x, _, _ = draw(grid, [(1, 1, Bt)], d)
    rng = np.random.default_rng(2)
    nT, k = 5, 2
    idx = np.sort(np.stack([rng.choice(nT, k, replace=False) for _ in range(nT)]), 1)
    idx = idx.astype(np.int32)[None, None]
    tile_mask = np.zeros((nT, nT), np.int64)
    for i in range(nT):
        tile_mask[i, idx[0, 0, i]] = 1
    allowed = np.kron(tile_mask, np.ones((Bt, Bt), np.int64)).astype(bool)
    O, lse, toks = oracle.sparse_attention(x["Q"], x["K"], x["V"], idx, grid, [(1, 1, Bt)], 0.5)
    Qf, Kf, Vf = (bf.bits_to_f64(x[n])[0, 0] for n in "QKV")
    logits = np.where(allowed, 0.5 * Qf @ Kf.T, -np.inf)
    P = np.exp(logits - logits.max(1, keepdims=True))
    P /= P.sum(1, keepdims=True)
    np.testing.assert_allclose(O.reshape(-1, d), P @ Vf, rtol=1e-11, atol=1e-12)


def test_attention_renormalisation(oracle):
    """Kept probabilities are the dense ones scaled by Z/Z_hat = exp(lse_dense - lse) >= 1."""
    grid, shapes, d = (4, 4, 4), [(2, 2, 2)], 8
    w, x, Wq, Wk = draw(grid, shapes, d)
    r = oracle.mask_prep(x["Q"], x["K"], Wq, Wk, grid, shapes, 3)
    scale = 1 / math.sqrt(d)
    O, lse, toks = oracle.sparse_attention(x["Q"], x["K"], x["V"], r["idx"], grid, shapes, scale)
    _, lse_dense = oracle.teacher(x["Q"], x["K"], grid, shapes, scale)
    Qf, Kf, Vf = (bf.bits_to_f64(x[n])[0, 0] for n in "QKV")
    P = bf.dense_probs(Qf, Kf, scale)
    allowed = bf.token_mask(r["mask"][0, 0], grid, shapes[0])
    for u in range(O.shape[0]):
        rows = toks[u]
        ratio = np.exp(lse_dense[0, 0][rows] - lse[u])
        assert np.all(ratio >= 1.0)
        kept = np.where(allowed[rows], P[rows], 0.0) * ratio[:, None]
        np.testing.assert_allclose(kept.sum(1), 1.0, rtol=1e-12)
        np.testing.assert_allclose(O[u], kept @ Vf, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- teacher
@pytest.mark.parametrize("grid,shapes,d", SMALL_CASES[:2])
def test_teacher_is_tile_max_of_dense_probs(oracle, grid, shapes, d):
    w, x, _, _ = draw(grid, shapes, d)
    scale = 1 / math.sqrt(d)
    T, lse = oracle.teacher(x["Q"], x["K"], grid, shapes, scale)
    Qf, Kf = bf.bits_to_f64(x["Q"]), bf.bits_to_f64(x["K"])
    np.testing.assert_allclose(T, bf.teacher(Qf, Kf, grid, shapes, scale), rtol=1e-12)
    assert np.all(T > 0) and np.all(T <= 1)
    for h in range(w.H):
        P = bf.dense_probs(Qf[0, h], Kf[0, h], scale)
        np.testing.assert_allclose(T[0, h].max(1), P[bf.token_of_tile_row(grid, shapes[h])]
                                   .max(axis=(1, 2)), rtol=1e-12)


# ---------------------------------------------------------------- workload recipe
def test_workload_tables():
    assert (workloads.tiny().nT, workloads.tiny().k) == (8, 2)
    assert (workloads.p480().nT, workloads.p480().k) == (240, 24)
    assert (workloads.p720().nT, workloads.p720().k) == (600, 30)
    assert (workloads.long_video().nT, workloads.long_video().k) == (1920, 96)
    assert workloads.long_video().N == 245760
    ks = [workloads.sweep(64, s).k for s in workloads.SWEEP_SPARSITY]
    assert ks == [1920, 960, 384, 192, 96, 38]
    assert [workloads.sweep(T, 95).N for T in workloads.SWEEP_T] == \
        [15360, 30720, 76800, 122880, 245760]
    for w in [workloads.p720(), workloads.long_video()] + workloads.sweep_points():
        for s in w.tile_shapes:
            assert int(np.prod(s)) == 128
            assert w.T % s[0] == 0 and w.Hs % s[1] == 0 and w.Ws % s[2] == 0
    assert abs(workloads.long_video().sparse_flops() - 4.948e13) / 4.948e13 < 1e-3


def test_generator_is_seeded():
    w = workloads.tiny()
    a, b = workloads.generate(w), workloads.generate(w)
    for n in ("Q", "K", "V", "Wq", "Wk"):
        assert torch.equal(a[n], b[n])
    c = workloads.generate(workloads.tiny(seed=1))
    assert not torch.equal(a["Q"], c["Q"])


# ---------------------------------------------------------------- tile recall
def test_tile_recall_hand_cases(oracle):
    pred = np.array([[0, 2, 5], [1, 2, 3], [4, 6, 7]], np.int32)
    ref = np.array([[2, 3, 5], [1, 2, 3], [0, 1, 2]], np.int32)
    per, mean = oracle.tile_recall(pred, ref)
    np.testing.assert_array_equal(per, [2 / 3, 1.0, 0.0])
    assert mean == (2 + 3 + 0) / 9


def test_tile_recall_brute_force(oracle):
    rng = np.random.default_rng(4)
    nT, k = 40, 7
    pred = np.sort(np.stack([rng.permutation(nT)[:k] for _ in range(50)]), 1).astype(np.int32)
    ref = np.sort(np.stack([rng.permutation(nT)[:k] for _ in range(50)]), 1).astype(np.int32)
    per, mean = oracle.tile_recall(pred, ref)
    want = np.array([len(set(a) & set(b)) / k for a, b in zip(pred, ref)])
    np.testing.assert_array_equal(per, want)
    assert abs(mean - want.mean()) < 1e-15
    per_self, mean_self = oracle.tile_recall(ref, ref)
    assert mean_self == 1.0 and np.all(per_self == 1.0)


# ---------------------------------------------------------------- KL distillation
def _distill_case(seed=0, B=1, H=2, nT=6, d=4):
    rng = np.random.default_rng(seed)
    sq = rng.standard_normal((B, H, nT, 3, d))
    sk = rng.standard_normal((B, H, nT, 3, d))
    Wq = (rng.standard_normal((H, d, d)) / 2).astype(np.float32)
    Wk = (rng.standard_normal((H, d, d)) / 2).astype(np.float32)
    T = rng.uniform(0.01, 1.0, (B, H, nT, nT))
    return sq, sk, Wq, Wk, T


@pytest.mark.parametrize("tau,B", [(0.7, 1), (1.0, 2), (3.0, 1)])
def test_distill_gradient_matches_finite_differences(oracle, tau, B):
    """Central differences of the loss (computed from its definition) pin dL/dW."""
    sq, sk, Wq, Wk, T = _distill_case(B=B)
    _, dWq, dWk = oracle.distill_kl(sq, sk, Wq, Wk, T, tau)
    scale = max(np.abs(dWq).max(), np.abs(dWk).max())
    eps = np.float32(2.0 ** -12)
    for side in ("q", "k"):
        W, dW = (Wq, dWq) if side == "q" else (Wk, dWk)
        for (h, a, b) in [(0, 0, 0), (1, 2, 3), (0, 3, 1), (1, 1, 2), (0, 2, 2)]:
            Wp, Wm = W.copy(), W.copy()
            Wp[h, a, b] = np.float32(W[h, a, b] + eps)
            Wm[h, a, b] = np.float32(W[h, a, b] - eps)
            step = float(Wp[h, a, b]) - float(Wm[h, a, b])
            args_p = (Wp, Wk) if side == "q" else (Wq, Wp)
            args_m = (Wm, Wk) if side == "q" else (Wq, Wm)
            Lp = oracle.distill_kl(sq, sk, *args_p, T, tau, grads=False)
            Lm = oracle.distill_kl(sq, sk, *args_m, T, tau, grads=False)
            fd = (Lp - Lm) / step
            assert abs(fd - dW[h, a, b]) <= 1e-4 * scale + 1e-10, (side, h, a, b, fd, dW[h, a, b])


@pytest.mark.parametrize("tau,B,seed", [(0.7, 1, 0), (1.0, 2, 11), (3.0, 1, 4)])
def test_distill_loss_matches_definition(oracle, tau, B, seed):
    """The loss value against the brute-force KL written from the definition:
    direction KL(target || estimator) and the mean over the B*H*nT rows.  A
    reversed divergence or a sum over rows changes the value (the teacher rows
    here are far from the estimator's, so the two directions differ)."""
    sq, sk, Wq, Wk, T = _distill_case(seed=seed, B=B)
    L = oracle.distill_kl(sq, sk, Wq, Wk, T, tau, grads=False)
    ref = bf.distill_kl(sq, sk, Wq, Wk, T, tau)
    assert abs(L - ref) <= 1e-12 * max(1.0, abs(ref)), (L, ref)
    # a teacher with zero entries: those terms contribute nothing
    Tz = T.copy()
    Tz[..., ::3] = 0.0
    Lz = oracle.distill_kl(sq, sk, Wq, Wk, Tz, tau, grads=False)
    assert abs(Lz - bf.distill_kl(sq, sk, Wq, Wk, Tz, tau)) <= 1e-12 * max(1.0, abs(Lz))


def test_distill_zero_when_target_equals_prediction(oracle):
    sq, sk, Wq, Wk, _ = _distill_case(seed=3)
    tau = 1.7
    S = oracle.score(oracle.project(sq, Wq), oracle.project(sk, Wk))
    T = np.exp(S / tau - (S / tau).max(-1, keepdims=True)) * 5.0  # any positive row scale
    L, dWq, dWk = oracle.distill_kl(sq, sk, Wq, Wk, T, tau)
    assert abs(L) < 1e-14
    assert np.abs(dWq).max() < 1e-12 and np.abs(dWk).max() < 1e-12


def test_distill_invariances_and_positivity(oracle):
    sq, sk, Wq, Wk, T = _distill_case(seed=5)
    L = oracle.distill_kl(sq, sk, Wq, Wk, T, 1.0, grads=False)
    assert L > 0
    # the teacher enters only through its row-normalised distribution
    T2 = T * np.random.default_rng(1).uniform(0.5, 3.0, T.shape[:-1] + (1,))
    assert abs(oracle.distill_kl(sq, sk, Wq, Wk, T2, 1.0, grads=False) - L) < 1e-13
    # S / tau is what matters: scaling Wq by 2 and tau by 2 leaves the loss unchanged
    L2 = oracle.distill_kl(sq, sk, (Wq * 2).astype(np.float32), Wk, T, 2.0, grads=False)
    assert abs(L2 - L) < 1e-12


# ---------------------------------------------------------------- head-aware tile search
def test_tile_search_brute_force(oracle):
    grid, d, k = (2, 4, 8), 8, 2
    cands = [(1, 2, 4), (2, 2, 2), (1, 4, 2)]
    w, x, Wq, Wk = draw(grid, [cands[0], cands[0]], d, B=2)
    scale = 1 / math.sqrt(d)
    err, best, _ = oracle.tile_search(x["Q"], x["K"], x["V"], Wq, Wk, grid, cands, k, scale)
    Qf, Kf, Vf = (bf.bits_to_f64(x[n]) for n in "QKV")
    full = np.stack([np.stack([bf.masked_attention(Qf[b, h], Kf[b, h], Vf[b, h],
                                                    np.ones((w.N, w.N), bool), scale)[0]
                               for h in range(2)]) for b in range(2)])
    for c, shape in enumerate(cands):
        shapes = [shape, shape]
        S = bf.scores(bf.tripool(Qf, grid, shapes), bf.tripool(Kf, grid, shapes), Wq, Wk)
        mask, _ = bf.topk(S, k)
        Os, _ = bf.sparse_attention(Qf, Kf, Vf, mask, grid, shapes, scale)
        np.testing.assert_allclose(err[c], ((full - Os) ** 2).sum(axis=(2, 3)), rtol=1e-9,
                                   atol=1e-12)
    np.testing.assert_array_equal(best, np.argmin(err.sum(axis=1), axis=0))


def test_tile_search_all_tiles_has_zero_error(oracle):
    grid, d = (2, 4, 8), 8
    cands = [(1, 2, 4), (2, 2, 2)]
    w, x, Wq, Wk = draw(grid, [cands[0]], d)
    err, best, _ = oracle.tile_search(x["Q"], x["K"], x["V"], Wq, Wk, grid, cands, 8, 0.3)
    assert np.abs(err).max() < 1e-24
    assert best.tolist() == [0]


# ------------------------------------------------------------------ fp8 weights
# OCP FP8 E4M3 ("e4m3fn") format facts: bias 7, 3 mantissa bits, no infinities,
# S.1111.111 is NaN, largest finite 1.75 * 2^8 = 448, smallest normal 2^-6,
# smallest subnormal 2^-9.
def test_e4m3_format_facts(oracle):
    o = oracle
    assert o.e4m3_decode(0x7E) == 448.0 and o.e4m3_decode(0xFE) == -448.0
    assert np.isnan(o.e4m3_decode(0x7F)) and np.isnan(o.e4m3_decode(0xFF))
    assert o.e4m3_decode(0x08) == 2.0 ** -6 and o.e4m3_decode(0x07) == 7 * 2.0 ** -9
    assert o.e4m3_decode(0x01) == 2.0 ** -9
    assert o.e4m3_decode(0x38) == 1.0 and o.e4m3_decode(0x3C) == 1.5
    z = o.e4m3_decode(0x80)
    assert z == 0.0 and np.signbit(z)
    vals = [o.e4m3_decode(c) for c in range(127)]
    assert all(b > a for a, b in zip(vals, vals[1:]))


def test_e4m3_round_trip_midpoints_and_saturation(oracle):
    o = oracle
    for c in list(range(127)) + list(range(128, 255)):
        assert o.e4m3_encode(o.e4m3_decode(c)) == c
    for c in range(126):
        a, b = o.e4m3_decode(c), o.e4m3_decode(c + 1)
        mid = np.float32((a + b) / 2)          # one extra bit: exact in fp32
        assert float(mid) == (a + b) / 2
        even = c if c % 2 == 0 else c + 1
        assert o.e4m3_encode(mid) == even
        assert o.e4m3_encode(-mid) == 0x80 | even
        assert o.e4m3_encode(np.nextafter(mid, np.float32(0))) == c
        assert o.e4m3_encode(np.nextafter(mid, np.float32(1000))) == c + 1
    for x in (448.0, 449.0, 463.9, 464.0, 1e4, 3e38):
        assert o.e4m3_encode(x) == 0x7E and o.e4m3_encode(-x) == 0xFE


def test_e4m3_matches_library_conversion(oracle):
    """Round to nearest even, as torch's float8_e4m3fn conversion does (|x| <= 448)."""
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.uniform(-448, 448, 4000), rng.standard_normal(4000),
                        rng.standard_normal(2000) * 2.0 ** -7,
                        rng.standard_normal(1000) * 2.0 ** -10]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(v) for v in x], dtype=np.uint8)
    np.testing.assert_array_equal(got, ref)


def test_e4m3_quantize_per_head(oracle):
    rng = np.random.default_rng(12)
    W = (rng.standard_normal((4, 16, 16)) / 4).astype(np.float32)
    W[1] *= 1e-3                               # small values, subnormal codes
    W[2] = 0.0                                 # all-zero head: scale 1, zero codes
    W[3, 5, 7] = -7.5                          # a single large value sets the scale
    codes, scale = oracle.quantize_e4m3(W)
    for h in range(4):
        amax = np.abs(W[h]).max()
        want = np.float32(amax) / np.float32(448.0) if amax > 0 else np.float32(1.0)
        assert scale[h] == want
    assert np.all(codes[2] == 0)
    assert codes[3, 5, 7] == 0xFE
    Wd = oracle.dequantize_e4m3(codes, scale)
    assert Wd.dtype == np.float32 and Wd[3, 5, 7] == np.float32(np.float32(-448.0) * scale[3])
    for h in (0, 1, 3):
        s = float(scale[h])
        y = np.abs(W[h].astype(np.float64)) / s
        # half a code step: 2^(e-4) in a normal binade, 2^-10 below 2^-6; plus fp32 rounding
        step = np.where(y >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(y, 1e-30))) - 4), 2.0 ** -10)
        err = np.abs(Wd[h].astype(np.float64) - W[h].astype(np.float64))
        assert np.all(err <= s * step * (1 + 2.0 ** -20) + np.abs(W[h]) * 2.0 ** -23)
    # decoding the codes by the format definition gives the same weights
    dec = np.vectorize(oracle.e4m3_decode)(codes.astype(np.int64)).astype(np.float32)
    np.testing.assert_array_equal(Wd, (dec * scale[:, None, None]).astype(np.float32))
