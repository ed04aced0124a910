"""GPU parity of the fp8 (E4M3) estimator weights.

News page ("Veda from ByteDance, HKU and USTC: an open method that speeds up
video generation fivefold", "Why this matters for users"): the predictor is
distributed in fp8.  Codes, per-head scales and dequantised fp32 weights are
integer / correctly rounded results, so they must match the oracle bit for
bit; the mask computed with the dequantised weights then follows the usual
mask rule against the oracle's mask prep with the oracle's dequantised weights.
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


def _weights(H, d, seed):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((H, d, d)) / np.sqrt(d)).astype(np.float32)
    if H > 1:
        W[1] *= 1e-4          # tiny head: many subnormal codes
    if H > 2:
        W[2] = 0.0            # all-zero head
    if H > 3:
        W[3, 0, 0] = 40.0     # one outlier sets the scale
        W[3, 1, 1] = -0.0
    return W


@pytest.mark.parametrize("H,d", [(4, 128), (5, 64), (40, 128)])
def test_quantize_and_dequantize_bit_exact(vb, oracle, H, d):
    W = _weights(H, d, 3 + H)
    Wt = torch.from_numpy(W).cuda()
    W8 = torch.empty((H, d, d), dtype=torch.uint8, device="cuda")
    sc = torch.empty((H,), dtype=torch.float32, device="cuda")
    vb.veda_quantize_fp8(Wt, W8, sc)
    Wd = torch.empty_like(Wt)
    vb.veda_dequantize_fp8(W8, sc, Wd)
    torch.cuda.synchronize()
    codes_o, scale_o = oracle.quantize_e4m3(W)
    np.testing.assert_array_equal(sc.cpu().numpy(), scale_o)
    np.testing.assert_array_equal(W8.cpu().numpy(), codes_o)
    np.testing.assert_array_equal(Wd.cpu().numpy(), oracle.dequantize_e4m3(codes_o, scale_o))


def test_mask_with_fp8_weights(vb, oracle):
    """The 480P-like layer's mask with fp8 estimator weights, against the oracle."""
    w = workloads.p480()
    t = {n: v.cuda() for n, v in workloads.generate(w, device="cpu").items()}
    prob = vb.Problem.from_workload(w)
    H, d = w.H, w.d
    deq = {}
    for name in ("Wq", "Wk"):
        W8 = torch.empty((H, d, d), dtype=torch.uint8, device="cuda")
        sc = torch.empty((H,), dtype=torch.float32, device="cuda")
        vb.veda_quantize_fp8(t[name], W8, sc)
        deq[name] = torch.empty_like(t[name])
        vb.veda_dequantize_fp8(W8, sc, deq[name])
    g = ph.gpu_mask_prep(vb, prob, t["Q"], t["K"], deq["Wq"], deq["Wk"])
    Qb, Kb = ph.to_host_bits(t["Q"]), ph.to_host_bits(t["K"])
    Wq_o = oracle.dequantize_e4m3(*oracle.quantize_e4m3(t["Wq"].cpu().numpy()))
    Wk_o = oracle.dequantize_e4m3(*oracle.quantize_e4m3(t["Wk"].cpu().numpy()))
    np.testing.assert_array_equal(deq["Wq"].cpu().numpy(), Wq_o)
    heads = list(range(H))
    ora = ph.oracle_mask_prep_heads(oracle, w, Qb, Kb, Wq_o, Wk_o, heads)
    ph.check_masks(g["mask"].cpu().numpy(), g["idx"].cpu().numpy(), ora["S"], ora["mask"],
                   ora["idx"], w.k, label=f"fp8 weights {w.name}")
    # tile recall of the fp8-weight mask against the fp32-weight mask (GPU kernel
    # against the oracle's count on the same index lists)
    g32 = ph.gpu_mask_prep(vb, prob, t["Q"], t["K"], t["Wq"], t["Wk"])
    rows = torch.empty((w.B, H, w.nT), dtype=torch.float32, device="cuda")
    mean = torch.empty((1,), dtype=torch.float64, device="cuda")
    ws = vb.alloc_workspace(prob)
    vb.veda_tile_recall(prob, g["idx"], g32["idx"], rows, mean, ws)
    torch.cuda.synchronize()
    _, mean_o = oracle.tile_recall(g["idx"].cpu().numpy(), g32["idx"].cpu().numpy())
    assert mean.item() == mean_o
    assert 0.0 < mean_o <= 1.0


def test_fp8_argument_errors(vb):
    z8 = torch.zeros((16,), dtype=torch.uint8, device="cuda")
    zf = torch.zeros((16,), dtype=torch.float32, device="cuda")
    lib = vb.load_library()
    assert lib.veda_quantize_fp8(zf.data_ptr(), 0, 4, z8.data_ptr(), zf.data_ptr(), None) != 0
    assert lib.veda_dequantize_fp8(z8.data_ptr(), zf.data_ptr(), 1, 0, zf.data_ptr(), None) != 0
    assert lib.veda_quantize_fp8(None, 1, 4, z8.data_ptr(), zf.data_ptr(), None) != 0
