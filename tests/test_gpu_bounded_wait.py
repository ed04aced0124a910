"""Failure detection without a GPU fault: a device wait that runs out.

With VEDA_TEST_WITHHOLD_ARRIVE set, one softmax warp of every CTA skips its
first "P ready" arrival, so the tensor-core issuer's bounded wait (limit set to
300 ms through VEDA_WAIT_LIMIT_MS) expires.  The CTA then raises its abort
flag, the other roles leave their waits, in-flight copies and products are
drained, tensor memory is freed and VEDA_ERR_TIMEOUT lands in the status word.
The context stays usable: the next call computes correct results.  Both
attention kernels are covered: the persistent one (short key lists) and the
one-CTA-per-query-tile one (k above 64).
"""
import os

import numpy as np
import pytest
import torch

import parity_helpers as ph
import workloads

pytestmark = pytest.mark.gpu

CASES = [
    ("persistent_k2", workloads.tiny),
    ("per_tile_k80", lambda: workloads.custom("wb", 1, 2, 128, (8, 32, 64), [(2, 8, 8)], 80)),
]


@pytest.mark.parametrize("name,make", CASES)
def test_timeout_is_reported_and_context_survives(oracle, name, make):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tile_sparse_attention_b200 as vb
    vb.load_library()
    w = make()
    t = {n: v.cuda() for n, v in workloads.generate(w, device="cpu").items()}
    prob = vb.Problem.from_workload(w)
    idx = torch.stack([torch.arange(w.k, dtype=torch.int32)] * (w.H * w.nT)).reshape(
        1, w.H, w.nT, w.k).cuda().contiguous()
    O = torch.empty_like(t["Q"])
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device="cuda")
    ws = vb.alloc_workspace(prob)
    os.environ["VEDA_WAIT_LIMIT_MS"] = "300"
    os.environ["VEDA_TEST_WITHHOLD_ARRIVE"] = "1"
    try:
        vb.veda_sparse_attn(prob, t["Q"], t["K"], t["V"], idx, O, lse, ws)
        status = vb.veda_get_status(ws)
    finally:
        del os.environ["VEDA_TEST_WITHHOLD_ARRIVE"]
        del os.environ["VEDA_WAIT_LIMIT_MS"]
    assert status == 6  # VEDA_ERR_TIMEOUT
    # the same call without the hook succeeds and matches the oracle
    vb.veda_sparse_attn(prob, t["Q"], t["K"], t["V"], idx, O, lse, ws)
    assert vb.veda_get_status(ws) == 0
    bits = {n: ph.to_host_bits(t[n]) for n in "QKV"}
    units = workloads.sample_units(w, min(w.nT, 8), seed=5)
    O_o, lse_o, toks = oracle.sparse_attention(bits["Q"], bits["K"], bits["V"], idx.cpu().numpy(),
                                               w.grid, w.tile_shapes, w.scale, units=units)
    ph.check_attention(ph.to_host_bits(O), lse.cpu().numpy(), units, O_o, lse_o, toks)
