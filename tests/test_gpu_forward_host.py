"""veda_forward_host: the layer from pinned host buffers, pipelined over head
chunks, gives exactly the results of one veda_forward call (every step is
independent per batch entry and head, and each chunk runs the same kernels on
its own heads)."""
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tile_sparse_attention_b200 as m
    m.load_library()
    return m


def _run(vb, w, head_chunk, draw="cpu"):
    t = {n: v.cuda() for n, v in workloads.generate(w, device=draw).items()}
    prob = vb.Problem.from_workload(w)
    B, H, N, d = w.B, w.H, w.N, w.d
    ws = vb.alloc_workspace(prob)
    O_ref = torch.empty_like(t["Q"])
    lse_ref = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    vb.veda_forward(prob, t["Q"], t["K"], t["V"], t["Wq"], t["Wk"], O_ref, lse_ref, None, None, ws)
    host = {n: t[n].cpu().pin_memory() for n in ("Q", "K", "V", "Wq", "Wk")}
    hO = torch.empty(O_ref.shape, dtype=torch.bfloat16).pin_memory()
    hlse = torch.empty(lse_ref.shape, dtype=torch.float32).pin_memory()
    dev = {n: torch.empty_like(t[n]) for n in ("Q", "K", "V", "Wq", "Wk")}
    dO = torch.empty_like(O_ref)
    dlse = torch.empty_like(lse_ref)
    ws2 = vb.alloc_workspace(prob)
    vb.veda_forward_host(prob, host["Q"], host["K"], host["V"], host["Wq"], host["Wk"], hO, hlse,
                         dev["Q"], dev["K"], dev["V"], dev["Wq"], dev["Wk"], dO, dlse, ws2,
                         head_chunk)
    torch.cuda.current_stream().synchronize()
    assert vb.veda_get_status(ws2) == 0
    assert torch.equal(hO, O_ref.cpu()), "O differs from veda_forward"
    assert torch.equal(hlse, lse_ref.cpu()), "lse differs from veda_forward"


@pytest.mark.parametrize("name,make,chunk", [
    ("tiny_1", workloads.tiny, 1),
    ("480p_default", workloads.p480, 0),
    ("480p_5", workloads.p480, 5),
    ("720p_7", workloads.p720, 7),
    ("720p_all", workloads.p720, 40),
    ("b2_ragged", lambda: workloads.custom("b2", 2, 3, 64, (3, 16, 40), [(1, 8, 8)], 7), 2),
])
def test_forward_host_equals_forward(vb, name, make, chunk):
    _run(vb, make(), chunk)


def test_forward_host_long_video_default_chunk(vb):
    """The benchmarked end-to-end call: 245,760 tokens, 32 heads, 6 GB of host
    input, the default of one head per chunk (inputs drawn on the device)."""
    _run(vb, workloads.long_video(), 0, draw="cuda")


def test_forward_host_rejects_bad_chunk(vb):
    w = workloads.tiny()
    prob = vb.Problem.from_workload(w)
    z = torch.zeros((64,), dtype=torch.bfloat16)
    zf = torch.zeros((64,), dtype=torch.float32)
    dz = torch.zeros((64,), dtype=torch.bfloat16, device="cuda")
    dzf = torch.zeros((64,), dtype=torch.float32, device="cuda")
    ws = torch.zeros((4096,), dtype=torch.uint8, device="cuda")
    with pytest.raises(vb.VedaError):
        vb.veda_forward_host(prob, z, z, z, zf, zf, z, None, dz, dz, dz, dzf, dzf, dz, None, ws, 3)
