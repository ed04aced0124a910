"""C-ABI checks that need no GPU: the library builds for sm_100a, loads, exports
every entry point that include/veda.h declares, and rejects invalid arguments
on the host (documented status codes, nothing launched, no CUDA call made)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "veda.h")


@pytest.fixture(scope="module")
def lib():
    from tile_sparse_attention_b200 import build as b
    import tile_sparse_attention_b200 as vb
    b.build()
    return vb.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(veda_[a-z_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("veda_tripool", "veda_tile_score", "veda_topk_mask", "veda_sparse_attn",
              "veda_forward", "veda_workspace_size", "veda_get_status", "veda_version",
              "veda_last_error"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} missing from libveda.so"


def _problem(vb, **kw):
    args = dict(B=1, H=2, d=128, grid=(4, 16, 32), tile_shapes=[(2, 8, 8)], k=3)
    args.update(kw)
    return vb.Problem(args["B"], args["H"], args["d"], args["grid"], args["tile_shapes"],
                      args["k"], args.get("scale", 0.0))


def _call_tripool(lib, prob, ptr=0x10000):
    p = ctypes.c_void_p(ptr)
    return lib.veda_tripool(ctypes.byref(prob.c), p, p, p, p, None)


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), 3),                                   # unsupported head dim
    (dict(tile_shapes=[(3, 8, 8)]), 2),                # grid not divisible
    (dict(tile_shapes=[(2, 8, 8), (1, 8, 8)]), 2),     # tile sizes differ
    (dict(tile_shapes=[(1, 4, 8)]), 3),                # tile size 32 unsupported
    (dict(H=300, tile_shapes=[(2, 8, 8)]), 3),         # too many heads
])
def test_problem_validation(lib, kw, code):
    import tile_sparse_attention_b200 as vb
    assert _call_tripool(lib, _problem(vb, **kw)) == code
    assert lib.veda_last_error()


def test_k_and_scale_validation(lib):
    import tile_sparse_attention_b200 as vb
    n = ctypes.c_size_t(0)
    assert lib.veda_workspace_size(ctypes.byref(_problem(vb, k=0).c), ctypes.byref(n)) == 1
    assert lib.veda_workspace_size(ctypes.byref(_problem(vb, k=17).c), ctypes.byref(n)) == 1
    assert lib.veda_workspace_size(ctypes.byref(_problem(vb, scale=-1.0).c), ctypes.byref(n)) == 1
    assert lib.veda_workspace_size(ctypes.byref(_problem(vb, k=16).c), ctypes.byref(n)) == 0
    assert n.value > 256


def test_pointer_validation(lib):
    import tile_sparse_attention_b200 as vb
    prob = _problem(vb)
    assert _call_tripool(lib, prob, ptr=0x10008) == 4          # misaligned
    p = ctypes.c_void_p(0x10000)
    assert lib.veda_tripool(ctypes.byref(prob.c), None, p, p, p, None) == 1   # NULL Q
    assert lib.veda_sparse_attn(ctypes.byref(prob.c), p, p, p, None, p, None, None, None) == 1


def test_workspace_size_matches_layout(lib):
    import tile_sparse_attention_b200 as vb
    prob = _problem(vb, B=2, H=3, tile_shapes=[(2, 8, 8)], k=5)
    nT, d = 16, 128
    stats = 2 * 3 * nT * 3 * d * 4
    proj = 2 * 3 * nT * 9 * d * 4
    S = 2 * 3 * nT * nT * 4
    idx = 2 * 3 * nT * 5 * 4
    r256 = lambda x: (x + 255) // 256 * 256
    want = 256 + 2 * r256(proj) + 2 * r256(stats) + r256(S) + r256(idx)
    assert vb.veda_workspace_size(prob) == want
