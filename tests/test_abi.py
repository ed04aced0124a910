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


# Every entry point that takes device buffers, with each required pointer in
# turn made NULL (VEDA_ERR_INVALID_ARG = 1) and each device pointer made
# misaligned (VEDA_ERR_ALIGN = 4).  The other pointers are a fake, 16-byte
# aligned address that is never dereferenced: validation fails before any
# copy or launch, and on a machine without a GPU a CUDA call would have
# returned VEDA_ERR_CUDA (5) instead.
#   D required device pointer   N nullable device pointer
#   H required host pointer     h nullable host pointer (left NULL)
#   C host candidate tilings    i / f: an integer / float argument
ENTRY_POINTS = {
    "veda_tripool": "PDDDDs",
    "veda_tile_score": "PDDDDDDs",
    "veda_topk_mask": "PDNDs",
    "veda_mask_fused": "PDDDDNDDs",
    "veda_sparse_attn": "PDDDNDNDs",
    "veda_forward": "PDDDDDDNNNDs",
    "veda_forward_host": "PHHHHHHhDDDDDDNDis",
    "veda_tile_search": "PCiDDDDDDDDDDs",
    "veda_teacher": "PDDDDDDDs",
    "veda_tile_recall": "PDDNDDs",
    "veda_distill_kl": "PDDDDDDfDDDDs",
    "veda_tile_score_noalloc": "PDDDDDs",
    "veda_noalloc_get_status": "sH",
}
FAKE, MISALIGNED = 0x10000, 0x10008


def _entry_args(vb, spec, bad=None, how=None):
    prob = _problem(vb)  # grid 4x16x32, tiles (2,8,8): nT = 16, k = 3
    cands = (ctypes.c_int32 * 3)(2, 8, 8)
    args = []
    for i, kind in enumerate(spec):
        if i == bad:
            args.append(None if how == "null" else ctypes.c_void_p(MISALIGNED))
        elif kind == "P":
            args.append(ctypes.byref(prob.c))
        elif kind == "C":
            args.append(ctypes.cast(cands, ctypes.c_void_p))
        elif kind == "i":
            args.append(1)
        elif kind == "f":
            args.append(1.0)
        elif kind in "sh":
            args.append(None)
        else:
            args.append(None if kind == "N" else ctypes.c_void_p(FAKE))
    return prob, cands, args


@pytest.mark.parametrize("name", sorted(ENTRY_POINTS))
def test_every_entry_point_rejects_bad_pointers_before_launch(lib, name):
    import torch
    import tile_sparse_attention_b200 as vb
    if torch.cuda.is_available():
        # the fake addresses must never reach a device: this check runs where
        # no GPU is visible, so a call that got past validation fails with
        # VEDA_ERR_CUDA instead of launching
        pytest.skip("uses fake device addresses; runs only without a visible GPU")
    spec = ENTRY_POINTS[name]
    fn = getattr(lib, name)
    for i, kind in enumerate(spec):
        if kind in "DHC":
            _, _, args = _entry_args(vb, spec, bad=i, how="null")
            assert fn(*args) == 1, f"{name}: NULL argument {i}"
            assert lib.veda_last_error()
        if kind in "DN":
            _, _, args = _entry_args(vb, spec, bad=i, how="misaligned")
            assert fn(*args) == 4, f"{name}: misaligned argument {i}"
