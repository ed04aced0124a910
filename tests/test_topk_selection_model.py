"""The Top-k kernel's selection, replayed in float32 on the CPU.

topk.cu selects the k largest scores of a row without sorting it:
  1. every score goes to one of 256 buckets spread linearly over [row min, row
     max], computed as t = fl(fl(x - min) * inv) with inv = min(256 / range,
     FLT_MAX) (0 for a zero or non-finite range) and bucket = min(int(t), 255);
  2. a histogram gives the bucket b* of the k-th largest score and the count of
     scores above it; inside b* the threshold is found exactly on
     order-preserving keys (pairwise ranks for up to 32 candidates, an 8-bit
     radix select otherwise);
  3. scores above the threshold are kept, and of those equal to it the
     lowest-index ones.
The argument for exactness is that the bucket is a non-decreasing function of
the score under correctly rounded fp32 subtraction and multiplication, and that
equal scores (-0.0 and +0.0 included) share a bucket.  This module replays those
steps with numpy float32 arithmetic on rows built to stress the argument and
checks the result against a stable sort (larger score first, ties to the lower
index), the rule of "Attention Structure Distillation", Execution, in "Veda:
Scalable Video Diffusion via Distilled Sparse Attention" (project page).
"""
import numpy as np
import pytest

F = np.float32
FMAX = np.finfo(np.float32).max


def order_key(x):
    u = int(np.array(x, dtype=np.float32).view(np.uint32))
    if (u << 1) & 0xFFFFFFFF == 0:
        u = 0  # -0.0 -> +0.0
    return (~u & 0xFFFFFFFF) if u & 0x80000000 else (u | 0x80000000)


def bucket(x, mn, inv):
    with np.errstate(all="ignore"):
        t = F(F(F(x) - F(mn)) * F(inv))
    return int(t) if t < F(255) else 255


def select_bin(hist, kr):
    run = 0
    for b in range(len(hist) - 1, -1, -1):
        if run + hist[b] >= kr:
            return b, run
        run += hist[b]
    raise AssertionError("rank beyond the histogram's total")


def radix_threshold(keys, kr):
    kmin, kmax = min(keys), max(keys)
    top = (kmin ^ kmax).bit_length()
    pmask = 0 if top == 32 else (~((1 << top) - 1)) & 0xFFFFFFFF
    prefix = kmin & pmask
    hi = top
    while hi > 0:
        shift = hi - 8 if hi >= 8 else 0
        dmask = 255 if hi >= 8 else (1 << hi) - 1
        hist = [0] * 256
        for key in keys:
            if key & pmask == prefix:
                hist[(key >> shift) & dmask] += 1
        digit, above = select_bin(hist, kr)
        kr -= above
        prefix |= digit << shift
        pmask |= dmask << shift
        hi -= 8
    return prefix, kr


def kernel_selection(row, k, cap=256):
    """Returns (ascending kept indices, which threshold branch ran)."""
    row = row.astype(np.float32)
    mn, mx = F(np.min(row)), F(np.max(row))
    with np.errstate(all="ignore"):
        rng = F(mx - mn)
        inv = F(min(F(256) / rng, FMAX)) if (rng > 0 and rng <= FMAX) else F(0)
    bk = [bucket(x, mn, inv) for x in row]
    hist = [0] * 256
    for b in bk:
        hist[b] += 1
    bstar, above = select_bin(hist, k)
    kr = k - above
    cand = [order_key(row[j]) for j in range(len(row)) if bk[j] == bstar]
    if len(cand) <= 32:
        branch = "ranks"
        hits = {(m, sum(o > m for o in cand)) for m in cand
                if sum(o > m for o in cand) < kr <= sum(o >= m for o in cand)}
        assert len({m for m, _ in hits}) == 1
        thr, gt = hits.pop()
        kr -= gt
    else:
        branch = "radix" if len(cand) <= cap else "radix over the row"
        thr, kr = radix_threshold(cand, kr)
    kept, equal_seen = [], 0
    for j, x in enumerate(row):
        key = order_key(x)
        if key > thr:
            kept.append(j)
        elif key == thr:
            if equal_seen < kr:
                kept.append(j)
            equal_seen += 1
    return kept, branch


def stable_topk(row, k):
    order = sorted(range(len(row)), key=lambda j: (-float(row[j]), j))
    return sorted(order[:k])


def rows():
    rnd = np.random.default_rng(3)
    for nT, k in ((240, 24), (37, 5), (600, 30), (8, 8), (1920, 96), (33, 1), (300, 299)):
        base = rnd.standard_normal(nT).astype(np.float32)
        yield "gaussian", base, k
        r = base.copy(); r[::5] = r[0]; r[1] = -0.0; r[2] = 0.0
        yield "ties and signed zeros", r, k
        yield "quantised", (np.round(base * 4) / 4).astype(np.float32), k
        r = base.copy(); r[nT // 3] = 3e38; r[nT // 2] = -3e38
        yield "range beyond fp32", r, k
        yield "constant", np.full(nT, 1.5, np.float32), k
        yield "sub-normal spacing", (rnd.integers(0, 5, nT) * 1e-45).astype(np.float32), k
        r = base.copy(); r[nT // 4] = 1e30
        yield "one outlier", r, k
    yield "outlier, long row", np.concatenate([[1e30], rnd.standard_normal(1999)]).astype(np.float32), 100
    yield "many equal at the threshold", \
        (np.round(rnd.standard_normal(2000) * 64) / 64).astype(np.float32), 500


def test_selection_matches_stable_sort_on_stress_rows():
    branches = set()
    for name, row, k in rows():
        kept, branch = kernel_selection(row, k)
        branches.add(branch)
        assert kept == stable_topk(row, k), name
    assert branches == {"ranks", "radix", "radix over the row"}


@pytest.mark.parametrize("seed", range(3))
def test_bucket_is_monotone_and_equal_scores_share_it(seed):
    rnd = np.random.default_rng(seed)
    x = np.sort(np.concatenate([rnd.standard_normal(3000), [-0.0, 0.0, 0.0, -0.0],
                                rnd.standard_normal(50) * 1e-40]).astype(np.float32))
    mn, mx = F(x[0]), F(x[-1])
    inv = F(min(F(256) / F(mx - mn), FMAX))
    b = [bucket(v, mn, inv) for v in x]
    assert all(b[i] <= b[i + 1] for i in range(len(b) - 1))
    assert bucket(F(-0.0), mn, inv) == bucket(F(0.0), mn, inv)
    assert b[0] == 0 and b[-1] == 255
