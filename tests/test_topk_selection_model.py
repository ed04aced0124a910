"""The Top-k kernels' selection, replayed in float32 on the CPU.

topk.cu selects the k largest scores of a row without sorting it.  For rows
longer than 2048 scores (the shared-memory kernel):
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


# ---------------------------------------------------------------- rows of up to 2048 scores
# (up to 1024 when a row does not start on a 16-byte boundary) topk.cu keeps
# such a row in registers: lane l holds the groups of four scores
# l, l + 32, ... (G = ceil(nT / 128) per lane, padding read as NaN), buckets are
# 7-bit, floor(127 * sat(fl(fl(x - min) * fl(1 / range)))) with NaN sent to 0 by
# the saturation, packed four per 32-bit word as 0x80 | bucket; byte-parallel
# counts drive a binary search for b*; the candidates' threshold is exact as
# above; the emitted list comes from per-word selected bytes and a prefix over
# lanes computed on four byte-sized counts per word.

M32 = 0xFFFFFFFF


def bucket7(x, mn, inv):
    with np.errstate(all="ignore"):
        t = F(F(F(x) - F(mn)) * F(inv))
    t = 0.0 if np.isnan(t) else min(max(float(t), 0.0), 1.0)
    return int(np.floor(127.0 * t))  # exact: 127 t needs 31 bits


def register_kernel_selection(row, k, rnd, cap=256):
    """Replays topk_reg_kernel on one row; returns (kept indices, branch, mask)."""
    row = row.astype(np.float32)
    nT = len(row)
    G = (nT + 127) // 128
    vals = np.full(128 * G, np.nan, np.float32)
    vals[:nT] = row
    mn, mx = F(np.nanmin(vals)), F(np.nanmax(vals))
    with np.errstate(all="ignore"):
        rng = F(mx - mn)
        inv = F(min(F(F(1) / rng), FMAX)) if (rng > 0 and rng <= FMAX) else F(0)
    # pk[u][lane]: word of group g = 32 u + lane
    pk = [[0] * 32 for _ in range(G)]
    for u in range(G):
        for lane in range(32):
            g = 32 * u + lane
            w = 0
            for e in range(4):
                w |= bucket7(vals[4 * g + e], mn, inv) << (8 * e)
            pk[u][lane] = w | 0x80808080

    def count_ge(P):
        T = P * 0x01010101
        tot = 0
        for lane in range(32):
            acc = 0
            for u in range(G):
                acc = (acc + ((((pk[u][lane] - T) & M32) & 0x80808080) >> 7)) & M32
            tot += ((acc * 0x01010101) & M32) >> 24
        return tot

    lo, hi, above = 0, 128, 0
    for _ in range(7):
        mid = (lo + hi) >> 1
        c = count_ge(mid)
        if c >= k:
            lo = mid
        else:
            hi, above = mid, c
    bstar, kr = lo, k - above
    Bs = bstar * 0x01010101
    cand, cm = [], [[False] * 32 for _ in range(G)]
    for u in range(G):
        for lane in range(32):
            z = (pk[u][lane] ^ Bs) & 0x7F7F7F7F
            eq = (~((z + 0x7F7F7F7F) & M32)) & 0x80808080
            if eq:
                cm[u][lane] = True
                for e in range(4):
                    j = 4 * (32 * u + lane) + e
                    if (eq >> (8 * e + 7)) & 1 and j < nT:
                        cand.append((order_key(row[j]), j))
    rnd.shuffle(cand)  # the kernel appends in atomic order
    c = len(cand)
    keys = [key for key, _ in cand]
    if c <= 32:
        branch = "ranks"
        hits = {(m, sum(o > m for o in keys)) for m in keys
                if sum(o > m for o in keys) < kr <= sum(o >= m for o in keys)}
        assert len({m for m, _ in hits}) == 1
        thr, gt = hits.pop()
        kr -= gt
    elif c <= cap:
        branch = "radix"
        thr, kr = radix_threshold(keys, kr)
    else:
        branch = "radix over the row"
        thr, kr = radix_threshold(
            [order_key(row[j]) for j in range(nT) if bucket7(row[j], mn, inv) == bstar], kr)
    bitmap = set()
    if c <= cap:
        neq = sum(key == thr for key in keys)
        for key, j in cand:
            keep = key > thr
            if key == thr:
                keep = True if neq == kr else \
                    sum(1 for o, i in cand if o == thr and i < j) < kr
            if keep:
                bitmap.add(j)
    else:
        seen = 0
        for j in range(nT):
            if bucket7(row[j], mn, inv) != bstar:
                continue
            key = order_key(row[j])
            if key > thr or (key == thr and seen < kr):
                bitmap.add(j)
            seen += key == thr
    T = (bstar + 1) * 0x01010101
    msel = [[0] * 32 for _ in range(G)]
    for u in range(G):
        for lane in range(32):
            m = ((pk[u][lane] - T) & M32) & 0x80808080
            if cm[u][lane]:
                g = 32 * u + lane
                nib = sum(1 << e for e in range(4) if 4 * g + e in bitmap)
                m |= (((nib * 0x00204081) & M32) & 0x01010101) << 7
            msel[u][lane] = m
    # prefix over lanes: four byte-sized counts per word, one scan per word
    out = [None] * k
    run = 0
    for q in range((G + 3) // 4):
        sw = [0] * 32
        for lane in range(32):
            for u in range(4 * q, min(G, 4 * q + 4)):
                sw[lane] |= bin(msel[u][lane]).count("1") << (8 * (u & 3))
        incl, acc = [], 0
        for lane in range(32):
            acc += sw[lane]
            assert all(((acc >> (8 * f)) & 0xFF) <= 128 for f in range(4))  # no carries
            incl.append(acc)
        tot = incl[31]
        for u in range(4 * q, min(G, 4 * q + 4)):
            for lane in range(32):
                pos = run + (((incl[lane] - sw[lane]) >> (8 * (u & 3))) & 0xFF)
                m = msel[u][lane]
                for e in range(4):
                    if (m >> (8 * e + 7)) & 1:
                        assert pos < k
                        out[pos] = 4 * (32 * u + lane) + e
                        pos += 1
            run += (tot >> (8 * (u & 3))) & 0xFF
    assert run == k and None not in out
    mask = np.zeros(nT, np.uint8)
    for u in range(G):
        for lane in range(32):
            for e in range(4):
                j = 4 * (32 * u + lane) + e
                if j < nT:
                    mask[j] = (msel[u][lane] >> (8 * e + 7)) & 1
    return out, branch, mask


def test_register_selection_matches_stable_sort_on_stress_rows():
    rnd = np.random.default_rng(5)
    branches = set()
    for name, row, k in rows():
        if len(row) > 2048:
            continue
        kept, branch, mask = register_kernel_selection(row, k, rnd)
        branches.add(branch)
        want = stable_topk(row, k)
        assert kept == want, name
        assert np.flatnonzero(mask).tolist() == want, name
    assert branches == {"ranks", "radix", "radix over the row"}


@pytest.mark.parametrize("seed", range(3))
def test_bucket7_is_monotone_and_equal_scores_share_it(seed):
    rnd = np.random.default_rng(seed)
    x = np.sort(np.concatenate([rnd.standard_normal(3000), [-0.0, 0.0, 0.0, -0.0],
                                rnd.standard_normal(50) * 1e-40]).astype(np.float32))
    mn, mx = F(x[0]), F(x[-1])
    inv = F(min(F(F(1) / F(mx - mn)), FMAX))
    b = [bucket7(v, mn, inv) for v in x]
    assert all(b[i] <= b[i + 1] for i in range(len(b) - 1))
    assert bucket7(F(-0.0), mn, inv) == bucket7(F(0.0), mn, inv)
    assert b[0] == 0 and b[-1] == 127
    assert bucket7(F(np.nan), mn, inv) == 0  # padding


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
