"""Barrier protocols of the three attention kernels, of the persistent score
GEMM (score_tc.cu: a TMA ring running on across blocks of S, two tensor-memory
accumulators drained by four epilogue warps) and of the projection
(proj_tc.cu: two raw buffers filled one half ahead, a shared lo buffer, two
accumulators), checked by random interleaving.

The tile-skipping attention kernels (sparse_attn.cu: one CTA per query tile;
sparse_attn_persistent.cu: persistent CTAs looping over query tiles with one
key-tile stream; sparse_attn_dual.cu: one query tile per CTA, two softmax
groups on alternate 64-key chunks) hand work between TMA producer threads, one
tcgen05-issuing thread and softmax warps through mbarriers waited on by phase
parity.  This module models those protocols -- the roles, the barriers and
their arrival counts, a tensor pipe that executes in issue order, copies that
land in any order -- and runs them under many random interleavings, checking
that

* every role finishes (no deadlock);
* every wait for completion c of a barrier happens while completion c - 1
  has occurred and c + 1 has not (a parity wait is exact only then: two
  phases behind it waits for ever, one phase ahead it passes at once);
* every product reads what it should: the ring stage holds K_g / V_g, the
  S/P buffer holds S_g / P_g, tensor memory holds Q of the right query tile;
* a query tile's output accumulator is read by the epilogue only after its
  last P V product, and before the next tile's first one overwrites it.

It models the kernels' protocol, not their code: a change to the barriers of
a kernel has to be made here as well.  A planted mistake (a producer that
refills a ring stage without waiting for its release) must trip a check.
"""
import random

import pytest


class Bar:
    """An mbarrier: `count` arrivals complete a phase; `done` counts completions."""

    def __init__(self, count):
        self.count = count
        self.pending = count
        self.done = 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, "more arrivals than the barrier's count"
        if self.pending == 0:
            self.done += 1
            self.pending = self.count


def passed(bar, c):
    """A wait for completion number c of `bar`.  The kernels wait on parity c & 1,
    which is right only while completion c - 1 has happened and c + 1 has not:
    a waiter two phases behind would wait for ever, and one that starts while
    completion c - 1 is still pending would pass at once."""
    assert bar.done <= c + 1, f"wait for completion {c} trails the barrier ({bar.done} done)"
    assert bar.done >= c, f"wait for completion {c} runs ahead of the barrier ({bar.done} done)"
    return bar.done >= c + 1


def run(roles, tma, tc, rnd):
    """Roles are generators that yield the predicate they wait on.  Each step
    advances one ready role, lands one pending copy (any of them) or executes
    the tensor pipe's oldest operation, chosen at random."""
    waits = {}
    live = []
    for r in roles:
        w = next(r, None)
        if w is not None:
            waits[r] = w
            live.append(r)
    while live or tma or tc:
        moves = [r for r in live if waits[r]()]
        if tma:
            moves.append("tma")
        if tc:
            moves.append("tc")
        assert moves, "deadlock: no role can proceed"
        m = rnd.choice(moves)
        if m == "tma":
            tma.pop(rnd.randrange(len(tma)))()
        elif m == "tc":
            tc.pop(0)()
        else:
            w = next(m, None)
            if w is None:
                live.remove(m)
            else:
                waits[m] = w


# ------------------------------------------------------------------ per query tile
def model_per_tile(k, NS, seed, p_rescale=0.3, release_wait=True):
    """sparse_attn.cu: Q staged and copied to tensor memory once; a K/V ring of NS
    stages, each released by one commit after P_j V_j; two S/P buffers; the
    issuer runs P_j V_j and then Q K_{j+2}^T."""
    rnd = random.Random(seed)
    bq, bq_tmem = Bar(1), Bar(4)
    k_full = [Bar(1) for _ in range(NS)]
    v_full = [Bar(1) for _ in range(NS)]
    kv_empty = [Bar(1) for _ in range(NS)]
    s_full, p_full = [Bar(1), Bar(1)], [Bar(4), Bar(4)]
    tma, tc = [], []
    st = {"K": [None] * NS, "V": [None] * NS, "Qs": False, "Qt": [False] * 4,
          "S": [None, None], "P": [[None, None] for _ in range(4)], "O": 0}

    def producer():
        def q_landed():
            st["Qs"] = True
            bq.arrive()
        tma.append(q_landed)
        for j in range(k):
            s, n = j % NS, j // NS
            if n > 0 and release_wait:
                yield lambda: passed(kv_empty[s], n - 1)

            def kl(s=s, j=j):
                st["K"][s] = j
                k_full[s].arrive()

            def vl(s=s, j=j):
                st["V"][s] = j
                v_full[s].arrive()
            tma.append(kl)
            tma.append(vl)

    def issuer():
        yield lambda: passed(bq_tmem, 0)

        def issue_qk(j):
            s, b = j % NS, j & 1
            yield lambda: passed(k_full[s], j // NS)

            def op():
                assert st["K"][s] == j, "Q K^T read a ring stage that no longer holds its K tile"
                assert all(st["Qt"]), "Q K^T before Q reached tensor memory"
                st["S"][b] = j
            tc.append(op)
            tc.append(s_full[b].arrive)
        yield from issue_qk(0)
        if k > 1:
            yield from issue_qk(1)
        for j in range(k):
            s, b = j % NS, j & 1
            yield lambda: passed(p_full[b], j >> 1)
            yield lambda: passed(v_full[s], j // NS)

            def op(j=j, s=s, b=b):
                assert st["V"][s] == j, "P V read a ring stage that no longer holds its V tile"
                assert all(st["P"][w][b] == j for w in range(4)), "P V read a stale P buffer"
                assert st["O"] == j
                st["O"] = j + 1
            tc.append(op)
            tc.append(kv_empty[s].arrive)
            if j + 2 < k:
                yield from issue_qk(j + 2)

    def softmax(w):
        yield lambda: passed(bq, 0)
        assert st["Qs"]
        st["Qt"][w] = True
        bq_tmem.arrive()
        for j in range(k):
            b = j & 1
            yield lambda: passed(s_full[b], j >> 1)
            assert st["S"][b] == j, "the softmax read a stale S buffer"
            if j > 0 and rnd.random() < p_rescale:  # O rescale: P_{j-1} V_{j-1} landed first
                yield lambda: passed(kv_empty[(j - 1) % NS], (j - 1) // NS)
                assert st["O"] == j
            st["P"][w][b] = j
            p_full[b].arrive()
        yield lambda: passed(kv_empty[(k - 1) % NS], (k - 1) // NS)
        assert st["O"] == k, "the epilogue read O before the last P V product"

    run([producer(), issuer()] + [softmax(w) for w in range(4)], tma, tc, rnd)


# ------------------------------------------------------------------ persistent
def model_persistent(n_tiles, k, NS, seed, p_rescale=0.3):
    """sparse_attn_persistent.cu: the CTA's query tiles n = 0..n_tiles-1 form one
    key-tile stream g = n*k + j for the K/V ring and the two S/P buffers; Q of
    tile n is staged in shared memory and copied to tensor-memory buffer n & 1
    (q_full / q_free / q_tmem), Q of tile n+1 right after the last P of tile n,
    so tile n+1's first products can run during tile n's epilogue."""
    rnd = random.Random(seed)
    total = n_tiles * k
    q_full, q_free = Bar(1), Bar(4)
    q_tmem = [Bar(4), Bar(4)]
    k_full = [Bar(1) for _ in range(NS)]
    v_full = [Bar(1) for _ in range(NS)]
    kv_empty = [Bar(1) for _ in range(NS)]
    s_full, p_full = [Bar(1), Bar(1)], [Bar(4), Bar(4)]
    tma, tc = [], []
    st = {"K": [None] * NS, "V": [None] * NS, "Qs": None,
          "Qt": [[None, None] for _ in range(4)], "S": [None, None],
          "P": [[None, None] for _ in range(4)], "O": (None, 0), "O_read": [-1] * 4}

    def producer():
        for n in range(n_tiles):
            if n > 0:
                yield lambda: passed(q_free, n - 1)

            def q_landed(n=n):
                st["Qs"] = n
                q_full.arrive()
            tma.append(q_landed)
            for j in range(k):
                g = n * k + j
                s, f = g % NS, g // NS
                if f > 0:
                    yield lambda: passed(kv_empty[s], f - 1)

                def kl(s=s, g=g):
                    st["K"][s] = g
                    k_full[s].arrive()

                def vl(s=s, g=g):
                    st["V"][s] = g
                    v_full[s].arrive()
                tma.append(kl)
                tma.append(vl)

    def issuer():
        cnt = {"g": 0, "n": 0, "j": 0}  # the next Q K^T: stream index, query tile, key tile

        def issue_next_qk():
            g, n = cnt["g"], cnt["n"]
            s, b = g % NS, g & 1
            if cnt["j"] == 0:
                yield lambda: passed(q_tmem[n & 1], n >> 1)
            yield lambda: passed(k_full[s], g // NS)

            def op():
                assert st["K"][s] == g, "Q K^T read a ring stage that no longer holds its K tile"
                assert all(st["Qt"][w][n & 1] == n for w in range(4)), \
                    "Q K^T read a tensor-memory Q buffer that does not hold its query tile"
                st["S"][b] = g
            tc.append(op)
            tc.append(s_full[b].arrive)
            cnt["g"] += 1
            cnt["j"] += 1
            if cnt["j"] == k:
                cnt["j"] = 0
                cnt["n"] += 1
        if total > 0:
            yield from issue_next_qk()
        if total > 1:
            yield from issue_next_qk()
        for g in range(total):
            s, b, n, j = g % NS, g & 1, g // k, g % k
            yield lambda: passed(p_full[b], g >> 1)
            yield lambda: passed(v_full[s], g // NS)

            def op(g=g, s=s, b=b, n=n, j=j):
                assert st["V"][s] == g, "P V read a ring stage that no longer holds its V tile"
                assert all(st["P"][w][b] == g for w in range(4)), "P V read a stale P buffer"
                if j == 0:
                    assert all(r == n - 1 for r in st["O_read"]), \
                        "the first P V of a tile overwrote O before the epilogue read it"
                    st["O"] = (n, 1)
                else:
                    assert st["O"] == (n, j)
                    st["O"] = (n, j + 1)
            tc.append(op)
            tc.append(kv_empty[s].arrive)
            if cnt["g"] < total:
                yield from issue_next_qk()

    def softmax(w):
        def copy_q(n):
            yield lambda: passed(q_full, n)
            assert st["Qs"] == n, "the staging buffer does not hold Q of this tile"
            st["Qt"][w][n & 1] = n
            q_tmem[n & 1].arrive()
            q_free.arrive()
        if n_tiles > 0:
            yield from copy_q(0)
        for n in range(n_tiles):
            for j in range(k):
                g = n * k + j
                b = g & 1
                yield lambda: passed(s_full[b], g >> 1)
                assert st["S"][b] == g, "the softmax read a stale S buffer"
                if j > 0 and rnd.random() < p_rescale:
                    yield lambda: passed(kv_empty[(g - 1) % NS], (g - 1) // NS)
                    assert st["O"] == (n, j)
                st["P"][w][b] = g
                p_full[b].arrive()
            if n + 1 < n_tiles:
                yield from copy_q(n + 1)
            g_last = n * k + k - 1
            yield lambda: passed(kv_empty[g_last % NS], g_last // NS)
            assert st["O"] == (n, k), "the epilogue read O before the tile's last P V product"
            st["O_read"][w] = n

    run([producer(), issuer()] + [softmax(w) for w in range(4)], tma, tc, rnd)


# ------------------------------------------------------------------ two softmax groups
def model_dual(k, seed, p_rescale=0.3, release_wait=True, q_gate=True, pv_wait=True,
               free_wait=True, NS=6):
    """sparse_attn_dual.cu: one query tile; its selected key tiles are processed
    in 64-key chunks n = 0..2k-1 from one ring (two producers taking alternate
    key tiles, each with its own 3 stages; Q staged in the last stage, gated by
    q_tmem); three S/P buffers (chunk n in buffer n % 3); softmax group
    g = n % 2 takes alternate chunks and accumulates its own O_g.  One thread
    issues S(0..2), then per chunk: wait P(n), O_g += P(n) V (commits: stage
    release, pv_done[g], and o_done[g] after the group's last), then
    S(n + 3) = Q K^T into the buffer P(n) V read.  A group rescales O_g only
    after pv_done[g] reports its previous P V, and reads O_g (both groups'
    accumulators, after a barrier of the eight warps) after o_done[g].
    free_wait=False plants S(n + 3) ahead of P(n) V in the issue order."""
    rnd = random.Random(seed)
    chunks = 2 * k
    q_full, q_tmem = Bar(1), Bar(8)
    kv_full = [Bar(1) for _ in range(NS)]  # K and V halves land on one barrier
    kv_empty = [Bar(1) for _ in range(NS)]
    s_full = [Bar(1) for _ in range(3)]
    p_full = [Bar(4) for _ in range(3)]
    pv_done = [Bar(1), Bar(1)]
    o_done = [Bar(1), Bar(1)]
    tma, tc = [], []
    st = {"K": [None] * NS, "V": [None] * NS, "Qt": [False] * 8, "S": [None] * 3,
          "P": [[None] * 4 for _ in range(3)], "Pread": [-1] * 3, "O": [0, 0],
          "read": [False, False]}
    mine = [False, False]
    R = NS // 2

    def stage(n):
        j, hh = n >> 1, n & 1
        m = 2 * (j >> 1) + hh
        return R * (j & 1) + m % R, m // R

    def q_loader():
        def q_landed():
            st["K"][NS - 1] = "Q"
            q_full.arrive()
        tma.append(q_landed)
        yield lambda: passed(q_full, 0)

    def producer(par):
        for j in range(par, k, 2):
            for hh in range(2):
                n = 2 * j + hh
                s, u = stage(n)
                if u > 0 and release_wait:
                    yield lambda: passed(kv_empty[s], u - 1)
                elif u == 0 and s == NS - 1 and q_gate:
                    yield lambda: passed(q_tmem, 0)

                def kvl(s=s, n=n):
                    # the barrier completes once both copies landed
                    st["K"][s] = n
                    st["V"][s] = n
                    kv_full[s].arrive()
                tma.append(kvl)

    def issue_qk(n):
        s, u = stage(n)
        b = n % 3
        yield lambda: passed(kv_full[s], u)

        def op(n=n, s=s, b=b):
            assert st["K"][s] == n, "Q K^T read a ring stage that no longer holds its K half"
            assert all(st["Qt"]), "Q K^T before Q reached tensor memory"
            assert n < 3 or st["Pread"][b] == n - 3, \
                "S overwrote a P buffer before its P V product read it"
            st["S"][b] = n
        tc.append(op)
        tc.append(s_full[b].arrive)

    def issuer():
        yield lambda: passed(q_tmem, 0)
        for n in range(min(3, chunks)):
            yield from issue_qk(n)
        for n in range(chunks):
            s, u = stage(n)
            b, g = n % 3, n % 2
            yield lambda: passed(p_full[b], n // 3)  # V landed with K (S(n) waited)
            if not free_wait and n + 3 < chunks:  # planted: S(n + 3) ahead of P(n) V
                yield from issue_qk(n + 3)

            def op(n=n, s=s, b=b, g=g):
                assert st["V"][s] == n, "P V read a ring stage that no longer holds its V half"
                assert all(st["P"][b][w] == n for w in range(4)), "P V read a stale P buffer"
                assert st["S"][b] == n, "the P buffer was overwritten before P V read it"
                assert st["O"][g] == n // 2
                assert not st["read"][g], "P V after the epilogue read O"
                st["Pread"][b] = n
                st["O"][g] += 1
            tc.append(op)
            tc.append(kv_empty[s].arrive)
            tc.append(pv_done[g].arrive)
            if n + 2 >= chunks:
                tc.append(o_done[g].arrive)
            if free_wait and n + 3 < chunks:
                yield from issue_qk(n + 3)

    def softmax(g, w):
        yield lambda: passed(q_full, 0)
        assert st["K"][NS - 1] == "Q", "the Q staging was overwritten before the copy"
        st["Qt"][4 * g + w] = True
        q_tmem.arrive()
        i = 0
        for n in range(g, chunks, 2):
            b = n % 3
            yield lambda: passed(s_full[b], n // 3)
            assert st["S"][b] == n, "the softmax read a stale S buffer"
            if i > 0 and rnd.random() < p_rescale:  # O_g rescale
                if pv_wait:
                    yield lambda: passed(pv_done[g], i - 1)
                assert st["O"][g] == i, "O rescaled before the group's previous P V landed"
            st["P"][b][w] = n
            p_full[b].arrive()
            i += 1
        yield lambda: passed(o_done[g], 0)
        assert st["O"][g] == i, "the epilogue read O before the group's last P V product"
        # the merge reads both accumulators, after both groups passed this point
        # (a barrier over the eight softmax warps)
        mine[g] = True
        yield lambda: all(mine)
        assert st["O"] == [(chunks + 1) // 2, chunks // 2]
        st["read"][g] = True

    run([q_loader(), producer(0), producer(1), issuer()]
        + [softmax(g, w) for g in range(2) for w in range(4)], tma, tc, rnd)


@pytest.mark.parametrize("k", [1, 2, 3, 4, 7])
def test_dual_protocol(k):
    for seed in range(30):
        model_dual(k, seed)


def test_dual_planted_mistakes_are_caught():
    for kw in (dict(release_wait=False), dict(q_gate=False), dict(pv_wait=False),
               dict(free_wait=False)):
        caught = 0
        for seed in range(40):
            try:
                model_dual(5, seed, **kw)
            except AssertionError:
                caught += 1
        assert caught > 0, kw


@pytest.mark.parametrize("NS", [2, 3, 4])
@pytest.mark.parametrize("k", [1, 2, 3, 5, 8])
def test_per_query_tile_protocol(k, NS):
    for seed in range(25):
        model_per_tile(k, NS, seed)


@pytest.mark.parametrize("NS", [3, 4])
@pytest.mark.parametrize("k", [1, 2, 3, 5])
@pytest.mark.parametrize("n_tiles", [0, 1, 2, 3, 5])
def test_persistent_protocol(n_tiles, k, NS):
    for seed in range(12):
        model_persistent(n_tiles, k, NS, seed)


def test_a_planted_refill_race_is_caught():
    """Without the wait for a stage's release, some interleaving overwrites a K or
    V tile before its product reads it."""
    caught = 0
    for seed in range(40):
        try:
            model_per_tile(8, 2, seed, release_wait=False)
        except AssertionError:
            caught += 1
    assert caught > 0


# ------------------------------------------------------------------ score GEMM
def model_score(n_blocks, KB, NS, seed, release_wait=True, acc_wait=True):
    """score_tc.cu: a persistent CTA computes n_blocks blocks of S, each KB K
    blocks long; the TMA ring of NS stages runs on across blocks; block lt is
    accumulated in tensor-memory accumulator lt & 1, released by the four
    epilogue warps once they have read it back."""
    rnd = random.Random(seed)
    full = [Bar(1) for _ in range(NS)]
    empty = [Bar(1) for _ in range(NS)]
    acc_full, acc_empty = [Bar(1), Bar(1)], [Bar(4), Bar(4)]
    tma, tc = [], []
    st = {"ring": [None] * NS, "acc": [None, None]}  # acc: (block, products so far)
    written = []

    def producer():
        g = 0
        for lt in range(n_blocks):
            for kb in range(KB):
                s, n = g % NS, g // NS
                if n > 0 and release_wait:
                    yield lambda s=s, n=n: passed(empty[s], n - 1)

                def landed(s=s, lt=lt, kb=kb):
                    st["ring"][s] = (lt, kb)
                    full[s].arrive()
                tma.append(landed)
                g += 1

    def issuer():
        g = 0
        for lt in range(n_blocks):
            a, use = lt & 1, lt >> 1
            if use > 0 and acc_wait:
                yield lambda a=a, use=use: passed(acc_empty[a], use - 1)
            for kb in range(KB):
                s = g % NS
                yield lambda s=s, g=g: passed(full[s], g // NS)

                def mma(s=s, lt=lt, kb=kb, a=a):
                    assert st["ring"][s] == (lt, kb), "product reads the wrong ring stage"
                    if kb == 0:
                        st["acc"][a] = (lt, 1)
                    else:
                        assert st["acc"][a] == (lt, kb), "accumulator overwritten mid-block"
                        st["acc"][a] = (lt, kb + 1)
                tc.append(mma)
                tc.append(lambda s=s: empty[s].arrive())
                g += 1
            tc.append(lambda a=a: acc_full[a].arrive())

    def epilogue(w):
        for lt in range(n_blocks):
            a, use = lt & 1, lt >> 1
            yield lambda a=a, use=use: passed(acc_full[a], use)
            assert st["acc"][a] == (lt, KB), "epilogue reads an incomplete block"
            yield lambda: True  # the read takes time: other roles may move
            assert st["acc"][a] == (lt, KB), "accumulator overwritten while being read"
            written.append((w, lt))
            acc_empty[a].arrive()

    run([producer(), issuer()] + [epilogue(w) for w in range(4)], tma, tc, rnd)
    assert sorted(written) == [(w, lt) for w in range(4) for lt in range(n_blocks)]


@pytest.mark.parametrize("n_blocks,KB,NS", [(1, 3, 4), (2, 1, 4), (5, 3, 4), (7, 2, 6), (4, 9, 4),
                                            (6, 1, 2)])
def test_score_protocol(n_blocks, KB, NS):
    for seed in range(300):
        model_score(n_blocks, KB, NS, seed)


@pytest.mark.parametrize("mistake", ["release_wait", "acc_wait"])
def test_score_planted_mistakes_are_caught(mistake):
    caught = 0
    for seed in range(300):
        try:
            model_score(5, 3, 4, seed, **{mistake: False})
        except AssertionError:
            caught += 1
    assert caught > 0, f"dropping {mistake} went unnoticed"


# ------------------------------------------------------------------ projection
def model_projection(n_blocks, halves, seed, acc_wait=True, done_wait=True, full_wait=True):
    """proj_tc.cu: warps 0..3 (one role: they act together) take each half of
    a block's statistics from one of two raw buffers (the next half's copy goes
    out once this half's products are issued), split it into a shared lo
    buffer, and issue its products into accumulator lb & 1; warps 4..7 read a
    finished accumulator back and release it."""
    rnd = random.Random(seed)
    full, done = Bar(1), Bar(1)
    acc_full, acc_empty = [Bar(1), Bar(1)], [Bar(4), Bar(4)]
    tma, tc = [], []
    st = {"raw": [None, None], "lo": None, "acc": [None, None]}
    written = []

    def load(lb, hk, g):
        def landed():
            st["raw"][g & 1] = (lb, hk)
            full.arrive()
        tma.append(landed)

    def main():
        g = 0
        if n_blocks:
            load(0, 0, 0)
        for lb in range(n_blocks):
            a, use = lb & 1, lb >> 1
            if use > 0 and acc_wait:
                yield lambda a=a, use=use: passed(acc_empty[a], use - 1)
            for hk in range(halves):
                if full_wait:
                    yield lambda g=g: passed(full, g)
                st["lo"] = st["raw"][g & 1]  # the split reads the raw half, writes lo

                def mma(lb=lb, hk=hk, g=g, a=a):
                    assert st["raw"][g & 1] == (lb, hk), "products read the wrong raw half"
                    assert st["lo"] == (lb, hk), "products read the wrong lo half"
                    if hk == 0:
                        st["acc"][a] = (lb, 1)
                    else:
                        assert st["acc"][a] == (lb, hk), "accumulator overwritten mid-block"
                        st["acc"][a] = (lb, hk + 1)
                tc.append(mma)
                tc.append(done.arrive)
                if hk + 1 == halves:
                    tc.append(lambda a=a: acc_full[a].arrive())
                if hk + 1 < halves:
                    load(lb, hk + 1, g + 1)
                elif lb + 1 < n_blocks:
                    load(lb + 1, 0, g + 1)
                if done_wait:
                    yield lambda g=g: passed(done, g)
                g += 1

    def epilogue(w):
        for lb in range(n_blocks):
            a, use = lb & 1, lb >> 1
            yield lambda a=a, use=use: passed(acc_full[a], use)
            assert st["acc"][a] == (lb, halves), "epilogue reads an incomplete block"
            yield lambda: True
            assert st["acc"][a] == (lb, halves), "accumulator overwritten while being read"
            written.append((w, lb))
            acc_empty[a].arrive()

    run([main()] + [epilogue(w) for w in range(4)], tma, tc, rnd)
    assert sorted(written) == [(w, lb) for w in range(4) for lb in range(n_blocks)]


@pytest.mark.parametrize("n_blocks,halves", [(1, 2), (2, 1), (5, 2), (7, 1), (4, 2)])
def test_projection_protocol(n_blocks, halves):
    for seed in range(300):
        model_projection(n_blocks, halves, seed)


@pytest.mark.parametrize("mistake", ["acc_wait", "done_wait", "full_wait"])
def test_projection_planted_mistakes_are_caught(mistake):
    caught = 0
    for seed in range(300):
        try:
            model_projection(5, 2, seed, **{mistake: False})
        except AssertionError:
            caught += 1
    assert caught > 0, f"dropping {mistake} went unnoticed"
