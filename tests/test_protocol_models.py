"""Models of two kernels' barrier protocols, run on the CPU with random
interleavings and asynchronous completions.

Each role of a kernel is a generator that yields while it waits; copies and
MMAs complete at random later points; mbarriers count arrivals and
transaction bytes per phase and answer parity waits the way the hardware
does (a parity wait passes while the barrier's current phase has the other
parity).  The assertions are the protocols' invariants: no buffer is
overwritten before its reader is done, every wait passes on the phase it
means, no count-1 barrier gets two arrivals in one phase, and nothing
deadlocks.  These are models of the designs in csrc/sparse_attn.cuh and
csrc/token_tc.cuh, not of their code line by line.
"""
import random

import pytest


class Bar:
    """An mbarrier: `n` arrivals and the announced bytes complete a phase."""

    def __init__(self, n, name):
        self.n, self.cnt, self.tx, self.ph, self.name = n, 0, 0, 0, name

    def arrive(self, expect=0):
        assert self.cnt < self.n, ("more arrivals than the count in one phase", self.name)
        self.cnt += 1
        self.tx += expect
        self._check()

    def complete_tx(self, b):
        self.tx -= b
        self._check()

    def _check(self):
        if self.cnt == self.n and self.tx == 0:
            self.cnt = 0
            self.ph += 1

    def passes(self, parity):
        return (self.ph & 1) != parity


def _wait(cond):
    while not cond():
        yield


def _run(gens, events, rnd, limit=400000):
    alive = list(gens)
    steps = 0
    while alive or events:
        steps += 1
        assert steps < limit, "no progress: deadlock"
        if events and (not alive or rnd.random() < 0.3):
            events.pop(rnd.randrange(len(events)))()
            continue
        g = rnd.choice(alive)
        try:
            next(g)
        except StopIteration:
            alive.remove(g)


# ---------------------------------------------------------------- attention

def _attention(T, seed, stages=4, gather_warps=4, soft_warps=4, send_before_read=False):
    """Two CTAs.  Per CTA: a logit-MMA issuer, an output-MMA issuer, gather
    warps, softmax warps.  A softmax warp reads the peer's rows of tile i,
    then sends its own rows of tile i+1's partial logits, then works on tile
    i; the peer's buffer for a tile parity is written again two tiles later.
    send_before_read swaps the first two steps (a planted mistake)."""
    rnd = random.Random(seed)
    events = []

    class CTA:
        def __init__(self):
            self.q_full = Bar(soft_warps, "q_full")
            self.kv_full = [Bar(gather_warps, "kv_full") for _ in range(stages)]
            self.kv_empty = [Bar(1, "kv_empty") for _ in range(stages)]
            self.s_full, self.s_empty = Bar(1, "s_full"), Bar(soft_warps, "s_empty")
            self.p_full, self.pv_done = Bar(soft_warps, "p_full"), Bar(1, "pv_done")
            self.x_full = [[Bar(1, "x_full") for _ in range(2)] for _ in range(2)]   # [parity][key half]
            self.stage = [None] * stages
            self.S, self.S_read = None, True
            self.P, self.P_busy = None, False
            self.x = [[[None] * soft_warps for _ in range(2)] for _ in range(2)]     # tile held, per warp rows
            self.x_read = [[[True] * soft_warps for _ in range(2)] for _ in range(2)]

    C = [CTA(), CTA()]

    def roles(me):
        b, pb = C[me], C[1 - me]

        def qk():
            yield from _wait(lambda: b.q_full.passes(0))
            for k in range(T):
                st = k % stages
                yield from _wait(lambda: b.kv_full[st].passes((k // stages) & 1))
                if k >= 1:
                    yield from _wait(lambda: b.s_empty.passes((k - 1) & 1))
                assert b.stage[st] == k and b.S_read, ("logit MMA inputs", me, k)

                def fin(k=k):
                    b.S, b.S_read = k, False
                    b.s_full.arrive()
                events.append(fin)
                yield

        def pv():
            for j in range(T):
                yield from _wait(lambda: b.p_full.passes(j & 1))
                st = j % stages
                assert b.stage[st] == j and b.P == j, ("output MMA inputs", me, j)
                b.P_busy = True

                def fin(st=st):
                    b.P_busy = False
                    b.stage[st] = None
                    b.kv_empty[st].arrive()
                    b.pv_done.arrive()
                events.append(fin)
                yield

        def gather():
            for k in range(T):
                st = k % stages
                yield from _wait(lambda: b.kv_empty[st].passes(((k // stages) & 1) ^ 1))
                assert b.stage[st] in (None, k), ("key stage overwritten", me, k)
                b.kv_full[st].arrive(expect=1)

                def fin(k=k, st=st):
                    b.stage[st] = k
                    b.kv_full[st].complete_tx(1)
                events.append(fin)
                yield

        def send(tile, w):
            xb = tile & 1
            for hf in range(2):
                assert pb.x_read[xb][hf][w], ("peer rows overwritten before read", me, tile)
            for hf in range(2):
                def fin(hf=hf):
                    pb.x[xb][hf][w] = tile
                    pb.x_read[xb][hf][w] = False
                    pb.x_full[xb][hf].complete_tx(1)
                events.append(fin)

        def load_send(tile, w):
            yield from _wait(lambda: b.s_full.passes(tile & 1))
            assert b.S == tile
            yield
            b.s_empty.arrive()
            if w == 0:
                b.S_read = True
                for hf in range(2):
                    b.x_full[tile & 1][hf].arrive(expect=soft_warps)
            send(tile, w)

        def softmax(w):
            b.q_full.arrive()
            yield
            if T:
                yield from load_send(0, w)
            for i in range(T):
                xb = i & 1
                if send_before_read and i + 1 < T:
                    yield from load_send(i + 1, w)
                for hf in range(2):
                    yield from _wait(lambda: b.x_full[xb][hf].passes((i >> 1) & 1))
                    assert b.x[xb][hf][w] == i, ("peer rows of another tile", me, i)
                yield
                for hf in range(2):
                    b.x_read[xb][hf][w] = True
                if not send_before_read and i + 1 < T:
                    yield from load_send(i + 1, w)
                yield
                if i >= 1:
                    yield from _wait(lambda: b.pv_done.passes((i - 1) & 1))
                assert not b.P_busy, ("P overwritten while the output MMA reads it", me, i)
                if w == 0:
                    b.P = i
                yield
                b.p_full.arrive()
            if T:
                yield from _wait(lambda: b.pv_done.passes((T - 1) & 1))

        return [qk(), pv()] + [gather() for _ in range(gather_warps)] + [softmax(w) for w in range(soft_warps)]

    _run(roles(0) + roles(1), events, rnd)


@pytest.mark.parametrize("T", [0, 1, 2, 3, 5, 9])
def test_attention_exchange_pipeline(T):
    for seed in range(25):
        _attention(T, seed)


def _fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    return False


def test_attention_model_catches_a_send_before_the_read():
    """The negative control: sending tile i+1 before reading tile i lets the
    peer overwrite rows not yet read (caught in some interleavings)."""
    assert any(_fails(lambda: _attention(T, seed, send_before_read=True)) for T in (3, 5, 9) for seed in range(25))


def test_attention_pipeline_needs_more_than_one_key_stage():
    """With one key stage the logit MMA of tile i+1 waits for the output MMA
    of tile i, which waits for the softmax of tile i, which waits for tile
    i+1's logits: a deadlock."""
    assert _fails(lambda: _attention(3, 0, stages=1))


# ---------------------------------------------------------------- refinement key stages

def _refinement_stages(S, tiles, seed, shared_empty):
    """Two TMA issuers and two MMA issuers; tile g goes to issuer g % 2 and to
    stage g % S.  The issuer of tile g waits until the MMA of tile g - S is
    done with the stage: on one barrier per stage shared by both issuers
    (shared_empty), or on a barrier of its own per stage, which the MMA of
    tile g - S completes for the issuer of tile g."""
    rnd = random.Random(seed)
    events = []
    k_full = [[Bar(1, "k_full") for _ in range(S)] for _ in range(2)]
    k_empty = [[Bar(1, "k_empty") for _ in range(S)] for _ in range(2)]
    k_empty_shared = [Bar(1, "k_empty") for _ in range(S)]
    stage = [None] * S

    def tma(me):
        eph, kph = 0, 0
        for g in range(tiles):
            st = g % S
            if g % 2 == me:
                if shared_empty:
                    yield from _wait(lambda: k_empty_shared[st].passes(kph ^ 1))
                    assert g < S or k_empty_shared[st].ph >= g // S, ("stale phase passed", g)
                elif g >= S:
                    bar, par = k_empty[me][st], (eph >> st) & 1
                    yield from _wait(lambda: bar.passes(par))
                    eph ^= 1 << st
                assert stage[st] is None, ("stage overwritten", g)
                k_full[me][st].arrive(expect=1)
                stage[st] = ("loading", g)

                def fin(g=g, st=st):
                    stage[st] = ("ready", g)
                    k_full[me][st].complete_tx(1)
                events.append(fin)
                yield
            if st == S - 1:
                kph ^= 1

    def mma(me):
        fph = 0
        for g in range(tiles):
            st = g % S
            if g % 2 == me:
                bar, par = k_full[me][st], (fph >> st) & 1
                yield from _wait(lambda: bar.passes(par))
                fph ^= 1 << st
                assert stage[st] == ("ready", g), ("MMA reads another tile", g, stage[st])

                def fin(st=st):
                    stage[st] = None
                    if shared_empty:
                        k_empty_shared[st].arrive()
                    else:
                        k_empty[(me + S) % 2][st].arrive()
                events.append(fin)
                yield

    _run([tma(0), tma(1), mma(0), mma(1)], events, rnd)


@pytest.mark.parametrize("S", [2, 3, 4])
def test_refinement_stage_barrier_per_issuer(S):
    for tiles in (1, 2, 5, 7, 13, 30):
        for seed in range(20):
            _refinement_stages(S, tiles, seed, shared_empty=False)


def test_refinement_stage_barrier_shared_by_two_issuers_fails():
    """The negative control: with one 'stage free' barrier per stage shared by
    both issuers and an odd stage count, some interleaving lets an issuer pass
    its parity wait on a phase two uses old."""
    failures = 0
    for tiles in (7, 13, 30):
        for seed in range(40):
            try:
                _refinement_stages(3, tiles, seed, shared_empty=True)
            except AssertionError:
                failures += 1
    assert failures > 0
