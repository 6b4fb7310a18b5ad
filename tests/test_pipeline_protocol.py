"""A model of the attention kernel's mbarrier protocol, run under randomized
schedules on the CPU, so that a change to the pipeline cannot deadlock the
kernel (which would surface on the GPU only as a bounded-wait timeout).

Roles, as in the kernel: a TMA producer over the K/V ring (4 stages with two
S buffers per query tile, 2 with one); one MMA issuer per query tile (S_t(j)
into S buffer j % sbuf, PV_t(j) reading P_t(j), S_t(j + sbuf) issued after
PV_t(j)); one softmax group per query tile that may wait for PV_t(j - 1)
before rescaling O. Barriers complete phases; a wait
names a parity and succeeds once the current phase's parity differs, exactly
the try_wait.parity rule, so a barrier that runs two phases ahead of its
waiter is a lost wake-up. Each issuer's commits complete in issue order.
"""
import random

import pytest


class Barrier:
    def __init__(self, name, count=1):
        self.name, self.count, self.pending, self.phase = name, count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, self.name
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def passed(self, parity):
        return (self.phase & 1) != parity


def simulate(nkv, rng, sbuf=2, p_full_per_buffer=True, rescale_at=()):
    ns = 4 if sbuf == 2 else 2
    bar = Barrier
    q_full = bar("q_full")
    kv_full = [bar(f"kv_full{s}") for s in range(ns)]
    kv_empty = [bar(f"kv_empty{s}", 2) for s in range(ns)]
    s_full = [[bar(f"s_full{t}{b}") for b in range(sbuf)] for t in range(2)]
    if p_full_per_buffer:
        p_full = [[bar(f"p_full{t}{b}") for b in range(sbuf)] for t in range(2)]
        p_wait = lambda t, j: (p_full[t][j % sbuf], (j // sbuf) & 1)
    else:  # one barrier per tile: the lost-wake-up layout
        one = [bar(f"p_full{t}") for t in range(2)]
        p_full = [[one[t]] * sbuf for t in range(2)]
        p_wait = lambda t, j: (one[t], j & 1)
    pv_done = [bar(f"pv_done{t}") for t in range(2)]
    o_full = [bar(f"o_full{t}") for t in range(2)]
    drain = [bar(f"drain{t}") for t in range(2)]
    pipe = {0: [], 1: []}

    def producer():
        q_full.arrive()
        for j in range(nkv):
            st = j % ns
            yield kv_empty[st], ((j // ns) & 1) ^ 1
            kv_full[st].arrive()

    def issuer(t):
        def issue_s(j):
            yield kv_full[j % ns], (j // ns) & 1
            pipe[t].append(s_full[t][j % sbuf])

        yield q_full, 0
        for j in range(min(sbuf, nkv)):
            yield from issue_s(j)
        for j in range(nkv):
            yield p_wait(t, j)
            pipe[t].extend([pv_done[t], kv_empty[j % ns]])
            if j + 1 == nkv:
                pipe[t].append(o_full[t])
            if j + sbuf < nkv:
                yield from issue_s(j + sbuf)
        pipe[t].append(drain[t])
        yield drain[t], 0

    def softmax(t):
        for j in range(nkv):
            yield s_full[t][j % sbuf], (j // sbuf) & 1
            if j > 0 and (t, j) in rescale_at:
                yield pv_done[t], (j - 1) & 1
            p_full[t][j % sbuf].arrive()
        yield o_full[t], 0

    roles = {"producer": producer(), "mma0": issuer(0), "mma1": issuer(1),
             "softmax0": softmax(0), "softmax1": softmax(1)}
    waiting = dict.fromkeys(roles)
    finished = set()
    idle = 0
    while idle < 300 and len(finished) < len(roles):
        progressed = False
        for t in (0, 1):
            if pipe[t] and rng.random() < 0.5:
                pipe[t].pop(0).arrive()
                progressed = True
        order = list(roles.items())
        rng.shuffle(order)
        for name, gen in order:
            if name in finished or rng.random() < 0.3:
                continue
            w = waiting[name]
            if w is not None and not w[0].passed(w[1]):
                continue
            try:
                waiting[name] = next(gen)
            except StopIteration:
                finished.add(name)
            progressed = True
        idle = 0 if progressed else idle + 1
    return {n: (w[0].name, w[1], w[0].phase) for n, w in waiting.items()
            if n not in finished and w is not None}


@pytest.mark.parametrize("sbuf", [1, 2])
@pytest.mark.parametrize("nkv", [1, 2, 3, 5, 8, 17, 33])
def test_attention_pipeline_never_stalls(nkv, sbuf):
    rng = random.Random(nkv)
    for _ in range(60):
        rescale = {(t, j) for t in range(2) for j in range(1, nkv) if rng.random() < 0.3}
        stuck = simulate(nkv, rng, sbuf=sbuf, rescale_at=rescale)
        assert not stuck, f"stalled with {nkv} KV tiles: {stuck}"


def test_one_p_barrier_per_tile_would_lose_wakeups():
    """With a single P barrier per query tile, a softmax group that finishes
    two steps before its issuer looks moves the barrier two phases and the
    issuer's parity wait never succeeds: the reason for one per S buffer."""
    rng = random.Random(7)
    stalls = sum(bool(simulate(8, rng, p_full_per_buffer=False)) for _ in range(60))
    assert stalls > 0
