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


# ---------------------------------------------------------------------------
# The paired-CTA GEMM: two producers (one per CTA) whose loads complete on the
# first CTA's FULL barrier (two arrivals plus the bytes), one MMA issuer whose
# commits arrive on both CTAs' EMPTY / TFULL, one epilogue per CTA arriving on
# the first CTA's TEMPTY; then the exit drain. Failures elsewhere in the grid
# are modelled as an abort flag raised at a random moment, after which waits
# that honour it give up.

class TxBarrier(Barrier):
    def __init__(self, name, count=1):
        super().__init__(name, count)
        self.tx = 0

    def arrive(self, tx=0):
        self.tx += tx
        self.pending -= 1
        assert self.pending >= 0, self.name
        self._maybe_complete()

    def complete_tx(self, tx):
        self.tx -= tx
        self._maybe_complete()

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count


def simulate_pair(tiles, kblocks, rng, stages=6, abort_at=None, stats=None):
    full = [TxBarrier(f"full{s}", 2) for s in range(stages)]
    empty = [[Barrier(f"empty{r}{s}") for s in range(stages)] for r in range(2)]
    tfull = [[Barrier(f"tfull{r}{a}") for a in range(2)] for r in range(2)]
    tempty = [Barrier(f"tempty{a}", 2) for a in range(2)]
    drain = Barrier("drain")
    mma_pipe, copies = [], []  # commits in issue order; loads in flight
    issued = [0, 0]
    state = {"abort": False, "ticks": 0}

    def wait(bar, parity, honor_abort=True):
        while not bar.passed(parity):
            if honor_abort and state["abort"]:
                return False
            yield bar, parity, honor_abort
        return True

    def producer(r):
        i = 0
        for _ in range(tiles):
            for _ in range(kblocks):
                ok = yield from wait(empty[r][i % stages], ((i // stages) & 1) ^ 1)
                if not ok:
                    return
                full[i % stages].arrive(tx=1)
                copies.append(full[i % stages])
                i += 1
                issued[r] = i

    def mma():
        i, acc, acc_phase = 0, 0, 0
        for _ in range(tiles):
            if not (yield from wait(tempty[acc], acc_phase ^ 1)):
                break
            stop = False
            for _ in range(kblocks):
                if not (yield from wait(full[i % stages], (i // stages) & 1)):
                    stop = True
                    break
                mma_pipe.append([empty[0][i % stages], empty[1][i % stages]])
                i += 1
            if stop:
                break
            mma_pipe.append([tfull[0][acc], tfull[1][acc]])
            acc ^= 1
            acc_phase ^= acc == 0
        mma_pipe.append([drain])
        yield from wait(drain, 0, honor_abort=False)

    def epilogue(r):
        acc, acc_phase = 0, 0
        for _ in range(tiles):
            if not (yield from wait(tfull[r][acc], acc_phase)):
                return
            tempty[acc].arrive()
            acc ^= 1
            acc_phase ^= acc == 0

    def run(roles):
        waiting = {n: None for n in roles}
        live = dict(roles)
        idle = 0
        while live and idle < 400:
            state["ticks"] += 1
            if abort_at is not None and state["ticks"] >= abort_at:
                state["abort"] = True
            progressed = False
            if mma_pipe and rng.random() < 0.5:
                for b in mma_pipe.pop(0):
                    b.arrive()
                progressed = True
            if copies and rng.random() < 0.5:
                copies.pop(rng.randrange(len(copies))).complete_tx(1)
                progressed = True
            for name in rng.sample(list(live), len(live)):
                if rng.random() < 0.3:  # this role is late this time
                    continue
                w = waiting[name]
                if w is not None and not w[0].passed(w[1]) and not (w[2] and state["abort"]):
                    continue
                try:
                    waiting[name] = next(live[name])
                except StopIteration:
                    del live[name]
                progressed = True
            idle = 0 if progressed else idle + 1
        return live

    stuck = run({"producer0": producer(0), "producer1": producer(1), "mma": mma(),
                 "epilogue0": epilogue(0), "epilogue1": epilogue(1)})
    if stuck:
        return f"roles stuck: {sorted(stuck)}"

    def drain_loads():
        lo, hi = min(issued), max(issued)
        for i in range(lo, hi):
            full[i % stages].arrive()
        for i in range(max(hi - stages, 0), hi):
            yield from wait(full[i % stages], (i // stages) & 1, honor_abort=False)

    if stats is not None:
        stats.append(tuple(issued))
    stuck = run({"drain": drain_loads()})
    if stuck:
        return f"drain stuck, issued {issued}"
    if copies:
        return f"{len(copies)} loads still in flight at exit"
    if mma_pipe:
        return "MMA commits still pending at exit"
    return None


@pytest.mark.parametrize("tiles,kblocks", [(1, 1), (1, 5), (3, 2), (4, 7), (7, 13)])
def test_pair_gemm_pipeline_completes(tiles, kblocks):
    rng = random.Random(tiles * 100 + kblocks)
    for _ in range(40):
        assert simulate_pair(tiles, kblocks, rng) is None


@pytest.mark.parametrize("tiles,kblocks", [(2, 3), (4, 7), (6, 11)])
def test_pair_gemm_drains_every_load_after_an_abort(tiles, kblocks):
    """Wherever the abort lands, the roles unwind, the drain ends, and no load
    or commit is left in flight when the CTAs exit."""
    rng = random.Random(tiles * 7 + kblocks)
    stats = []
    for trial in range(120):
        res = simulate_pair(tiles, kblocks, rng, abort_at=rng.randrange(1, 60 + 10 * tiles * kblocks),
                            stats=stats)
        assert res is None, res
    # with more loads than stages, the case the drain's stand-in arrivals
    # exist for (one producer stopped before the other) did come up
    if tiles * kblocks > 6:
        assert any(a != b for a, b in stats)
