"""Randomised model of the mbarrier protocols of the two tensor-core attention kernels.

Each role of one CTA (TMA loader, table writer, MMA issuer, the softmax warps) is a generator
that follows the kernel's sequence of waits and arrivals; MMA commits and TMA completions land
later, each stream in issue order.  A seeded random scheduler with per-role speeds interleaves
them.  The checks: no deadlock; a parity wait passes only when exactly the phase it waits for
has completed (so it can neither pass on, nor miss, another phase); every arrival of one phase
belongs to one tile.  mbarrier semantics modelled: a phase completes when its count of
arrivals is reached; try_wait.parity(p) passes iff the current phase parity differs from p.

Modelled: the BF16 kernel (3 stages, P and row-max hand-over barriers per tile parity), the
TF32 kernel (2 stages, P over S in TMEM, S(t+1) after PV(t) completes) and the streaming kernel
for windows of more than 144 slots (Q by unit parity, K/V ring, S double-buffered in TMEM, P
hand-over per block parity).  The single-barrier variants of the BF16 and streaming protocols
must be caught.
"""
import random

import pytest

STAGES = 3


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.done = name, count, count, 0
        self.tile = None

    def arrive(self, tile, n=1):
        if self.tile is None:
            self.tile = tile
        assert self.tile == tile, f"{self.name}: phase {self.done} mixes tiles {self.tile} and {tile}"
        self.pending -= n
        assert self.pending >= 0, f"{self.name}: too many arrivals"
        if self.pending == 0:
            self.done += 1
            self.pending = self.count
            self.tile = None


def model(ntiles, has_tail=True, variant="kernel", seed=0, max_steps=2_000_000):
    """The BF16 kernel: 3 stages; one P buffer per row group (main rows, tail rows), handed to
    the PV MMA on p_full / p_full_t and released on p_empty / p_empty_t; the softmax warps
    finish tile t-1 (the epilogue) after handing over P(t).  variant="no_p_empty" drops the
    release waits (P placed so that it would not need them) while keeping single hand-over
    barriers: the combination that lets a warp lap another."""
    rng = random.Random(seed)
    n_soft_warps = 9 if has_tail else 8
    nsoft = 32 * n_soft_warps
    B = {}

    def mk(name, count):
        B[name] = Bar(name, count)

    for s in range(STAGES):
        mk(f"load{s}", 1)
        mk(f"empty{s}", 1 + nsoft)
        mk(f"table{s}", 32)
    for n, c in (("s_full", 1), ("s_empty", nsoft), ("p_full", 256), ("p_empty", 1), ("p_full_t", 32),
                 ("p_empty_t", 1), ("o_full", 1), ("o_empty", nsoft)):
        mk(n, c)
    for par in range(2):
        for h in range(2):
            mk(f"xmax{par}{h}", 128)

    def tma():
        for it in range(ntiles):
            s = it % STAGES
            yield ("wait", f"empty{s}", ((it // STAGES) & 1) ^ 1, it // STAGES - 1)
            yield ("tma", f"load{s}", it)

    def table():
        for it in range(ntiles):
            s = it % STAGES
            yield ("wait", f"empty{s}", ((it // STAGES) & 1) ^ 1, it // STAGES - 1)
            yield ("arrive", f"table{s}", it, 32)

    def mma():
        for j in range(ntiles + 1):
            if j < ntiles:
                s = j % STAGES
                yield ("wait", f"load{s}", (j // STAGES) & 1, j // STAGES)
                yield ("wait", "s_empty", (j & 1) ^ 1, j - 1)
                yield ("commit", [("s_full", j)])
            if j > 0:
                jt = j - 1
                s = jt % STAGES
                yield ("wait", "p_full", jt & 1, jt)
                yield ("wait", "o_empty", (jt & 1) ^ 1, jt - 1)
                yield ("commit", [("p_empty", jt)])
                if has_tail:
                    yield ("wait", "p_full_t", jt & 1, jt)
                    yield ("commit", [("p_empty_t", jt)])
                yield ("commit", [("o_full", jt), (f"empty{s}", jt)])

    def softmax(w):
        tail = w == 8
        half = 0 if tail else (w >> 2) & 1
        prev = None
        for it in range(ntiles + 1):
            if it < ntiles:
                s = it % STAGES
                yield ("wait", f"table{s}", (it // STAGES) & 1, it // STAGES)
                yield ("arrive", f"empty{s}", it, 32)
                yield ("wait", "s_full", it & 1, it)
                yield ("arrive", "s_empty", it, 32)
                if not tail:
                    par = it & 1
                    yield ("arrive", f"xmax{par}{half}", it, 32)
                    yield ("wait", f"xmax{par}{half ^ 1}", (it >> 1) & 1, it >> 1)
                if variant != "no_p_empty":
                    yield ("wait", "p_empty_t" if tail else "p_empty", (it & 1) ^ 1, it - 1)
                yield ("arrive", "p_full_t" if tail else "p_full", it, 32)
            if prev is not None:
                yield ("wait", "o_full", prev & 1, prev)
                yield ("arrive", "o_empty", prev, 32)
            if it < ntiles:
                prev = it

    actors = {"tma": tma(), "table": table(), "mma": mma()}
    for w in range(n_soft_warps):
        actors[f"w{w}"] = softmax(w)
    return run(actors, B, rng, max_steps)


def run(actors, B, rng, max_steps):
    """Random interleaving of the actors with in-order tensor-core and TMA completion streams."""
    cur = {k: None for k in actors}
    asyncq, tmaq, finished = [], [], set()
    weight = {k: rng.choice([0.05, 0.3, 1.0, 1.0, 3.0]) for k in actors}
    steps = 0
    while len(finished) < len(actors) or asyncq or tmaq:
        steps += 1
        assert steps < max_steps
        runnable = []
        for k, g in actors.items():
            if k in finished:
                continue
            if cur[k] is None:
                try:
                    cur[k] = next(g)
                except StopIteration:
                    finished.add(k)
                    continue
            op = cur[k]
            if op[0] == "wait":
                b = B[op[1]]
                if (b.done & 1) != op[2]:
                    assert b.done == op[3] + 1, f"{k}: wait on {op[1]} for phase {op[3]} passed with {b.done} done"
                else:
                    assert b.done == op[3], f"{k}: wait on {op[1]} for phase {op[3]} blocked with {b.done} done"
                    continue
            runnable.append(k)
        choices = runnable + (["async"] if asyncq else []) + (["tmaq"] if tmaq else [])
        if not choices and len(finished) == len(actors):
            break
        if not choices:
            raise AssertionError("deadlock: " + ", ".join(f"{k}:{cur[k]}" for k in actors if k not in finished))
        k = rng.choices(choices, weights=[weight.get(c, 0.5) for c in choices])[0]
        if k in ("async", "tmaq"):
            q = asyncq if k == "async" else tmaq
            bar, tile = q.pop(0)
            B[bar].arrive(tile)
            continue
        op = cur[k]
        cur[k] = None
        if op[0] == "arrive":
            B[op[1]].arrive(op[2], op[3])
        elif op[0] == "commit":
            asyncq.extend(op[1])
        elif op[0] == "tma":
            tmaq.append((op[1], op[2]))
    return steps


def model_tf32(ntiles, has_tail=True, seed=0, max_steps=2_000_000):
    """The TF32 kernel: 2 stages, P over S in TMEM, S(t+1) after PV(t) completes."""
    rng = random.Random(seed)
    ST = 2
    nw = 9 if has_tail else 8
    nsoft = 32 * nw
    B = {}

    def mk(name, count):
        B[name] = Bar(name, count)

    for s in range(ST):
        mk(f"load{s}", 1); mk(f"empty{s}", 1 + nsoft); mk(f"table{s}", 32)
    for n, c in (("s_full", 1), ("p_full", 256), ("p_full_t", 32), ("o_full", 1), ("o_empty", nsoft),
                 ("pv_done", 1), ("xmax0", 128), ("xmax1", 128)):
        mk(n, c)

    def tma():
        for it in range(ntiles):
            s = it % ST
            yield ("wait", f"empty{s}", ((it // ST) & 1) ^ 1, it // ST - 1)
            yield ("tma", f"load{s}", it)

    def table():
        for it in range(ntiles):
            s = it % ST
            yield ("wait", f"empty{s}", ((it // ST) & 1) ^ 1, it // ST - 1)
            yield ("arrive", f"table{s}", it, 32)

    def issue_s(j):
        s = j % ST
        yield ("wait", f"load{s}", (j // ST) & 1, j // ST)
        if j > 0:
            yield ("wait", "pv_done", (j - 1) & 1, j - 1)
            yield ("sync_pv", j - 1)     # the waiter itself observed PV(j-1) complete
        yield ("commit", [("s_full", j)])

    def mma():
        if ntiles:
            yield from issue_s(0)
        for t in range(ntiles):
            s = t % ST
            yield ("wait", "p_full", t & 1, t)
            yield ("wait", "o_empty", (t & 1) ^ 1, t - 1)
            if has_tail:
                yield ("wait", "p_full_t", t & 1, t)
            yield ("commit", [("o_full", t), (f"empty{s}", t), ("pv_done", t)])
            if t + 1 < ntiles:
                yield from issue_s(t + 1)

    def softmax(w):
        tail = w == 8
        half = (w >> 2) & 1
        prev = None
        for it in range(ntiles + 1):
            if it < ntiles:
                s = it % ST
                yield ("wait", f"table{s}", (it // ST) & 1, it // ST)
                yield ("arrive", f"empty{s}", it, 32)
                yield ("wait", "s_full", it & 1, it)
                if not tail:
                    yield ("arrive", f"xmax{half}", it, 32)
                    yield ("wait", f"xmax{half ^ 1}", it & 1, it)
                yield ("arrive", "p_full_t" if tail else "p_full", it, 32)
            if prev is not None:
                yield ("wait", "o_full", prev & 1, prev)
                yield ("arrive", "o_empty", prev, 32)
            if it < ntiles:
                prev = it

    actors = {"tma": tma(), "table": table(), "mma": mma()}
    for w in range(nw):
        actors[f"w{w}"] = softmax(w)
    return run(actors, B, rng, max_steps)


def test_bf16_protocol_holds_under_random_schedules():
    for seed in range(120):
        for tail in (True, False):
            model(ntiles=1 + seed % 13, has_tail=tail, seed=seed)


def test_dropping_the_p_release_wait_is_caught():
    """Without the p_empty waits a softmax warp can arrive for tile t+1 before another has
    arrived for tile t, and the tail warp can complete tile t+1's P before the MMA warp has
    waited for tile t's: the model must find it."""
    fails = 0
    for seed in range(60):
        try:
            model(ntiles=2 + seed % 12, has_tail=True, variant="no_p_empty", seed=seed)
        except AssertionError:
            fails += 1
    assert fails > 0


def test_tf32_protocol_holds_under_random_schedules():
    for seed in range(120):
        for tail in (True, False):
            model_tf32(ntiles=1 + seed % 11, has_tail=tail, seed=seed)


def model_stream(nunits, nblk, seed=0, variant="kernel", max_steps=2_000_000, stages=4):
    """The streaming kernel (windows of more than 144 slots): Q blocks by unit parity, K/V
    blocks through a ring of `stages` stages (4 in the kernel), S double-buffered by block parity in TMEM with P written
    back over it (S(j + 2) waits for PV(j)), P handed over on a barrier per block parity, one
    O accumulator read out by every softmax thread before the next PV.  variant="single_p_full"
    hands P over on one barrier, which a fast row can lap."""
    rng = random.Random(seed)
    S = stages
    B = {}

    def mk(name, count):
        B[name] = Bar(name, count)

    for b in range(2):
        mk(f"q_full{b}", 1); mk(f"q_free{b}", 1); mk(f"s_full{b}", 1); mk(f"s_free{b}", 1)
        mk(f"p_full{b}", 256)
    for s in range(S):
        mk(f"kv_full{s}", 1); mk(f"kv_empty{s}", 1 + 256); mk(f"tab_full{s}", 32)
    mk("o_full", 1); mk("o_empty", 256)
    for par in range(2):
        for h in range(2):
            mk(f"xmax{par}{h}", 128)
    nblocks = nunits * nblk

    def pfull(j):   # barrier name, parity, phase index of block j's P hand-over
        if variant == "single_p_full":
            return "p_full0", j & 1, j
        return f"p_full{j & 1}", (j >> 1) & 1, j >> 1

    def tma():
        j = 0
        for ui in range(nunits):
            qp = ui & 1
            yield ("wait", f"q_free{qp}", ((ui >> 1) & 1) ^ 1, (ui >> 1) - 1)
            yield ("tma", f"q_full{qp}", ui)
            for _ in range(nblk):
                s = j % S
                yield ("wait", f"kv_empty{s}", ((j // S) & 1) ^ 1, j // S - 1)
                yield ("tma", f"kv_full{s}", j)
                j += 1

    def table():
        for j in range(nblocks):
            s = j % S
            yield ("wait", f"kv_empty{s}", ((j // S) & 1) ^ 1, j // S - 1)
            yield ("arrive", f"tab_full{s}", j, 32)

    def mma():
        for jj in range(nblocks + 1):
            if jj < nblocks:
                ui, kb = divmod(jj, nblk)
                s, buf, qp = jj % S, jj & 1, ui & 1
                if kb == 0:
                    yield ("wait", f"q_full{qp}", (ui >> 1) & 1, ui >> 1)
                yield ("wait", f"kv_full{s}", (jj // S) & 1, jj // S)
                yield ("wait", f"s_free{buf}", ((jj >> 1) & 1) ^ 1, (jj >> 1) - 1)
                yield ("commit", [(f"s_full{buf}", jj)] + ([(f"q_free{qp}", ui)] if kb == nblk - 1 else []))
            if jj > 0:
                t = jj - 1
                name, par, ph = pfull(t)
                yield ("wait", name, par, ph)
                yield ("wait", "o_empty", (t & 1) ^ 1, t - 1)
                yield ("commit", [("o_full", t), (f"kv_empty{t % S}", t), (f"s_free{t & 1}", t)])

    def softmax(w):
        half = w >> 2
        j = 0
        for _ in range(nunits):
            for kb in range(nblk):
                s, buf = j % S, j & 1
                yield ("wait", f"tab_full{s}", (j // S) & 1, j // S)
                yield ("arrive", f"kv_empty{s}", j, 32)
                yield ("wait", f"s_full{buf}", (j >> 1) & 1, j >> 1)
                yield ("arrive", f"xmax{buf}{half}", j, 32)
                yield ("wait", f"xmax{buf}{half ^ 1}", (j >> 1) & 1, j >> 1)
                name, _, _ = pfull(j)
                yield ("arrive", name, j, 32)
                if kb > 0:
                    yield ("wait", "o_full", (j - 1) & 1, j - 1)
                    yield ("arrive", "o_empty", j - 1, 32)
                j += 1
            yield ("wait", "o_full", (j - 1) & 1, j - 1)
            yield ("arrive", "o_empty", j - 1, 32)

    actors = {"tma": tma(), "table": table(), "mma": mma()}
    for w in range(8):
        actors[f"w{w}"] = softmax(w)
    return run(actors, B, rng, max_steps)


def test_stream_protocol_holds_under_random_schedules():
    for seed in range(100):
        model_stream(nunits=1 + seed % 5, nblk=1 + seed % 4, seed=seed, stages=3 + seed % 2)


def test_stream_single_p_full_is_caught():
    """With one P hand-over barrier a softmax warp can arrive for block j + 1 before a warp of
    another row has arrived for block j (nothing between the two needs PV(j)): caught."""
    fails = 0
    for seed in range(60):
        try:
            model_stream(nunits=2 + seed % 3, nblk=2 + seed % 3, seed=seed, variant="single_p_full")
        except AssertionError:
            fails += 1
    assert fails > 0
