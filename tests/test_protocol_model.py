"""A model of the dense attention kernel's synchronisation protocol, run
under random interleavings on the CPU (race detection without a GPU).

The kernel (attn_dual_kernel.cuh) coordinates a Q/K producer, a V producer,
one MMA-issuing thread, two softmax groups and the epilogue through
mbarriers whose waits name a phase only by its parity.  The model keeps the
kernel's barrier set and the parity each wait uses, gives every barrier the
PTX semantics (a parity wait returns once the phase of that parity has
completed, so it is only unambiguous while the barrier is at most one phase
behind or ahead), runs the tensor pipe in issue order, completes TMA copies
in any order, and explores random schedules.  At every wait that returns it
checks that the event the wait stands for has really happened, and at every
buffer access that nothing else still needs the buffer:

* a K or V ring slot is refilled only after the MMA that read it executed;
* the softmax reads S of tile j only after Q.K^T(j) executed, and O of its
  group is rescaled only while no P.V into it is waiting in the pipe;
* P.V(j) reads the P of tile j and the V of tile j;
* the epilogue reads O only after every P.V into it executed.

A run that deadlocks, or reaches a check that fails, fails the test.  The
planted-defect tests check that the model reports each of a few defects,
among them the two this barrier scheme once had in the sparse kernel.

The second model is the persistent sparse kernel (attn_kernel.cuh): one
softmax group, one O accumulator, and a CTA that loops over work items
(query groups) with one tile counter for all of them, so barriers carry
phases across items; the Q buffer is refilled for the next item once the
current item's last Q.K^T has executed (a "Q empty" barrier), and the next
item's first P.V, which overwrites O, must not run before the epilogue has
read it.  The third is the group-score kernel (colsum_kernel.cuh), whose
reducing warps hand each S buffer back to the MMA thread explicitly.  The
fourth is one K/V ring fed by several producer warps, as in the sparse
kernels: it holds while each warp's copies carry part of every phase's
transaction bytes, and a variant in which one warp's plain arrival completes
each phase leaves the other warps waiting on phases that never come.
"""
import random

import pytest


class Barrier:
    """mbarrier: `count` arrivals plus a transaction byte count per phase."""

    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.completed = 0          # phases completed so far

    def _settle(self):
        if self.pending == 0 and self.tx == 0:
            self.completed += 1
            self.pending = self.count

    def arrive(self, n=1):
        self.pending -= n
        assert self.pending >= 0, "more arrivals than the barrier's count"
        self._settle()

    def arrive_expect_tx(self, nbytes):
        self.tx += nbytes
        self.arrive()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        self._settle()

    def parity_done(self, parity):
        # try_wait.parity: the phase of this parity has completed
        return (self.completed & 1) != parity


class ProtocolError(AssertionError):
    pass


def check(cond, what):
    if not cond:
        raise ProtocolError(what)


class Kernel:
    """State of one CTA: barriers, buffers, the tensor pipe, copies in flight."""

    def __init__(self, T, NK, NV, defect=None):
        self.T, self.NK, self.NV = T, NK, NV
        self.q = Barrier(1)
        self.kfull = [Barrier(1) for _ in range(NK)]
        self.kempty = [Barrier(1) for _ in range(NK)]
        self.vfull = [Barrier(1) for _ in range(NV)]
        self.vempty = [Barrier(1) for _ in range(NV)]
        self.sfull = [Barrier(1), Barrier(1)]
        p = [Barrier(1), Barrier(1)]
        pv = [Barrier(1), Barrier(1)]
        # planted defects: one barrier for both parities
        self.p = [p[0], p[0]] if defect == "one_p" else p
        self.pv = [pv[0], pv[0]] if defect == "one_pv" else pv
        self.empty_flip = 0 if defect == "empty_parity" else 1
        self.drain = Barrier(1)
        self.kslot = [None] * NK          # tile whose K the slot holds (None: loading / empty)
        self.vslot = [None] * NV
        self.S = [None, None]             # ("S", j) after Q.K^T(j), ("P", j) after the softmax
        self.pipe = []                    # issued, not yet executed: ("QK", j) / ("PV", j) / ("commit", bar)
        self.done = set()                 # executed MMAs
        self.copies = []                  # (kind, slot, tile, barrier) in flight
        self.pv_into = [[], []]           # P.V tiles issued into O_g
        self.merged = 0

    # -- asynchronous engines ------------------------------------------------
    def step_pipe(self):
        op = self.pipe.pop(0)
        if op[0] == "commit":
            op[1].arrive()
            return
        kind, j = op
        if kind == "QK":
            s = j % self.NK
            check(self.kslot[s] == j, f"Q.K^T({j}) read a K slot holding {self.kslot[s]}")
            prev = self.S[j & 1]
            check(prev is None or (prev[0] == "P" and ("PV", prev[1]) in self.done),
                  f"Q.K^T({j}) overwrote S still holding {prev}")
            self.S[j & 1] = ("S", j)
        else:
            s = j % self.NV
            check(self.S[j & 1] == ("P", j), f"P.V({j}) read S holding {self.S[j & 1]}")
            check(self.vslot[s] == j, f"P.V({j}) read a V slot holding {self.vslot[s]}")
        self.done.add((kind, j))

    def step_copy(self, i):
        kind, slot, tile, bar = self.copies.pop(i)
        if kind == "K":
            self.kslot[slot] = tile
        elif kind == "V":
            self.vslot[slot] = tile
        bar.complete_tx(1)


def wait(bar, parity, event_ok, what):
    """Yielded by an actor: resume once the parity wait returns, then check
    the event it stands for."""
    return (bar, parity, event_ok, what)


def producer_k(K):
    yield from ()
    K.q.arrive_expect_tx(1)
    K.copies.append(("Q", 0, 0, K.q))
    for j in range(K.T):
        s = j % K.NK
        if j >= K.NK:
            t = j - K.NK
            yield wait(K.kempty[s], ((j // K.NK) & 1) ^ K.empty_flip, lambda t=t: ("QK", t) in K.done,
                       f"K slot of tile {t} free")
        K.kslot[s] = None
        K.kfull[s].arrive_expect_tx(1)
        K.copies.append(("K", s, j, K.kfull[s]))


def producer_v(K):
    yield from ()
    for j in range(K.T):
        s = j % K.NV
        if j >= K.NV:
            t = j - K.NV
            yield wait(K.vempty[s], ((j // K.NV) & 1) ^ K.empty_flip, lambda t=t: ("PV", t) in K.done,
                       f"V slot of tile {t} free")
        K.vslot[s] = None
        K.vfull[s].arrive_expect_tx(1)
        K.copies.append(("V", s, j, K.vfull[s]))


def mma(K):
    yield wait(K.q, 0, lambda: True, "Q loaded")

    def issue_qk(j):
        s = j % K.NK
        yield wait(K.kfull[s], (j // K.NK) & 1, lambda: K.kslot[s] == j, f"K of tile {j} landed")
        K.pipe += [("QK", j), ("commit", K.sfull[j & 1]), ("commit", K.kempty[s])]

    def issue_pv(j):
        s = j % K.NV
        yield wait(K.p[j & 1], (j >> 1) & 1, lambda: K.S[j & 1] == ("P", j), f"P of tile {j} ready")
        yield wait(K.vfull[s], (j // K.NV) & 1, lambda: K.vslot[s] == j, f"V of tile {j} landed")
        K.pipe += [("PV", j), ("commit", K.pv[j & 1]), ("commit", K.vempty[s])]
        K.pv_into[j & 1].append(j)

    yield from issue_qk(0)
    if K.T > 1:
        yield from issue_qk(1)
    for j in range(K.T):
        yield from issue_pv(j)
        if j + 2 < K.T:
            yield from issue_qk(j + 2)
    K.pipe.append(("commit", K.drain))
    yield wait(K.drain, 0, lambda: not any(op[0] != "commit" for op in K.pipe), "pipe drained")


def softmax_group(K, g, rng):
    last = -1
    for j in range(g, K.T, 2):
        yield wait(K.sfull[j & 1], (j >> 1) & 1, lambda j=j: K.S[j & 1] == ("S", j), f"S of tile {j}")
        if j >= 2 and rng.random() < 0.3:   # a row's max moved: O_g is rescaled in place
            check(all(("PV", t) in K.done for t in K.pv_into[g]),
                  f"group {g} rescaled O while a P.V into it was pending (tile {j})")
        K.S[j & 1] = ("P", j)
        K.p[j & 1].arrive()
        last = j
    if last >= 0:
        yield wait(K.pv[last & 1], (last >> 1) & 1, lambda: ("PV", last) in K.done, f"P.V of tile {last}")
    K.merged += 1
    yield ("merge",)                       # the two groups meet at a named barrier
    check(all(("PV", t) in K.done for t in range(K.T)), "epilogue read O before every P.V executed")


def run(T, NK, NV, seed, defect=None, max_steps=200000):
    rng = random.Random(seed)
    K = Kernel(T, NK, NV, defect)
    actors = {"k": producer_k(K), "v": producer_v(K), "mma": mma(K),
              "g0": softmax_group(K, 0, rng), "g1": softmax_group(K, 1, rng)}
    blocked = {name: None for name in actors}      # the wait an actor is parked on
    finished = set()

    def advance(name):
        try:
            blocked[name] = next(actors[name])
        except StopIteration:
            finished.add(name)
            blocked[name] = None

    for name in list(actors):
        advance(name)
    for _ in range(max_steps):
        if len(finished) == len(actors):
            return K
        moves = []
        for name, w in blocked.items():
            if name in finished or w is None:
                continue
            if w[0] == "merge":
                if K.merged == 2:
                    moves.append(("actor", name))
            elif w[0].parity_done(w[1]):
                moves.append(("actor", name))
        if K.pipe:
            moves.append(("pipe", None))
        moves += [("copy", i) for i in range(len(K.copies))]
        if not moves:
            raise ProtocolError(f"deadlock: waiting {[(n, w[3] if w and len(w) > 3 else w) for n, w in blocked.items() if n not in finished]}")
        kind, arg = rng.choice(moves)
        if kind == "pipe":
            K.step_pipe()
        elif kind == "copy":
            K.step_copy(arg)
        else:
            w = blocked[arg]
            if w[0] != "merge":
                check(w[2](), f"{arg}: wait for '{w[3]}' returned before it happened")
            advance(arg)
    raise ProtocolError("schedule did not finish")


@pytest.mark.parametrize("NK,NV", [(3, 3), (6, 6)])
@pytest.mark.parametrize("T", [1, 2, 3, 4, 7, 12])
def test_protocol_holds_under_random_schedules(T, NK, NV):
    for seed in range(60):
        K = run(T, NK, NV, seed)
        assert {("QK", j) for j in range(T)} | {("PV", j) for j in range(T)} <= K.done


@pytest.mark.parametrize("defect", ["one_p", "one_pv", "empty_parity"])
def test_model_catches_planted_defects(defect):
    """Each planted defect must be reported on some schedule: one "P ready"
    or one "P.V done" barrier for both tile parities (the defects this
    protocol once had: the MMA thread took a P phase for the wrong tile, the
    epilogue read O one P.V early), or the ring producers waiting on the
    wrong parity of a slot's empty barrier."""
    failures = 0
    for seed in range(200):
        try:
            run(8, 3, 3, seed, defect=defect)
        except ProtocolError:
            failures += 1
    assert failures > 0


# ---------------------------------------------------------------------------
# the persistent sparse kernel: several items per CTA, one tile counter
# ---------------------------------------------------------------------------

class SparseKernel(Kernel):
    def __init__(self, items, T, NK, NV, defect=None):
        super().__init__(items * T, NK, NV, defect)
        self.items, self.T_item = items, T
        self.qempty = Barrier(1)
        self.qbuf = None                   # item whose Q the buffer holds
        self.epi_done = set()              # items whose O the epilogue has read
        self.pv_issued = set()

    def step_pipe(self):
        op = self.pipe[0]
        if op[0] == "QK":
            it = op[1] // self.T_item
            check(self.qbuf == it, f"Q.K^T({op[1]}) read Q holding item {self.qbuf}")
        elif op[0] == "PV" and op[1] % self.T_item == 0 and op[1] > 0:
            it = op[1] // self.T_item
            check(it - 1 in self.epi_done, f"item {it}'s first P.V overwrote O before item {it - 1}'s epilogue read it")
        super().step_pipe()

    def step_copy(self, i):
        kind, slot, tile, bar = self.copies[i]
        if kind == "Q":
            self.qbuf = tile
        super().step_copy(i)


def sparse_producer_k(K):
    yield from ()
    issued = 0
    for it in range(K.items):
        if it > 0:
            last = it * K.T_item - 1
            yield wait(K.qempty, (it - 1) & 1, lambda last=last: ("QK", last) in K.done, f"Q of item {it - 1} consumed")
        K.qbuf = None
        K.q.arrive_expect_tx(1)
        K.copies.append(("Q", 0, it, K.q))
        for j in range(K.T_item):
            s = issued % K.NK
            if issued >= K.NK:
                t = issued - K.NK
                yield wait(K.kempty[s], ((issued // K.NK) & 1) ^ K.empty_flip, lambda t=t: ("QK", t) in K.done,
                           f"K slot of tile {t} free")
            K.kslot[s] = None
            K.kfull[s].arrive_expect_tx(1)
            K.copies.append(("K", s, issued, K.kfull[s]))
            issued += 1


def sparse_producer_v(K):
    yield from ()
    for gj in range(K.T):
        s = gj % K.NV
        if gj >= K.NV:
            t = gj - K.NV
            yield wait(K.vempty[s], ((gj // K.NV) & 1) ^ K.empty_flip, lambda t=t: ("PV", t) in K.done,
                       f"V slot of tile {t} free")
        K.vslot[s] = None
        K.vfull[s].arrive_expect_tx(1)
        K.copies.append(("V", s, gj, K.vfull[s]))


def sparse_mma(K):
    T = K.T_item

    def issue_qk(g, j):
        gj = g + j
        s = gj % K.NK
        yield wait(K.kfull[s], (gj // K.NK) & 1, lambda: K.kslot[s] == gj, f"K of tile {gj} landed")
        K.pipe += [("QK", gj), ("commit", K.sfull[gj & 1]), ("commit", K.kempty[s])]
        if j == T - 1:
            K.pipe.append(("commit", K.qempty))

    def issue_pv(g, j):
        gj = g + j
        s = gj % K.NV
        yield wait(K.p[gj & 1], (gj >> 1) & 1, lambda: K.S[gj & 1] == ("P", gj), f"P of tile {gj} ready")
        yield wait(K.vfull[s], (gj // K.NV) & 1, lambda: K.vslot[s] == gj, f"V of tile {gj} landed")
        K.pipe += [("PV", gj), ("commit", K.pv[gj & 1]), ("commit", K.vempty[s])]
        K.pv_issued.add(gj)

    for it in range(K.items):
        g = it * T
        yield wait(K.q, it & 1, lambda it=it: K.qbuf == it, f"Q of item {it} landed")
        yield from issue_qk(g, 0)
        if T > 1:
            yield from issue_qk(g, 1)
        for j in range(T):
            yield from issue_pv(g, j)
            if j + 2 < T:
                yield from issue_qk(g, j + 2)
    K.pipe.append(("commit", K.drain))
    yield wait(K.drain, 0, lambda: not any(op[0] != "commit" for op in K.pipe), "pipe drained")


def sparse_softmax(K, rng):
    T = K.T_item
    for it in range(K.items):
        g = it * T
        for j in range(T):
            gj = g + j
            yield wait(K.sfull[gj & 1], (gj >> 1) & 1, lambda gj=gj: K.S[gj & 1] == ("S", gj), f"S of tile {gj}")
            if j > 0 and rng.random() < 0.3:   # a row's max moved: wait for the previous P.V, rescale O
                yield wait(K.pv[(gj - 1) & 1], ((gj - 1) >> 1) & 1, lambda gj=gj: ("PV", gj - 1) in K.done,
                           f"P.V of tile {gj - 1}")
                check(all(("PV", t) in K.done for t in range(g, gj)) and gj not in K.pv_issued,
                      f"O rescaled at tile {gj} with a P.V into it pending")
            K.S[gj & 1] = ("P", gj)
            K.p[gj & 1].arrive()
        for t in range(max(0, T - 2), T):
            yield wait(K.pv[(g + t) & 1], ((g + t) >> 1) & 1, lambda u=g + t: ("PV", u) in K.done,
                       f"P.V of tile {g + t}")
        check(all(("PV", t) in K.done for t in range(g, g + T)), f"item {it}'s epilogue read O before its P.V finished")
        K.epi_done.add(it)


def run_sparse(items, T, NK, NV, seed, defect=None, max_steps=400000):
    rng = random.Random(seed)
    K = SparseKernel(items, T, NK, NV, defect)
    actors = {"k": sparse_producer_k(K), "v": sparse_producer_v(K), "mma": sparse_mma(K),
              "soft": sparse_softmax(K, rng)}
    blocked = {name: None for name in actors}
    finished = set()

    def advance(name):
        try:
            blocked[name] = next(actors[name])
        except StopIteration:
            finished.add(name)
            blocked[name] = None

    for name in list(actors):
        advance(name)
    for _ in range(max_steps):
        if len(finished) == len(actors):
            return K
        moves = [("actor", n) for n, w in blocked.items()
                 if n not in finished and w is not None and w[0].parity_done(w[1])]
        if K.pipe:
            moves.append(("pipe", None))
        moves += [("copy", i) for i in range(len(K.copies))]
        if not moves:
            raise ProtocolError(f"deadlock: waiting {[(n, w[3]) for n, w in blocked.items() if n not in finished]}")
        kind, arg = rng.choice(moves)
        if kind == "pipe":
            K.step_pipe()
        elif kind == "copy":
            K.step_copy(arg)
        else:
            w = blocked[arg]
            check(w[2](), f"{arg}: wait for '{w[3]}' returned before it happened")
            advance(arg)
    raise ProtocolError("schedule did not finish")


@pytest.mark.parametrize("NK,NV", [(3, 3), (6, 6)])
@pytest.mark.parametrize("items,T", [(1, 1), (3, 1), (3, 2), (4, 3), (3, 13)])
def test_sparse_protocol_holds_under_random_schedules(items, T, NK, NV):
    for seed in range(40):
        K = run_sparse(items, T, NK, NV, seed)
        assert K.epi_done == set(range(items))


@pytest.mark.parametrize("defect", ["one_p", "one_pv", "empty_parity"])
def test_sparse_model_catches_planted_defects(defect):
    failures = 0
    for seed in range(200):
        try:
            run_sparse(3, 5, 3, 3, seed, defect=defect)
        except ProtocolError:
            failures += 1
    assert failures > 0


# ---------------------------------------------------------------------------
# the group-score kernel: S buffers handed back by the reducing warps
# ---------------------------------------------------------------------------

class ColsumKernel:
    def __init__(self, T, NST, defect=None):
        self.T, self.NST = T, NST
        self.q = Barrier(1)
        self.kfull = [Barrier(1) for _ in range(NST)]
        self.kempty = [Barrier(1) for _ in range(NST)]
        self.sfull = [Barrier(1), Barrier(1)]
        sfree = [Barrier(1), Barrier(1)]
        self.sfree = [sfree[0], sfree[0]] if defect == "one_sfree" else sfree
        self.sfree_off = 0 if defect == "sfree_parity" else 1
        self.drain = Barrier(1)
        self.kslot = [None] * NST
        self.S = [None, None]            # ("S", j) written, ("read", j) reduced
        self.qready = False
        self.pipe, self.done, self.copies = [], set(), []

    def step_pipe(self):
        op = self.pipe.pop(0)
        if op[0] == "commit":
            op[1].arrive()
            return
        j = op[1]
        s = j % self.NST
        check(self.qready, "Q.K^T before Q landed")
        check(self.kslot[s] == j, f"Q.K^T({j}) read a K slot holding {self.kslot[s]}")
        prev = self.S[j & 1]
        check(prev is None or prev == ("read", j - 2), f"Q.K^T({j}) overwrote S holding {prev}")
        self.S[j & 1] = ("S", j)
        self.done.add(("QK", j))

    def step_copy(self, i):
        kind, slot, tile, bar = self.copies.pop(i)
        if kind == "K":
            self.kslot[slot] = tile
        else:
            self.qready = True
        bar.complete_tx(1)


def colsum_producer(K):
    yield from ()
    K.q.arrive_expect_tx(1)
    K.copies.append(("Q", 0, 0, K.q))
    for j in range(K.T):
        s = j % K.NST
        if j >= K.NST:
            t = j - K.NST
            yield wait(K.kempty[s], ((j // K.NST) & 1) ^ 1, lambda t=t: ("QK", t) in K.done, f"K slot of tile {t} free")
        K.kslot[s] = None
        K.kfull[s].arrive_expect_tx(1)
        K.copies.append(("K", s, j, K.kfull[s]))


def colsum_mma(K):
    yield wait(K.q, 0, lambda: K.qready, "Q landed")
    for j in range(K.T):
        s, b = j % K.NST, j & 1
        if j >= 2:
            yield wait(K.sfree[b], ((j >> 1) - K.sfree_off) & 1, lambda j=j: K.S[j & 1] == ("read", j - 2),
                       f"S of tile {j - 2} reduced")
        yield wait(K.kfull[s], (j // K.NST) & 1, lambda j=j, s=s: K.kslot[s] == j, f"K of tile {j} landed")
        K.pipe += [("QK", j), ("commit", K.sfull[b]), ("commit", K.kempty[s])]
    K.pipe.append(("commit", K.drain))
    yield wait(K.drain, 0, lambda: not any(op[0] != "commit" for op in K.pipe), "pipe drained")


def colsum_reducers(K):
    for j in range(K.T):
        b = j & 1
        yield wait(K.sfull[b], (j >> 1) & 1, lambda j=j: K.S[j & 1] == ("S", j), f"S of tile {j}")
        K.S[b] = ("read", j)
        K.sfree[b].arrive()


def run_colsum(T, NST, seed, defect=None, max_steps=200000):
    rng = random.Random(seed)
    K = ColsumKernel(T, NST, defect)
    actors = {"k": colsum_producer(K), "mma": colsum_mma(K), "red": colsum_reducers(K)}
    blocked = {name: None for name in actors}
    finished = set()

    def advance(name):
        try:
            blocked[name] = next(actors[name])
        except StopIteration:
            finished.add(name)
            blocked[name] = None

    for name in list(actors):
        advance(name)
    for _ in range(max_steps):
        if len(finished) == len(actors):
            return K
        moves = [("actor", n) for n, w in blocked.items()
                 if n not in finished and w is not None and w[0].parity_done(w[1])]
        if K.pipe:
            moves.append(("pipe", None))
        moves += [("copy", i) for i in range(len(K.copies))]
        if not moves:
            raise ProtocolError(f"deadlock: waiting {[(n, w[3]) for n, w in blocked.items() if n not in finished]}")
        kind, arg = rng.choice(moves)
        if kind == "pipe":
            K.step_pipe()
        elif kind == "copy":
            K.step_copy(arg)
        else:
            w = blocked[arg]
            check(w[2](), f"{arg}: wait for '{w[3]}' returned before it happened")
            advance(arg)
    raise ProtocolError("schedule did not finish")


@pytest.mark.parametrize("NST", [2, 4])
@pytest.mark.parametrize("T", [1, 2, 3, 8, 17])
def test_colsum_protocol_holds_under_random_schedules(T, NST):
    for seed in range(60):
        K = run_colsum(T, NST, seed)
        assert {("QK", j) for j in range(T)} <= K.done


@pytest.mark.parametrize("defect", ["one_sfree", "sfree_parity"])
def test_colsum_model_catches_planted_defects(defect):
    failures = 0
    for seed in range(200):
        try:
            run_colsum(9, 2, seed, defect=defect)
        except ProtocolError:
            failures += 1
    assert failures > 0



# ---------------------------------------------------------------------------
# one K/V ring fed by several producer warps (pair_kernel.cuh, attn_kernel.cuh)
# ---------------------------------------------------------------------------
#
# Every producer warp waits on a slot's empty barrier before issuing its share
# of the tile's gather4 copies; warp 0 alone makes the phase's one arrival,
# with the tile's transaction bytes.  Because each warp's copies carry part of
# those bytes, a slot's full phase, and so its next empty phase, cannot
# complete before every warp has passed its own wait: no warp falls two
# phases behind, where a parity wait would mistake a later phase for the one
# it waits on.  A producer scheme in which warp 0 completes each phase on its
# own (a plain arrival, the other warps issuing nothing) loses that coupling.

class Ring:
    def __init__(self, T, NS, W, coupled):
        self.T, self.NS, self.W, self.coupled = T, NS, W, coupled
        self.full = [Barrier(1) for _ in range(NS)]
        self.empty = [Barrier(1) for _ in range(NS)]
        self.landed = {}                   # tile -> copies landed
        self.arrived = set()               # tiles whose phase arrival warp 0 made
        self.consumed = set()
        self.copies = []                   # (slot, tile) in flight

    def step_copy(self, i):
        s, j = self.copies.pop(i)
        self.landed[j] = self.landed.get(j, 0) + 1
        self.full[s].complete_tx(1)


def ring_producer(R, w):
    yield from ()
    for j in range(R.T):
        s = j % R.NS
        t = j - R.NS
        yield wait(R.empty[s], ((j // R.NS) & 1) ^ 1, lambda t=t: t < 0 or t in R.consumed,
                   f"warp {w}: slot of tile {t} free")
        if w == 0:
            R.arrived.add(j)
            if R.coupled:
                R.full[s].arrive_expect_tx(R.W)
            else:
                R.full[s].arrive()
        if R.coupled:
            R.copies.append((s, j))


def ring_consumer(R):
    for j in range(R.T):
        s = j % R.NS
        ready = (lambda j=j: j in R.arrived and R.landed.get(j, 0) == R.W) if R.coupled else (lambda j=j: j in R.arrived)
        yield wait(R.full[s], (j // R.NS) & 1, ready, f"tile {j} in its slot")
        R.consumed.add(j)
        R.empty[s].arrive()


def run_ring(T, NS, W, coupled, seed, max_steps=200000):
    rng = random.Random(seed)
    R = Ring(T, NS, W, coupled)
    actors = {f"w{w}": ring_producer(R, w) for w in range(W)}
    actors["mma"] = ring_consumer(R)
    blocked = {name: None for name in actors}
    finished = set()

    def advance(name):
        try:
            blocked[name] = next(actors[name])
        except StopIteration:
            finished.add(name)
            blocked[name] = None

    for name in list(actors):
        advance(name)
    for _ in range(max_steps):
        if len(finished) == len(actors):
            return R
        moves = [("actor", n) for n, w in blocked.items()
                 if n not in finished and w is not None and w[0].parity_done(w[1])]
        moves += [("copy", i) for i in range(len(R.copies))]
        if not moves:
            raise ProtocolError(f"deadlock: waiting {[(n, w[3]) for n, w in blocked.items() if n not in finished]}")
        kind, arg = rng.choice(moves)
        if kind == "copy":
            R.step_copy(arg)
        else:
            w = blocked[arg]
            check(w[2](), f"{arg}: wait for '{w[3]}' returned before it happened")
            advance(arg)
    raise ProtocolError("schedule did not finish")


@pytest.mark.parametrize("NS", [2, 5])
@pytest.mark.parametrize("W", [3, 4])
def test_ring_producer_warps_coupled_by_transaction_bytes(NS, W):
    for seed in range(150):
        R = run_ring(12, NS, W, True, seed)
        assert R.consumed == set(range(12))


def test_ring_producer_warps_without_bytes_can_wait_forever():
    """warp 0's plain arrival alone completes each phase: some schedule
    leaves another producer warp waiting on a phase that never comes."""
    failures = 0
    for seed in range(300):
        try:
            run_ring(12, 2, 4, False, seed)
        except ProtocolError as e:
            assert "deadlock" in str(e)
            failures += 1
    assert failures > 0
