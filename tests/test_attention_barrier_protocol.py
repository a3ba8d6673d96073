"""The attention kernel's mbarrier protocol under every interleaving we try.

A model of the roles of ``attn_fwd_kernel`` (csrc/attn_sm100.cuh), each a
coroutine over the kernel's barriers in the kernel's own order:

* the loader: the TMA producer (one arrival with its bytes per tile), or, in
  window mode, the gathering loader (K(j) and V(j) published one step after
  they are issued, as its cp.async groups land);
* the MMA issuer: S(0) for each query tile, then per key tile PV, the next
  S, and the stage releases (with one query tile, V's stage is released
  right after its only PV product);
* one softmax group per query tile: Q ready, then per key tile S in, P out,
  and finally the O barrier;
* both producers' tails, which wait for the last stages' releases.

Waits are parity waits, as ``mbarrier.try_wait.parity`` does them, so a
producer that ran two phases ahead of a consumer would stall the model just
as it would stall the GPU.  Commits arrive immediately (on the GPU they
arrive once the products issued before them finish, which needs no other
event).  For NQ = 1, 2 (one and two K/V stages), both loaders and 1..7 key
tiles, random schedules must finish, and every wait must see the completion
of the tile it means.  The ordering the kernel had before the one-tile
release fix (V released only after the next QK^T) must deadlock with the
gathering loader, so the model is not vacuous."""
import random

import pytest


class Bar:
    def __init__(self, name):
        self.name = name
        self.completed = 0          # phases completed so far

    def arrive(self):
        self.completed += 1         # every barrier here expects one arrival per phase

    def parity_done(self, parity):
        return (self.completed & 1) != parity


class Model:
    def __init__(self, nq, n_kv, gather, vempty_early=True):
        self.nq, self.n_kv, self.gather = nq, n_kv, gather
        self.S = 2 if nq == 2 else 1
        self.vempty_early = vempty_early
        names = ["QFULL", "QREADY0", "QREADY1", "SFULL0", "SFULL1", "PFULL0", "PFULL1", "OFULL"]
        for s in range(2):
            names += [f"KFULL{s}", f"KEMPTY{s}", f"VFULL{s}", f"VEMPTY{s}"]
        self.bars = {n: Bar(n) for n in names}

    def stg(self, j):
        return j % self.S

    def phs(self, j):
        return (j // self.S) & 1

    def wait(self, name, parity, expect_completed=None):
        """Parity wait; once it passes, the barrier must have completed the
        phase the waiter means (not one more, which parity cannot tell)."""
        bar = self.bars[name]
        while not bar.parity_done(parity):
            yield name
        if expect_completed is not None:
            assert bar.completed == expect_completed, (
                f"{name}: waited for completion {expect_completed}, barrier at {bar.completed}")

    def arrive(self, name):
        self.bars[name].arrive()

    # ------------------------------------------------------------- roles
    def tma_loader(self):
        S, n = self.S, self.n_kv
        self.arrive("QFULL")
        for j in range(n):
            s, ph = self.stg(j), self.phs(j)
            if j >= S:
                yield from self.wait(f"KEMPTY{s}", ph ^ 1, j // S)
            self.arrive(f"KFULL{s}")
            if j >= S:
                yield from self.wait(f"VEMPTY{s}", ph ^ 1, j // S)
            self.arrive(f"VFULL{s}")
        yield from self.tail()

    def gather_loader(self):
        S, n = self.S, self.n_kv
        self.arrive("QFULL")        # Q rows are gathered by the softmax threads; modelled as ready
        for j in range(n + 1):
            s, ph = self.stg(j), self.phs(j)
            if j >= 1:
                self.arrive(f"KFULL{self.stg(j - 1)}")      # K(j-1) landed: publish
            if j < n and j >= S:
                yield from self.wait(f"KEMPTY{s}", ph ^ 1, j // S)
            if j >= 1:
                self.arrive(f"VFULL{self.stg(j - 1)}")      # V(j-1) landed: publish
            if j < n and j >= S:
                yield from self.wait(f"VEMPTY{s}", ph ^ 1, j // S)
        yield from self.tail()

    def tail(self):
        S, n = self.S, self.n_kv
        first = n - S if n > S else 0
        for j in range(first, n):
            yield from self.wait(f"KEMPTY{self.stg(j)}", self.phs(j), j // S + 1)
            yield from self.wait(f"VEMPTY{self.stg(j)}", self.phs(j), j // S + 1)

    def mma(self):
        nq, n = self.nq, self.n_kv
        yield from self.wait("QREADY0", 0, 1)
        if nq == 2:
            yield from self.wait("QREADY1", 0, 1)
        yield from self.wait("KFULL0", 0, 1)
        self.arrive("SFULL0")
        if nq == 2:
            self.arrive("SFULL1")
        self.arrive("KEMPTY0")
        for j in range(n):
            s, ph = self.stg(j), self.phs(j)
            more = j + 1 < n
            s2, ph2 = self.stg(j + 1), self.phs(j + 1)
            yield from self.wait(f"VFULL{s}", ph, j // self.S + 1)
            yield from self.wait("PFULL0", j & 1, j + 1)
            if nq == 1 and self.vempty_early:
                self.arrive(f"VEMPTY{s}")
            if more:
                yield from self.wait(f"KFULL{s2}", ph2, (j + 1) // self.S + 1)
                self.arrive("SFULL0")
            if nq == 2:
                yield from self.wait("PFULL1", j & 1, j + 1)
                self.arrive(f"VEMPTY{s}")
            elif not self.vempty_early:
                self.arrive(f"VEMPTY{s}")
            if more:
                if nq == 2:
                    self.arrive("SFULL1")
                self.arrive(f"KEMPTY{s2}")
        self.arrive("OFULL")

    def softmax(self, g):
        yield from self.wait("QFULL", 0, 1)
        self.arrive(f"QREADY{g}")
        for j in range(self.n_kv):
            yield from self.wait(f"SFULL{g}", j & 1, j + 1)
            self.arrive(f"PFULL{g}")
        yield from self.wait("OFULL", 0, 1)

    def roles(self):
        loader = self.gather_loader() if self.gather else self.tma_loader()
        return [loader, self.mma()] + [self.softmax(g) for g in range(self.nq)]


def _blocked_only(model, seed):
    """Random schedule of the roles; False if no barrier moves for a long
    time while roles are left (every live role waits: the GPU would stall)."""
    rng = random.Random(seed)
    live = model.roles()
    stall = 0
    while live:
        snapshot = tuple(b.completed for b in model.bars.values())
        i = rng.randrange(len(live))
        try:
            for _ in range(rng.randint(1, 4)):
                next(live[i])
        except StopIteration:
            live.pop(i)
            stall = 0
            continue
        if tuple(b.completed for b in model.bars.values()) == snapshot:
            stall += 1
            if stall > 200 * len(live):
                return False
        else:
            stall = 0
    return True


@pytest.mark.parametrize("nq", [1, 2])
@pytest.mark.parametrize("gather", [False, True], ids=["tma", "gather"])
@pytest.mark.parametrize("n_kv", [1, 2, 3, 4, 5, 7])
def test_barrier_protocol_completes(nq, gather, n_kv):
    for seed in range(60):
        m = Model(nq, n_kv, gather)
        assert _blocked_only(m, seed), f"stuck: nq={nq} gather={gather} n_kv={n_kv} seed={seed}"
        S = 2 if nq == 2 else 1
        # every stage was filled and released as often as tiles went through it
        for s in range(S):
            uses = len([j for j in range(n_kv) if j % S == s])
            assert m.bars[f"KFULL{s}"].completed == uses
            assert m.bars[f"VFULL{s}"].completed == uses
            assert m.bars[f"VEMPTY{s}"].completed == uses
        assert m.bars["OFULL"].completed == 1


@pytest.mark.parametrize("n_kv", [2, 3])
def test_late_v_release_with_one_stage_and_gathered_rows_deadlocks(n_kv):
    """The ordering before the fix: with one K/V stage and the gathering
    loader, releasing V only after the next QK^T waits on a K tile the loader
    publishes only after refilling V."""
    stuck = False
    for seed in range(60):
        m = Model(1, n_kv, gather=True, vempty_early=False)
        if not _blocked_only(m, seed):
            stuck = True
            break
    assert stuck


# --------------------------------------------------- split-tile epilogue

def _split_units(order_seed):
    """The two units of a split tile (each over half of the keys): every
    softmax thread stores its normalised partial row and (max, sum) to the
    scratch and fences; once the whole CTA has (B_EPI), one thread adds 1 to
    the tile's counter (cleared by the table kernel before the launch) and
    publishes the old value (B_EPI_GO); the unit that saw 1 merges both
    halves.  Each unit is a list of events over a shared state; the rows of
    a unit are modelled as two threads to let their stores interleave."""
    state = {"count": 0, "written": [[False, False], [False, False]], "merged_by": [],
             "seen": [None, None]}

    def unit(u):
        ev = []
        for row in range(2):
            ev.append(lambda st, row=row: st["written"][u].__setitem__(row, True))
        # B_EPI: all rows stored and fenced before the counting thread runs
        ev.append(("epi", u))
        def count(st):
            st["seen"][u] = st["count"]
            st["count"] += 1
        ev.append(count)
        def merge(st):
            if st["seen"][u] == 1:
                other = 1 - u
                assert all(st["written"][other]), "merged a half that was not fully stored"
                assert all(st["written"][u])
                st["merged_by"].append(u)
        ev.append(merge)
        return ev
    return state, [unit(0), unit(1)]


def test_split_tile_is_merged_once_and_only_when_complete():
    for seed in range(500):
        rng = random.Random(seed)
        state, units = _split_units(seed)
        pcs = [0, 0]
        while pcs != [len(units[0]), len(units[1])]:
            ready = []
            for u in (0, 1):
                if pcs[u] >= len(units[u]):
                    continue
                ev = units[u][pcs[u]]
                if isinstance(ev, tuple) and ev[0] == "epi" and not all(state["written"][u]):
                    continue
                ready.append(u)
            u = rng.choice(ready)
            ev = units[u][pcs[u]]
            if not isinstance(ev, tuple):
                ev(state)
            pcs[u] += 1
        assert state["count"] == 2
        assert len(state["merged_by"]) == 1
        assert sorted(state["seen"]) == [0, 1]
