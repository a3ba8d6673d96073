"""The context-parallel exchange protocols under concurrency, on the CPU.

Every GPU run here has one GPU, so the ranks' kernels never run at the same
time in the tests that execute them.  This test checks the protocols
themselves: it records the calls each rank's ``UlyssesAttention`` or
``RingAttention`` makes (through a recording backend), turns every call into
the copies, signals and waits the library performs for it, and runs P ranks
concurrently under many random interleavings (each rank's stream in order,
as on a GPU; a wait blocks until its counter reaches the count the call
states).  Each copy is split into a begin and an end event with other
ranks' events in between.  Checked: no interleaving deadlocks; every read
finds the data of the right call (and, for the ring, the right block); no
write starts on a buffer while another copy still reads or writes it; a
rank's output slice is complete when its last wait passes."""
import random

import pytest

from test_context_parallel_cpu import FakeBackend, FakeRingBackend


# ------------------------------------------------------------ simulator

class Race(AssertionError):
    pass


class World:
    """Counters (per region) and buffers (per region and part) shared by all
    simulated ranks."""

    def __init__(self):
        self.counters = {}
        self.buffers = {}

    def counter(self, region, name):
        return self.counters.get((region, name), 0)

    def add(self, region, name, n=1):
        self.counters[(region, name)] = self.counter(region, name) + n

    def buf(self, key):
        return self.buffers.setdefault(key, {"label": None, "readers": 0, "writers": 0})


def read_begin(world, key, expect):
    b = world.buf(key)
    if b["writers"]:
        raise Race(f"read of {key} while it is being written")
    if b["label"] != expect:
        raise Race(f"read of {key}: found {b['label']}, expected {expect}")
    b["readers"] += 1


def read_end(world, key):
    world.buf(key)["readers"] -= 1


def write_begin(world, key):
    b = world.buf(key)
    if b["readers"] or b["writers"]:
        raise Race(f"write of {key} while {b['readers']} reads / {b['writers']} writes are active")
    b["writers"] += 1


def write_end(world, key, label):
    b = world.buf(key)
    b["writers"] -= 1
    b["label"] = label


def run(programs, seed, max_events=200000):
    """programs: one list of events per rank; an event is ("wait", region,
    counter, n) or a callable(world).  Random interleaving; returns world."""
    world = World()
    rng = random.Random(seed)
    pcs = [0] * len(programs)
    for _ in range(max_events):
        ready = []
        for r, prog in enumerate(programs):
            if pcs[r] >= len(prog):
                continue
            ev = prog[pcs[r]]
            if isinstance(ev, tuple) and ev[0] == "wait":
                _, region, name, n = ev
                if world.counter(region, name) < n:
                    continue
            ready.append(r)
        if not ready:
            if all(pcs[r] >= len(p) for r, p in enumerate(programs)):
                return world
            raise AssertionError(f"deadlock: ranks at {pcs} of {[len(p) for p in programs]}")
        r = rng.choice(ready)
        ev = programs[r][pcs[r]]
        if not isinstance(ev, tuple):
            ev(world)
        pcs[r] += 1
    raise AssertionError("simulation did not finish")


# ------------------------------------------------------- Ulysses protocol

def ulysses_calls(world_size, rank, calls):
    """The calls rank `rank`'s UlyssesAttention makes for `calls` steps."""
    import torch
    from full_spatiotemporal_attention_b200.ulysses import UlyssesAttention
    import full_spatiotemporal_attention_b200 as va
    fake = FakeBackend(rank)
    handles = [f"handle-of-{0x10000 * (j + 1):#x}".encode() for j in range(world_size)]
    ua = UlyssesAttention(va.Grid.make(world_size, 2, 4), 1, 2 * world_size, world=world_size,
                          rank=rank, device="cpu", backend=fake, exchange=lambda h: handles)
    x = torch.zeros(ua.plan.local_shape, dtype=torch.bfloat16)
    fake.calls.clear()
    for _ in range(calls):
        ua(x, x, x)
    return [c for c in fake.calls], ua.regions


def region_rank(ptr):
    """Rank that owns a (possibly peer-mapped) fake region address."""
    return (ptr & 0xFFFFFF) // 0x10000 - 1


def ulysses_program(world_size, rank, calls):
    recorded, _ = ulysses_calls(world_size, rank, calls)
    prog = []
    epoch = [0]
    P = world_size
    for c in recorded:
        if c[0] == "scatter":
            regions = [region_rank(p) for p in c[1]]
            def begin(w, regions=regions):
                for j in regions:
                    write_begin(w, (j, "qkv", rank))
            def end(w, regions=regions):
                epoch[0] += 1
                for j in regions:
                    write_end(w, (j, "qkv", rank), epoch[0])
                for j in regions:
                    w.add(j, "scatter")       # one block per rank in this model
            prog += [begin, end]
        elif c[0] == "wait":
            _, region, phase, e, ws = c
            prog.append(("wait", region_rank(region), "scatter" if phase == 0 else "gather", e * ws))
        elif c[0] == "attn":
            def begin(w):
                for s in range(P):
                    read_begin(w, (rank, "qkv", s), epoch[0])
                write_begin(w, (rank, "o_heads", 0))
            def end(w):
                for s in range(P):
                    read_end(w, (rank, "qkv", s))
                write_end(w, (rank, "o_heads", 0), epoch[0])
            prog += [begin, end]
        elif c[0] == "gather":
            regions = [region_rank(p) for p in c[1]]
            def begin(w, regions=regions):
                read_begin(w, (rank, "o_heads", 0), epoch[0])
                for j in regions:
                    write_begin(w, (j, "o", rank))
            def end(w, regions=regions):
                read_end(w, (rank, "o_heads", 0))
                for j in regions:
                    write_end(w, (j, "o", rank), epoch[0])
                for j in regions:
                    w.add(j, "gather")
            prog += [begin, end]
            # after the gather wait (the next recorded call) the caller reads
            # its whole output slice: every rank's part of this call
        else:
            raise AssertionError(f"unexpected call {c}")
        if c[0] == "wait" and c[2] == 1:
            def consume_begin(w):
                for s in range(P):
                    read_begin(w, (rank, "o", s), epoch[0])
            def consume_end(w):
                for s in range(P):
                    read_end(w, (rank, "o", s))
            prog += [consume_begin, consume_end]
    return prog


@pytest.mark.parametrize("P", [1, 2, 3, 4, 8])
def test_ulysses_protocol_is_race_and_deadlock_free(P):
    programs = [ulysses_program(P, r, calls=3) for r in range(P)]
    for seed in range(150):
        world = run(programs, seed)
        for r in range(P):
            assert world.counter(r, "scatter") == 3 * P
            assert world.counter(r, "gather") == 3 * P


def test_ulysses_model_catches_a_missing_wait():
    """The model is not vacuous: drop the gather wait of rank 0 and some
    interleaving reads an unfinished output slice."""
    P = 3
    programs = [ulysses_program(P, r, calls=2) for r in range(P)]
    programs[0] = [e for e in programs[0] if not (isinstance(e, tuple) and e[2] == "gather")]
    with pytest.raises(Race):
        for seed in range(300):
            run(programs, seed)


# ---------------------------------------------------------- ring protocol

def ring_calls(world_size, rank, calls):
    import torch
    from full_spatiotemporal_attention_b200.ring import RingAttention
    import full_spatiotemporal_attention_b200 as va

    class Recorder(FakeRingBackend):
        def ring_attend(self, q_rot, k, v, acc, lse_in, lse_out, first, out=None):
            self.calls.append(("attend", 0 if k is self.owner.kbuf[0] else 1))

    fake = Recorder(rank)
    handles = [f"handle-of-{0x10000 * (j + 1):#x}".encode() for j in range(world_size)]
    ra = RingAttention(va.Grid.make(world_size, 2, 4), 1, 3, world=world_size, rank=rank,
                       device="cpu", backend=fake, exchange=lambda h: handles)
    fake.owner = ra
    x = torch.zeros((1, 3, 8, 128), dtype=torch.bfloat16)
    fake.calls.clear()
    for _ in range(calls):
        ra(x, x, x)
    return list(fake.calls)


def ring_program(P, rank, calls):
    recorded = ring_calls(P, rank, calls)
    prog = []
    state = {"call": 0, "step": 0}
    nxt = (rank + 1) % P
    for c in recorded:
        if c[0] == "load":
            def begin(w):
                state["call"] += 1
                state["step"] = 0
                write_begin(w, (rank, "kv", 0))
            def end(w):
                write_end(w, (rank, "kv", 0), (state["call"], rank))
            prog += [begin, end]
        elif c[0] == "wait":
            _, region, counter, count = c
            prog.append(("wait", region_rank(region), "full" if counter == 0 else "free", count))
        elif c[0] == "pass":
            _, region, next_region, buf = c
            assert region_rank(region) == rank and region_rank(next_region) == nxt
            def begin(w, buf=buf):
                expect = (state["call"], (rank - state["step"]) % P)
                read_begin(w, (rank, "kv", buf), expect)
                write_begin(w, (nxt, "kv", 1 - buf))
                state["passing"] = expect
            def end(w, buf=buf):
                read_end(w, (rank, "kv", buf))
                write_end(w, (nxt, "kv", 1 - buf), state["passing"])
                w.add(nxt, "full")
            prog += [begin, end]
        elif c[0] == "attend":
            # the block product reads the buffer; its merge ends the step
            buf = c[1]
            def begin(w, buf=buf):
                assert buf == state["step"] % 2
                read_begin(w, (rank, "kv", buf), (state["call"], (rank - state["step"]) % P))
            def end(w, buf=buf):
                read_end(w, (rank, "kv", buf))
                state["step"] += 1
            prog += [begin, end]
        elif c[0] == "free_signal":
            assert region_rank(c[1]) == (rank - 1) % P
            prog.append(lambda w: w.add((rank - 1) % P, "free"))
        else:
            raise AssertionError(f"unexpected call {c}")
    return prog


@pytest.mark.parametrize("P", [1, 2, 3, 4, 5, 8])
def test_ring_protocol_is_race_and_deadlock_free(P):
    programs = [ring_program(P, r, calls=3) for r in range(P)]
    for seed in range(150):
        world = run(programs, seed)
        for r in range(P):
            assert world.counter(r, "full") == 3 * (P - 1)
            assert world.counter(r, "free") == (3 * P if P > 1 else 0)


def test_ring_model_catches_a_missing_free_wait():
    """Drop rank 0's free waits: some interleaving overwrites a block its
    neighbour still reads."""
    P = 3
    programs = [ring_program(P, r, calls=3) for r in range(P)]
    programs[0] = [e for e in programs[0] if not (isinstance(e, tuple) and e[2] == "free")]
    with pytest.raises(Race):
        for seed in range(300):
            run(programs, seed)


def _lower_waits(program, name, by=1):
    return [("wait", e[1], e[2], e[3] - by) if isinstance(e, tuple) and e[2] == name else e
            for e in program]


@pytest.mark.parametrize("name", ["scatter", "gather"])
def test_ulysses_model_catches_a_short_count(name):
    """A wait count one short of what va3d_ulysses_wait computes lets some
    interleaving read a slice that has not landed."""
    P = 3
    programs = [ulysses_program(P, r, calls=2) for r in range(P)]
    programs[1] = _lower_waits(programs[1], name)
    with pytest.raises(Race):
        for seed in range(400):
            run(programs, seed)


@pytest.mark.parametrize("name", ["full", "free"])
def test_ring_model_catches_a_short_count(name):
    P = 4
    programs = [ring_program(P, r, calls=2) for r in range(P)]
    programs[2] = _lower_waits(programs[2], name)
    with pytest.raises(Race):
        for seed in range(400):
            run(programs, seed)
