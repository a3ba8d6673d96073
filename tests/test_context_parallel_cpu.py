"""Host logic of context parallelism (Ulysses and ring forms) on the CPU.

The exchanges themselves run in the library's kernels (tested on a GPU with
emulated ranks).  Here ``UlyssesAttention`` and ``RingAttention`` run over a
fake backend that records every call (two gloo ranks for the Ulysses form):
the IPC handles travel through ``all_gather_object``, each rank must map
exactly the regions it needs in rank order, and every call must issue its
copies, waits, products and merges in order with the right counts."""
import json
import os
import socket
import sys

import pytest

from conftest import ROOT

sys.path.insert(0, ROOT)


def test_plan_shapes_and_limits():
    from full_spatiotemporal_attention_b200.ulysses import make_plan
    p = make_plan(1, 40, 75600, 8, 3)
    assert p.heads_per_rank == 5 and p.tokens_per_rank == 9450
    assert p.local_shape == (1, 40, 9450, 128)
    assert p.head_shard_shape == (1, 5, 75600, 128)
    assert p.token_range == (28350, 37800) and p.head_range == (15, 20)
    # the token slices tile the sequence and the head groups tile the heads
    slices = [make_plan(1, 24, 119056, 8, r) for r in range(8)]
    assert [s.token_range for s in slices] == [(r * 14882, (r + 1) * 14882) for r in range(8)]
    assert slices[-1].token_range[1] == 119056
    assert [s.head_range for s in slices] == [(3 * r, 3 * r + 3) for r in range(8)]
    for bad in ((1, 12, 32760, 8, 0), (1, 12, 32761, 4, 0), (1, 8, 32, 9, 0), (1, 8, 32, 2, 2),
                (0, 8, 32, 2, 0)):
        with pytest.raises(ValueError):
            make_plan(*bad)


class FakeBackend:
    """Stands in for the binding: regions are integers, views are CPU tensors."""
    PHASE_SCATTER, PHASE_GATHER = 0, 1

    def __init__(self, rank):
        import full_spatiotemporal_attention_b200 as va
        self.Grid = va.Grid          # a plain ctypes structure, no device involved
        self.rank = rank
        self.calls = []

    def ulysses_region_bytes(self, B, H, N, world):
        return 1 << 20

    def region_alloc(self, nbytes):
        self.calls.append(("alloc", nbytes))
        return 0x10000 * (self.rank + 1)

    def region_free(self, ptr):
        self.calls.append(("free", ptr))

    def ipc_export(self, ptr):
        return f"handle-of-{ptr:#x}".encode()

    def ipc_open(self, handle):
        ptr = int(handle.decode().rsplit("-", 1)[1], 16) + 0x7000000
        self.calls.append(("open", ptr))
        return ptr

    def ipc_close(self, ptr):
        self.calls.append(("close", ptr))

    def ulysses_offsets(self, B, H, N, world):
        return 256, 512, 768, 1024

    def region_view(self, ptr, off, shape, device):
        import torch
        return torch.zeros(shape, dtype=torch.bfloat16)

    def workspace_bytes(self, B, H, N, grid, k_rotated=False):
        return 4096

    def ulysses_scatter(self, q, k, v, regions, rank, grid, k_rotated=False):
        self.calls.append(("scatter", list(regions), rank, k_rotated))

    def ulysses_wait(self, region, phase, epoch, world, B, H, N, device=None):
        self.calls.append(("wait", region, phase, epoch, world))

    def attn_factorized_fwd(self, q, k, v, grid, spatial=True, temporal=True, out_spatial=None,
                            out_temporal=None, workspace=None):
        self.calls.append(("factorised", tuple(q.shape), [grid.T, grid.H, grid.W], spatial,
                           temporal))
        return out_spatial, out_temporal

    def attn3d_full_fwd(self, q, k, v, grid, k_rotated=False, out=None, workspace=None):
        self.calls.append(("attn", tuple(q.shape), k_rotated))
        return out

    def ulysses_gather(self, o, regions, rank, heads):
        self.calls.append(("gather", list(regions), rank, heads))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    from datetime import timedelta
    import torch
    import torch.distributed as dist
    from full_spatiotemporal_attention_b200.ulysses import UlyssesAttention
    import full_spatiotemporal_attention_b200 as va

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    fake = FakeBackend(rank)
    g = va.Grid.make(2, 4, 4)
    ua = UlyssesAttention(g, 1, 4, device="cpu", backend=fake)
    x = torch.zeros(ua.plan.local_shape, dtype=torch.bfloat16)
    ua(x, x, x)
    ua(x, x, x, k_rotated=True)
    ua.close(barrier=dist.barrier)
    with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
        json.dump({"calls": fake.calls, "regions": ua.regions,
                   "plan": [ua.plan.world, ua.plan.rank]}, f)
    dist.destroy_process_group()


def test_two_ranks_map_regions_and_sequence_calls(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    own = [0x10000 * (r + 1) for r in range(world)]
    for r, out in enumerate(res):
        assert out["plan"] == [world, r]
        # own region at its own index, every peer's mapped region at the peer's
        expect = [own[j] if j == r else own[j] + 0x7000000 for j in range(world)]
        assert out["regions"] == expect
        calls = [c for c in out["calls"] if c[0] not in ("alloc", "open")]
        one = lambda epoch, rot: [
            ["scatter", expect, r, rot],
            ["wait", own[r], 0, epoch, world],
            ["attn", [1, 2, 32, 128], True],
            ["gather", expect, r, 4],
            ["wait", own[r], 1, epoch, world]]
        peers = [own[j] + 0x7000000 for j in range(world) if j != r]
        assert calls == one(1, False) + one(2, True) + [["close", p] for p in peers] + \
            [["free", own[r]]]


def test_single_rank_needs_no_exchange():
    import torch
    from full_spatiotemporal_attention_b200.ulysses import UlyssesAttention
    import full_spatiotemporal_attention_b200 as va
    fake = FakeBackend(0)

    def no_exchange(_):
        raise AssertionError("one rank exchanges nothing")
    ua = UlyssesAttention(va.Grid.make(2, 4, 4), 1, 2, world=1, rank=0, device="cpu",
                          backend=fake, exchange=no_exchange)
    assert ua.regions == [0x10000]
    with pytest.raises(ValueError, match="shape"):
        bad = torch.zeros((1, 2, 31, 128), dtype=torch.bfloat16)
        ua(bad, bad, bad)
    ua.close()
    assert fake.calls[-1] == ("free", 0x10000)
    ua.close()   # idempotent


def test_factorised_call_sequence():
    """Spatial pass on the rank's own frames (local grid, no exchange), then
    the raw keys exchanged as they are and the temporal pass on whole
    sequences of the rank's heads."""
    import torch
    from full_spatiotemporal_attention_b200.ulysses import UlyssesAttention
    import full_spatiotemporal_attention_b200 as va
    fake = FakeBackend(1)
    g = va.Grid.make(6, 4, 4)                       # 96 tokens, 2 frames per rank
    ua = UlyssesAttention(g, 1, 6, world=3, rank=1, device="cpu", backend=fake,
                          exchange=lambda h: [b"handle-of-0x10000", h, b"handle-of-0x30000"])
    x = torch.zeros(ua.plan.local_shape, dtype=torch.bfloat16)
    fake.calls.clear()
    ua.factorised(x, x, x)
    regions = [0x10000 + 0x7000000, 0x20000, 0x30000 + 0x7000000]
    assert [list(c) for c in fake.calls] == [
        ["factorised", (1, 6, 32, 128), [2, 4, 4], True, False],
        ["scatter", regions, 1, True],
        ["wait", 0x20000, 0, 1, 3],
        ["factorised", (1, 2, 96, 128), [6, 4, 4], False, True],
        ["gather", regions, 1, 6],
        ["wait", 0x20000, 1, 1, 3]]
    # frames that do not split over the ranks, or text tokens
    ua2 = UlyssesAttention(va.Grid.make(5, 4, 4, n_text=1), 1, 3, world=3, rank=0, device="cpu",
                           backend=FakeBackend(0), exchange=lambda h: [h, h, h])
    y = torch.zeros(ua2.plan.local_shape, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="whole frames"):
        ua2.factorised(y, y, y)


def test_failed_exchange_releases_the_region():
    from full_spatiotemporal_attention_b200.ulysses import UlyssesAttention
    import full_spatiotemporal_attention_b200 as va
    fake = FakeBackend(1)
    with pytest.raises(RuntimeError, match="entries"):
        UlyssesAttention(va.Grid.make(2, 4, 4), 1, 2, world=2, rank=1, device="cpu",
                         backend=fake, exchange=lambda h: [h])
    assert fake.calls[-1] == ("free", 0x20000)


class FakeRingBackend(FakeBackend):
    RING_FULL, RING_FREE = 0, 1

    def ring_region_bytes(self, B, H, N, world):
        return 1 << 20

    def ring_offsets(self, B, H, N, world):
        return 256, 512, 768, 1024

    def cross_workspace_bytes(self, B, H, Nq, Nkv):
        return 4096

    def ring_load(self, q, k, v, q_rot, region, world, rank, grid, k_rotated=False):
        self.calls.append(("load", region, world, rank, k_rotated))

    def ring_wait(self, region, counter, count, world, B, H, N, device=None):
        self.calls.append(("wait", region, counter, count))

    def ring_pass(self, region, next_region, buf, world, B, H, N, device=None):
        self.calls.append(("pass", region, next_region, buf))

    def attn_cross_fwd(self, q, k, v, out=None, lse=None, workspace=None):
        self.calls.append(("product",))
        return out, lse

    def ring_free(self, prev_region, device=None):
        self.calls.append(("free_signal", prev_region))

    def ring_merge(self, o_blk, lse_blk, acc, lse_in, lse_out, first, out=None):
        self.calls.append(("merge", first, out is not None))

    def ring_attend(self, q_rot, k, v, acc, lse_in, lse_out, first, out=None):
        self.calls.append(("attend", first, out is not None))


def test_ring_call_sequence():
    """Rank 1 of 3: neighbours mapped (next = rank 2, previous = rank 0); per
    call one load, then per step the free wait and pass (not at the last
    step), the product with its merge into the accumulator (one call; the
    last one writes the output), the free signal to the previous rank and
    the full wait (not at the last step), with counts that grow across
    calls."""
    import torch
    from full_spatiotemporal_attention_b200.ring import RingAttention
    import full_spatiotemporal_attention_b200 as va
    fake = FakeRingBackend(1)
    handles = [b"handle-of-0x10000", None, b"handle-of-0x30000"]
    ra = RingAttention(va.Grid.make(3, 4, 4), 1, 2, world=3, rank=1, device="cpu", backend=fake,
                       exchange=lambda h: [handles[0], h, handles[2]])
    own, nxt, prv = 0x20000, 0x30000 + 0x7000000, 0x10000 + 0x7000000
    assert (ra.region, ra.next_region, ra.prev_region) == (own, nxt, prv)
    x = torch.zeros((1, 2, 16, 128), dtype=torch.bfloat16)
    for c in (1, 2):
        fake.calls.clear()
        assert ra(x, x, x) is ra.out
        expect = [("load", own, 3, 1, False)]
        for s in range(3):
            if s < 2:
                expect += [("wait", own, 1, (c - 1) * 3 + s), ("pass", own, nxt, s % 2)]
            expect += [("attend", s == 0, s == 2), ("free_signal", prv)]
            if s < 2:
                expect += [("wait", own, 0, (c - 1) * 2 + s + 1)]
        assert fake.calls == expect
    ra.close()
    assert fake.calls[-3:] == [("close", nxt), ("close", prv), ("free", own)]


def test_ring_two_ranks_share_one_neighbour():
    """With two ranks the next and the previous rank are the same one: it is
    mapped once and unmapped once."""
    from full_spatiotemporal_attention_b200.ring import RingAttention
    import full_spatiotemporal_attention_b200 as va
    fake = FakeRingBackend(0)
    ra = RingAttention(va.Grid.make(2, 4, 4), 1, 1, world=2, rank=0, device="cpu", backend=fake,
                       exchange=lambda h: [h, b"handle-of-0x20000"])
    assert ra.next_region == ra.prev_region == 0x20000 + 0x7000000
    ra.close()
    assert [c for c in fake.calls if c[0] in ("open", "close")] == [
        ("open", 0x20000 + 0x7000000), ("close", 0x20000 + 0x7000000)]
    with pytest.raises(ValueError, match="split"):
        RingAttention(va.Grid.make(1, 3, 3), 1, 1, world=2, rank=0, device="cpu",
                      backend=FakeRingBackend(0), exchange=lambda h: [h, h])
