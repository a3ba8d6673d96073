"""Host logic of Ulysses context parallelism on the CPU.

The exchange itself runs in the library's kernels (tested on a GPU with
emulated ranks).  Here two gloo ranks run ``UlyssesAttention`` over a fake
backend that records every call: the IPC handles travel through
``all_gather_object``, each rank must map exactly its peers' regions in rank
order, and every call must scatter, wait, attend, gather and wait with the
right epoch."""
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


def test_failed_exchange_releases_the_region():
    from full_spatiotemporal_attention_b200.ulysses import UlyssesAttention
    import full_spatiotemporal_attention_b200 as va
    fake = FakeBackend(1)
    with pytest.raises(RuntimeError, match="entries"):
        UlyssesAttention(va.Grid.make(2, 4, 4), 1, 2, world=2, rank=1, device="cpu",
                         backend=fake, exchange=lambda h: [h])
    assert fake.calls[-1] == ("free", 0x20000)
