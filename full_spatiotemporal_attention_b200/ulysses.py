"""Ulysses context parallelism for full 3D attention, one process per GPU.

Each rank holds a contiguous token slice [rank*N/P, (rank+1)*N/P) of every
head (the sequence-parallel layout: with absolute (t, h, w) coordinates each
rank can turn its own tokens, handbook "A video model's architecture",
section "Position: RoPE in three dimensions").  One call:

1. ``ulysses_scatter``: every rank writes its slice of head group j
   (heads/P heads) into rank j's region over peer memory, keys turned by 3D
   RoPE at their global positions on the way;
2. ``ulysses_wait`` (scatter phase): a bounded device-side wait until all P
   ranks' slices have landed;
3. ``attn3d_full_fwd`` on whole sequences of this rank's heads (keys already
   rotated; queries turned in the attention kernel's prologue);
4. ``ulysses_gather``: the output's token slices go back to their owners;
5. ``ulysses_wait`` (gather phase).

Every step runs in the library's kernels; this class only owns the regions,
exchanges their IPC handles once (``torch.distributed.all_gather_object``)
and sequences the calls.  The returned O shard is a view into this rank's
region, valid until the next call.
"""
from __future__ import annotations

from dataclasses import dataclass

MAX_WORLD = 8


@dataclass(frozen=True)
class UlyssesPlan:
    """Shapes of one rank's part of the exchange."""
    batch: int
    heads: int
    N: int
    world: int
    rank: int

    @property
    def heads_per_rank(self):
        return self.heads // self.world

    @property
    def tokens_per_rank(self):
        return self.N // self.world

    @property
    def local_shape(self):
        """Sequence shard in and out: [B, heads, N/P, 128]."""
        return (self.batch, self.heads, self.tokens_per_rank, 128)

    @property
    def head_shard_shape(self):
        """Whole sequences of this rank's heads: [B, heads/P, N, 128]."""
        return (self.batch, self.heads_per_rank, self.N, 128)

    @property
    def token_range(self):
        n = self.tokens_per_rank
        return self.rank * n, (self.rank + 1) * n

    @property
    def head_range(self):
        h = self.heads_per_rank
        return self.rank * h, (self.rank + 1) * h


def make_plan(batch, heads, N, world, rank):
    if not 1 <= world <= MAX_WORLD:
        raise ValueError(f"world must be 1..{MAX_WORLD}, got {world}")
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside 0..{world - 1}")
    if batch < 1 or heads < 1 or N < 1:
        raise ValueError("batch, heads and N must be positive")
    if heads % world:
        raise ValueError(f"{heads} heads do not split over {world} ranks")
    if N % world:
        raise ValueError(f"{N} tokens do not split over {world} ranks")
    return UlyssesPlan(batch, heads, N, world, rank)


def _all_gather_object(obj, group):
    import torch.distributed as dist
    out = [None] * dist.get_world_size(group)
    dist.all_gather_object(out, obj, group=group)
    return out


class UlyssesAttention:
    """Full 3D attention over a sequence split across `world` ranks.

    ``backend`` is the binding module (default: the library); ``exchange``
    maps this rank's picklable value to the list of every rank's values
    (default: ``all_gather_object`` over ``group``)."""

    def __init__(self, grid, batch, heads, *, world=None, rank=None, group=None, device=None,
                 backend=None, exchange=None):
        import torch
        if backend is None:
            import full_spatiotemporal_attention_b200 as backend
        self.va = backend
        if world is None or rank is None:
            import torch.distributed as dist
            if dist.is_available() and dist.is_initialized():
                world, rank = dist.get_world_size(group), dist.get_rank(group)
            else:
                world, rank = 1, 0
        self.grid = grid
        self.plan = make_plan(batch, heads, grid.N, world, rank)
        self.device = torch.device(device) if device is not None else torch.device(
            "cuda", torch.cuda.current_device())
        p = self.plan
        nbytes = self.va.ulysses_region_bytes(p.batch, p.heads, p.N, p.world)
        if nbytes == 0:
            raise ValueError(f"unsupported Ulysses sizes: {p}")
        self.region = self.va.region_alloc(nbytes)
        self._opened = []
        try:
            if p.world > 1:
                exchange = exchange or (lambda obj: _all_gather_object(obj, group))
                handles = exchange(self.va.ipc_export(self.region))
                if len(handles) != p.world:
                    raise RuntimeError(f"handle exchange returned {len(handles)} entries for "
                                       f"{p.world} ranks")
                regions = []
                for j, h in enumerate(handles):
                    if j == p.rank:
                        regions.append(self.region)
                    else:
                        ptr = self.va.ipc_open(h)
                        self._opened.append(ptr)
                        regions.append(ptr)
                self.regions = regions
            else:
                self.regions = [self.region]
            off_q, off_k, off_v, off_o = self.va.ulysses_offsets(p.batch, p.heads, p.N, p.world)
            view = self.va.region_view
            self.qh = view(self.region, off_q, p.head_shard_shape, self.device)
            self.kh = view(self.region, off_k, p.head_shard_shape, self.device)
            self.vh = view(self.region, off_v, p.head_shard_shape, self.device)
            self.o_shard = view(self.region, off_o, p.local_shape, self.device)
            self.o_heads = torch.empty(p.head_shard_shape, dtype=torch.bfloat16, device=self.device)
            self.workspace = torch.empty(
                max(self.va.workspace_bytes(p.batch, p.heads_per_rank, p.N, grid, k_rotated=True),
                    256), dtype=torch.uint8, device=self.device)
        except BaseException:
            self._release()
            raise
        # calls made of each phase; every rank makes the same sequence
        self.epochs = [0, 0]

    @property
    def epoch(self):
        return self.epochs[self.va.PHASE_GATHER]

    def scatter(self, q, k, v, *, k_rotated=False):
        """Steps 1-2: this rank's slice out to every rank, then wait for all
        ranks' slices of this rank's heads."""
        p, va = self.plan, self.va
        for t, name in ((q, "q"), (k, "k"), (v, "v")):
            if tuple(t.shape) != p.local_shape:
                raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {p.local_shape}")
        va.ulysses_scatter(q, k, v, self.regions, p.rank, self.grid, k_rotated=k_rotated)
        self.epochs[va.PHASE_SCATTER] += 1
        va.ulysses_wait(self.region, va.PHASE_SCATTER, self.epochs[va.PHASE_SCATTER], p.world,
                        p.batch, p.heads, p.N, self.device)

    def attend(self):
        """Step 3: full attention over whole sequences of this rank's heads."""
        self.va.attn3d_full_fwd(self.qh, self.kh, self.vh, self.grid, k_rotated=True,
                                out=self.o_heads, workspace=self.workspace)

    def gather(self):
        """Steps 4-5: output token slices back to their owners; returns this
        rank's slice (a view into the region)."""
        p, va = self.plan, self.va
        va.ulysses_gather(self.o_heads, self.regions, p.rank, p.heads)
        self.epochs[va.PHASE_GATHER] += 1
        va.ulysses_wait(self.region, va.PHASE_GATHER, self.epochs[va.PHASE_GATHER], p.world,
                        p.batch, p.heads, p.N, self.device)
        return self.o_shard

    def factorised(self, q, k, v, *, out_spatial=None):
        """Factorised attention of this rank's slice: (o_spatial, o_temporal),
        each [B, heads, N/P, 128].  The slice must hold whole frames (P divides
        T'): the spatial pass then runs on the rank's own frames with no
        exchange (a frame's t rotation is the same for all its tokens and
        cancels in q.k, so local frame numbers give the global result), and
        the temporal pass, which needs every frame of a position, runs on
        whole sequences of this rank's heads after a Ulysses exchange of the
        raw keys (its kernel turns only their t range).  o_temporal is a view
        into the region, valid until the next call."""
        p, va = self.plan, self.va
        g = self.grid
        if g.n_text != 0 or g.T % p.world != 0:
            raise ValueError(f"factorised slices need whole frames and no text: T'={g.T} "
                             f"over {p.world} ranks, n_text={g.n_text}")
        local = va.Grid.make(g.T // p.world, g.H, g.W, 0, (g.d_t, g.d_h, g.d_w), g.theta)
        out_spatial, _ = va.attn_factorized_fwd(q, k, v, local, temporal=False,
                                                out_spatial=out_spatial)
        self.scatter(q, k, v, k_rotated=True)   # raw keys copied as they are
        va.attn_factorized_fwd(self.qh, self.kh, self.vh, g, spatial=False,
                               out_temporal=self.o_heads, workspace=self._temporal_workspace())
        return out_spatial, self.gather()

    def _temporal_workspace(self):
        if getattr(self, "_tws", None) is None:
            import torch
            p = self.plan
            self._tws = torch.empty(
                max(self.va.workspace_bytes(p.batch, p.heads_per_rank, p.N, self.grid), 256),
                dtype=torch.uint8, device=self.device)
        return self._tws

    def __call__(self, q, k, v, *, k_rotated=False):
        """q, k, v: this rank's token slice [B, heads, N/P, 128] bf16; returns
        its slice of the attention output (a view into the region, valid until
        the next call)."""
        self.scatter(q, k, v, k_rotated=k_rotated)
        self.attend()
        return self.gather()

    def _release(self):
        for ptr in self._opened:
            self.va.ipc_close(ptr)
        self._opened = []
        if self.region is not None:
            self.va.region_free(self.region)
            self.region = None

    def close(self, barrier=None):
        """Unmap the peers' regions and free this rank's.  Every rank must have
        finished its last call first (pass ``barrier``, e.g.
        ``torch.distributed.barrier``, to make sure no peer still writes here)."""
        import torch
        if self.region is None:
            return
        if self.device.type == "cuda":
            torch.cuda.synchronize(self.device)
        if barrier is not None:
            barrier()
        self.qh = self.kh = self.vh = self.o_shard = None
        self._release()
