"""Ring context parallelism for full 3D attention, one process per GPU.

Rank r holds tokens [r*N/P, (r+1)*N/P) of every head.  Unlike the Ulysses
form it splits no heads, so it serves any head count (12 heads on 8 GPUs).
One call:

1. ``ring_load``: this rank's Q and K turned at their global positions (Q
   into ``q_rot``, K with V into the region's block buffer 0);
2. for s = 0 .. P-1: the product of ``q_rot`` with the block in buffer
   s % 2, merged into an fp32 accumulator by log-sum-exp weights in the
   attention kernel's own epilogue (``ring_attend``; the last step writes the
   bf16 output), while the same block is copied into the next rank's buffer
   (s + 1) % 2 (``ring_pass``, on a side stream so that the copy overlaps the
   product);
3. ordering by the region counters: before a pass, wait until the next rank
   has finished the products that read that buffer (``free``); after a
   product, signal the previous rank (``ring_free``); before the next
   product, wait until the block has landed (``full``).

Every step runs in the library's kernels; this class owns the buffers,
exchanges IPC handles once and sequences the calls.
"""
from __future__ import annotations

from .ulysses import MAX_WORLD, _all_gather_object


class RingAttention:
    """Full 3D attention over a sequence split across `world` ranks, K/V
    blocks passed around the ring.  ``backend`` and ``exchange`` as for
    ``UlyssesAttention``."""

    def __init__(self, grid, batch, heads, *, world=None, rank=None, group=None, device=None,
                 backend=None, exchange=None, overlap=True):
        import torch
        if backend is None:
            import full_spatiotemporal_attention_b200 as backend
        self.va = va = backend
        if world is None or rank is None:
            import torch.distributed as dist
            if dist.is_available() and dist.is_initialized():
                world, rank = dist.get_world_size(group), dist.get_rank(group)
            else:
                world, rank = 1, 0
        if not 1 <= world <= MAX_WORLD or not 0 <= rank < world:
            raise ValueError(f"rank {rank} of {world} (1..{MAX_WORLD} ranks)")
        if grid.N % world:
            raise ValueError(f"{grid.N} tokens do not split over {world} ranks")
        self.grid, self.batch, self.heads, self.world, self.rank = grid, batch, heads, world, rank
        self.N, self.n_loc = grid.N, grid.N // world
        self.device = torch.device(device) if device is not None else torch.device(
            "cuda", torch.cuda.current_device())
        nbytes = va.ring_region_bytes(batch, heads, self.N, world)
        if nbytes == 0:
            raise ValueError("unsupported ring sizes")
        self.region = va.region_alloc(nbytes)
        self._opened = []
        try:
            self.prev_region = self.next_region = self.region
            if world > 1:
                exchange = exchange or (lambda obj: _all_gather_object(obj, group))
                handles = exchange(va.ipc_export(self.region))
                if len(handles) != world:
                    raise RuntimeError(f"handle exchange returned {len(handles)} entries for "
                                       f"{world} ranks")
                nxt, prv = (rank + 1) % world, (rank - 1) % world
                self.next_region = va.ipc_open(handles[nxt])
                self._opened.append(self.next_region)
                if prv != nxt:
                    self.prev_region = va.ipc_open(handles[prv])
                    self._opened.append(self.prev_region)
                else:
                    self.prev_region = self.next_region
            shape = (batch, heads, self.n_loc, 128)
            k0, v0, k1, v1 = va.ring_offsets(batch, heads, self.N, world)
            view = va.region_view
            self.kbuf = [view(self.region, k0, shape, self.device),
                         view(self.region, k1, shape, self.device)]
            self.vbuf = [view(self.region, v0, shape, self.device),
                         view(self.region, v1, shape, self.device)]
            bf, f32 = torch.bfloat16, torch.float32
            self.q_rot = torch.empty(shape, dtype=bf, device=self.device)
            self.out = torch.empty(shape, dtype=bf, device=self.device)
            self.acc = torch.empty(shape, dtype=f32, device=self.device)
            self.lse = [torch.empty(shape[:3], dtype=f32, device=self.device) for _ in range(2)]
            self.side = torch.cuda.Stream(self.device) if (overlap and world > 1 and
                                                           self.device.type == "cuda") else None
        except BaseException:
            self._release()
            raise
        self.calls = 0

    def _shape_args(self):
        return self.world, self.batch, self.heads, self.N

    def __call__(self, q, k, v, *, k_rotated=False):
        """q, k, v: this rank's token slice [B, heads, N/P, 128] bf16; returns
        its slice of the attention output (a buffer reused by the next call)."""
        import contextlib
        import torch
        va, P = self.va, self.world
        shape = (self.batch, self.heads, self.n_loc, 128)
        for t, name in ((q, "q"), (k, "k"), (v, "v")):
            if tuple(t.shape) != shape:
                raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {shape}")
        c = self.calls + 1
        va.ring_load(q, k, v, self.q_rot, self.region, P, self.rank, self.grid, k_rotated=k_rotated)
        for s in range(P):
            cur = s % 2
            if s < P - 1:
                if self.side is not None:
                    self.side.wait_stream(torch.cuda.current_stream(self.device))
                ctx = torch.cuda.stream(self.side) if self.side is not None else contextlib.nullcontext()
                with ctx:
                    # the next rank has finished every product that read the
                    # buffer this pass overwrites
                    va.ring_wait(self.region, va.RING_FREE, (c - 1) * P + s, *self._shape_args(),
                                 device=self.device)
                    va.ring_pass(self.region, self.next_region, cur, *self._shape_args(),
                                 device=self.device)
            va.ring_attend(self.q_rot, self.kbuf[cur], self.vbuf[cur], self.acc,
                           self.lse[(s + 1) % 2], self.lse[s % 2], first=(s == 0),
                           out=self.out if s == P - 1 else None)
            if self.side is not None and s < P - 1:
                torch.cuda.current_stream(self.device).wait_stream(self.side)
            if P > 1:
                va.ring_free(self.prev_region, device=self.device)
            if s < P - 1:
                va.ring_wait(self.region, va.RING_FULL, (c - 1) * (P - 1) + s + 1,
                             *self._shape_args(), device=self.device)
        self.calls = c
        return self.out

    def _release(self):
        for ptr in self._opened:
            self.va.ipc_close(ptr)
        self._opened = []
        if self.region is not None:
            self.va.region_free(self.region)
            self.region = None

    def close(self, barrier=None):
        """Unmap the neighbours' regions and free this rank's (after every
        rank's last call: pass ``barrier``)."""
        import torch
        if self.region is None:
            return
        if self.device.type == "cuda":
            torch.cuda.synchronize(self.device)
        if barrier is not None:
            barrier()
        self.kbuf = self.vbuf = None
        self._release()
