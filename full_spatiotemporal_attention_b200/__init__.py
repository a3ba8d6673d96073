"""B200-native 3D-RoPE video self-attention: thin Python binding of libva3d.so.

Every step of the hot path runs in the library's sm_100a kernels; this module
only checks tensor properties and passes pointers, sizes and the current CUDA
stream to the C ABI declared in ``include/va3d.h``.  There is no fallback: if
the library is missing or a tensor is not a contiguous bf16 CUDA tensor of
shape [B, heads, N, 128], the call raises.

Entry points (same names as the C ABI):

* ``rope3d_apply(x, grid)``                 3D RoPE of a [B, heads, N, 128] tensor
* ``attn3d_full_fwd(q, k, v, grid)``        full 3D (or joint video+text) attention
* ``attn_factorized_fwd(q, k, v, grid)``    spatial and temporal passes
* ``attn_cross_fwd(q, k, v)``               video-to-text cross-attention (no RoPE)
* ``attn_window_fwd(q, k, v, grid, window)`` local 3D-window attention
* ``ulysses_scatter / ulysses_gather / ulysses_wait`` and the region / IPC
  calls: the exchange steps of Ulysses context parallelism (composed by
  ``ulysses.UlyssesAttention``)
* ``grid_from_video(frames, height, width)``  token grid of a clip
* ``workspace_bytes(...)``, ``device_error()``
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libva3d.so")

VA3D_OK = 0
VA3D_K_ROTATED = 1
HEAD_DIM = 128

SYMBOLS = ("va3d_status_string", "va3d_version", "va3d_grid_from_video",
           "va3d_workspace_bytes", "rope3d_apply", "attn3d_full_fwd",
           "attn_factorized_fwd", "va3d_device_error", "attn3d_full_fwd_noalloc",
           "va3d_cross_workspace_bytes", "attn_cross_fwd", "attn_window_fwd",
           "va3d_watchdog_selftest", "va3d_ulysses_region_bytes", "va3d_ulysses_offsets",
           "va3d_region_alloc", "va3d_region_free", "va3d_ipc_export", "va3d_ipc_open",
           "va3d_ipc_close", "va3d_ulysses_scatter", "va3d_ulysses_gather", "va3d_ulysses_wait",
           "va3d_ring_region_bytes", "va3d_ring_offsets", "va3d_ring_load", "va3d_ring_pass",
           "va3d_ring_free", "va3d_ring_wait", "va3d_ring_merge", "va3d_ring_attend")


class VA3DError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {status} ({_status_string(status)})")


class Grid(ctypes.Structure):
    """va3d_grid_t: post-patch grid T', H', W', appended text tokens, RoPE split, theta."""
    _fields_ = [("T", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
                ("n_text", ctypes.c_int),
                ("d_t", ctypes.c_int), ("d_h", ctypes.c_int), ("d_w", ctypes.c_int),
                ("theta", ctypes.c_double)]

    @classmethod
    def make(cls, T, H, W, n_text=0, dims=(44, 42, 42), theta=10000.0):
        return cls(T, H, W, n_text, dims[0], dims[1], dims[2], theta)

    @property
    def n_video(self):
        return self.T * self.H * self.W

    @property
    def N(self):
        return self.n_video + self.n_text

    def __repr__(self):
        return (f"Grid(T={self.T}, H={self.H}, W={self.W}, n_text={self.n_text}, "
                f"dims=({self.d_t}, {self.d_h}, {self.d_w}), theta={self.theta})")


def _load():
    # Build (or rebuild, when the sources changed) with nvcc first; without
    # nvcc and without a library built from these sources the import fails.
    from . import build as _build
    try:
        _build.build()
    except (OSError, RuntimeError) as e:
        raise ImportError(f"{LIB_PATH} could not be built from the current sources "
                          f"(nvcc for sm_100a): {e}") from e
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, u, sz, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_size_t, ctypes.c_float
    gp = ctypes.POINTER(Grid)
    lib.va3d_status_string.argtypes = [i]
    lib.va3d_status_string.restype = ctypes.c_char_p
    lib.va3d_version.restype = i
    lib.va3d_grid_from_video.argtypes = [i, i, i, i, i, i, i, gp]
    lib.va3d_workspace_bytes.argtypes = [i, i, i, i, gp, u]
    lib.va3d_workspace_bytes.restype = sz
    lib.rope3d_apply.argtypes = [vp, vp, i, i, i, i, gp, vp]
    lib.attn3d_full_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, gp, f, u, vp, sz, vp]
    lib.attn_factorized_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, gp, f, u, vp, sz, vp]
    lib.va3d_device_error.argtypes = [i]
    lib.va3d_watchdog_selftest.argtypes = [vp]
    lib.attn3d_full_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, gp, f, u, vp]
    lib.va3d_cross_workspace_bytes.argtypes = [i, i, i, i, i]
    lib.va3d_cross_workspace_bytes.restype = sz
    lib.attn_cross_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, vp, sz, vp]
    lib.attn_window_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, gp, i, i, i, f, u, vp, sz, vp]
    szp, vpp = ctypes.POINTER(sz), ctypes.POINTER(vp)
    lib.va3d_ulysses_region_bytes.argtypes = [i, i, i, i, i]
    lib.va3d_ulysses_region_bytes.restype = sz
    lib.va3d_ulysses_offsets.argtypes = [i, i, i, i, i, szp, szp, szp, szp]
    lib.va3d_region_alloc.argtypes = [sz, vpp]
    lib.va3d_region_free.argtypes = [vp]
    lib.va3d_ipc_export.argtypes = [vp, ctypes.c_char_p]
    lib.va3d_ipc_open.argtypes = [ctypes.c_char_p, vpp]
    lib.va3d_ipc_close.argtypes = [vp]
    lib.va3d_ulysses_scatter.argtypes = [vp, vp, vp, vpp, i, i, i, i, i, i, gp, u, vp]
    lib.va3d_ulysses_gather.argtypes = [vp, vpp, i, i, i, i, i, i, vp]
    lib.va3d_ulysses_wait.argtypes = [vp, i, ctypes.c_ulonglong, i, i, i, i, i, vp]
    lib.va3d_ring_region_bytes.argtypes = [i, i, i, i, i]
    lib.va3d_ring_region_bytes.restype = sz
    lib.va3d_ring_offsets.argtypes = [i, i, i, i, i, szp, szp, szp, szp]
    lib.va3d_ring_load.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, gp, u, vp]
    lib.va3d_ring_pass.argtypes = [vp, vp, i, i, i, i, i, i, vp]
    lib.va3d_ring_free.argtypes = [vp, vp]
    lib.va3d_ring_wait.argtypes = [vp, i, ctypes.c_ulonglong, i, i, i, i, i, vp]
    lib.va3d_ring_merge.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, vp]
    lib.va3d_ring_attend.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp]
    return lib


lib = _load()


def _status_string(status):
    return lib.va3d_status_string(int(status)).decode()


def version():
    return lib.va3d_version()


def grid_from_video(frames, height, width, dims=(44, 42, 42), n_text=0):
    """Token grid of a clip: T' = 1 + (frames-1)/4, H' = height/16, W' = width/16."""
    g = Grid()
    rc = lib.va3d_grid_from_video(frames, height, width, dims[0], dims[1], dims[2], n_text,
                                  ctypes.byref(g))
    if rc != VA3D_OK:
        raise VA3DError("va3d_grid_from_video", rc)
    return g


def workspace_bytes(B, heads, N, grid, k_rotated=False):
    return int(lib.va3d_workspace_bytes(B, heads, N, HEAD_DIM, ctypes.byref(grid),
                                        VA3D_K_ROTATED if k_rotated else 0))


# ---------------------------------------------------------------- tensors

def _torch():
    import torch
    return torch


def _check(t, name, shape=None):
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
    if t.dim() != 4 or t.shape[-1] != HEAD_DIM:
        raise ValueError(f"{name} must be [B, heads, N, {HEAD_DIM}], got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t


def _stream(t):
    return ctypes.c_void_p(_torch().cuda.current_stream(t.device).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _run(name, device, *args):
    """Call C entry point `name` with `device` current (the library launches on
    the current device and takes its per-device state from it), raising
    VA3DError on a non-zero status."""
    with _torch().cuda.device(device):
        rc = getattr(lib, name)(*args)
    if rc != VA3D_OK:
        raise VA3DError(name, rc)


def _check_lse(lse, shape):
    torch = _torch()
    if lse is not None and (not isinstance(lse, torch.Tensor) or lse.dtype != torch.float32
                            or tuple(lse.shape) != tuple(shape) or not lse.is_contiguous()
                            or not lse.is_cuda):
        raise ValueError(f"lse must be a contiguous CUDA float32 {list(shape)} tensor")
    return lse


def _device(device=None):
    """`device` as a torch.device (the current CUDA device when None)."""
    torch = _torch()
    return torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)


def _cur_stream(device=None):
    return ctypes.c_void_p(_torch().cuda.current_stream(device).cuda_stream)


def _same_device(ref, *ts):
    for t in ts:
        if t is not None and t.device != ref.device:
            raise ValueError(f"tensors must be on one device: {t.device} != {ref.device}")


# Workspaces the binding keeps for calls that pass none, one per (device,
# stream), grown on demand: calls on one stream are ordered, so they can share
# one buffer, and calls on different streams never do.
_WORKSPACES = {}


def release_workspaces():
    """Drop the workspaces kept for calls that passed none (synchronise first
    if calls that use them may still be running)."""
    _WORKSPACES.clear()


def _workspace(q, grid, k_rotated, workspace):
    B, H, N, _ = q.shape
    need = workspace_bytes(B, H, N, grid, k_rotated)
    if workspace is None:
        torch = _torch()
        key = (q.device.index, torch.cuda.current_stream(q.device).cuda_stream)
        workspace = _WORKSPACES.get(key)
        if workspace is None or workspace.numel() < need:
            workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
            _WORKSPACES[key] = workspace
    if workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace holds {workspace.numel()} bytes, needs {need}")
    return workspace


def rope3d_apply(x, grid, out=None):
    """3D RoPE of x [B, heads, N, 128] (bf16, CUDA); out may be x (in place)."""
    _check(x, "x")
    if out is None:
        out = _torch().empty_like(x)
    _check(out, "out", x.shape)
    _same_device(x, out)
    B, H, N, D = x.shape
    _run("rope3d_apply", x.device, _ptr(x), _ptr(out), B, H, N, D, ctypes.byref(grid), _stream(x))
    return out


def attn3d_full_fwd(q, k, v, grid, *, scale=None, return_lse=False, k_rotated=False,
                    out=None, lse=None, workspace=None):
    """Full 3D attention (joint video+text when grid.n_text > 0).

    Returns o [B, heads, N, 128] bf16 (and lse [B, heads, N] fp32 if asked)."""
    torch = _torch()
    _check(q, "q")
    _check(k, "k", q.shape)
    _check(v, "v", q.shape)
    B, H, N, D = q.shape
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", q.shape)
    if return_lse and lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _check_lse(lse, (B, H, N))
    ws = _workspace(q, grid, k_rotated, workspace)
    _same_device(q, k, v, out, lse, ws)
    _run("attn3d_full_fwd", q.device, _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, D,
         ctypes.byref(grid), float(scale or 0.0), VA3D_K_ROTATED if k_rotated else 0, _ptr(ws),
         ws.numel() * ws.element_size(), _stream(q))
    return (out, lse) if (return_lse or lse is not None) else out


def attn3d_full_fwd_noalloc(q, k, v, grid, *, scale=None, return_lse=False, k_rotated=False,
                            out=None, lse=None):
    """attn3d_full_fwd using the library's built-in 64 MiB scratch instead of a
    workspace (for callers that cannot allocate device memory); calls that
    overlap in time on the GPU race on that scratch."""
    torch = _torch()
    _check(q, "q")
    _check(k, "k", q.shape)
    _check(v, "v", q.shape)
    B, H, N, D = q.shape
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", q.shape)
    if return_lse and lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _check_lse(lse, (B, H, N))
    _same_device(q, k, v, out, lse)
    _run("attn3d_full_fwd_noalloc", q.device, _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
         B, H, N, D, ctypes.byref(grid), float(scale or 0.0), VA3D_K_ROTATED if k_rotated else 0,
         _stream(q))
    return (out, lse) if (return_lse or lse is not None) else out


def attn_factorized_fwd(q, k, v, grid, *, spatial=True, temporal=True, scale=None,
                        k_rotated=False, out_spatial=None, out_temporal=None, workspace=None):
    """Factorised attention: (o_spatial, o_temporal); a skipped pass returns None."""
    torch = _torch()
    _check(q, "q")
    _check(k, "k", q.shape)
    _check(v, "v", q.shape)
    B, H, N, D = q.shape
    if spatial and out_spatial is None:
        out_spatial = torch.empty_like(q)
    if temporal and out_temporal is None:
        out_temporal = torch.empty_like(q)
    if not spatial:
        out_spatial = None
    if not temporal:
        out_temporal = None
    for t, nm in ((out_spatial, "out_spatial"), (out_temporal, "out_temporal")):
        if t is not None:
            _check(t, nm, q.shape)
    ws = _workspace(q, grid, k_rotated, workspace)
    _same_device(q, k, v, out_spatial, out_temporal, ws)
    _run("attn_factorized_fwd", q.device, _ptr(q), _ptr(k), _ptr(v), _ptr(out_spatial),
         _ptr(out_temporal), B, H, N, D, ctypes.byref(grid), float(scale or 0.0),
         VA3D_K_ROTATED if k_rotated else 0, _ptr(ws), ws.numel() * ws.element_size(), _stream(q))
    return out_spatial, out_temporal


def attn_window_fwd(q, k, v, grid, window, *, scale=None, return_lse=False, k_rotated=False,
                    out=None, lse=None, workspace=None):
    """Local 3D-window attention: tokens attend inside non-overlapping windows
    of ``window = (wt, wh, ww)`` tokens (each dividing the grid), 3D RoPE as in
    full attention.  Returns o (and lse if asked)."""
    torch = _torch()
    _check(q, "q")
    _check(k, "k", q.shape)
    _check(v, "v", q.shape)
    B, H, N, D = q.shape
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", q.shape)
    if return_lse and lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _check_lse(lse, (B, H, N))
    ws = _workspace(q, grid, k_rotated, workspace)
    _same_device(q, k, v, out, lse, ws)
    wt, wh, ww = (int(x) for x in window)
    _run("attn_window_fwd", q.device, _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, D,
         ctypes.byref(grid), wt, wh, ww, float(scale or 0.0), VA3D_K_ROTATED if k_rotated else 0,
         _ptr(ws), ws.numel() * ws.element_size(), _stream(q))
    return (out, lse) if (return_lse or lse is not None) else out


def cross_workspace_bytes(B, heads, Nq, Nkv):
    return int(lib.va3d_cross_workspace_bytes(B, heads, Nq, Nkv, HEAD_DIM))


def attn_cross_fwd(q, k, v, *, scale=None, return_lse=False, out=None, lse=None,
                   workspace=None):
    """Cross-attention of video queries q [B, heads, Nq, 128] to text keys and
    values k, v [B, heads, Nkv, 128]; no RoPE.  Returns o [B, heads, Nq, 128]
    (and lse [B, heads, Nq] fp32 if asked)."""
    torch = _torch()
    _check(q, "q")
    _check(k, "k")
    B, H, Nq, D = q.shape
    Nkv = k.shape[2]
    if k.shape[:2] != q.shape[:2]:
        raise ValueError(f"k has shape {tuple(k.shape)}, expected [{B}, {H}, Nkv, {D}]")
    _check(v, "v", k.shape)
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", q.shape)
    if return_lse and lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _check_lse(lse, (B, H, Nq))
    _same_device(q, k, v, out, lse, workspace)
    # the workspace is optional here (it only lets the last partial wave split)
    _run("attn_cross_fwd", q.device, _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Nq,
         Nkv, D, float(scale or 0.0), _ptr(workspace),
         workspace.numel() * workspace.element_size() if workspace is not None else 0, _stream(q))
    return (out, lse) if (return_lse or lse is not None) else out


# ------------------------------------------- Ulysses context parallelism

IPC_HANDLE_BYTES = 64
PHASE_SCATTER, PHASE_GATHER = 0, 1


def ulysses_region_bytes(B, heads, N, world):
    """Bytes of one rank's exchange region (0 if the sizes are not supported)."""
    return int(lib.va3d_ulysses_region_bytes(B, heads, N, HEAD_DIM, world))


def ulysses_offsets(B, heads, N, world):
    """(off_q, off_k, off_v, off_o): byte offsets of Qh, Kh, Vh and the O shard."""
    offs = [ctypes.c_size_t() for _ in range(4)]
    rc = lib.va3d_ulysses_offsets(B, heads, N, HEAD_DIM, world, *(ctypes.byref(o) for o in offs))
    if rc != VA3D_OK:
        raise VA3DError("va3d_ulysses_offsets", rc)
    return tuple(int(o.value) for o in offs)


def region_alloc(nbytes):
    """Device memory (cudaMalloc, zeroed) on the current device; returns its address."""
    p = ctypes.c_void_p()
    rc = lib.va3d_region_alloc(int(nbytes), ctypes.byref(p))
    if rc != VA3D_OK:
        raise VA3DError("va3d_region_alloc", rc)
    return int(p.value)


def region_free(ptr):
    rc = lib.va3d_region_free(ctypes.c_void_p(ptr))
    if rc != VA3D_OK:
        raise VA3DError("va3d_region_free", rc)


def ipc_export(ptr):
    """CUDA IPC handle of a region, as bytes."""
    buf = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    rc = lib.va3d_ipc_export(ctypes.c_void_p(ptr), buf)
    if rc != VA3D_OK:
        raise VA3DError("va3d_ipc_export", rc)
    return buf.raw


def ipc_open(handle):
    """Map a peer's region from its handle; returns the address in this process."""
    if len(handle) != IPC_HANDLE_BYTES:
        raise ValueError(f"an IPC handle has {IPC_HANDLE_BYTES} bytes, got {len(handle)}")
    p = ctypes.c_void_p()
    rc = lib.va3d_ipc_open(bytes(handle), ctypes.byref(p))
    if rc != VA3D_OK:
        raise VA3DError("va3d_ipc_open", rc)
    return int(p.value)


def ipc_close(ptr):
    rc = lib.va3d_ipc_close(ctypes.c_void_p(ptr))
    if rc != VA3D_OK:
        raise VA3DError("va3d_ipc_close", rc)


def _ptr_array(regions):
    return (ctypes.c_void_p * len(regions))(*[ctypes.c_void_p(int(r)) for r in regions])


def ulysses_scatter(q, k, v, regions, rank, grid, *, k_rotated=False):
    """Send this rank's token slice q, k, v [B, heads, N/world, 128] to every
    rank's region (world = len(regions)); keys turned at their global
    positions unless k_rotated."""
    _check(q, "q")
    _check(k, "k", q.shape)
    _check(v, "v", q.shape)
    B, H, n_loc, D = q.shape
    world = len(regions)
    _same_device(q, k, v)
    _run("va3d_ulysses_scatter", q.device, _ptr(q), _ptr(k), _ptr(v), _ptr_array(regions), world,
         rank, B, H, n_loc * world, D, ctypes.byref(grid), VA3D_K_ROTATED if k_rotated else 0,
         _stream(q))


def ulysses_gather(o_heads, regions, rank, heads):
    """Send this rank's attention output o_heads [B, heads/world, N, 128] back
    as token slices into every rank's O shard."""
    _check(o_heads, "o_heads")
    B, hpw, N, D = o_heads.shape
    world = len(regions)
    if hpw * world != heads:
        raise ValueError(f"o_heads holds {hpw} heads, expected {heads} / {world}")
    _run("va3d_ulysses_gather", o_heads.device, _ptr(o_heads), _ptr_array(regions), world, rank, B,
         heads, N, D, _stream(o_heads))


def ulysses_wait(region, phase, epoch, world, B, heads, N, device=None):
    """Stream-ordered, bounded wait for every peer's signals of call `epoch`."""
    _run("va3d_ulysses_wait", _device(device), ctypes.c_void_p(region), phase, int(epoch), world, B,
         heads, N, HEAD_DIM, _cur_stream(device))


# ----------------------------------------------- ring context parallelism

RING_FULL, RING_FREE = 0, 1


def ring_region_bytes(B, heads, N, world):
    return int(lib.va3d_ring_region_bytes(B, heads, N, HEAD_DIM, world))


def ring_offsets(B, heads, N, world):
    """(off_k0, off_v0, off_k1, off_v1) inside a ring region."""
    offs = [ctypes.c_size_t() for _ in range(4)]
    rc = lib.va3d_ring_offsets(B, heads, N, HEAD_DIM, world, *(ctypes.byref(o) for o in offs))
    if rc != VA3D_OK:
        raise VA3DError("va3d_ring_offsets", rc)
    return tuple(int(o.value) for o in offs)


def ring_load(q, k, v, q_rot, region, world, rank, grid, *, k_rotated=False):
    """Turn this rank's slice q, k [B, heads, N/world, 128] at global
    positions into q_rot and the region's block buffer 0 (with v)."""
    _check(q, "q")
    _check(k, "k", q.shape)
    _check(v, "v", q.shape)
    _check(q_rot, "q_rot", q.shape)
    B, H, n_loc, D = q.shape
    _same_device(q, k, v, q_rot)
    _run("va3d_ring_load", q.device, _ptr(q), _ptr(k), _ptr(v), _ptr(q_rot), ctypes.c_void_p(region),
         world, rank, B, H, n_loc * world, D, ctypes.byref(grid),
         VA3D_K_ROTATED if k_rotated else 0, _stream(q))


def ring_pass(region, next_region, buf, world, B, heads, N, device=None):
    _run("va3d_ring_pass", _device(device), ctypes.c_void_p(region), ctypes.c_void_p(next_region),
         buf, world, B, heads, N, HEAD_DIM, _cur_stream(device))


def ring_free(prev_region, device=None):
    _run("va3d_ring_free", _device(device), ctypes.c_void_p(prev_region), _cur_stream(device))


def ring_wait(region, counter, count, world, B, heads, N, device=None):
    _run("va3d_ring_wait", _device(device), ctypes.c_void_p(region), counter, int(count), world, B,
         heads, N, HEAD_DIM, _cur_stream(device))


def ring_merge(o_blk, lse_blk, acc, lse_in, lse_out, *, first, out=None):
    """Merge a block's (o_blk, lse_blk) into the fp32 accumulator (acc,
    lse_in) -> (acc, lse_out); with `out`, also write the merged bf16 output."""
    torch = _torch()
    _check(o_blk, "o_blk")
    B, H, n, D = o_blk.shape
    if acc.dtype != torch.float32 or tuple(acc.shape) != (B, H, n, D) or not acc.is_contiguous():
        raise ValueError("acc must be a contiguous float32 tensor shaped like o_blk")
    for t, nm in ((lse_blk, "lse_blk"), (lse_out, "lse_out")) + (() if first else ((lse_in, "lse_in"),)):
        if t.dtype != torch.float32 or tuple(t.shape) != (B, H, n) or not t.is_contiguous():
            raise ValueError(f"{nm} must be a contiguous float32 [B, heads, n] tensor")
    if out is not None:
        _check(out, "out", o_blk.shape)
    _same_device(o_blk, lse_blk, acc, lse_out, out, None if first else lse_in)
    _run("va3d_ring_merge", o_blk.device, _ptr(o_blk), _ptr(lse_blk), _ptr(acc),
         None if first else _ptr(lse_in), _ptr(lse_out), _ptr(out), B, H, n, 1 if first else 0,
         _stream(o_blk))


def ring_attend(q_rot, k, v, acc, lse_in, lse_out, *, first, out=None, scale=None):
    """One ring block step: attention of q_rot [B, heads, n, 128] over the
    block k, v [B, heads, n_keys, 128] (no RoPE), merged into the fp32
    accumulator (acc, lse_in) -> (acc, lse_out) inside the attention kernel;
    with `out`, the merged output is also written as bf16."""
    torch = _torch()
    _check(q_rot, "q_rot")
    _check(k, "k")
    B, H, n, D = q_rot.shape
    if k.shape[:2] != q_rot.shape[:2]:
        raise ValueError(f"k has shape {tuple(k.shape)}, expected [{B}, {H}, n_keys, {D}]")
    _check(v, "v", k.shape)
    if (not isinstance(acc, torch.Tensor) or acc.dtype != torch.float32
            or tuple(acc.shape) != (B, H, n, D) or not acc.is_contiguous()):
        raise ValueError("acc must be a contiguous float32 tensor shaped like q_rot")
    _check_lse(lse_out, (B, H, n))
    if not first:
        _check_lse(lse_in, (B, H, n))
    if out is not None:
        _check(out, "out", q_rot.shape)
    _same_device(q_rot, k, v, acc, lse_out, out, None if first else lse_in)
    _run("va3d_ring_attend", q_rot.device, _ptr(q_rot), _ptr(k), _ptr(v), _ptr(acc),
         None if first else _ptr(lse_in), _ptr(lse_out), _ptr(out), B, H, n, k.shape[2], D,
         float(scale or 0.0), 1 if first else 0, _stream(q_rot))


class _DeviceMemory:
    """__cuda_array_interface__ of a stretch of a region, for a zero-copy tensor view."""

    def __init__(self, ptr, shape):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": "<i2",
                                         "data": (int(ptr), False), "version": 3,
                                         "strides": None}


def region_view(ptr, offset, shape, device):
    """bf16 tensor of `shape` over region memory at ptr + offset (no copy; the
    region must outlive it)."""
    torch = _torch()
    t = torch.as_tensor(_DeviceMemory(ptr + offset, shape), device=device)
    return t.view(torch.bfloat16)


def watchdog_selftest():
    """Launch the watchdog probe on the current device (its wait times out by
    design after 2 s); read the result with device_error()."""
    rc = lib.va3d_watchdog_selftest(ctypes.c_void_p(_torch().cuda.current_stream().cuda_stream))
    if rc != VA3D_OK:
        raise VA3DError("va3d_watchdog_selftest", rc)


def device_error(reset=True):
    """Watchdog code recorded on the current device (0 = none); synchronises."""
    rc = lib.va3d_device_error(1 if reset else 0)
    if rc < 0:
        raise VA3DError("va3d_device_error", rc)
    return rc
