"""Oracle for 3D-RoPE video self-attention: plain, slow, obviously correct.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(the C-ABI library and its Python binding) never imports, links or executes
anything here, and this package never imports the product.

Two layers:

* page helpers in pure Python, restating the closed forms the handbook page
  ("A video model's architecture: spatiotemporal attention and the 3D VAE")
  prints: ``video_tokens`` (section "The latents: the extra time axis"),
  ``attn_flops`` and ``linear_flops`` (section "How attention sees time:
  factorised or full"), ``rope_3d_dims`` (section "Position: RoPE in three
  dimensions");
* the fp64 C oracle (``va3d_oracle.c``) for RoPE and attention, reached with
  ctypes: ``rope3d``, ``attention`` (full, spatial, temporal, joint),
  ``window_attention`` (local 3D windows) and ``cross_attention`` (video
  queries over text keys).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "va3d_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

FULL, SPATIAL, TEMPORAL = 0, 1, 2
MODES = {"full": FULL, "spatial": SPATIAL, "temporal": TEMPORAL}


# ---------------------------------------------------------------------------
# Page helpers (closed forms printed by the handbook page)
# ---------------------------------------------------------------------------

def video_tokens(frames, h, w, ft=4, fs=8, pt=1, ps=2, latent_ch=16):
    """Latent grid, token count and token width for a clip.

    Handbook, "The latents: the extra time axis": the first frame is encoded
    on its own and every ``ft`` further frames become one latent frame;
    space shrinks by ``fs``; patches of ``pt x ps x ps`` become tokens (floor
    division, as the page's function does).  Returns
    ``((T, H_lat, W_lat), tokens, token_dim)`` where ``H_lat, W_lat`` are the
    latent (pre-patch) sizes, as the page prints them.
    """
    T = 1 + (frames - 1) // ft
    H, W = h // fs, w // fs
    tokens = (T // pt) * (H // ps) * (W // ps)
    return (T, H, W), tokens, latent_ch * pt * ps * ps


def patch_grid(frames, h, w, ft=4, fs=8, pt=1, ps=2):
    """Post-patch token grid (T', H', W') = (T/pt, H_lat/ps, W_lat/ps)."""
    (T, H, W), _, _ = video_tokens(frames, h, w, ft, fs, pt, ps)
    return T // pt, H // ps, W // ps


def attn_flops(T, H, W, d, layers, mode):
    """Attention FLOPs per denoising step (handbook, "How attention sees time").

    ``T, H, W`` are latent sizes (patch 2 applied inside, as on the page);
    ``d`` is the model width (heads x head_dim).  Factorised: spatial term
    T*4*n_sp^2*d plus temporal term n_sp*4*T^2*d; full: 4*(T*n_sp)^2*d.
    """
    n_sp = (H // 2) * (W // 2)
    if mode == "factorised":
        per_layer = T * 4 * n_sp ** 2 * d + n_sp * 4 * T ** 2 * d
    elif mode == "full":
        per_layer = 4 * (T * n_sp) ** 2 * d
    else:
        raise ValueError(mode)
    return layers * per_layer


def linear_flops(tokens, d, layers):
    """Linear-layer FLOPs per step, 24*N*d^2 per layer (same section)."""
    return layers * 24 * tokens * d * d


def rope_3d_dims(head_dim=128, axes=(16, 56, 56)):
    """Head-dim allocation of 3D RoPE; the three ranges must fill the head
    (handbook, "Position: RoPE in three dimensions")."""
    assert sum(axes) == head_dim
    return {"t": axes[0], "h": axes[1], "w": axes[2]}


def token_coords(i, T, H, W):
    """(t, h, w) of video token i: t-major, w fastest (the handbook's shard
    listing enumerates ``for t, for h, for w``)."""
    return i // (H * W), (i // W) % H, i % W


# ---------------------------------------------------------------------------
# C oracle
# ---------------------------------------------------------------------------

class _Grid(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
                ("n_text", ctypes.c_int),
                ("d_t", ctypes.c_int), ("d_h", ctypes.c_int), ("d_w", ctypes.c_int),
                ("theta", ctypes.c_double),
                ("off_t", ctypes.c_int), ("off_h", ctypes.c_int), ("off_w", ctypes.c_int)]


@dataclass(frozen=True)
class Grid:
    """Token grid and RoPE split: T', H', W', appended text tokens, (d_t, d_h, d_w)."""
    T: int
    H: int
    W: int
    n_text: int = 0
    dims: tuple = (44, 42, 42)
    theta: float = 10000.0
    offset: tuple = (0, 0, 0)

    @property
    def n_video(self):
        return self.T * self.H * self.W

    @property
    def N(self):
        return self.n_video + self.n_text

    def _c(self):
        return _Grid(self.T, self.H, self.W, self.n_text, *self.dims, self.theta, *self.offset)


def build(force=False):
    """Compile the C oracle with gcc (plain -O2, no fast-math, OpenMP)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-std=c11", "-Wall", "-o", _LIB, _SRC, "-lm"]
    subprocess.check_call(cmd)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        lib.oracle_rope3d.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_long,
                                      ctypes.c_long, ctypes.c_int, ctypes.POINTER(_Grid)]
        lib.oracle_attention.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_long, ctypes.c_long, ctypes.c_int,
                                         ctypes.POINTER(_Grid), ctypes.c_int, ctypes.c_double,
                                         ctypes.c_int, ctypes.c_void_p, ctypes.c_long,
                                         ctypes.c_void_p, ctypes.c_void_p]
        lib.oracle_token_coords.argtypes = [ctypes.POINTER(_Grid), ctypes.c_long,
                                            ctypes.POINTER(ctypes.c_int),
                                            ctypes.POINTER(ctypes.c_int),
                                            ctypes.POINTER(ctypes.c_int)]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_window_attention.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                ctypes.c_long, ctypes.c_long, ctypes.c_int,
                                                ctypes.POINTER(_Grid), ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, ctypes.c_double, ctypes.c_int,
                                                ctypes.c_void_p, ctypes.c_long, ctypes.c_void_p,
                                                ctypes.c_void_p]
        lib.oracle_window_attention.restype = ctypes.c_int
        lib.oracle_cross_attention.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.c_long, ctypes.c_long, ctypes.c_long,
                                               ctypes.c_int, ctypes.c_double, ctypes.c_void_p,
                                               ctypes.c_long, ctypes.c_void_p, ctypes.c_void_p]
        lib.oracle_cross_attention.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads():
    """OpenMP threads the oracle uses."""
    return int(_load().oracle_num_threads())


def _bits(a):
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (uint16)")
    return a


def c_token_coords(grid: Grid, i: int):
    t, h, w = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    g = grid._c()
    text = _load().oracle_token_coords(ctypes.byref(g), i, ctypes.byref(t), ctypes.byref(h),
                                       ctypes.byref(w))
    return None if text else (t.value, h.value, w.value)


def rope3d(x_bits, grid: Grid):
    """fp64 3D RoPE of bf16 bits shaped [..., N, head_dim]."""
    x = _bits(x_bits)
    N, D = x.shape[-2], x.shape[-1]
    BH = int(np.prod(x.shape[:-2])) if x.ndim > 2 else 1
    y = np.empty(x.shape, dtype=np.float64)
    g = grid._c()
    rc = _load().oracle_rope3d(x.ctypes.data, y.ctypes.data, BH, N, D, ctypes.byref(g))
    if rc != 0:
        raise ValueError(f"oracle_rope3d rejected the arguments ({rc})")
    return y


def attention(q_bits, k_bits, v_bits, grid: Grid, mode="full", rows=None, scale=None,
              rotate=True, want_lse=False):
    """fp64 attention for query ``rows`` (all rows when None).

    Inputs are bf16 bits [..., N, head_dim] (leading dims flattened to BH).
    Returns out [BH, len(rows), head_dim] (and lse [BH, len(rows)]).
    """
    q, k, v = _bits(q_bits), _bits(k_bits), _bits(v_bits)
    N, D = q.shape[-2], q.shape[-1]
    BH = int(np.prod(q.shape[:-2])) if q.ndim > 2 else 1
    if rows is None:
        rows = np.arange(N, dtype=np.int64)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.empty((BH, rows.size, D), dtype=np.float64)
    lse = np.empty((BH, rows.size), dtype=np.float64) if want_lse else None
    g = grid._c()
    rc = _load().oracle_attention(q.ctypes.data, k.ctypes.data, v.ctypes.data, BH, N, D,
                                  ctypes.byref(g), MODES[mode] if isinstance(mode, str) else mode,
                                  float(scale) if scale else 0.0, 1 if rotate else 0,
                                  rows.ctypes.data, rows.size, out.ctypes.data,
                                  lse.ctypes.data if want_lse else None)
    if rc != 0:
        raise ValueError(f"oracle_attention rejected the arguments ({rc})")
    return (out, lse) if want_lse else out


def window_attention(q_bits, k_bits, v_bits, grid: Grid, window, rows=None, scale=None,
                     rotate=True, want_lse=False):
    """fp64 local 3D-window attention (anthology record sota-390, the W.A.L.T
    comparison): the grid is cut into non-overlapping windows of
    ``window = (wt, wh, ww)`` tokens and every token attends to its own window,
    3D RoPE as in full attention.  Returns out [BH, len(rows), d] (and lse)."""
    q, k, v = _bits(q_bits), _bits(k_bits), _bits(v_bits)
    N, D = q.shape[-2], q.shape[-1]
    BH = int(np.prod(q.shape[:-2])) if q.ndim > 2 else 1
    if rows is None:
        rows = np.arange(N, dtype=np.int64)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.empty((BH, rows.size, D), dtype=np.float64)
    lse = np.empty((BH, rows.size), dtype=np.float64) if want_lse else None
    g = grid._c()
    wt, wh, ww = (int(x) for x in window)
    rc = _load().oracle_window_attention(q.ctypes.data, k.ctypes.data, v.ctypes.data, BH, N, D,
                                         ctypes.byref(g), wt, wh, ww,
                                         float(scale) if scale else 0.0, 1 if rotate else 0,
                                         rows.ctypes.data, rows.size, out.ctypes.data,
                                         lse.ctypes.data if want_lse else None)
    if rc != 0:
        raise ValueError(f"oracle_window_attention rejected the arguments ({rc})")
    return (out, lse) if want_lse else out


def cross_attention(q_bits, k_bits, v_bits, rows=None, scale=None, want_lse=False):
    """fp64 text cross-attention of a Wan block ("04 HunyuanVideo and Wan",
    section 3.1): query rows of q [..., Nq, d] attend to all keys of
    k, v [..., Nkv, d]; no rotation.  Returns out [BH, len(rows), d] (and lse)."""
    q, k, v = _bits(q_bits), _bits(k_bits), _bits(v_bits)
    Nq, D = q.shape[-2], q.shape[-1]
    Nkv = k.shape[-2]
    BH = int(np.prod(q.shape[:-2])) if q.ndim > 2 else 1
    if k.shape != v.shape or k.shape[-1] != D or int(np.prod(k.shape[:-2])) != BH:
        raise ValueError("k and v must be [..., Nkv, d] with q's leading dims")
    if rows is None:
        rows = np.arange(Nq, dtype=np.int64)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.empty((BH, rows.size, D), dtype=np.float64)
    lse = np.empty((BH, rows.size), dtype=np.float64) if want_lse else None
    rc = _load().oracle_cross_attention(q.ctypes.data, k.ctypes.data, v.ctypes.data, BH, Nq, Nkv,
                                        D, float(scale) if scale else 0.0, rows.ctypes.data,
                                        rows.size, out.ctypes.data,
                                        lse.ctypes.data if want_lse else None)
    if rc != 0:
        raise ValueError(f"oracle_cross_attention rejected the arguments ({rc})")
    return (out, lse) if want_lse else out


def full_flops(N, heads, head_dim=128):
    """4*N^2*d*heads: the FLOP count of one full-attention forward."""
    return 4 * N * N * head_dim * heads


def factorised_flops(T, H, W, heads, head_dim=128):
    """4*d*heads*(T*(HW)^2 + HW*T^2): spatial plus temporal pass."""
    hw = H * W
    return 4 * head_dim * heads * (T * hw * hw + hw * T * T)


def default_scale(head_dim=128):
    return 1.0 / math.sqrt(head_dim)
