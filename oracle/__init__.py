"""Oracle for 3D-RoPE video self-attention: plain, slow, obviously correct.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(the C-ABI library and its Python binding) never imports, links or executes
anything here, and this package never imports the product.

Two layers:

* page helpers in pure Python, written from the closed forms the handbook page
  ("A video model's architecture: spatiotemporal attention and the 3D VAE")
  states: ``latent_shape``, ``patch_grid``, ``token_count`` and
  ``token_width`` (section "The latents: the extra time axis"),
  ``attention_flops`` and ``linear_flops`` (section "How attention sees time:
  factorised or full"), ``rope_ranges`` (section "Position: RoPE in three
  dimensions");
* the fp64 C oracle (``va3d_oracle.c``) for RoPE and attention, reached with
  ctypes: ``rope3d``, ``attention`` (full, spatial, temporal, joint),
  ``window_attention`` (local 3D windows) and ``cross_attention`` (video
  queries over text keys).
"""
from __future__ import annotations

import ctypes
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
# Page helpers: the handbook's closed forms for the token grid and the cost
# model, written from its formulas
# ---------------------------------------------------------------------------

# Handbook, "The latents: the extra time axis": the causal 3D VAE keeps the
# first frame and folds every 4 further frames into one latent frame, divides
# height and width by 8, and emits 16 channels; the DiT then cuts latents into
# 1 x 2 x 2 patches (one token each).
VAE_TIME_STRIDE = 4
VAE_SPACE_STRIDE = 8
LATENT_CHANNELS = 16
PATCH = (1, 2, 2)


def latent_shape(frames, height, width):
    """Latent (T, H_lat, W_lat) of a clip: 1 + floor((frames - 1) / 4) frames
    and floor(height / 8) x floor(width / 8) (the page divides with floors)."""
    return (1 + (frames - 1) // VAE_TIME_STRIDE, height // VAE_SPACE_STRIDE,
            width // VAE_SPACE_STRIDE)


def patch_grid(frames, height, width):
    """Token grid (T', H', W'): the latent shape divided by the patch size."""
    return tuple(n // p for n, p in zip(latent_shape(frames, height, width), PATCH))


def token_count(frames, height, width):
    """Video tokens T' * H' * W' of a clip."""
    t, h, w = patch_grid(frames, height, width)
    return t * h * w


def token_width():
    """Values per token before the patch embedding: channels x patch volume (64)."""
    return LATENT_CHANNELS * PATCH[0] * PATCH[1] * PATCH[2]


def attention_flops(grid, width, layers, mode):
    """Attention FLOPs of one denoising step (handbook, "How attention sees
    time: factorised or full").  ``grid`` is the token grid (T', H', W'),
    ``width`` the model width (heads x head_dim).  Full attention costs
    4 (T'H'W')^2 width per layer; the factorised form costs 4 width
    (T' (H'W')^2 + H'W' T'^2): T' spatial sequences of H'W' tokens plus H'W'
    temporal sequences of T' tokens."""
    t, h, w = grid
    s = h * w
    if mode == "full":
        per_layer = 4 * (t * s) ** 2 * width
    elif mode == "factorised":
        per_layer = 4 * width * (t * s * s + s * t * t)
    else:
        raise ValueError(f"mode must be 'full' or 'factorised', not {mode!r}")
    return layers * per_layer


def linear_flops(tokens, width, layers):
    """Linear-layer FLOPs of one step, 24 tokens width^2 per layer (same section)."""
    return layers * 24 * tokens * width * width


def rope_ranges(split, head_dim=128):
    """Head-dim ranges [start, end) turned by t, h and w (handbook, "Position:
    RoPE in three dimensions"): three contiguous ranges in t, h, w order that
    together fill the head, each of an even width (it holds whole pairs)."""
    if len(split) != 3 or sum(split) != head_dim or any(d < 0 or d % 2 for d in split):
        raise ValueError(f"a 3D RoPE split needs three even widths summing to {head_dim}: {split}")
    d_t, d_h, _ = split
    return {"t": (0, d_t), "h": (d_t, d_t + d_h), "w": (d_t + d_h, head_dim)}


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
