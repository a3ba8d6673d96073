"""Seeded synthetic workloads for 3D-RoPE video attention.

The only module shared by the CUDA path's tests/bench and the oracle: it
produces input bit patterns and workload descriptions and holds none of the
attention arithmetic.  Values come from a counter-based generator
(splitmix64 + Box-Muller, ``gen.c``), so they are identical on every machine
and thread count.

Workloads (all B=1, head_dim 128, theta 10000, scale 1/sqrt(128), bf16 Q/K/V
drawn from N(0, 1)):

========  ================================  =====  ================  ==================
name      grid T' x H' x W' (+ text)        heads  RoPE (t, h, w)    structure
========  ================================  =====  ================  ==================
tiny      2 x 4 x 4 = 32                    2      (44, 42, 42)      brute-force size
c17f480   5 x 30 x 52 = 7,800               12     (44, 42, 42)      17 frames 480x832
c81f480   21 x 30 x 52 = 32,760             12     (44, 42, 42)      81 frames 480x832
c81f720   21 x 45 x 80 = 75,600             40     (44, 42, 42)      K x2 on 10 % tokens
joint720  33 x 45 x 80 + 256 = 119,056      24     (16, 56, 56)      256 text tokens
========  ================================  =====  ================  ==================
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB = os.path.join(_HERE, "libseeded.so")

# stream ids of the tensors of one workload
Q_STREAM, K_STREAM, V_STREAM, SHARPEN_STREAM, ROWS_STREAM = 1, 2, 3, 4, 5


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    W: int
    heads: int
    dims: tuple
    n_text: int = 0
    batch: int = 1
    head_dim: int = 128
    theta: float = 10000.0
    seed: int = 1000
    sharpen_frac: float = 0.0   # fraction of tokens whose K is scaled by 2
    description: str = ""
    n_kv: int = 0               # > 0: cross-attention to n_kv separate key/value tokens

    @property
    def n_video(self):
        return self.T * self.H * self.W

    @property
    def N(self):
        return self.n_video + self.n_text

    @property
    def shape(self):
        return (self.batch, self.heads, self.N, self.head_dim)

    @property
    def kv_shape(self):
        n = self.n_kv if self.n_kv > 0 else self.N
        return (self.batch, self.heads, n, self.head_dim)


WORKLOADS = {
    "tiny": Workload("tiny", 2, 4, 4, 2, (44, 42, 42), seed=1001,
                     description="tiny grid 2x4x4, 2 heads"),
    "c17f480": Workload("c17f480", 5, 30, 52, 12, (44, 42, 42), seed=1002,
                        description="17-frame 480x832 clip, 5x30x52 = 7,800 tokens, 12 heads"),
    "c81f480": Workload("c81f480", 21, 30, 52, 12, (44, 42, 42), seed=1003,
                        description="81-frame 480x832 clip, 21x30x52 = 32,760 tokens, 12 heads"),
    "c81f720": Workload("c81f720", 21, 45, 80, 40, (44, 42, 42), seed=1004, sharpen_frac=0.1,
                        description="81-frame 720x1280 clip, 21x45x80 = 75,600 tokens, 40 heads, "
                                    "K x2 on 10% of tokens"),
    "joint720": Workload("joint720", 33, 45, 80, 24, (16, 56, 56), n_text=256, seed=1005,
                         description="129-frame 720x1280 clip, 33x45x80 = 118,800 video tokens "
                                     "+ 256 text tokens, 24 heads"),
    "cross720": Workload("cross720", 21, 45, 80, 40, (44, 42, 42), seed=1007, n_kv=512,
                         description="text cross-attention: 21x45x80 = 75,600 video queries "
                                     "x 512 text keys, 40 heads"),
    "refimg720": Workload("refimg720", 21, 45, 80, 40, (44, 42, 42), n_text=3 * 4096, seed=1006,
                          description="81-frame 720x1280 clip, 21x45x80 = 75,600 video tokens "
                                      "+ 3 reference images x 4,096 tokens = 87,888 tokens, "
                                      "40 heads"),
}


def build(force=False):
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11",
                           "-Wall", "-o", _LIB, _SRC, "-lm"])
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        lib.seeded_normal_bf16.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                                           ctypes.c_uint64, ctypes.c_double, ctypes.c_void_p]
        lib.seeded_uniform.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                                       ctypes.c_uint64, ctypes.c_void_p]
        _lib = lib
    return _lib


def normal_bf16(seed, stream, shape, scale=1.0, first=0):
    """bf16 bit patterns (uint16) of scale * N(0,1), element e = counter first+e."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    _load().seeded_normal_bf16(seed, stream, first, n, float(scale), out.ctypes.data)
    return out.reshape(shape)


def uniform(seed, stream, n, first=0):
    out = np.empty(int(n), dtype=np.float64)
    _load().seeded_uniform(seed, stream, first, int(n), out.ctypes.data)
    return out


def sharpened_tokens(w: Workload):
    """Boolean mask over token indices whose K rows are doubled (shared by heads)."""
    if w.sharpen_frac <= 0:
        return np.zeros(w.N, dtype=bool)
    return uniform(w.seed, SHARPEN_STREAM, w.kv_shape[2]) < w.sharpen_frac


def qkv(w: Workload):
    """(q, k, v) as uint16 bf16 bits: q [B, heads, N, head_dim], k and v
    [B, heads, N or n_kv, head_dim]."""
    q = normal_bf16(w.seed, Q_STREAM, w.shape)
    k = normal_bf16(w.seed, K_STREAM, w.kv_shape)
    v = normal_bf16(w.seed, V_STREAM, w.kv_shape)
    sel = sharpened_tokens(w)
    if sel.any():
        # doubling is exact in bf16: add one to the exponent field of nonzero finite values
        idx = np.nonzero(sel)[0]
        rows = k[:, :, idx, :]
        exp = (rows >> 7) & 0xFF
        bump = (exp != 0) & (exp < 0xFE)
        rows = np.where(bump, rows + np.uint16(1 << 7), rows).astype(np.uint16)
        k[:, :, idx, :] = rows
    return q, k, v


def sample_rows(w: Workload, count=512):
    """Seeded query rows for sampled parity: the structural rows (first/last
    row, every tile boundary tail, every frame boundary, and for joint
    workloads at least 64 text rows) plus seeded uniform picks up to count."""
    N = w.N
    must = {0, N - 1}
    for tile in (128, 256):
        last = (N // tile) * tile
        must.update({max(0, last - 1), min(N - 1, last)})
    hw = w.H * w.W
    for t in range(w.T):
        must.update({t * hw, min(N - 1, t * hw + hw - 1)})
    if w.n_text:
        nv = w.n_video
        text = np.linspace(nv, N - 1, num=min(64, w.n_text)).astype(np.int64)
        must.update(int(x) for x in text)
    must = sorted(x for x in must if 0 <= x < N)
    rest = count - len(must)
    picks = []
    if rest > 0:
        u = uniform(w.seed, ROWS_STREAM, 4 * rest + 16)
        cand = (u * N).astype(np.int64)
        have = set(must)
        for c in cand:
            c = int(min(c, N - 1))
            if c not in have:
                have.add(c)
                picks.append(c)
                if len(picks) == rest:
                    break
    return np.array(sorted(must + picks), dtype=np.int64)
