"""Robustness checks of the CUDA path that need no sanitizer and fault nothing.

* Guard bands: every output (and the workspace) sits between bands of
  sentinel values; after each entry point runs on ragged shapes, the bands
  must be untouched, so no kernel writes outside its buffers.
* Watchdog: a probe kernel waits on an arrival that never comes; the bounded
  wait must give up, record its code in the device error word and return,
  and the context must stay usable afterwards.
"""
import numpy as np
import pytest

import oracle
import seeded_inputs as si
from conftest import bf16_bits_to_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

GUARD = 2048                      # elements of sentinel on each side (4 KB of bf16)
SENT16 = -24415                   # 0xA0A1 as int16: a bf16 value no kernel writes here
SENT32 = -1.2345e-33


@pytest.fixture(scope="module")
def va():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from full_spatiotemporal_attention_b200 import build
    build.build()
    import full_spatiotemporal_attention_b200 as va
    return va


class Guarded:
    """A contiguous tensor of `shape` inside a buffer with sentinel bands."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape))
        self.buf = torch.empty(n + 2 * GUARD, dtype=dtype, device="cuda")
        if dtype == torch.bfloat16:
            self.buf.view(torch.int16).fill_(SENT16)
        else:
            self.buf.fill_(SENT32)
        self.t = self.buf[GUARD:GUARD + n].view(shape)
        self.n = n

    def bands_intact(self):
        lo, hi = self.buf[:GUARD], self.buf[GUARD + self.n:]
        if self.buf.dtype == torch.bfloat16:
            lo, hi = lo.view(torch.int16), hi.view(torch.int16)
            return bool((lo == SENT16).all()) and bool((hi == SENT16).all())
        return bool((lo == SENT32).all()) and bool((hi == SENT32).all())


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16).cuda()


def guarded_workspace(nbytes):
    buf = torch.full((nbytes + 4096,), 0xAB, dtype=torch.uint8, device="cuda")
    return buf, buf[:nbytes]


def tail_intact(buf, nbytes):
    return bool((buf[nbytes:] == 0xAB).all())


def grid_of(va, w):
    return va.Grid.make(w.T, w.H, w.W, w.n_text, w.dims, w.theta)


RAGGED = [si.Workload("g_255", 3, 5, 17, 3, (44, 42, 42), seed=21),
          si.Workload("g_joint", 2, 6, 10, 2, (16, 56, 56), n_text=37, seed=22),
          si.Workload("g_b2", 2, 7, 9, 2, (44, 42, 42), batch=2, seed=23)]


@pytest.mark.parametrize("w", RAGGED, ids=lambda w: w.name)
def test_rope_and_full_attention_stay_inside_their_buffers(va, w):
    q, k, v = (dev(x) for x in si.qkv(w))
    g = grid_of(va, w)
    y = Guarded(w.shape, torch.bfloat16)
    va.rope3d_apply(k, g, out=y.t)
    o = Guarded(w.shape, torch.bfloat16)
    lse = Guarded(w.shape[:3], torch.float32)
    need = va.workspace_bytes(w.batch, w.heads, w.N, g)
    wsbuf, ws = guarded_workspace(need)
    va.attn3d_full_fwd(q, k, v, g, out=o.t, lse=lse.t, workspace=ws)
    torch.cuda.synchronize()
    assert y.bands_intact() and o.bands_intact() and lse.bands_intact()
    assert tail_intact(wsbuf, need)
    assert bool(torch.isfinite(o.t.float()).all())
    assert va.device_error() == 0


def test_factorised_window_and_cross_stay_inside_their_buffers(va):
    w = RAGGED[0]
    q, k, v = (dev(x) for x in si.qkv(w))
    g = grid_of(va, w)
    need = va.workspace_bytes(w.batch, w.heads, w.N, g)
    os_, ot = Guarded(w.shape, torch.bfloat16), Guarded(w.shape, torch.bfloat16)
    wsbuf, ws = guarded_workspace(need)
    va.attn_factorized_fwd(q, k, v, g, out_spatial=os_.t, out_temporal=ot.t, workspace=ws)
    torch.cuda.synchronize()
    assert os_.bands_intact() and ot.bands_intact() and tail_intact(wsbuf, need)

    ow, lw = Guarded(w.shape, torch.bfloat16), Guarded(w.shape[:3], torch.float32)
    wsbuf, ws = guarded_workspace(need)
    va.attn_window_fwd(q, k, v, g, (3, 5, 1), out=ow.t, lse=lw.t, workspace=ws)
    torch.cuda.synchronize()
    assert ow.bands_intact() and lw.bands_intact() and tail_intact(wsbuf, need)

    xw = si.Workload("g_cross", 1, 1, 300, 3, (44, 42, 42), seed=24, n_kv=129)
    xq, xk, xv = (dev(x) for x in si.qkv(xw))
    ox, lx = Guarded(xw.shape, torch.bfloat16), Guarded(xw.shape[:3], torch.float32)
    xneed = va.cross_workspace_bytes(1, 3, 300, 129)
    wsbuf, ws = guarded_workspace(xneed)
    va.attn_cross_fwd(xq, xk, xv, out=ox.t, lse=lx.t, workspace=ws)
    torch.cuda.synchronize()
    assert ox.bands_intact() and lx.bands_intact() and tail_intact(wsbuf, xneed)
    assert va.device_error() == 0


def test_watchdog_gives_up_and_the_context_stays_usable(va):
    assert va.device_error(reset=True) in (0,)
    va.watchdog_selftest()
    torch.cuda.synchronize()
    assert va.device_error(reset=True) == 4          # VA3D_DEVERR_TIMEOUT_SELFTEST
    assert va.device_error() == 0                    # the reset cleared it
    # the same context still computes correct results
    w = si.WORKLOADS["tiny"]
    q, k, v = si.qkv(w)
    o = va.attn3d_full_fwd(dev(q), dev(k), dev(v), grid_of(va, w))
    ref = oracle.attention(q, k, v, oracle.Grid(w.T, w.H, w.W, w.n_text, w.dims, w.theta))
    got = bf16_bits_to_f64(o.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))
    assert np.abs(got.reshape(ref.shape) - ref).max() <= 1.5e-2
    assert va.device_error() == 0
