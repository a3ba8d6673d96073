"""Ulysses context parallelism through the C ABI, on one GPU.

Ranks are emulated on the one device: every "rank" gets its own region (all
local memory), the copy kernels of all ranks are launched one after the
other on one stream, and each wait is launched only after every signal it
counts has been made, so no kernel ever waits on a concurrent one.  The
exchanged tensors are compared bit for bit with the slices they must hold,
and the assembled output with the fp64 oracle."""
import numpy as np
import pytest

import oracle
import seeded_inputs as si
from test_gpu_parity import check, custom, dev, host, ogrid, vgrid

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def va():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from full_spatiotemporal_attention_b200 import build
    build.build()
    import full_spatiotemporal_attention_b200 as va
    return va


def bits_equal(a, b):
    return torch.equal(a.contiguous().view(torch.int16), b.contiguous().view(torch.int16))


def ulps_apart(a, b):
    """Largest distance in bf16 units in the last place (sign-magnitude bits
    mapped to a monotone integer line; +0 and -0 coincide)."""
    def key(t):
        x = t.contiguous().view(torch.int16).to(torch.int32)
        return torch.where(x >= 0, x, -(x & 0x7FFF))
    return int((key(a) - key(b)).abs().max())


def emulate(va, w, world, calls=1):
    """Run `calls` exchanges of `world` emulated ranks; returns the regions'
    views after the last one and the assembled output [B, heads, N, 128]."""
    q, k, v = (dev(x) for x in si.qkv(w))
    g = vgrid(va, w)
    B, H, N = w.batch, w.heads, w.N
    hpw, nl = H // world, N // world
    nbytes = va.ulysses_region_bytes(B, H, N, world)
    regions = [va.region_alloc(nbytes) for _ in range(world)]
    try:
        offs = va.ulysses_offsets(B, H, N, world)
        views = [[va.region_view(r, off, (B, hpw, N, 128), q.device) for off in offs[:3]]
                 for r in regions]
        shards = [va.region_view(r, offs[3], (B, H, nl, 128), q.device) for r in regions]
        o_heads = [torch.empty((B, hpw, N, 128), dtype=torch.bfloat16, device=q.device)
                   for _ in range(world)]
        ws = torch.empty(va.workspace_bytes(B, hpw, N, g, k_rotated=True), dtype=torch.uint8,
                         device=q.device)
        for epoch in range(1, calls + 1):
            for r in range(world):
                sl = slice(r * nl, (r + 1) * nl)
                va.ulysses_scatter(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(),
                                   v[:, :, sl].contiguous(), regions, r, g)
            for r in range(world):
                va.ulysses_wait(regions[r], va.PHASE_SCATTER, epoch, world, B, H, N)
            for r in range(world):
                qh, kh, vh = views[r]
                va.attn3d_full_fwd(qh, kh, vh, g, k_rotated=True, out=o_heads[r], workspace=ws)
            for r in range(world):
                va.ulysses_gather(o_heads[r], regions, r, H)
            for r in range(world):
                va.ulysses_wait(regions[r], va.PHASE_GATHER, epoch, world, B, H, N)
        torch.cuda.synchronize()
        assert va.device_error() == 0
        # copies out of the regions before they are freed
        got = {"views": [[t.clone() for t in vs] for vs in views],
               "o": torch.cat([s.clone() for s in shards], dim=2)}
    finally:
        torch.cuda.synchronize()
        for r in regions:
            va.region_free(r)
    return q, k, v, g, got


CASES = [(si.WORKLOADS["tiny"], 2), (si.WORKLOADS["c17f480"], 4),
         (custom("u_joint", 2, 6, 10, heads=4, n_text=40, dims=(16, 56, 56)), 2),
         (custom("u_b2", 3, 4, 6, heads=6, batch=2), 3),
         (custom("u_w8", 2, 4, 4, heads=8), 8)]


@pytest.mark.parametrize("w,world", CASES, ids=lambda x: getattr(x, "name", str(x)))
def test_exchange_moves_exact_slices(va, w, world):
    q, k, v, g, got = emulate(va, w, world)
    # keys turned by the single-GPU pre-pass: the same fp32 angles and the
    # same rotation, so at most one bf16 rounding apart (the compiler may
    # contract the two products of a rotated element into an FMA differently
    # in the two kernels); text keys (no rotation) are copied exactly
    kr = va.rope3d_apply(k, g)
    hpw = w.heads // world
    nv = w.T * w.H * w.W
    for r in range(world):
        hs = slice(r * hpw, (r + 1) * hpw)
        qh, kh, vh = got["views"][r]
        assert bits_equal(qh, q[:, hs]), f"Qh of rank {r}"
        assert bits_equal(vh, v[:, hs]), f"Vh of rank {r}"
        assert ulps_apart(kh, kr[:, hs]) <= 1, f"Kh of rank {r}"
        assert bits_equal(kh[:, :, nv:], k[:, hs, nv:]), f"text keys of rank {r}"


@pytest.mark.parametrize("w,world", CASES, ids=lambda x: getattr(x, "name", str(x)))
def test_context_parallel_output_matches_oracle(va, w, world):
    q, k, v, g, got = emulate(va, w, world)
    qb, kb, vb = si.qkv(w)
    ref = oracle.attention(qb, kb, vb, ogrid(w))
    check(host(got["o"]).reshape(ref.shape), ref, f"ulysses {w.name} x{world}")
    # the single-GPU call on the same inputs: both within the bar of the
    # oracle, hence within twice the bar of each other
    single = va.attn3d_full_fwd(q, k, v, g)
    diff = (single.float() - got["o"].float()).abs().max().item()
    assert diff <= 2 * 1.5e-2


def test_counters_across_calls(va):
    """Three calls in a row: every wait finds its epoch complete."""
    w = si.WORKLOADS["tiny"]
    _, _, _, _, got = emulate(va, w, 2, calls=3)
    qb, kb, vb = si.qkv(w)
    ref = oracle.attention(qb, kb, vb, ogrid(w))
    check(host(got["o"]).reshape(ref.shape), ref, "ulysses tiny x2, third call")


def test_keys_that_come_rotated_are_copied(va):
    w = si.WORKLOADS["tiny"]
    q, k, v = (dev(x) for x in si.qkv(w))
    g = vgrid(va, w)
    kr = va.rope3d_apply(k, g)
    B, H, N = w.batch, w.heads, w.N
    region = va.region_alloc(va.ulysses_region_bytes(B, H, N, 1))
    try:
        va.ulysses_scatter(q, kr, v, [region], 0, g, k_rotated=True)
        va.ulysses_wait(region, va.PHASE_SCATTER, 1, 1, B, H, N)
        off_k = va.ulysses_offsets(B, H, N, 1)[1]
        kh = va.region_view(region, off_k, (B, H, N, 128), q.device).clone()
        assert bits_equal(kh, kr)   # copied, not turned again
        assert va.device_error() == 0
    finally:
        torch.cuda.synchronize()
        va.region_free(region)


def test_single_rank_class_end_to_end(va):
    from full_spatiotemporal_attention_b200.ulysses import UlyssesAttention
    w = si.WORKLOADS["c17f480"]
    q, k, v = (dev(x) for x in si.qkv(w))
    ua = UlyssesAttention(vgrid(va, w), w.batch, w.heads, world=1, rank=0)
    try:
        for _ in range(2):
            o = ua(q, k, v)
        qb, kb, vb = si.qkv(w)
        rows = si.sample_rows(w)
        ref = oracle.attention(qb, kb, vb, ogrid(w), rows=rows)
        got = host(o)[..., rows, :].reshape(ref.shape)
        check(got, ref, "ulysses class world 1")
        assert ua.epoch == 2 and va.device_error() == 0
    finally:
        ua.close()


def test_wait_gives_up_and_reports(va):
    """A wait whose signals never come (nothing scatters into this region)
    ends after its 2 s limit with VA3D_DEVERR_TIMEOUT_PEER; the context stays
    usable."""
    va.device_error(reset=True)
    region = va.region_alloc(va.ulysses_region_bytes(1, 2, 32, 2))
    try:
        va.ulysses_wait(region, va.PHASE_SCATTER, 1, 2, 1, 2, 32)
        assert va.device_error(reset=True) == 5
        # still usable afterwards
        x = torch.ones(4, device="cuda")
        assert float((x * 2).sum()) == 8.0
    finally:
        torch.cuda.synchronize()
        va.region_free(region)
