"""Context parallelism (Ulysses and ring forms) through the C ABI, on one GPU.

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


def emulate_factorised(va, w, world):
    """The factorised context-parallel step of `world` emulated ranks: the
    spatial pass on each rank's own frames, the temporal pass after a
    Ulysses exchange of the raw keys.  Returns (o_spatial, o_temporal), each
    assembled to [B, heads, N, 128]."""
    q, k, v = (dev(x) for x in si.qkv(w))
    g = vgrid(va, w)
    B, H, N = w.batch, w.heads, w.N
    hpw, nl = H // world, N // world
    local = va.Grid.make(w.T // world, w.H, w.W, 0, w.dims, w.theta)
    nbytes = va.ulysses_region_bytes(B, H, N, world)
    regions = [va.region_alloc(nbytes) for _ in range(world)]
    try:
        offs = va.ulysses_offsets(B, H, N, world)
        views = [[va.region_view(r, off, (B, hpw, N, 128), q.device) for off in offs[:3]]
                 for r in regions]
        shards = [va.region_view(r, offs[3], (B, H, nl, 128), q.device) for r in regions]
        o_heads = [torch.empty((B, hpw, N, 128), dtype=torch.bfloat16, device=q.device)
                   for _ in range(world)]
        slices = [[x[:, :, r * nl:(r + 1) * nl].contiguous() for x in (q, k, v)]
                  for r in range(world)]
        o_sp = [va.attn_factorized_fwd(*slices[r], local, temporal=False)[0] for r in range(world)]
        for r in range(world):
            va.ulysses_scatter(*slices[r], regions, r, g, k_rotated=True)
        for r in range(world):
            va.ulysses_wait(regions[r], va.PHASE_SCATTER, 1, world, B, H, N)
        for r in range(world):
            qh, kh, vh = views[r]
            va.attn_factorized_fwd(qh, kh, vh, g, spatial=False, out_temporal=o_heads[r])
        for r in range(world):
            va.ulysses_gather(o_heads[r], regions, r, H)
        for r in range(world):
            va.ulysses_wait(regions[r], va.PHASE_GATHER, 1, world, B, H, N)
        torch.cuda.synchronize()
        assert va.device_error() == 0
        o_tp = torch.cat([s_.clone() for s_ in shards], dim=2)
    finally:
        torch.cuda.synchronize()
        for r in regions:
            va.region_free(r)
    return torch.cat(o_sp, dim=2), o_tp


@pytest.mark.parametrize("w,world", [(si.WORKLOADS["tiny"], 2),
                                     (custom("uf_6", 6, 5, 7, heads=6), 3),
                                     (custom("uf_b2", 4, 3, 9, heads=4, batch=2), 2),
                                     (si.WORKLOADS["c17f480"], 1)],
                         ids=lambda x: getattr(x, "name", str(x)))
def test_factorised_context_parallel_matches_oracle(va, w, world):
    o_sp, o_tp = emulate_factorised(va, w, world)
    qb, kb, vb = si.qkv(w)
    for mode, got in (("spatial", o_sp), ("temporal", o_tp)):
        ref = oracle.attention(qb, kb, vb, ogrid(w), mode=mode)
        check(host(got).reshape(ref.shape), ref, f"factorised CP {mode} {w.name} x{world}")


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
        o_s, o_t = ua.factorised(q, k, v)
        for mode, got in (("spatial", o_s), ("temporal", o_t)):
            ref = oracle.attention(qb, kb, vb, ogrid(w), mode=mode, rows=rows)
            check(host(got)[..., rows, :].reshape(ref.shape), ref, f"class factorised {mode}")
        assert ua.epoch == 3 and va.device_error() == 0
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


# ------------------------------------------------------------ ring form

def emulate_ring(va, w, world, calls=1, fold=True):
    """`calls` ring calls of `world` emulated ranks, every rank's launches in
    turn on one stream (each wait launched after the signals it counts).
    fold: each step is one va3d_ring_attend (merge in the attention kernel's
    epilogue, as RingAttention runs it); otherwise attn_cross_fwd with its
    LSE, then va3d_ring_merge.
    Returns the assembled output [B, heads, N, 128] and LSE [B, heads, N]."""
    q, k, v = (dev(x) for x in si.qkv(w))
    g = vgrid(va, w)
    B, H, N = w.batch, w.heads, w.N
    nl = N // world
    shape = (B, H, nl, 128)
    regions = [va.region_alloc(va.ring_region_bytes(B, H, N, world)) for _ in range(world)]
    try:
        offs = va.ring_offsets(B, H, N, world)
        kbuf = [[va.region_view(r, offs[0], shape, q.device), va.region_view(r, offs[2], shape, q.device)]
                for r in regions]
        vbuf = [[va.region_view(r, offs[1], shape, q.device), va.region_view(r, offs[3], shape, q.device)]
                for r in regions]
        new = lambda dt, shp: [torch.empty(shp, dtype=dt, device=q.device) for _ in range(world)]
        q_rot, o_blk, out = new(torch.bfloat16, shape), new(torch.bfloat16, shape), new(torch.bfloat16, shape)
        acc = new(torch.float32, shape)
        lse_blk = new(torch.float32, shape[:3])
        lse = [new(torch.float32, shape[:3]) for _ in range(2)]
        ws = torch.empty(max(va.cross_workspace_bytes(B, H, nl, nl), 256), dtype=torch.uint8,
                         device=q.device)
        sl = [[x[:, :, r * nl:(r + 1) * nl].contiguous() for x in (q, k, v)] for r in range(world)]
        for c in range(1, calls + 1):
            for r in range(world):
                va.ring_load(*sl[r], q_rot[r], regions[r], world, r, g)
            for s in range(world):
                cur = s % 2
                if s < world - 1:
                    for r in range(world):
                        va.ring_wait(regions[r], va.RING_FREE, (c - 1) * world + s, world, B, H, N)
                        va.ring_pass(regions[r], regions[(r + 1) % world], cur, world, B, H, N)
                for r in range(world):
                    if fold:
                        va.ring_attend(q_rot[r], kbuf[r][cur], vbuf[r][cur], acc[r],
                                       lse[(s + 1) % 2][r], lse[s % 2][r], first=(s == 0),
                                       out=out[r] if s == world - 1 else None)
                    else:
                        va.attn_cross_fwd(q_rot[r], kbuf[r][cur], vbuf[r][cur], out=o_blk[r],
                                          lse=lse_blk[r], workspace=ws)
                        va.ring_merge(o_blk[r], lse_blk[r], acc[r], lse[(s + 1) % 2][r],
                                      lse[s % 2][r], first=(s == 0),
                                      out=out[r] if s == world - 1 else None)
                    if world > 1:
                        va.ring_free(regions[(r - 1) % world])
                if s < world - 1:
                    for r in range(world):
                        va.ring_wait(regions[r], va.RING_FULL, (c - 1) * (world - 1) + s + 1, world,
                                     B, H, N)
        torch.cuda.synchronize()
        assert va.device_error() == 0
        final = lse[(world - 1) % 2]
        return torch.cat(out, dim=2), torch.cat(final, dim=2)
    finally:
        torch.cuda.synchronize()
        for r in regions:
            va.region_free(r)


RING_CASES = [(si.WORKLOADS["tiny"], 2), (si.WORKLOADS["c17f480"], 4),
              (si.WORKLOADS["c17f480"], 8),     # 12 heads over 8 ranks: no head split
              (custom("r_joint", 2, 6, 10, heads=4, n_text=40, dims=(16, 56, 56)), 5),
              (custom("r_b2", 3, 4, 6, heads=3, batch=2), 3),
              (si.WORKLOADS["tiny"], 1)]


@pytest.mark.parametrize("w,world", RING_CASES, ids=lambda x: getattr(x, "name", str(x)))
def test_ring_matches_oracle(va, w, world):
    o, lse = emulate_ring(va, w, world)
    qb, kb, vb = si.qkv(w)
    ref, ref_lse = oracle.attention(qb, kb, vb, ogrid(w), want_lse=True)
    check(host(o).reshape(ref.shape), ref, f"ring {w.name} x{world}")
    np.testing.assert_allclose(lse.cpu().numpy().reshape(ref_lse.shape), ref_lse, atol=2e-3, rtol=0)


@pytest.mark.parametrize("w,world", [RING_CASES[1], RING_CASES[3], RING_CASES[4]],
                         ids=lambda x: getattr(x, "name", str(x)))
def test_ring_two_call_merge_matches_oracle(va, w, world):
    """The separate merge kernel (attn_cross_fwd + va3d_ring_merge) computes
    the same as the folded step."""
    o, lse = emulate_ring(va, w, world, fold=False)
    qb, kb, vb = si.qkv(w)
    ref, ref_lse = oracle.attention(qb, kb, vb, ogrid(w), want_lse=True)
    check(host(o).reshape(ref.shape), ref, f"ring {w.name} x{world}")
    np.testing.assert_allclose(lse.cpu().numpy().reshape(ref_lse.shape), ref_lse, atol=2e-3, rtol=0)


def test_ring_counters_across_calls(va):
    w = custom("r_calls", 3, 4, 6, heads=2)
    o, _ = emulate_ring(va, w, 3, calls=3)
    qb, kb, vb = si.qkv(w)
    ref = oracle.attention(qb, kb, vb, ogrid(w))
    check(host(o).reshape(ref.shape), ref, "ring x3, third call")


def test_ring_class_single_rank(va):
    from full_spatiotemporal_attention_b200.ring import RingAttention
    w = si.WORKLOADS["c17f480"]
    q, k, v = (dev(x) for x in si.qkv(w))
    ra = RingAttention(vgrid(va, w), w.batch, w.heads, world=1, rank=0)
    try:
        for _ in range(2):
            o = ra(q, k, v)
        qb, kb, vb = si.qkv(w)
        rows = si.sample_rows(w)
        ref = oracle.attention(qb, kb, vb, ogrid(w), rows=rows)
        check(host(o)[..., rows, :].reshape(ref.shape), ref, "ring class world 1")
        assert ra.calls == 2 and va.device_error() == 0
    finally:
        ra.close()
