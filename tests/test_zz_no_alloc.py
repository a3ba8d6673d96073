"""attn3d_full_fwd_noalloc: the entry point for callers that cannot allocate.

Some callers hold only the device pointers of their inputs and outputs (a
plugin inside a host framework that owns all device memory, or code on a path
where cudaMalloc is not allowed) and so cannot hand the library a workspace.
For them the library keeps its scratch in a 64 MiB static device array.  These
tests call that entry point through the C ABI and check that two calls in a
row give what the workspace entry point gives, within the parity tolerance
the other GPU tests use.  The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest

import seeded_inputs as si

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

MAX_ABS, MEAN_ABS = 1.5e-2, 2e-3


@pytest.fixture(scope="module")
def va():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from full_spatiotemporal_attention_b200 import build
    build.build()
    import full_spatiotemporal_attention_b200 as va
    return va


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16).cuda()


def _call_noalloc(va, q, k, v, o, lse, g, flags=0):
    B, H, N, D = q.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return va.lib.attn3d_full_fwd_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(o.data_ptr()),
        ctypes.c_void_p(lse.data_ptr()) if lse is not None else None,
        B, H, N, D, ctypes.byref(g), 0.0, flags, stream)


def _close(a, b):
    d = (a.float() - b.float()).abs()
    return float(d.max()) <= MAX_ABS and float(d.mean()) <= MEAN_ABS


def test_noalloc_matches_workspace_entry_point_two_calls_in_a_row(va):
    w = si.WORKLOADS["c17f480"]          # 7,800 tokens x 12 heads: 24 MB of scratch
    q, k, v = (_dev(x) for x in si.qkv(w))
    g = va.Grid.make(w.T, w.H, w.W, w.n_text, w.dims, w.theta)
    ref, ref_lse = va.attn3d_full_fwd(q, k, v, g, return_lse=True)
    for _ in range(2):
        o = torch.full_like(q, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        assert _call_noalloc(va, q, k, v, o, lse, g) == 0
        torch.cuda.synchronize()
        assert _close(o, ref)
        assert float((lse - ref_lse).abs().max()) <= 2e-3
    assert va.device_error() == 0


def test_noalloc_after_a_different_problem_and_with_rotated_keys(va):
    # a different grid in between leaves other contents in the shared scratch
    t = si.WORKLOADS["tiny"]
    qt, kt, vt = (_dev(x) for x in si.qkv(t))
    gt = va.Grid.make(t.T, t.H, t.W, t.n_text, t.dims, t.theta)
    ot = torch.empty_like(qt)
    assert _call_noalloc(va, qt, kt, vt, ot, None, gt) == 0
    assert _close(ot, va.attn3d_full_fwd(qt, kt, vt, gt))

    w = si.Workload("joint_small", 2, 6, 10, 2, (16, 56, 56), n_text=37, seed=11)
    q, k, v = (_dev(x) for x in si.qkv(w))
    g = va.Grid.make(w.T, w.H, w.W, w.n_text, w.dims, w.theta)
    ref = va.attn3d_full_fwd(q, k, v, g)
    kr = va.rope3d_apply(k, g)
    for flags, key in ((0, k), (va.VA3D_K_ROTATED, kr)):
        o = torch.empty_like(q)
        assert _call_noalloc(va, q, key, v, o, None, g, flags) == 0
        torch.cuda.synchronize()
        assert _close(o, ref)


def test_noalloc_limit_counts_only_the_table_and_rotated_keys(va):
    # 7 heads x 32,760 tokens: the table and rotated keys take 58.7 MB, under
    # the 64 MiB array; the split-tail scratch a workspace would add (34 MB
    # for 896 tiles) is optional, so the call is taken and matches the
    # workspace entry point.  8 heads need 67.1 MB and are refused.
    w = si.WORKLOADS["c81f480"]
    g = va.Grid.make(w.T, w.H, w.W, w.n_text, w.dims, w.theta)
    q, k, v = (_dev(x[:, :7]) for x in si.qkv(w))
    assert va.workspace_bytes(1, 7, w.N, g) > (64 << 20)
    ref = va.attn3d_full_fwd(q, k, v, g)
    for _ in range(2):
        o = torch.full_like(q, float("nan"))
        assert _call_noalloc(va, q, k, v, o, None, g) == 0
        torch.cuda.synchronize()
        assert _close(o, ref)
    x = torch.zeros(1, 1, 1, 128, dtype=torch.bfloat16, device="cuda")
    p = ctypes.c_void_p(x.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert va.lib.attn3d_full_fwd_noalloc(p, p, p, p, None, 1, 8, w.N, 128, ctypes.byref(g), 0.0,
                                          0, stream) == -7
    assert va.device_error() == 0


def test_noalloc_binding_checks_lse(va):
    w = si.WORKLOADS["tiny"]
    q, k, v = (_dev(x) for x in si.qkv(w))
    g = va.Grid.make(w.T, w.H, w.W, w.n_text, w.dims, w.theta)
    B, H, N, _ = q.shape
    for bad in (torch.empty((B, H, N), dtype=torch.bfloat16, device="cuda"),
                torch.empty((B, H, N - 1), dtype=torch.float32, device="cuda"),
                torch.empty((B, H, 2 * N), dtype=torch.float32, device="cuda")[..., ::2],
                torch.empty((B, H, N), dtype=torch.float32)):
        with pytest.raises(ValueError):
            va.attn3d_full_fwd_noalloc(q, k, v, g, lse=bad)


def test_noalloc_rejects_problems_beyond_its_scratch(va):
    w = si.WORKLOADS["c81f480"]          # needs 100 MB of rotated keys > 64 MiB
    g = va.Grid.make(w.T, w.H, w.W, w.n_text, w.dims, w.theta)
    x = torch.zeros(1, 1, 1, 128, dtype=torch.bfloat16, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = ctypes.c_void_p(x.data_ptr())
    rc = va.lib.attn3d_full_fwd_noalloc(p, p, p, p, None, 1, w.heads, w.N, 128, ctypes.byref(g),
                                        0.0, 0, stream)
    assert rc == -7                      # VA3D_ERR_SCRATCH_LIMIT, nothing launched
    assert "64 MiB" in va.lib.va3d_status_string(rc).decode()
    # with pre-rotated keys only the angle table is needed, which fits
    assert va.workspace_bytes(1, w.heads, w.N, g, k_rotated=True) < (64 << 20)
