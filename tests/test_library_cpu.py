"""Host-side checks of the C-ABI library: it builds, loads without a GPU,
exports every entry point the header declares, rejects bad arguments before
touching a device, and has no CPU fallback."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "va3d.h")
PKG = os.path.join(ROOT, "full_spatiotemporal_attention_b200")


@pytest.fixture(scope="module")
def va():
    from full_spatiotemporal_attention_b200 import build
    build.build()
    import full_spatiotemporal_attention_b200 as va
    return va


def header_functions():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^(?:const\s+char\s*\*|int|size_t)\s*(\w+)\s*\(", txt, re.M)))


def test_header_declares_the_boundary():
    names = header_functions()
    for must in ("rope3d_apply", "attn3d_full_fwd", "attn_factorized_fwd", "attn_cross_fwd",
                 "attn_window_fwd", "va3d_watchdog_selftest",
                 "va3d_grid_from_video", "va3d_workspace_bytes", "va3d_cross_workspace_bytes",
                 "va3d_status_string", "va3d_device_error", "va3d_version"):
        assert must in names


def test_library_exports_every_declared_symbol(va):
    out = subprocess.run(["nm", "-D", "--defined-only", va.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    for name in header_functions():
        assert name in exported, name
        getattr(va.lib, name)           # resolvable through ctypes too
    assert set(va.SYMBOLS) == set(header_functions())


def test_library_needs_no_driver_to_load(va):
    out = subprocess.run(["ldd", va.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out      # driver entry points are resolved at run time


def test_grid_from_video_matches_oracle(va):
    import oracle
    for frames, h, w in [(81, 480, 832), (81, 720, 1280), (129, 720, 1280), (17, 480, 832),
                         (1, 16, 16), (5, 64, 32)]:
        g = va.grid_from_video(frames, h, w)
        assert (g.T, g.H, g.W) == oracle.patch_grid(frames, h, w)
        assert (g.d_t, g.d_h, g.d_w, g.theta) == (44, 42, 42, 10000.0)
    g = va.grid_from_video(129, 720, 1280, dims=(16, 56, 56), n_text=256)
    assert g.N == 118800 + 256


@pytest.mark.parametrize("frames,h,w", [(80, 480, 832), (81, 1080, 1920), (81, 480, 840),
                                        (0, 480, 832), (81, 8, 832)])
def test_grid_from_video_rejects_off_grid_clips(va, frames, h, w):
    with pytest.raises(va.VA3DError):
        va.grid_from_video(frames, h, w)


def test_workspace_bytes(va):
    g = va.Grid.make(21, 30, 52)
    tab = 8 * (21 * 22 + 30 * 21 + 52 * 21)
    tab = (tab + 255) // 256 * 256
    # scratch for splitting the last wave's tiles over two key halves: at most
    # 128 tiles x (two 256x128 fp32 partials + two 256-row (max, sum) + counter)
    split = (min(128, 12 * 128) * (2 * 256 * 128 * 4 + 2 * 256 * 8 + 4) + 255) // 256 * 256
    assert va.workspace_bytes(1, 12, 32760, g) == tab + 12 * 32760 * 256 + split
    assert va.workspace_bytes(1, 12, 32760, g, k_rotated=True) == tab + split
    tiny = va.Grid.make(2, 4, 4)
    tab_tiny = (8 * (2 * 22 + 4 * 21 + 4 * 21) + 255) // 256 * 256
    split_tiny = (2 * (2 * 256 * 128 * 4 + 2 * 256 * 8 + 4) + 255) // 256 * 256
    assert va.workspace_bytes(1, 2, 32, tiny, k_rotated=True) == tab_tiny + split_tiny
    assert va.workspace_bytes(1, 12, 32761, g) == 0          # N inconsistent with the grid
    bad = va.Grid.make(21, 30, 52, dims=(44, 42, 40))
    assert va.workspace_bytes(1, 12, 32760, bad) == 0


def test_cross_workspace_bytes(va):
    per = 2 * 256 * 128 * 4 + 2 * 256 * 8 + 4
    assert va.cross_workspace_bytes(1, 40, 75600, 512) == (128 * per + 255) // 256 * 256
    assert va.cross_workspace_bytes(2, 2, 1000, 129) == (16 * per + 255) // 256 * 256
    assert va.cross_workspace_bytes(1, 2, 32, 0) == 0
    assert va.lib.va3d_cross_workspace_bytes(1, 2, 32, 8, 64) == 0


def test_status_strings(va):
    for code in range(0, -7, -1):
        assert va.lib.va3d_status_string(code)
    assert va.lib.va3d_version() >= 100


def test_bad_arguments_rejected_before_any_device_call(va):
    lib = va.lib
    g = va.Grid.make(2, 4, 4)
    # 256-byte aligned, so that p + 16 is 16-byte but never 256-byte aligned
    buf = ctypes.create_string_buffer(4096 + 256)
    p = ctypes.c_void_p((ctypes.addressof(buf) + 255) // 256 * 256)
    gp = ctypes.byref(g)
    # head_dim other than 128
    assert lib.attn3d_full_fwd(p, p, p, p, None, 1, 2, 32, 64, gp, 0.0, 0, p, 4096, None) == -2
    # null input
    assert lib.attn3d_full_fwd(None, p, p, p, None, 1, 2, 32, 128, gp, 0.0, 0, p, 4096, None) == -1
    # N inconsistent with the grid
    assert lib.attn3d_full_fwd(p, p, p, p, None, 1, 2, 33, 128, gp, 0.0, 0, p, 4096, None) == -1
    # misaligned output
    q = ctypes.c_void_p(p.value + 2)
    assert lib.attn3d_full_fwd(p, p, p, q, None, 1, 2, 32, 128, gp, 0.0, 0, p, 4096, None) == -3
    # workspace too small
    assert lib.attn3d_full_fwd(p, p, p, p, None, 1, 2, 32, 128, gp, 0.0, 0, p, 16, None) == -4
    # unknown flag
    assert lib.attn3d_full_fwd(p, p, p, p, None, 1, 2, 32, 128, gp, 0.0, 8, p, 1 << 20, None) == -1
    # factorised passes take no text tokens; temporal needs T' <= 64
    gt = va.Grid.make(2, 4, 4, n_text=3)
    assert lib.attn_factorized_fwd(p, p, p, p, p, 1, 2, 35, 128, ctypes.byref(gt), 0.0, 0, p,
                                   1 << 20, None) == -1
    gl = va.Grid.make(65, 1, 1)
    assert lib.attn_factorized_fwd(p, p, p, None, p, 1, 1, 65, 128, ctypes.byref(gl), 0.0, 0, p,
                                   1 << 20, None) == -2
    # cross-attention: no keys, head_dim, misaligned output or workspace
    assert lib.attn_cross_fwd(p, p, p, p, None, 1, 2, 32, 0, 128, 0.0, None, 0, None) == -1
    assert lib.attn_cross_fwd(p, p, p, p, None, 1, 2, 32, 8, 64, 0.0, None, 0, None) == -2
    assert lib.attn_cross_fwd(p, p, p, q, None, 1, 2, 32, 8, 128, 0.0, None, 0, None) == -3
    assert lib.attn_cross_fwd(p, p, p, p, None, 1, 2, 32, 8, 128, 0.0,
                              ctypes.c_void_p(p.value + 16), 4096, None) in (-3,)
    assert lib.attn_cross_fwd(None, p, p, p, None, 1, 2, 32, 8, 128, 0.0, None, 0, None) == -1
    # window attention: window must divide the grid; no text tokens
    gw = va.Grid.make(2, 4, 4)
    assert lib.attn_window_fwd(p, p, p, p, None, 1, 2, 32, 128, ctypes.byref(gw), 1, 3, 4, 0.0, 0,
                               p, 1 << 20, None) == -1
    assert lib.attn_window_fwd(p, p, p, p, None, 1, 2, 32, 128, ctypes.byref(gw), 0, 2, 4, 0.0, 0,
                               p, 1 << 20, None) == -1
    gwt = va.Grid.make(2, 4, 4, n_text=2)
    assert lib.attn_window_fwd(p, p, p, p, None, 1, 2, 34, 128, ctypes.byref(gwt), 1, 2, 4, 0.0, 0,
                               p, 1 << 20, None) == -1
    assert lib.attn_window_fwd(p, p, p, p, None, 1, 2, 32, 64, ctypes.byref(gw), 1, 2, 4, 0.0, 0,
                               p, 1 << 20, None) == -2
    # odd RoPE range
    godd = va.Grid.make(2, 4, 4, dims=(43, 43, 42))
    assert lib.rope3d_apply(p, p, 1, 2, 32, 128, ctypes.byref(godd), None) == -1


def test_empty_inputs_are_rejected(va):
    """No tokens, no heads or no batch: every entry point returns
    VA3D_ERR_INVALID before touching a device (there is nothing to compute,
    and a zero-sized launch would be an error)."""
    lib = va.lib
    buf = ctypes.create_string_buffer(4096 + 256)
    p = ctypes.c_void_p((ctypes.addressof(buf) + 255) // 256 * 256)
    g0 = va.Grid.make(0, 4, 4)
    g = va.Grid.make(2, 4, 4)
    for B, H, N, grid in ((1, 2, 0, g0), (1, 0, 32, g), (0, 2, 32, g)):
        gp = ctypes.byref(grid)
        assert lib.attn3d_full_fwd(p, p, p, p, None, B, H, N, 128, gp, 0.0, 0, p, 4096, None) == -1
        assert lib.attn_factorized_fwd(p, p, p, p, p, B, H, N, 128, gp, 0.0, 0, p, 4096, None) == -1
        assert lib.attn_window_fwd(p, p, p, p, None, B, H, N, 128, gp, 1, 2, 2, 0.0, 0, p, 4096,
                                   None) == -1
        assert lib.rope3d_apply(p, p, B, H, N, 128, gp, None) == -1
        assert lib.va3d_workspace_bytes(B, H, N, 128, gp, 0) == 0
    assert lib.attn_cross_fwd(p, p, p, p, None, 1, 2, 0, 8, 128, 0.0, None, 0, None) == -1
    assert lib.attn_cross_fwd(p, p, p, p, None, 1, 2, 32, 0, 128, 0.0, None, 0, None) == -1
    assert lib.va3d_grid_from_video(0, 480, 832, 44, 42, 42, 0, ctypes.byref(va.Grid())) == -1


def test_ulysses_region_layout(va):
    """Region = 256-byte header, Qh, Kh, Vh [B, heads/P, N, 128] and the O
    shard [B, heads, N/P, 128], bf16 rows of 256 bytes."""
    B, H, N, P = 2, 12, 7800, 4
    head_shard = B * (H // P) * N * 256
    seq_shard = B * H * (N // P) * 256
    assert va.ulysses_offsets(B, H, N, P) == (256, 256 + head_shard, 256 + 2 * head_shard,
                                              256 + 3 * head_shard)
    assert va.ulysses_region_bytes(B, H, N, P) == 256 + 3 * head_shard + seq_shard
    # one rank holds everything twice over: whole sequences and its (whole) shard
    assert va.ulysses_region_bytes(1, 2, 32, 1) == 256 + 4 * 2 * 32 * 256
    # heads or tokens that do not split, or more ranks than one node holds
    for args in ((1, 12, 7800, 8), (1, 12, 7801, 4), (1, 16, 32, 9), (1, 16, 32, 0)):
        assert va.ulysses_region_bytes(*args) == 0
    with pytest.raises(va.VA3DError):
        va.ulysses_offsets(1, 12, 7800, 8)


def test_ulysses_bad_arguments_rejected_before_any_device_call(va):
    lib = va.lib
    g = va.Grid.make(2, 4, 4)
    gp = ctypes.byref(g)
    buf = ctypes.create_string_buffer(4096 + 256)
    p = ctypes.c_void_p((ctypes.addressof(buf) + 255) // 256 * 256)
    regions = (ctypes.c_void_p * 2)(p, p)
    # heads not divisible by world; tokens not divisible; head_dim; world range
    assert lib.va3d_ulysses_scatter(p, p, p, regions, 2, 0, 1, 3, 32, 128, gp, 0, None) == -2
    assert lib.va3d_ulysses_scatter(p, p, p, regions, 2, 0, 1, 2, 32, 64, gp, 0, None) == -2
    assert lib.va3d_ulysses_scatter(p, p, p, regions, 9, 0, 1, 18, 36, 128, gp, 0, None) == -2
    assert lib.va3d_ulysses_scatter(p, p, p, regions, 0, 0, 1, 2, 32, 128, gp, 0, None) == -2
    # grid inconsistent with N; rank out of range; missing region; unknown flag
    assert lib.va3d_ulysses_scatter(p, p, p, regions, 2, 0, 1, 2, 34, 128, gp, 0, None) == -1
    assert lib.va3d_ulysses_scatter(p, p, p, regions, 2, 2, 1, 2, 32, 128, gp, 0, None) == -1
    holes = (ctypes.c_void_p * 2)(p, None)
    assert lib.va3d_ulysses_scatter(p, p, p, holes, 2, 0, 1, 2, 32, 128, gp, 0, None) == -1
    assert lib.va3d_ulysses_scatter(p, p, p, regions, 2, 0, 1, 2, 32, 128, gp, 4, None) == -1
    # a region must be 256-byte aligned, tensors 16-byte aligned
    odd = (ctypes.c_void_p * 2)(p, ctypes.c_void_p(p.value + 16))
    assert lib.va3d_ulysses_scatter(p, p, p, odd, 2, 0, 1, 2, 32, 128, gp, 0, None) == -3
    q = ctypes.c_void_p(p.value + 2)
    assert lib.va3d_ulysses_scatter(q, p, p, regions, 2, 0, 1, 2, 32, 128, gp, 0, None) == -3
    assert lib.va3d_ulysses_gather(q, regions, 2, 0, 1, 2, 32, 128, None) == -3
    assert lib.va3d_ulysses_gather(p, regions, 2, 5, 1, 2, 32, 128, None) == -1
    # wait: phase, epoch 0, alignment
    assert lib.va3d_ulysses_wait(p, 2, 1, 2, 1, 2, 32, 128, None) == -1
    assert lib.va3d_ulysses_wait(p, 0, 0, 2, 1, 2, 32, 128, None) == -1
    assert lib.va3d_ulysses_wait(ctypes.c_void_p(p.value + 8), 0, 1, 2, 1, 2, 32, 128, None) == -3
    # set-up calls
    assert lib.va3d_region_alloc(0, ctypes.byref(ctypes.c_void_p())) == -1
    assert lib.va3d_ipc_export(None, ctypes.create_string_buffer(64)) == -1
    assert lib.va3d_ipc_open(None, ctypes.byref(ctypes.c_void_p())) == -1
    with pytest.raises(ValueError, match="64 bytes"):
        va.ipc_open(b"short")


def test_ring_region_layout_and_bad_arguments(va):
    """Ring region = 256-byte header, then K0, V0, K1, V1 of [B, heads, N/P, 128]."""
    blk = 2 * 12 * (7800 // 8) * 256
    assert va.ring_offsets(2, 12, 7800, 8) == (256, 256 + blk, 256 + 2 * blk, 256 + 3 * blk)
    assert va.ring_region_bytes(2, 12, 7800, 8) == 256 + 4 * blk
    # no head split, so 12 heads over 8 ranks is fine; tokens must split
    assert va.ring_region_bytes(1, 12, 7801, 8) == 0
    assert va.ring_region_bytes(1, 12, 7800, 9) == 0
    lib = va.lib
    g = va.Grid.make(2, 4, 4)
    gp = ctypes.byref(g)
    buf = ctypes.create_string_buffer(4096 + 256)
    p = ctypes.c_void_p((ctypes.addressof(buf) + 255) // 256 * 256)
    q16 = ctypes.c_void_p(p.value + 16)
    assert lib.va3d_ring_load(p, p, p, p, p, 2, 2, 1, 2, 32, 128, gp, 0, None) == -1    # rank
    assert lib.va3d_ring_load(p, p, p, p, p, 3, 0, 1, 2, 32, 128, gp, 0, None) == -2    # 32 % 3
    assert lib.va3d_ring_load(p, p, p, p, q16, 2, 0, 1, 2, 32, 128, gp, 0, None) == -3  # region
    assert lib.va3d_ring_load(p, p, p, p, p, 2, 0, 1, 2, 34, 128, gp, 0, None) == -1    # grid
    assert lib.va3d_ring_pass(p, p, 2, 2, 1, 2, 32, 128, None) == -1                   # buffer
    assert lib.va3d_ring_pass(p, q16, 0, 2, 1, 2, 32, 128, None) == -3
    assert lib.va3d_ring_wait(p, 2, 1, 2, 1, 2, 32, 128, None) == -1
    assert lib.va3d_ring_free(None, None) == -1
    # merge: a distinct LSE output unless first; alignment
    assert lib.va3d_ring_merge(p, p, p, p, p, None, 1, 2, 16, 0, None) == -1
    assert lib.va3d_ring_merge(p, p, p, None, q16, None, 1, 2, 16, 0, None) == -1      # no lse_in
    assert lib.va3d_ring_merge(ctypes.c_void_p(p.value + 2), p, p, p, ctypes.c_void_p(p.value + 64),
                               None, 1, 2, 16, 0, None) == -3
    # folded step: the same LSE rules, sizes and alignment, checked before any launch
    assert lib.va3d_ring_attend(p, p, p, p, p, p, None, 1, 2, 16, 16, 128, 0.0, 0, None) == -1
    assert lib.va3d_ring_attend(p, p, p, p, None, q16, None, 1, 2, 16, 16, 128, 0.0, 0, None) == -1
    assert lib.va3d_ring_attend(p, p, p, p, None, None, None, 1, 2, 16, 16, 128, 0.0, 1, None) == -1
    assert lib.va3d_ring_attend(p, p, p, p, None, q16, None, 1, 2, 16, 16, 64, 0.0, 1, None) == -2
    assert lib.va3d_ring_attend(p, p, p, p, None, q16, None, 1, 2, 0, 16, 128, 0.0, 1, None) == -1
    assert lib.va3d_ring_attend(ctypes.c_void_p(p.value + 2), p, p, p, None, q16, None, 1, 2, 16, 16,
                                128, 0.0, 1, None) == -3


def test_binding_has_no_cpu_path(va):
    import torch
    g = va.Grid.make(2, 4, 4)
    x = torch.zeros(1, 2, 32, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        va.attn3d_full_fwd(x, x, x, g)
    with pytest.raises(ValueError, match="CUDA"):
        va.rope3d_apply(x, g)
    with pytest.raises(ValueError, match="CUDA"):
        va.attn_factorized_fwd(x, x, x, g)
    with pytest.raises(ValueError, match="CUDA"):
        va.attn_cross_fwd(x, x, x)
    with pytest.raises(ValueError, match="CUDA"):
        va.attn_window_fwd(x, x, x, g, (1, 2, 2))


def test_product_and_oracle_share_nothing():
    """The CUDA path never refers to the oracle or the input generator, and
    the oracle never refers to the product."""
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in txt.lower(), f
                assert "seeded_inputs" not in txt, f
    for f in os.listdir(os.path.join(ROOT, "oracle")):
        if f.endswith((".py", ".c")):
            txt = open(os.path.join(ROOT, "oracle", f)).read()
            assert "full_spatiotemporal_attention_b200" not in txt
            assert "va3d.h" not in txt and "libva3d" not in txt
