"""Pins of the oracle to what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: values the
pages print (``tests/golden``), an independent library routine (torch's
scaled_dot_product_attention, transformers' Llama rotary embedding), an
explicit matrix formulation, closed-form special cases, or invariants.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import Grid
import seeded_inputs as si
from conftest import bf16_bits_to_f64, f64_to_bf16_bits


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def _rows(path):
    out = []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                out.append(line)
    return out


def _rand_bits(shape, seed, scale=1.0):
    return si.normal_bf16(seed, 77, shape, scale=scale)


def _coords(grid):
    n = np.arange(grid.n_video)
    return oracle.token_coords(n, grid.T, grid.H, grid.W)


def _llama_inv_freq(dim, theta=10000.0):
    """Inverse frequencies from transformers' Llama rotary embedding (fp32)."""
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaRotaryEmbedding
    cfg = LlamaConfig(head_dim=dim, hidden_size=2 * dim, num_attention_heads=2,
                      rope_parameters={"rope_type": "default", "rope_theta": theta})
    inv, _ = LlamaRotaryEmbedding.compute_default_rope_parameters(cfg)
    return inv.double()


def _explicit_R(pos, dims, theta=10000.0):
    """Block-diagonal R_3D(t, y, x) as an explicit 128x128 matrix, one 2x2
    rotation block per pair, frequencies from the Llama ladder."""
    D = sum(dims)
    R = np.zeros((D, D))
    off = 0
    for a, d in enumerate(dims):
        inv = _llama_inv_freq(d, theta).numpy() if d else np.zeros(0)
        for j in range(d // 2):
            phi = pos[a] * inv[j]
            c, s = math.cos(phi), math.sin(phi)
            i0 = off + 2 * j
            R[i0, i0], R[i0, i0 + 1] = c, -s
            R[i0 + 1, i0], R[i0 + 1, i0 + 1] = s, c
        off += d
    return R


def _sdpa(q, k, v, mask=None, scale=None):
    """torch fp64 scaled_dot_product_attention on [BH, N, D] arrays."""
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(x)).double() for x in (q, k, v))
    m = None if mask is None else torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=m, scale=scale)
    return o.numpy()


def _mode_mask(grid, mode):
    t, h, w = _coords(grid)
    if mode == "spatial":
        return t[:, None] == t[None, :]
    if mode == "temporal":
        return (h[:, None] == h[None, :]) & (w[:, None] == w[None, :])
    return np.ones((grid.N, grid.N), dtype=bool)


# ---------------------------------------------------------------------------
# token grid and FLOP model: values printed on the pages
# ---------------------------------------------------------------------------

def test_token_table_matches_printed(golden_dir):
    for line in _rows(os.path.join(golden_dir, "token_table.txt")):
        clip, lat, tokens, dim, ratio = [p.split() for p in line.split("|")]
        frames, h, w = map(int, clip)
        assert oracle.latent_shape(frames, h, w) == tuple(map(int, lat))
        n = oracle.token_count(frames, h, w)
        assert n == int(tokens[0])
        assert oracle.token_width() == int(dim[0])
        assert round(n / 4096) == int(ratio[0])


def test_flops_table_matches_printed(golden_dir):
    for line in _rows(os.path.join(golden_dir, "flops_table.txt")):
        left, right = line.split("|")
        frames, h, w, d, layers = map(int, left.split())
        fact, full, ratio, lin = map(int, right.split())
        grid, n = oracle.patch_grid(frames, h, w), oracle.token_count(frames, h, w)
        f1 = oracle.attention_flops(grid, d, layers, "factorised")
        f2 = oracle.attention_flops(grid, d, layers, "full")
        assert round(f1 / 1e12) == fact
        assert round(f2 / 1e12) == full
        assert round(f2 / f1) == ratio
        assert round(oracle.linear_flops(n, d, layers) / 1e12) == lin


def test_page_arithmetic(golden_dir):
    vals = {}
    for line in _rows(os.path.join(golden_dir, "page_arithmetic.txt")):
        key, *rest = line.split()
        vals[key] = [float(x) for x in rest]
    pixels = 81 * 832 * 480
    assert pixels == vals["pixels"][0]
    assert round(pixels ** 2 / 1e15, 3) == vals["raw_pairs_quadrillion"][0]
    n = oracle.token_count(81, 480, 832)
    assert n == vals["tokens"][0]
    assert int(pixels ** 2 / n ** 2) == vals["attention_cut"][0]
    assert round(pixels ** 2 * 2 / 1e12) == vals["raw_score_TB_one_head"][0]
    assert round(n * n * 2 / 1e9, 2) == vals["score_GB_one_head"][0]
    assert round(pixels * 3 / 1e6, 2) == vals["raw_floats_M"][0]
    T, H, W = oracle.latent_shape(81, 480, 832)
    assert round(T * H * W * oracle.LATENT_CHANNELS / 1e6, 2) == vals["latent_floats_M"][0]
    assert [d // 2 for d in (44, 42, 42)] == vals["rope_pairs_t_h_w"]
    # exercises: 480p -> 720p growth and reference-image tokens
    n480 = oracle.token_count(81, 480, 832)
    n720 = oracle.token_count(81, 720, 1280)
    assert (n480, n720) == (vals["tokens_480p"][0], vals["tokens_720p"][0])
    assert round(n720 / n480, 1) == vals["token_growth"][0]
    assert round((n720 / n480) ** 2, 1) == vals["attention_growth"][0]
    seq = n720 + 3 * int(vals["reference_image_tokens"][0])
    assert seq == vals["sequence_with_3_refs"][0]
    # the reference-image workload is that request's shape
    import seeded_inputs as si
    ref_w = si.WORKLOADS["refimg720"]
    assert ref_w.n_video == n720 and ref_w.N == vals["sequence_with_3_refs"][0]
    assert round(((seq / n720) ** 2 - 1) * 100) == vals["attention_cost_rise_percent"][0]
    # the diffusers DiT example: 3 latent frames of 8x8, patch 2, plus 4 text tokens
    lt, lhw = int(vals["dit_latent_T"][0]), int(vals["dit_latent_HW"][0])
    n_img = lt * (lhw // 2) * (lhw // 2)
    assert n_img + int(vals["dit_text_tokens"][0]) == vals["dit_sequence"][0]


def test_frame_rule_examples():
    # handbook VAE example: 9 frames of 32x32 -> 3 latent frames of 4x4 (compression 8)
    assert oracle.latent_shape(9, 32, 32) == (3, 4, 4)
    # CogVideoX guide: 49 frames -> 13 latent frames
    assert oracle.latent_shape(49, 480, 720)[0] == 13
    # the configurations of this build
    assert oracle.patch_grid(81, 480, 832) == (21, 30, 52)
    assert oracle.patch_grid(81, 720, 1280) == (21, 45, 80)
    assert oracle.patch_grid(129, 720, 1280) == (33, 45, 80)
    assert oracle.patch_grid(17, 480, 832) == (5, 30, 52)


def test_rope_ranges():
    # HunyuanVideo's (16, 56, 56) and Wan2.1's (44, 42, 42) both fill the head
    assert oracle.rope_ranges((16, 56, 56)) == {"t": (0, 16), "h": (16, 72), "w": (72, 128)}
    r = oracle.rope_ranges((44, 42, 42))
    assert [(b - a) // 2 for a, b in r.values()] == [22, 21, 21]
    for bad in ((44, 42, 40), (43, 43, 42), (128,), (64, 64, 0, 0)):
        with pytest.raises(ValueError):
            oracle.rope_ranges(bad)


def test_shard_listing_matches_printed(golden_dir):
    T, H, W, P = 2, 2, 3, 3
    toks = [oracle.token_coords(i, T, H, W) for i in range(T * H * W)]
    shards = [toks[r * len(toks) // P:(r + 1) * len(toks) // P] for r in range(P)]
    for line in _rows(os.path.join(golden_dir, "shard_listing.txt")):
        card, rest = line.split(":")
        printed = [tuple(int(x) for x in tok.strip("()").split(",")) for tok in rest.split()]
        assert shards[int(card)] == printed
    # the C oracle decodes coordinates the same way
    g = Grid(T, H, W)
    assert [oracle.c_token_coords(g, i) for i in range(T * H * W)] == toks


# ---------------------------------------------------------------------------
# 3D RoPE
# ---------------------------------------------------------------------------

GRIDS = [Grid(2, 4, 4, dims=(44, 42, 42)), Grid(3, 5, 7, dims=(16, 56, 56)),
         Grid(2, 3, 3, n_text=5, dims=(44, 42, 42))]


@pytest.mark.parametrize("grid", GRIDS)
def test_rope_preserves_norm(grid):
    x = _rand_bits((2, grid.N, 128), 11)
    y = oracle.rope3d(x, grid)
    xn = np.linalg.norm(bf16_bits_to_f64(x), axis=-1)
    yn = np.linalg.norm(y, axis=-1)
    np.testing.assert_allclose(yn, xn, rtol=1e-12, atol=0)


@pytest.mark.parametrize("grid", GRIDS)
def test_rope_identity_at_origin_and_for_text(grid):
    x = _rand_bits((1, grid.N, 128), 12)
    y = oracle.rope3d(x, grid)
    xf = bf16_bits_to_f64(x)
    np.testing.assert_array_equal(y[0, 0], xf[0, 0])           # position (0, 0, 0)
    np.testing.assert_array_equal(y[0, grid.n_video:], xf[0, grid.n_video:])  # text tokens


@pytest.mark.parametrize("dims", [(44, 42, 42), (16, 56, 56)])
def test_rope_axis_matches_llama_rotary(dims):
    """Each axis range is a 1D rotary embedding of that axis' coordinate.

    Compared with transformers' Llama rotary embedding (its own frequency
    ladder, its rotate-half pairing), after mapping the adjacent pairs of our
    convention onto the half split.
    """
    from transformers.models.llama.modeling_llama import apply_rotary_pos_emb
    grid = Grid(3, 5, 6, dims=dims)
    x = _rand_bits((1, grid.N, 128), 13)
    xf = bf16_bits_to_f64(x)[0]
    y = oracle.rope3d(x, grid)[0]
    t, h, w = _coords(grid)
    off = 0
    for a, d in enumerate(dims):
        pos = (t, h, w)[a]
        inv = _llama_inv_freq(d)
        freqs = torch.from_numpy(pos.astype(np.float64))[:, None] * inv[None, :]
        emb = torch.cat((freqs, freqs), dim=-1)
        cos, sin = emb.cos()[None], emb.sin()[None]
        sub = xf[:, off:off + d]
        half = np.concatenate([sub[:, 0::2], sub[:, 1::2]], axis=1)   # adjacent -> half split
        th = torch.from_numpy(half)[None, None]
        rq, _ = apply_rotary_pos_emb(th, th, cos, sin)
        rq = rq[0, 0].numpy()
        back = np.empty_like(sub)
        back[:, 0::2], back[:, 1::2] = rq[:, :d // 2], rq[:, d // 2:]
        # fp32 inverse frequencies on the library side bound the agreement
        np.testing.assert_allclose(y[:, off:off + d], back, atol=5e-5, rtol=0)
        off += d


@pytest.mark.parametrize("dims", [(44, 42, 42), (16, 56, 56)])
def test_rope_relative_position_identity(dims):
    """<R(p_i) q, R(p_j) k> = q^T R(p_j - p_i) k with R the explicit
    block-diagonal matrix of the CogVideoX guide's 3D RoPE section."""
    grid = Grid(4, 5, 6, dims=dims)
    x = _rand_bits((2, grid.N, 128), 14)
    rot = oracle.rope3d(x, grid)
    qf, kf = bf16_bits_to_f64(x)
    t, h, w = _coords(grid)
    rng = np.random.default_rng(0)
    for _ in range(40):
        i, j = rng.integers(0, grid.N, size=2)
        lhs = rot[0, i] @ rot[1, j]
        R = _explicit_R((t[j] - t[i], h[j] - h[i], w[j] - w[i]), dims)
        rhs = qf[i] @ R @ kf[j]
        assert abs(lhs - rhs) < 1e-4 * max(1.0, abs(rhs))   # library ladder is fp32


def test_rope_T1_reduces_to_2d_and_HW1_to_1d():
    # T' = 1: every token has t = 0, so the time range is untouched (2D RoPE)
    g = Grid(1, 6, 7, dims=(44, 42, 42))
    x = _rand_bits((1, g.N, 128), 15)
    y = oracle.rope3d(x, g)
    np.testing.assert_array_equal(y[..., :44], bf16_bits_to_f64(x)[..., :44])
    assert np.abs(y[..., 44:] - bf16_bits_to_f64(x)[..., 44:]).max() > 1e-3
    # H' = W' = 1: only the time range turns (1D temporal RoPE)
    g = Grid(9, 1, 1, dims=(44, 42, 42))
    x = _rand_bits((1, g.N, 128), 16)
    y = oracle.rope3d(x, g)
    np.testing.assert_array_equal(y[..., 44:], bf16_bits_to_f64(x)[..., 44:])
    assert np.abs(y[..., :44] - bf16_bits_to_f64(x)[..., :44]).max() > 1e-3


@pytest.mark.parametrize("dims", [(44, 42, 42), (16, 56, 56)])
def test_temporal_pass_needs_only_the_time_range_turned(dims):
    """Within one (h, w) position the h and w rotations of a query and a key
    are the same orthogonal map and cancel in their dot product, so the
    temporal pass's scores equal those of queries and keys turned by t only
    (the same tokens on a T' x 1 x 1 grid), with the other dims untouched."""
    T, H, W = 5, 3, 4
    g = Grid(T, H, W, dims=dims)
    x = _rand_bits((2, g.N, 128), 17)
    rot = oracle.rope3d(x, g)
    g_t = Grid(T, 1, 1, dims=dims)
    rng = np.random.default_rng(3)
    for _ in range(10):
        h, w = int(rng.integers(0, H)), int(rng.integers(0, W))
        idx = np.array([(t * H + h) * W + w for t in range(T)])
        only_t = oracle.rope3d(x[:, idx], g_t)          # token t of the column at (t, 0, 0)
        np.testing.assert_array_equal(only_t[..., dims[0]:], bf16_bits_to_f64(x[:, idx])[..., dims[0]:])
        full_scores = rot[0, idx] @ rot[1, idx].T
        t_scores = only_t[0] @ only_t[1].T
        np.testing.assert_allclose(full_scores, t_scores, atol=1e-9, rtol=1e-9)


def test_rope_pairs_are_adjacent():
    """A unit vector in dim o+2j of a range only mixes with dim o+2j+1."""
    g = Grid(3, 3, 3, dims=(44, 42, 42))
    D = 128
    e = np.zeros((g.N, D), dtype=np.float64)
    e[:, 44 + 2 * 5] = 1.0      # pair 5 of the h range
    y = oracle.rope3d(f64_to_bf16_bits(e)[None], g)[0]
    others = np.delete(y, [44 + 10, 44 + 11], axis=1)
    assert np.all(others == 0.0)
    np.testing.assert_allclose(y[:, 54] ** 2 + y[:, 55] ** 2, 1.0, rtol=1e-12)


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("mode", ["full", "spatial", "temporal"])
def test_attention_unrotated_equals_sdpa(mode):
    g = Grid(2, 4, 4)
    q, k, v = (_rand_bits((2, g.N, 128), s) for s in (21, 22, 23))
    o = oracle.attention(q, k, v, g, mode=mode, rotate=False)
    ref = _sdpa(bf16_bits_to_f64(q), bf16_bits_to_f64(k), bf16_bits_to_f64(v),
                mask=_mode_mask(g, mode))
    np.testing.assert_allclose(o, ref, atol=1e-12, rtol=0)


@pytest.mark.parametrize("grid", [Grid(2, 4, 4), Grid(3, 4, 5, dims=(16, 56, 56)),
                                  Grid(2, 3, 4, n_text=7)])
def test_attention_rotated_equals_sdpa_on_rotated(grid):
    q, k, v = (_rand_bits((2, grid.N, 128), s) for s in (31, 32, 33))
    o, lse = oracle.attention(q, k, v, grid, want_lse=True)
    qr, kr = oracle.rope3d(q, grid), oracle.rope3d(k, grid)
    ref = _sdpa(qr, kr, bf16_bits_to_f64(v))
    np.testing.assert_allclose(o, ref, atol=1e-12, rtol=0)
    scores = np.einsum("bid,bjd->bij", qr, kr) / math.sqrt(128)
    ref_lse = torch.logsumexp(torch.from_numpy(scores), dim=-1).numpy()
    np.testing.assert_allclose(lse, ref_lse, atol=1e-12, rtol=0)


@pytest.mark.parametrize("mode", ["full", "spatial", "temporal"])
def test_constant_values_give_constant_output(mode):
    g = Grid(3, 4, 4)
    q, k = (_rand_bits((1, g.N, 128), s) for s in (41, 42))
    row = _rand_bits((1, 1, 128), 43)
    v = np.repeat(row, g.N, axis=1)
    o = oracle.attention(q, k, v, g, mode=mode)
    np.testing.assert_allclose(o[0], np.repeat(bf16_bits_to_f64(row)[0], g.N, 0),
                               atol=1e-13, rtol=1e-13)


@pytest.mark.parametrize("mode", ["full", "spatial", "temporal"])
def test_zero_query_averages_allowed_values(mode):
    g = Grid(3, 4, 5)
    q = np.zeros((1, g.N, 128), dtype=np.uint16)
    k, v = (_rand_bits((1, g.N, 128), s) for s in (51, 52))
    o = oracle.attention(q, k, v, g, mode=mode)[0]
    vf = bf16_bits_to_f64(v)[0]
    t, h, w = _coords(g)
    for i in range(g.N):
        if mode == "full":
            sel = np.ones(g.N, dtype=bool)
        elif mode == "spatial":
            sel = t == t[i]
        else:
            sel = (h == h[i]) & (w == w[i])
        np.testing.assert_allclose(o[i], vf[sel].mean(axis=0), atol=1e-13, rtol=0)


@pytest.mark.parametrize("mode", ["spatial", "temporal"])
def test_factorised_equals_masked_full(mode):
    """Spatial attention = full attention under the block-diagonal mask
    [t_i = t_j]; temporal = full under [(h_i, w_i) = (h_j, w_j)]."""
    g = Grid(3, 5, 6)
    q, k, v = (_rand_bits((2, g.N, 128), s) for s in (61, 62, 63))
    o = oracle.attention(q, k, v, g, mode=mode)
    qr, kr = oracle.rope3d(q, g), oracle.rope3d(k, g)
    ref = _sdpa(qr, kr, bf16_bits_to_f64(v), mask=_mode_mask(g, mode))
    np.testing.assert_allclose(o, ref, atol=1e-12, rtol=0)


def test_spatial_pass_equals_per_frame_2d_rope():
    """Within one frame the time rotation cancels: the spatial pass of 3D
    RoPE equals attention with only (h, w) rotated."""
    g = Grid(3, 4, 5)
    q, k, v = (_rand_bits((1, g.N, 128), s) for s in (64, 65, 66))
    o = oracle.attention(q, k, v, g, mode="spatial")
    g2d = Grid(1, 4, 5)
    hw = g.H * g.W
    for t in range(g.T):
        sl = slice(t * hw, (t + 1) * hw)
        o2 = oracle.attention(q[:, sl], k[:, sl], v[:, sl], g2d)
        np.testing.assert_allclose(o[:, sl], o2, atol=1e-12, rtol=0)


@pytest.mark.parametrize("mode", ["full", "spatial", "temporal"])
def test_translation_invariance(mode):
    """Attention weights depend only on coordinate differences."""
    g = Grid(3, 4, 5)
    q, k, v = (_rand_bits((1, g.N, 128), s) for s in (71, 72, 73))
    o = oracle.attention(q, k, v, g, mode=mode)
    gs = Grid(3, 4, 5, offset=(7, 11, 13))
    o2 = oracle.attention(q, k, v, gs, mode=mode)
    np.testing.assert_allclose(o, o2, atol=1e-9, rtol=0)


def test_brute_force_tiny_all_modes():
    """Tiny grid, every row of every mode, against an explicit N x N score
    matrix built with explicit R_3D matrices per token."""
    w = si.WORKLOADS["tiny"]
    g = Grid(w.T, w.H, w.W, dims=w.dims)
    q, k, v = si.qkv(w)
    q, k, v = (x.reshape(w.heads, w.N, 128) for x in (q, k, v))
    t, h, ww = _coords(g)
    Rs = [_explicit_R((t[i], h[i], ww[i]), w.dims) for i in range(g.N)]
    qf, kf, vf = bf16_bits_to_f64(q), bf16_bits_to_f64(k), bf16_bits_to_f64(v)
    for mode in ("full", "spatial", "temporal"):
        o = oracle.attention(q, k, v, g, mode=mode)
        mask = _mode_mask(g, mode)
        for b in range(w.heads):
            qr = np.stack([Rs[i] @ qf[b, i] for i in range(g.N)])
            kr = np.stack([Rs[i] @ kf[b, i] for i in range(g.N)])
            S = qr @ kr.T / math.sqrt(128)
            S = np.where(mask, S, -np.inf)
            P = np.exp(S - S.max(axis=1, keepdims=True))
            P /= P.sum(axis=1, keepdims=True)
            # the explicit R uses the fp32 library ladder: agreement to ~1e-5
            np.testing.assert_allclose(o[b], P @ vf[b], atol=2e-5, rtol=0)


def test_sampled_rows_match_all_rows():
    g = Grid(3, 4, 6, n_text=9, dims=(16, 56, 56))
    q, k, v = (_rand_bits((2, g.N, 128), s) for s in (81, 82, 83))
    full = oracle.attention(q, k, v, g)
    rows = np.array([0, 5, g.n_video - 1, g.n_video, g.N - 1])
    part = oracle.attention(q, k, v, g, rows=rows)
    np.testing.assert_array_equal(part, full[:, rows])


def test_joint_text_rows_attend_to_everything():
    g = Grid(2, 3, 4, n_text=6)
    q, k, v = (_rand_bits((1, g.N, 128), s) for s in (91, 92, 93))
    o = oracle.attention(q, k, v, g)
    # the text rows of q are not rotated: compare with SDPA on (q, rotated k)
    kr = oracle.rope3d(k, g)
    ref = _sdpa(bf16_bits_to_f64(q)[:, g.n_video:], kr, bf16_bits_to_f64(v))
    np.testing.assert_allclose(o[:, g.n_video:], ref, atol=1e-12, rtol=0)


def test_oracle_rejects_bad_arguments():
    g = Grid(2, 2, 2, dims=(44, 42, 40))
    x = np.zeros((1, 8, 128), dtype=np.uint16)
    with pytest.raises(ValueError):
        oracle.rope3d(x, g)
    g = Grid(2, 2, 2, n_text=1)
    x = np.zeros((1, 9, 128), dtype=np.uint16)
    with pytest.raises(ValueError):
        oracle.attention(x, x, x, g, mode="spatial")     # factorised passes have no text
    with pytest.raises(ValueError):
        oracle.attention(x, x, x, Grid(2, 2, 2))          # N mismatch


# ---------------------------------------------------------------------------
# local 3D-window attention (W.A.L.T blocks, anthology record sota-390)
# ---------------------------------------------------------------------------

def _window_mask(grid, win):
    t, h, w = _coords(grid)
    wt, wh, ww = win
    return ((t[:, None] // wt == t[None, :] // wt) & (h[:, None] // wh == h[None, :] // wh)
            & (w[:, None] // ww == w[None, :] // ww))


@pytest.mark.parametrize("win", [(2, 2, 3), (1, 4, 2), (4, 1, 6), (2, 4, 6)])
def test_window_equals_masked_full(win):
    """Window attention = full attention under the mask 'same window'."""
    g = Grid(4, 4, 6)
    q, k, v = (_rand_bits((2, g.N, 128), s) for s in (131, 132, 133))
    o, lse = oracle.window_attention(q, k, v, g, win, want_lse=True)
    qr, kr = oracle.rope3d(q, g), oracle.rope3d(k, g)
    mask = _window_mask(g, win)
    np.testing.assert_allclose(o, _sdpa(qr, kr, bf16_bits_to_f64(v), mask=mask), atol=1e-12, rtol=0)
    s = torch.from_numpy(qr @ kr.transpose(0, 2, 1) / math.sqrt(128))
    s = s.masked_fill(~torch.from_numpy(mask), -math.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), atol=1e-12, rtol=0)


def test_window_special_cases_reduce_to_the_other_modes():
    g = Grid(3, 4, 5)
    q, k, v = (_rand_bits((1, g.N, 128), s) for s in (134, 135, 136))
    pairs = [((3, 4, 5), "full"), ((1, 4, 5), "spatial"), ((3, 1, 1), "temporal")]
    for win, mode in pairs:
        np.testing.assert_allclose(oracle.window_attention(q, k, v, g, win),
                                   oracle.attention(q, k, v, g, mode=mode), atol=1e-13, rtol=0)
    # one-token windows: every row copies its own value
    o = oracle.window_attention(q, k, v, g, (1, 1, 1))
    np.testing.assert_array_equal(o, bf16_bits_to_f64(v))
    # windows are defined on grid coordinates, RoPE on relative ones: a shift
    # of every position leaves the output unchanged
    gs = Grid(3, 4, 5, offset=(5, 9, 2))
    np.testing.assert_allclose(oracle.window_attention(q, k, v, gs, (3, 2, 5)),
                               oracle.window_attention(q, k, v, g, (3, 2, 5)), atol=1e-9, rtol=0)


def test_window_brute_force_tiny():
    g = Grid(2, 4, 4)
    q, k, v = (_rand_bits((1, g.N, 128), s) for s in (137, 138, 139))
    win = (1, 2, 4)
    o = oracle.window_attention(q, k, v, g, win)[0]
    t, h, w = _coords(g)
    Rs = [_explicit_R((t[i], h[i], w[i]), (44, 42, 42)) for i in range(g.N)]
    qf, kf, vf = (bf16_bits_to_f64(x)[0] for x in (q, k, v))
    qr = np.stack([Rs[i] @ qf[i] for i in range(g.N)])
    kr = np.stack([Rs[i] @ kf[i] for i in range(g.N)])
    for i in range(g.N):
        keys = [j for j in range(g.N) if t[j] == t[i] and h[j] // 2 == h[i] // 2]
        s_ = np.array([qr[i] @ kr[j] for j in keys]) / math.sqrt(128)
        p_ = np.exp(s_ - s_.max())
        np.testing.assert_allclose(o[i], (p_[:, None] * vf[keys]).sum(0) / p_.sum(), atol=2e-5,
                                   rtol=0)


def test_window_rejects_bad_arguments():
    g = Grid(3, 4, 6)
    x = np.zeros((1, g.N, 128), dtype=np.uint16)
    for win in [(2, 2, 3), (1, 3, 3), (1, 4, 5), (0, 1, 1)]:
        with pytest.raises(ValueError):
            oracle.window_attention(x, x, x, g, win)
    gt = Grid(3, 4, 6, n_text=2)
    xt = np.zeros((1, gt.N, 128), dtype=np.uint16)
    with pytest.raises(ValueError):
        oracle.window_attention(xt, xt, xt, gt, (1, 2, 3))


# ---------------------------------------------------------------------------
# text cross-attention (Wan block, "04 HunyuanVideo and Wan" section 3.1)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("nq,nkv", [(37, 11), (5, 300), (64, 1)])
def test_cross_attention_equals_sdpa(nq, nkv):
    q = _rand_bits((3, nq, 128), 101)
    k = _rand_bits((3, nkv, 128), 102)
    v = _rand_bits((3, nkv, 128), 103)
    o, lse = oracle.cross_attention(q, k, v, want_lse=True)
    qf, kf, vf = (bf16_bits_to_f64(x) for x in (q, k, v))
    np.testing.assert_allclose(o, _sdpa(qf, kf, vf), atol=1e-12, rtol=0)
    s = torch.from_numpy(qf @ kf.transpose(0, 2, 1) / math.sqrt(128))
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), atol=1e-12, rtol=0)


def test_cross_attention_special_cases():
    q = _rand_bits((2, 9, 128), 111, scale=3.0)
    k = _rand_bits((2, 1, 128), 112)
    v = _rand_bits((2, 1, 128), 113)
    # one key: every query copies its value
    o = oracle.cross_attention(q, k, v)
    np.testing.assert_array_equal(o, np.broadcast_to(bf16_bits_to_f64(v), o.shape))
    # zero queries average the values; permuting the keys (with their values)
    # changes nothing
    k = _rand_bits((2, 40, 128), 114)
    v = _rand_bits((2, 40, 128), 115)
    z = np.zeros((2, 4, 128), dtype=np.uint16)
    o = oracle.cross_attention(z, k, v)
    np.testing.assert_allclose(o, np.broadcast_to(bf16_bits_to_f64(v).mean(axis=1, keepdims=True),
                                                  o.shape), atol=1e-14, rtol=0)
    perm = np.random.default_rng(0).permutation(40)
    q = _rand_bits((2, 4, 128), 116)
    np.testing.assert_allclose(oracle.cross_attention(q, k[:, perm], v[:, perm]),
                               oracle.cross_attention(q, k, v), atol=1e-14, rtol=0)


def test_cross_attention_rows_and_self_attention_consistent():
    # with keys = the queries' own sequence and no rotation it is the
    # unrotated full attention
    g = Grid(2, 3, 5)
    q, k, v = (_rand_bits((2, g.N, 128), s) for s in (121, 122, 123))
    full = oracle.attention(q, k, v, g, rotate=False)
    np.testing.assert_allclose(oracle.cross_attention(q, k, v), full, atol=1e-13, rtol=0)
    rows = np.array([0, 7, g.N - 1])
    np.testing.assert_array_equal(oracle.cross_attention(q, k, v, rows=rows),
                                  oracle.cross_attention(q, k, v)[:, rows])
    with pytest.raises(ValueError):
        oracle.cross_attention(q, k, v, rows=np.array([g.N]))


# ---------------------------------------------------------------------------
# seeded inputs
# ---------------------------------------------------------------------------

def test_seeded_inputs_deterministic_and_normal():
    a = si.normal_bf16(5, 1, (1000, 128))
    b = si.normal_bf16(5, 1, (1000, 128))
    np.testing.assert_array_equal(a, b)
    tail = si.normal_bf16(5, 1, (10, 128), first=990 * 128)
    np.testing.assert_array_equal(a[990:], tail)
    x = bf16_bits_to_f64(a)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01
    assert not np.array_equal(a, si.normal_bf16(5, 2, (1000, 128)))


def test_sharpened_keys_are_exactly_doubled():
    w = si.Workload("s", 2, 8, 8, 2, (44, 42, 42), seed=9, sharpen_frac=0.1)
    q, k, v = si.qkv(w)
    base = si.normal_bf16(w.seed, si.K_STREAM, w.shape)
    sel = si.sharpened_tokens(w)
    assert 0.03 < sel.mean() < 0.2
    np.testing.assert_array_equal(bf16_bits_to_f64(k)[:, :, sel], 2 * bf16_bits_to_f64(base)[:, :, sel])
    np.testing.assert_array_equal(k[:, :, ~sel], base[:, :, ~sel])


def test_sample_rows_cover_structure():
    w = si.WORKLOADS["joint720"]
    rows = si.sample_rows(w, 512)
    assert rows.size == 512 and len(set(rows.tolist())) == 512
    assert 0 in rows and w.N - 1 in rows
    assert (rows >= w.n_video).sum() >= 64
