"""Parity of the sm_100a kernels (through the C ABI) with the fp64 oracle.

Bar (the tolerance set for bf16 outputs with fp32 accumulation):
max-abs error <= 1.5e-2 and mean-abs error <= 2e-3; in
addition the relative L2 error must stay <= 2e-2, which is the meaningful
gate at large N where outputs are small.  Small workloads compare every
row; the full-size workloads (the configuration the bench times) compare
512 seeded query rows per head, always including the first and last rows,
tile and frame boundaries and, for joint attention, at least 64 text rows.
"""
import numpy as np
import pytest

import oracle
import seeded_inputs as si
from conftest import bf16_bits_to_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

MAX_ABS, MEAN_ABS, REL_L2 = 1.5e-2, 2e-3, 2e-2


@pytest.fixture(scope="module")
def va():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from full_spatiotemporal_attention_b200 import build
    build.build()
    import full_spatiotemporal_attention_b200 as va
    assert torch.cuda.get_device_capability() == (10, 0), "kernels target sm_100a (B200)"
    return va


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16).cuda()


def host(t):
    return bf16_bits_to_f64(t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


def vgrid(va, w):
    return va.Grid.make(w.T, w.H, w.W, w.n_text, w.dims, w.theta)


def ogrid(w):
    return oracle.Grid(w.T, w.H, w.W, w.n_text, w.dims, w.theta)


def check(got, ref, label):
    err = np.abs(got - ref)
    max_abs, mean_abs = float(err.max()), float(err.mean())
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    assert np.isfinite(got).all(), f"{label}: non-finite output"
    assert max_abs <= MAX_ABS and mean_abs <= MEAN_ABS and rel <= REL_L2, (
        f"{label}: max_abs={max_abs:.3e} mean_abs={mean_abs:.3e} rel_l2={rel:.3e}")
    return max_abs, mean_abs, rel


def custom(name, T, H, W, heads=2, n_text=0, dims=(44, 42, 42), batch=1, seed=7):
    return si.Workload(name, T, H, W, heads, dims, n_text=n_text, batch=batch, seed=seed)


SMALL = [si.WORKLOADS["tiny"], si.WORKLOADS["c17f480"],
         custom("n1", 1, 1, 1), custom("n127", 1, 1, 127), custom("n129", 1, 3, 43),
         custom("n257", 1, 1, 257, dims=(16, 56, 56)), custom("odd", 3, 5, 17, heads=3),
         custom("batch2", 2, 7, 9, heads=2, batch=2),
         custom("joint_small", 2, 6, 10, heads=2, n_text=37, dims=(16, 56, 56)),
         custom("text1", 1, 4, 4, n_text=1), custom("mostly_text", 1, 2, 2, n_text=300)]

FACTORISED_SMALL = [si.WORKLOADS["tiny"], si.WORKLOADS["c17f480"], custom("f_odd", 3, 5, 17, heads=3),
                    custom("f_t1", 1, 9, 15), custom("f_t33", 33, 2, 3), custom("f_t64", 64, 1, 5),
                    custom("f_hw1", 7, 1, 1), custom("f_b2", 4, 6, 7, batch=2),
                    # frames padded to 16, 24 and 32 rows per position (8, 5 and 4
                    # positions per 128-row tile), position counts not a multiple
                    custom("f_t12", 12, 3, 5), custom("f_t21", 21, 2, 7, dims=(16, 56, 56)),
                    custom("f_t29", 29, 3, 3, heads=3)]

LARGE = ["c81f480", "c81f720", "joint720", "refimg720"]

# the local window timed on the 720p clip: 3 x 9 x 16 = 432 tokens
WINDOW_720 = (3, 9, 16)


# ------------------------------------------------------------------ RoPE

@pytest.mark.parametrize("w", [si.WORKLOADS["tiny"], si.WORKLOADS["c17f480"],
                               custom("r_joint", 2, 6, 10, n_text=37, dims=(16, 56, 56))],
                         ids=lambda w: w.name)
def test_rope3d_apply_matches_oracle(va, w):
    q, _, _ = si.qkv(w)
    x = dev(q)
    y = va.rope3d_apply(x, vgrid(va, w))
    ref = oracle.rope3d(q, ogrid(w))
    got = host(y)
    # One bf16 rounding of an fp32 result (one bf16 ulp), plus the fp32 angle
    # error: pos * inv_freq is rounded twice in fp32 (<= ~1e-5 rad for
    # positions below 100), which moves a pair by that angle times its norm.
    pair = np.sqrt(ref[..., 0::2] ** 2 + ref[..., 1::2] ** 2).repeat(2, axis=-1)
    bound = 2.0 ** -7 * np.abs(ref) + 2e-5 * pair + 1e-7
    err = np.abs(got - ref)
    assert (err <= bound).all(), float((err - bound).max())
    # in place gives the same bits
    va.rope3d_apply(x, vgrid(va, w), out=x)
    assert torch.equal(x.view(torch.int16), y.view(torch.int16))


# ------------------------------------------------------------- full / joint

@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_full_attention_all_rows(va, w):
    q, k, v = si.qkv(w)
    o, lse = va.attn3d_full_fwd(dev(q), dev(k), dev(v), vgrid(va, w), return_lse=True)
    ref, ref_lse = oracle.attention(q, k, v, ogrid(w), want_lse=True)
    check(host(o).reshape(ref.shape), ref, f"full {w.name}")
    np.testing.assert_allclose(lse.cpu().numpy().reshape(ref_lse.shape), ref_lse, atol=2e-3, rtol=0)
    assert va.device_error() == 0


@pytest.mark.parametrize("name", LARGE)
def test_full_attention_sampled_rows_full_size(va, name):
    w = si.WORKLOADS[name]
    q, k, v = si.qkv(w)
    rows = si.sample_rows(w, 512)
    o = va.attn3d_full_fwd(dev(q), dev(k), dev(v), vgrid(va, w))
    got = host(o[:, :, torch.from_numpy(rows).cuda(), :]).reshape(w.batch * w.heads, rows.size, 128)
    ref = oracle.attention(q, k, v, ogrid(w), rows=rows)
    check(got, ref, f"full {name}")
    if w.n_text:
        txt = rows >= w.n_video
        check(got[:, txt], ref[:, txt], f"full {name} text rows")
    assert va.device_error() == 0


def test_prerotated_keys_give_identical_output(va):
    w = si.WORKLOADS["c17f480"]
    q, k, v = (dev(x) for x in si.qkv(w))
    g = vgrid(va, w)
    o1 = va.attn3d_full_fwd(q, k, v, g)
    kr = va.rope3d_apply(k, g)
    o2 = va.attn3d_full_fwd(q, kr, v, g, k_rotated=True)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))


def test_scale_argument(va):
    """A caller-given scale.  Rounding the rotated Q and K to bf16 perturbs each
    logit in proportion to the scale, so the absolute bounds grow by
    scale / (1/sqrt(128)) (3.4x at 0.3); the relative L2 bound stays."""
    w = custom("scale", 2, 4, 6)
    q, k, v = si.qkv(w)
    o = va.attn3d_full_fwd(dev(q), dev(k), dev(v), vgrid(va, w), scale=0.3)
    ref = oracle.attention(q, k, v, ogrid(w), scale=0.3)
    got = host(o).reshape(ref.shape)
    amp = 0.3 * np.sqrt(128.0)
    err = np.abs(got - ref)
    assert err.max() <= MAX_ABS * amp and err.mean() <= MEAN_ABS * amp
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= REL_L2


def test_repeat_calls_are_deterministic(va):
    w = si.WORKLOADS["c17f480"]
    q, k, v = (dev(x) for x in si.qkv(w))
    g = vgrid(va, w)
    a = va.attn3d_full_fwd(q, k, v, g)
    b = va.attn3d_full_fwd(q, k, v, g)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


# -------------------------------------------------------------- factorised

@pytest.mark.parametrize("w", FACTORISED_SMALL, ids=lambda w: w.name)
def test_factorised_all_rows(va, w):
    q, k, v = si.qkv(w)
    os_, ot = va.attn_factorized_fwd(dev(q), dev(k), dev(v), vgrid(va, w))
    shape = (w.batch * w.heads, w.N, 128)
    check(host(os_).reshape(shape), oracle.attention(q, k, v, ogrid(w), mode="spatial"),
          f"spatial {w.name}")
    check(host(ot).reshape(shape), oracle.attention(q, k, v, ogrid(w), mode="temporal"),
          f"temporal {w.name}")
    assert va.device_error() == 0


@pytest.mark.parametrize("w", [si.WORKLOADS["c17f480"], custom("r_t12", 12, 3, 5),
                               custom("r_t21", 21, 2, 7), custom("r_t29", 29, 3, 3, heads=3),
                               custom("r_t40", 40, 2, 3)], ids=lambda w: w.name)
def test_factorised_with_prerotated_keys(va, w):
    """Keys turned by rope3d_apply and passed with k_rotated: the temporal
    pass then turns Q in full and runs all of QK^T in scaled fp16."""
    q, k, v = si.qkv(w)
    g = vgrid(va, w)
    qd, kd, vd = dev(q), dev(k), dev(v)
    kr = va.rope3d_apply(kd, g)
    os_, ot = va.attn_factorized_fwd(qd, kr, vd, g, k_rotated=True)
    shape = (w.batch * w.heads, w.N, 128)
    check(host(os_).reshape(shape), oracle.attention(q, k, v, ogrid(w), mode="spatial"),
          f"spatial {w.name}")
    check(host(ot).reshape(shape), oracle.attention(q, k, v, ogrid(w), mode="temporal"),
          f"temporal {w.name}")
    assert va.device_error() == 0


def test_factorised_sampled_rows_full_size(va):
    w = si.WORKLOADS["c81f720"]
    q, k, v = si.qkv(w)
    rows = si.sample_rows(w, 512)
    os_, ot = va.attn_factorized_fwd(dev(q), dev(k), dev(v), vgrid(va, w))
    idx = torch.from_numpy(rows).cuda()
    for mode, out in (("spatial", os_), ("temporal", ot)):
        got = host(out[:, :, idx, :]).reshape(w.heads, rows.size, 128)
        ref = oracle.attention(q, k, v, ogrid(w), mode=mode, rows=rows)
        check(got, ref, f"{mode} c81f720")


def _scale_bits(bits, k):
    """bf16 bit patterns times 2^k, exactly (exponent field + k; zeros kept)."""
    b = bits.astype(np.int32)
    nz = (b & 0x7FFF) != 0
    b = np.where(nz, b + (k << 7), b)
    return b.astype(np.uint16)


@pytest.mark.parametrize("k", [-14, -8, 8, 14])
def test_temporal_pass_at_extreme_magnitudes(va, k):
    """Queries times 2^k and keys times 2^-k leave every logit exactly as it
    was while moving the turned values out of fp16's comfortable range
    (k = +-14: the power-of-two-scaled path) or to its edges (k = +-8: the
    unscaled path with small operands near fp16's subnormals)."""
    w = si.WORKLOADS["c17f480"]
    q, kk, v = si.qkv(w)
    q, kk = _scale_bits(q, k), _scale_bits(kk, -k)
    _, ot = va.attn_factorized_fwd(dev(q), dev(kk), dev(v), vgrid(va, w), spatial=False)
    ref = oracle.attention(q, kk, v, ogrid(w), mode="temporal")
    check(host(ot).reshape(ref.shape), ref, f"temporal 2^{k}")
    assert va.device_error() == 0


@pytest.mark.parametrize("k", [-14, 14])
@pytest.mark.parametrize("w", [si.WORKLOADS["c17f480"], custom("x_t21", 21, 4, 7)], ids=lambda w: w.name)
@pytest.mark.parametrize("rotated", [False, True], ids=["raw_keys", "rotated_keys"])
def test_temporal_pass_fallback_for_both_key_forms(va, k, w, rotated):
    """Queries times 2^k and keys times 2^-k push the values written as fp16
    out of range, so every tile takes the scaled fallback: with raw keys and
    with keys that come rotated (rope3d_apply of the scaled keys), on 8- and
    32-row position tiles."""
    q, kk, v = si.qkv(w)
    q, kk = _scale_bits(q, k), _scale_bits(kk, -k)
    g = vgrid(va, w)
    kd = dev(kk)
    if rotated:
        kd = va.rope3d_apply(kd, g)
    _, ot = va.attn_factorized_fwd(dev(q), kd, dev(v), g, spatial=False, k_rotated=rotated)
    ref = oracle.attention(q, kk, v, ogrid(w), mode="temporal")
    check(host(ot).reshape(ref.shape), ref, f"temporal {w.name} 2^{k} rotated={rotated}")
    assert va.device_error() == 0


def test_factorised_single_pass_outputs(va):
    w = si.WORKLOADS["tiny"]
    q, k, v = (dev(x) for x in si.qkv(w))
    g = vgrid(va, w)
    s_only, none = va.attn_factorized_fwd(q, k, v, g, temporal=False)
    assert none is None
    none, t_only = va.attn_factorized_fwd(q, k, v, g, spatial=False)
    s2, t2 = va.attn_factorized_fwd(q, k, v, g)
    assert torch.equal(s_only.view(torch.int16), s2.view(torch.int16))
    assert torch.equal(t_only.view(torch.int16), t2.view(torch.int16))


# ------------------------------------------------------ local 3D windows

WINDOW_SMALL = [(si.WORKLOADS["tiny"], (1, 2, 4)), (si.WORKLOADS["tiny"], (2, 2, 2)),
                (si.WORKLOADS["tiny"], (1, 1, 1)), (si.WORKLOADS["c17f480"], (5, 6, 4)),
                (si.WORKLOADS["c17f480"], (1, 10, 26)), (si.WORKLOADS["c17f480"], (5, 15, 13)),
                (custom("w_odd", 3, 5, 17, heads=3), (3, 5, 1)),
                (custom("w_b2", 2, 7, 9, batch=2), (2, 7, 3)),
                # w extents that tile a 128-row tile exactly (8, 16, 32)
                (custom("w_tma", 3, 6, 32, heads=2), (1, 3, 16)),
                (custom("w_tma", 3, 6, 32, heads=2), (3, 6, 16)),
                (custom("w_tma", 3, 6, 32, heads=2), (3, 2, 8)),
                (custom("w_tma", 3, 6, 32, heads=2), (3, 3, 32)),
                (custom("w_tma_b2", 2, 4, 16, batch=2), (2, 4, 16)),
                (custom("w_tma_b2", 2, 4, 16, batch=2), (1, 2, 8))]


def window_keys(w, win, n):
    """Token indices of the window that holds token n."""
    hw = w.H * w.W
    t, rem = divmod(int(n), hw)
    h, x = divmod(rem, w.W)
    t0, h0, x0 = t // win[0] * win[0], h // win[1] * win[1], x // win[2] * win[2]
    return np.array([(tt * w.H + hh) * w.W + xx for tt in range(t0, t0 + win[0])
                     for hh in range(h0, h0 + win[1]) for xx in range(x0, x0 + win[2])])


def window_bounds(w, win, q, k, v, rows, want_o=True):
    """Per-element bound on |GPU - oracle| for window attention, derived from
    the kernel's arithmetic to first order.  The scores use Q~ and K~ rounded
    to bf16, so |ds_j| <= D_j = 2^-8 * scale * sum_i |q~_i| |k~_ji|; a score
    error moves o_c by sum_j p_j ds_j (v_jc - o_c) and the LSE by
    sum_j p_j ds_j.  P rounded to bf16 adds 2^-9 sum_j p_j |v_jc|, the
    polynomial exp2 (relative error 7.5e-5) 1.5e-4 sum_j p_j |v_jc - o_c|, the
    bf16 output 2^-9 |o_c|.  Returns (bound_o [BH, rows, 128] or None,
    bound_lse [BH, rows]).  Worst case over the rounding errors, so several
    times the typical error."""
    g = ogrid(w)
    scale = 1.0 / np.sqrt(128)
    BH = w.batch * w.heads
    qb, kb, vb = (x.reshape(BH, w.N, 128) for x in (q, k, v))
    bo = np.empty((BH, rows.size, 128)) if want_o else None
    bl = np.empty((BH, rows.size))
    # group the rows by window: rows of one window share its keys
    groups = {}
    for i, n in enumerate(rows):
        ks = window_keys(w, win, n)
        groups.setdefault(int(ks[0]), (ks, []))[1].append(i)
    for b in range(BH):
        qr = oracle.rope3d(qb[b:b + 1], g)[0]
        kr = oracle.rope3d(kb[b:b + 1], g)[0]
        vf = bf16_bits_to_f64(vb[b])
        for ks, idx in groups.values():
            idx = np.array(idx)
            qs = qr[rows[idx]]                              # [r, 128]
            sc = qs @ kr[ks].T * scale                       # [r, keys]
            p = np.exp(sc - sc.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            o = p @ vf[ks]                                   # [r, 128]
            D = 2.0 ** -8 * scale * (np.abs(qs) @ np.abs(kr[ks]).T)     # [r, keys]
            pd = p * D
            bl[b, idx] = pd.sum(axis=1) * 1.1 + 2e-4
            if want_o:
                dv = np.abs(vf[ks][None, :, :] - o[:, None, :])         # [r, keys, 128]
                bo[b, idx] = (np.einsum("rk,rkc->rc", pd, dv)
                              + 1.5e-4 * np.einsum("rk,rkc->rc", p, dv)
                              + 2.0 ** -9 * (p @ np.abs(vf[ks])) + 2.0 ** -9 * np.abs(o)) * 1.1 + 1e-6
    return bo, bl


def check_window(got, ref, bound, label):
    """Within the derived per-element bound, and the mean-abs and relative-L2
    bars of the other modes."""
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), f"{label}: non-finite output"
    worst = float((err / bound).max())
    assert worst <= 1.0, f"{label}: error reaches {worst:.2f} x the derived bound"
    rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    assert float(err.mean()) <= MEAN_ABS and rel <= REL_L2, (label, float(err.mean()), rel)
    return float(err.max()), worst


@pytest.mark.parametrize("w,win", WINDOW_SMALL, ids=lambda x: x.name if hasattr(x, "name") else
                         "x".join(map(str, x)))
def test_window_attention_all_rows(va, w, win):
    q, k, v = si.qkv(w)
    o, lse = va.attn_window_fwd(dev(q), dev(k), dev(v), vgrid(va, w), win, return_lse=True)
    ref, ref_lse = oracle.window_attention(q, k, v, ogrid(w), win, want_lse=True)
    # outputs: the bar of the other modes; LSE: the derived bound (with a
    # handful of keys per window there is no averaging of score errors)
    check(host(o).reshape(ref.shape), ref, f"window {w.name} {win}")
    _, bl = window_bounds(w, win, q, k, v, np.arange(w.N), want_o=False)
    lerr = np.abs(lse.cpu().numpy().reshape(ref_lse.shape) - ref_lse)
    assert (lerr <= bl).all(), float((lerr / bl).max())
    assert va.device_error() == 0


def test_window_gather_matches_the_tma_paths_bit_for_bit(va):
    """A window of the whole grid is full attention and a window of one frame
    the spatial pass: the gathered rows are then in natural order, so the
    outputs must equal the TMA-loaded paths bit for bit."""
    w = si.WORKLOADS["c17f480"]
    q, k, v = (dev(x) for x in si.qkv(w))
    g = vgrid(va, w)
    full = va.attn3d_full_fwd(q, k, v, g)
    win_full = va.attn_window_fwd(q, k, v, g, (w.T, w.H, w.W))
    assert torch.equal(full.view(torch.int16), win_full.view(torch.int16))
    sp, _ = va.attn_factorized_fwd(q, k, v, g, temporal=False)
    win_sp = va.attn_window_fwd(q, k, v, g, (1, w.H, w.W))
    assert torch.equal(sp.view(torch.int16), win_sp.view(torch.int16))


def test_window_rows_of_wide_frames_match_the_tile_paths_bit_for_bit(va):
    """A 32-wide grid: a window of one frame is the spatial pass and a window
    of the whole grid full attention, bit for bit."""
    # frames of 544 tokens (5 key tiles), so that both sides run the same
    # two-query-tile configuration and split the same tiles
    w = custom("w_tma_frame", 2, 17, 32, heads=2)
    q, k, v = (dev(x) for x in si.qkv(w))
    g = vgrid(va, w)
    full = va.attn3d_full_fwd(q, k, v, g)
    win_full = va.attn_window_fwd(q, k, v, g, (w.T, w.H, w.W))
    assert torch.equal(full.view(torch.int16), win_full.view(torch.int16))
    sp, _ = va.attn_factorized_fwd(q, k, v, g, temporal=False)
    win_sp = va.attn_window_fwd(q, k, v, g, (1, w.H, w.W))
    assert torch.equal(sp.view(torch.int16), win_sp.view(torch.int16))
    assert va.device_error() == 0


def test_window_attention_sampled_rows_full_size(va):
    w = si.WORKLOADS["c81f720"]
    win = WINDOW_720
    q, k, v = si.qkv(w)
    rows = si.sample_rows(w, 512)
    o = va.attn_window_fwd(dev(q), dev(k), dev(v), vgrid(va, w), win)
    got = host(o[:, :, torch.from_numpy(rows).cuda(), :]).reshape(w.batch * w.heads, rows.size, 128)
    ref = oracle.window_attention(q, k, v, ogrid(w), win, rows=rows)
    bo, _ = window_bounds(w, win, q, k, v, rows)
    check_window(got, ref, bo, f"window c81f720 {win}")
    assert va.device_error() == 0


# ------------------------------------------------------- text cross-attention

def cross_case(name, nq, nkv, heads=2, batch=1, seed=11):
    # queries on a 1 x 1 x nq "grid" (the grid does not enter cross-attention)
    return si.Workload(name, 1, 1, nq, heads, (44, 42, 42), batch=batch, seed=seed, n_kv=nkv)


CROSS_SMALL = [cross_case("x_1_1", 1, 1, heads=1), cross_case("x_32_7", 32, 7),
               cross_case("x_300_512", 300, 512, heads=3), cross_case("x_1000_129", 1000, 129, batch=2),
               cross_case("x_257_1", 257, 1), cross_case("x_7800_512", 7800, 512, heads=12),
               cross_case("x_130_1000", 130, 1000)]


@pytest.mark.parametrize("w", CROSS_SMALL, ids=lambda w: w.name)
def test_cross_attention_all_rows(va, w):
    q, k, v = si.qkv(w)
    o, lse = va.attn_cross_fwd(dev(q), dev(k), dev(v), return_lse=True)
    ref, ref_lse = oracle.cross_attention(q, k, v, want_lse=True)
    check(host(o).reshape(ref.shape), ref, f"cross {w.name}")
    np.testing.assert_allclose(lse.cpu().numpy().reshape(ref_lse.shape), ref_lse, atol=2e-3, rtol=0)
    # without scratch every tile runs whole: same result within the bar
    o2 = va.attn_cross_fwd(dev(q), dev(k), dev(v), workspace=torch.empty(0, dtype=torch.uint8,
                                                                         device="cuda"))
    check(host(o2).reshape(ref.shape), ref, f"cross {w.name} unsplit")
    assert va.device_error() == 0


def test_cross_attention_sampled_rows_full_size(va):
    w = si.WORKLOADS["cross720"]
    q, k, v = si.qkv(w)
    rows = si.sample_rows(w, 512)
    o = va.attn_cross_fwd(dev(q), dev(k), dev(v))
    got = host(o[:, :, torch.from_numpy(rows).cuda(), :]).reshape(w.batch * w.heads, rows.size, 128)
    ref = oracle.cross_attention(q, k, v, rows=rows)
    check(got, ref, "cross cross720")
    assert va.device_error() == 0


def test_binding_rejects_bad_tensors(va):
    g = va.Grid.make(2, 4, 4)
    x = torch.zeros(1, 2, 32, 128, dtype=torch.float16, device="cuda")
    with pytest.raises(TypeError):
        va.attn3d_full_fwd(x, x, x, g)
    y = torch.zeros(1, 2, 33, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(va.VA3DError):
        va.attn3d_full_fwd(y, y, y, g)    # N inconsistent with the grid
