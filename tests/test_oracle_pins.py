"""Pins of the CPU oracle to what the pages and the mathematics fix (no GPU).

Each test checks the oracle against something other than itself: a worked
example printed on a page (tests/golden, with its citation), a closed form, an
invariant, a special case that reduces to a library routine (torch conv2d /
grid_sample on the CPU in float64), or brute force in the pure-Python twin.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import gen
import oracle
from oracle import scalar

RNG = np.random.default_rng(1234)


def _zeros_offsets(N, Ho, Wo, G, K):
    return np.zeros((N, Ho, Wo, G, K, 2))


# --------------------------------------------------------------------------
# Worked examples printed on the pages
# --------------------------------------------------------------------------

def test_bilinear_worked_example(golden):
    g = golden("bilinear_worked_example.txt")
    grid = [g["grid_row0"], g["grid_row1"]]
    px, py = g["point"]
    _, w = scalar.corner_weights(px, py)
    order = [(0, 0), (1, 0), (0, 1), (1, 1)]
    assert [w[c] for c in order] == pytest.approx(g["weights"], abs=1e-15)
    contrib = [w[(i, j)] * grid[j][i] for (i, j) in order]
    assert contrib == pytest.approx(g["contributions"], abs=1e-15)
    assert sum(w.values()) == pytest.approx(1.0, abs=1e-15)
    assert scalar.bilinear_pixel(grid, px, py) == pytest.approx(g["value"], abs=1e-12)

    # the C oracle: a 2x2 single-channel map, one tap, output (0,0) moved by p
    x = np.array(grid, dtype=np.float64).reshape(1, 2, 2, 1)
    off = _zeros_offsets(1, 2, 2, 1, 1)
    off[0, 0, 0, 0, 0] = (px, py)
    mask = np.ones((1, 2, 2, 1, 1))
    out = oracle.dcn_forward_ref(x, off, mask, kh=1, kw=1, stride=1, pad=0, dil=1)
    assert out[0, 0, 0, 0] == pytest.approx(g["value"], abs=1e-12)
    # the other outputs did not move: identity
    assert out[0, 0, 1, 0] == 20 and out[0, 1, 0, 0] == 30 and out[0, 1, 1, 0] == 40


def test_spike_1d(golden):
    g = golden("spike_1d.txt")
    sig = np.array(g["signal"]).reshape(1, 1, 5, 1)
    mask = np.ones((1, 1, 5, 1, 1))
    for off_key, val_key in (("offset_rigid", "value_rigid"),
                             ("offset_learned", "value_learned")):
        off = _zeros_offsets(1, 1, 5, 1, 1)
        off[0, 0, int(g["p0"]), 0, 0, 0] = g[off_key]
        out = oracle.dcn_forward_ref(sig, off, mask, kh=1, kw=1, stride=1, pad=0, dil=1)
        assert out[0, 0, int(g["p0"]), 0] == g[val_key]


def _three_tap_row(values, logits, softmax_flag):
    """1x3 map read by a 1x3 window centred at output (1, 1), zero offsets."""
    x = np.array(values, dtype=np.float64).reshape(1, 1, 3, 1)
    # pad 1 in both directions: Ho = 3 (kh = 1), Wo = 3 (kw = 3)
    off = _zeros_offsets(1, 3, 3, 1, 3)
    mask = np.zeros((1, 3, 3, 1, 3))
    mask[0, 1, 1, 0, :] = logits            # k = ix * kh + iy = ix
    out = oracle.dcn_forward_ref(x, off, mask, kh=1, kw=3, stride=1, pad=1, dil=1,
                                 softmax_flag=softmax_flag)
    return out[0, 1, 1, 0]


def test_dcnv3_softmax_worked_example(golden):
    g = golden("dcnv3_softmax_k3.txt")
    z, v = g["logits"], g["sampled"]
    m = scalar.softmax(z)
    assert sum(math.exp(t) for t in z) == pytest.approx(g["exp_sum"], abs=5e-4)
    assert m == pytest.approx(g["modulation"], abs=g["page_rounding_m"])
    assert sum(m) == pytest.approx(1.0, abs=1e-15)
    y = _three_tap_row(v, z, softmax_flag=1)
    e = math.e
    exact = (2 + 8 * e ** 2 + 4 * e) / (1 + e ** 2 + e)      # closed form
    assert y == pytest.approx(exact, abs=1e-12)
    assert abs(y - g["value"]) <= g["page_rounding_y"]
    assert min(v) <= y <= max(v)                              # weighted average


def test_right_minus_left_unbounded(golden):
    g = golden("right_minus_left.txt")
    for _ in range(20):
        left, centre, right = RNG.uniform(-1, 1, 3)
        y = _three_tap_row([left, centre, right], g["weights_unbounded"], softmax_flag=0)
        assert y == right - left                      # exact: integer taps
    # a case whose result lies outside [min v, max v]
    y = _three_tap_row([0.5, 0.4, 0.2], g["weights_unbounded"], softmax_flag=0)
    assert y == pytest.approx(-0.3, abs=1e-15) and y < 0.2
    # softmax weights can only average
    for _ in range(20):
        vals = RNG.uniform(-1, 1, 3)
        y = _three_tap_row(vals, RNG.normal(0, 3, 3), softmax_flag=1)
        assert vals.min() - 1e-15 <= y <= vals.max() + 1e-15


def test_offset_counts(golden):
    g = golden("offset_counts.txt")
    C, K = int(g["C"]), int(g["K"])
    for G, n_off, n_log in ((1, g["G1_offsets"], g["G1_logits"]),
                            (4, g["G4_offsets"], g["G4_logits"])):
        w = gen.DcnWorkload("t", N=1, H=3, W=3, C=C, G=G)
        assert w.K == K
        inp = gen.dcn_inputs(w)
        per_loc_off = inp["offset"][0, 0, 0].numel()
        per_loc_mask = inp["mask"][0, 0, 0].numel()
        assert per_loc_off == n_off and per_loc_mask == n_log
    assert C // 4 == g["G4_channels_per_group"]


def test_msda_corner_quarter(golden):
    g = golden("msda_corner.txt")
    H, W = 3, 4
    value = np.zeros((1, H * W, 1, 1))
    value[0, 0, 0, 0] = g["first_cell"]
    for uv, expect in ((g["corner_uv"], g["corner_value"]), (g["far_uv"], g["far_value"])):
        loc = np.array(uv).reshape(1, 1, 1, 1, 1, 2)
        attn = np.ones((1, 1, 1, 1, 1))
        out = oracle.msda_forward_ref(value, [[H, W]], [0], loc, attn)
        assert out[0, 0, 0] == pytest.approx(expect, abs=1e-15)
    grid = [[g["first_cell"]] + [0.0] * (W - 1)] + [[0.0] * W for _ in range(H - 1)]
    assert scalar.bilinear_normalized(grid, *g["corner_uv"]) == pytest.approx(0.25)


def test_msda_joint_softmax_quarter(golden):
    g = golden("msda_joint_softmax.txt")
    L, K = int(g["levels"]), int(g["points"])
    w = scalar.normalize_weights([[0.0] * K for _ in range(L)])
    assert all(x == pytest.approx(g["weight_each"]) for lvl in w for x in lvl)
    per_level = [scalar.softmax([0.0] * K) for _ in range(L)]
    assert per_level[0][0] == pytest.approx(g["per_level_wrong"])
    # joint normalisation: total mass 1 for random logits too
    for _ in range(10):
        z = RNG.normal(0, 2, (3, 4)).tolist()
        w = scalar.normalize_weights(z)
        assert sum(map(sum, w)) == pytest.approx(1.0, abs=1e-14)


# --------------------------------------------------------------------------
# Invariants and closed forms
# --------------------------------------------------------------------------

def test_bilinear_weights_sum_and_convex_hull():
    for _ in range(200):
        px, py = RNG.uniform(-5, 5, 2)
        _, w = scalar.corner_weights(px, py)
        assert sum(w.values()) == pytest.approx(1.0, abs=1e-14)
        assert all(v >= 0 for v in w.values())
    # convex hull through the C oracle: interior reads of a random map
    H, W = 6, 7
    x = RNG.uniform(-1, 1, (1, H, W, 1))
    off = RNG.uniform(0.0, 1.0, (1, H, W, 1, 1, 2))
    off[0, :, W - 1] = 0.0        # keep every read inside the map
    off[0, H - 1, :] = 0.0
    out = oracle.dcn_forward_ref(x, off, np.ones((1, H, W, 1, 1)), kh=1, kw=1,
                                 stride=1, pad=0, dil=1)
    for oy in range(H - 1):
        for ox in range(W - 1):
            cell = x[0, oy:oy + 2, ox:ox + 2, 0]
            assert cell.min() - 1e-15 <= out[0, oy, ox, 0] <= cell.max() + 1e-15


def test_constant_map_softmax_and_unbounded():
    H = W = 9
    c = 0.37
    x = np.full((2, H, W, 8), c)
    w = gen.DcnWorkload("t", N=2, H=H, W=W, C=8, G=2)
    off = RNG.uniform(-0.9, 0.9, (2, H, W, 2, 9, 2))
    logits = RNG.normal(0, 1, (2, H, W, 2, 9))
    soft = oracle.dcn_forward_ref(x, off, logits, 3, 3, 1, 1, 1, softmax_flag=1)
    unb = oracle.dcn_forward_ref(x, off, logits, 3, 3, 1, 1, 1, softmax_flag=0)
    inner = (slice(None), slice(2, H - 2), slice(2, W - 2))   # every corner in bounds
    assert np.allclose(soft[inner], c, atol=1e-14, rtol=0)
    msum = logits.sum(axis=-1)                                 # [N, Ho, Wo, G]
    expect = c * np.repeat(msum, w.D, axis=-1)
    assert np.allclose(unb[inner], expect[inner], atol=1e-13, rtol=0)


def test_edge_straddle_and_far_outside():
    """x = 1 everywhere: a tap straddling the border reads the in-bounds weight
    sum (no clamping, no renormalisation); a tap far outside reads 0."""
    H, W = 4, 5
    x = np.ones((1, H, W, 1))
    off = _zeros_offsets(1, H, W, 1, 1)
    off[0, 0, 0, 0, 0] = (-0.25, -0.5)        # corners at x=-1/0, y=-1/0
    off[0, 1, 1, 0, 0] = (-30.0, 0.0)         # far outside
    off[0, 2, 2, 0, 0] = (1e30, -1e30)        # huge: no overflow, reads 0
    off[0, 3, 3, 0, 0] = (np.nan, 0.0)        # not finite: reads 0, no crash
    out = oracle.dcn_forward_ref(x, off, np.ones((1, H, W, 1, 1)), 1, 1, 1, 0, 1)
    assert out[0, 0, 0, 0] == pytest.approx(0.75 * 0.5, abs=1e-15)
    assert out[0, 1, 1, 0] == 0.0 and out[0, 2, 2, 0] == 0.0 and out[0, 3, 3, 0] == 0.0


def test_identity_zero_offsets_k1():
    for (N, H, W, C, G) in ((1, 3, 4, 6, 3), (2, 5, 5, 16, 1), (1, 1, 7, 4, 4)):
        x = RNG.uniform(-1, 1, (N, H, W, C))
        out = oracle.dcn_forward_ref(x, _zeros_offsets(N, H, W, G, 1),
                                     np.ones((N, H, W, G, 1)), 1, 1, 1, 0, 1)
        assert np.array_equal(out, x)


@pytest.mark.parametrize("kh,kw,stride,pad,dil,H,W", [
    (3, 3, 1, 1, 1, 7, 9), (3, 3, 2, 1, 1, 8, 7), (3, 3, 1, 2, 2, 6, 6),
    (5, 5, 1, 2, 1, 7, 5), (1, 3, 1, 0, 1, 4, 6), (3, 1, 2, 0, 3, 9, 4),
    (2, 3, 1, 1, 1, 5, 5),
])
def test_zero_offsets_match_grouped_conv(kh, kw, stride, pad, dil, H, W):
    """Zero offsets and pixel-independent m reduce DCN to a depthwise conv
    whose weight at (iy, ix) is m[g, k(ix, iy)] (torch conv2d, float64)."""
    N, C, G = 2, 6, 3
    D = C // G
    K = kh * kw
    Ho = oracle.out_size(H, kh, stride, pad, dil)
    Wo = oracle.out_size(W, kw, stride, pad, dil)
    x = RNG.uniform(-1, 1, (N, H, W, C))
    m = RNG.normal(0, 1, (G, K))
    mask = np.broadcast_to(m, (N, Ho, Wo, G, K)).copy()
    out = oracle.dcn_forward_ref(x, _zeros_offsets(N, Ho, Wo, G, K), mask,
                                 kh, kw, stride, pad, dil)
    weight = np.zeros((C, 1, kh, kw))
    for c in range(C):
        for ix in range(kw):
            for iy in range(kh):
                weight[c, 0, iy, ix] = m[c // D, ix * kh + iy]
    ref = F.conv2d(torch.from_numpy(x).permute(0, 3, 1, 2), torch.from_numpy(weight),
                   stride=stride, padding=pad, dilation=dil, groups=C)
    ref = ref.permute(0, 2, 3, 1).numpy()
    assert ref.shape == out.shape
    assert np.allclose(out, ref, atol=1e-13, rtol=0)


def test_integer_offsets_are_a_shifted_gather():
    N, H, W, C, G, kh, kw, stride, pad, dil = 2, 6, 7, 4, 2, 3, 3, 1, 1, 1
    D, K = C // G, kh * kw
    x = RNG.uniform(-1, 1, (N, H, W, C))
    off = RNG.integers(-3, 4, (N, H, W, G, K, 2)).astype(np.float64)
    m = RNG.normal(0, 1, (N, H, W, G, K))
    out = oracle.dcn_forward_ref(x, off, m, kh, kw, stride, pad, dil)
    ref = np.zeros_like(out)
    for n in range(N):
        for oy in range(H):
            for ox in range(W):
                for g in range(G):
                    for ix in range(kw):
                        for iy in range(kh):
                            k = ix * kh + iy
                            xx = ox * stride - pad + ix * dil + int(off[n, oy, ox, g, k, 0])
                            yy = oy * stride - pad + iy * dil + int(off[n, oy, ox, g, k, 1])
                            if 0 <= xx < W and 0 <= yy < H:
                                ref[n, oy, ox, g * D:(g + 1) * D] += (
                                    m[n, oy, ox, g, k] * x[n, yy, xx, g * D:(g + 1) * D])
    assert np.allclose(out, ref, atol=1e-14, rtol=0)


def test_bilinear_matches_grid_sample():
    """One tap per pixel with fractional offsets (some outside the map) equals
    torch grid_sample(align_corners=False, zeros) at u = (px + 1/2) / W."""
    N, H, W, C = 2, 5, 8, 3
    x = RNG.uniform(-1, 1, (N, H, W, C))
    off = RNG.uniform(-3.5, 3.5, (N, H, W, 1, 1, 2))
    out = oracle.dcn_forward_ref(x, off, np.ones((N, H, W, 1, 1)), 1, 1, 1, 0, 1)
    ox = np.arange(W)[None, None, :]
    oy = np.arange(H)[None, :, None]
    px = ox + off[..., 0, 0, 0]
    py = oy + off[..., 0, 0, 1]
    grid = np.stack([(2 * px + 1) / W - 1, (2 * py + 1) / H - 1], axis=-1)
    ref = F.grid_sample(torch.from_numpy(x).permute(0, 3, 1, 2), torch.from_numpy(grid),
                        mode="bilinear", padding_mode="zeros", align_corners=False)
    ref = ref.permute(0, 2, 3, 1).numpy()
    assert np.allclose(out, ref, atol=1e-13, rtol=0)


def test_groups_use_their_own_offsets_and_masks():
    N, H, W, C, G = 1, 5, 6, 8, 4
    D = C // G
    x = RNG.uniform(-1, 1, (N, H, W, C))
    off = RNG.normal(0, 1.5, (N, H, W, G, 9, 2))
    m = RNG.normal(0, 1, (N, H, W, G, 9))
    out = oracle.dcn_forward_ref(x, off, m, 3, 3, 1, 1, 1)
    for g in range(G):
        single = oracle.dcn_forward_ref(
            np.ascontiguousarray(x[..., g * D:(g + 1) * D]),
            np.ascontiguousarray(off[:, :, :, g:g + 1]),
            np.ascontiguousarray(m[:, :, :, g:g + 1]), 3, 3, 1, 1, 1)
        assert np.array_equal(out[..., g * D:(g + 1) * D], single)


def test_linearity_in_x_and_m():
    N, H, W, C, G = 1, 6, 6, 4, 2
    off = RNG.normal(0, 2, (N, H, W, G, 9, 2))
    x1, x2 = RNG.uniform(-1, 1, (2, N, H, W, C))
    m1, m2 = RNG.normal(0, 1, (2, N, H, W, G, 9))
    f = lambda x, m: oracle.dcn_forward_ref(x, off, m, 3, 3, 1, 1, 1)
    assert np.allclose(f(x1 + 2 * x2, m1), f(x1, m1) + 2 * f(x2, m1), atol=1e-13)
    assert np.allclose(f(x1, m1 - 3 * m2), f(x1, m1) - 3 * f(x1, m2), atol=1e-13)


# --------------------------------------------------------------------------
# MSDA against torch grid_sample and special cases
# --------------------------------------------------------------------------

def _msda_grid_sample(value, shapes, starts, loc, attn):
    """Independent MSDA core: grid_sample(2s - 1) per level, weighted by A."""
    N, S, M, D = value.shape
    _, Lq, _, L, K, _ = loc.shape
    v = torch.from_numpy(value)
    out = torch.zeros(N, M, D, Lq, dtype=torch.float64)
    for l, (h, w) in enumerate(shapes):
        lvl = v[:, starts[l]:starts[l] + h * w]                  # [N, h*w, M, D]
        lvl = lvl.permute(0, 2, 3, 1).reshape(N * M, D, h, w)
        grid = torch.from_numpy(loc[:, :, :, l]).permute(0, 2, 1, 3, 4)  # N,M,Lq,K,2
        grid = (2 * grid - 1).reshape(N * M, Lq, K, 2)
        s = F.grid_sample(lvl, grid, mode="bilinear", padding_mode="zeros",
                          align_corners=False)                   # [N*M, D, Lq, K]
        a = torch.from_numpy(attn[:, :, :, l]).permute(0, 2, 1, 3).reshape(N * M, 1, Lq, K)
        out += (s * a).sum(-1).reshape(N, M, D, Lq)
    return out.permute(0, 3, 1, 2).reshape(N, Lq, M * D).numpy()


def test_msda_matches_grid_sample():
    shapes = [(5, 7), (3, 4), (2, 2)]
    starts = gen.level_start_index(shapes)
    N, M, D, K, Lq = 2, 3, 4, 2, 6
    S = sum(h * w for h, w in shapes)
    value = RNG.uniform(-1, 1, (N, S, M, D))
    loc = RNG.uniform(-0.3, 1.3, (N, Lq, M, len(shapes), K, 2))
    attn = RNG.uniform(0, 1, (N, Lq, M, len(shapes), K))
    out = oracle.msda_forward_ref(value, shapes, starts, loc, attn)
    ref = _msda_grid_sample(value, shapes, starts, loc, attn)
    assert np.allclose(out, ref, atol=1e-13, rtol=0)


def test_msda_pixel_centres_read_the_value():
    shapes = [(4, 6), (2, 3)]
    starts = gen.level_start_index(shapes)
    S = sum(h * w for h, w in shapes)
    N, M, D = 1, 2, 3
    value = RNG.uniform(-1, 1, (N, S, M, D))
    for l, (h, w) in enumerate(shapes):
        for (i, j) in ((0, 0), (w - 1, h - 1), (w // 2, h // 3)):
            loc = np.zeros((N, 1, M, 2, 1, 2))
            attn = np.zeros((N, 1, M, 2, 1))
            loc[:, :, :, l, 0] = ((i + 0.5) / w, (j + 0.5) / h)
            attn[:, :, :, l, 0] = 1.0
            out = oracle.msda_forward_ref(value, shapes, starts, loc, attn)
            expect = value[0, starts[l] + j * w + i].reshape(-1)
            assert np.allclose(out[0, 0], expect, atol=1e-15)


def test_dcn_and_msda_bilinear_forms_agree():
    """The floor form of InternImage ch.2 and the tent form of Deformable DETR
    helper 2 are one function: pixel point (px, py) <-> (u, v) = ((px+1/2)/W, ...)."""
    H, W = 6, 9
    x = RNG.uniform(-1, 1, (1, H, W, 1))
    off = RNG.uniform(-2, 2, (1, H, W, 1, 1, 2))
    dcn = oracle.dcn_forward_ref(x, off, np.ones((1, H, W, 1, 1)), 1, 1, 1, 0, 1)
    oy, ox = np.meshgrid(np.arange(H), np.arange(W), indexing="ij")
    u = (ox + off[0, :, :, 0, 0, 0] + 0.5) / W
    v = (oy + off[0, :, :, 0, 0, 1] + 0.5) / H
    loc = np.stack([u, v], -1).reshape(1, H * W, 1, 1, 1, 2)
    ms = oracle.msda_forward_ref(x.reshape(1, H * W, 1, 1), [(H, W)], [0], loc,
                                 np.ones((1, H * W, 1, 1, 1)))
    assert np.allclose(dcn.reshape(-1), ms.reshape(-1), atol=1e-13)


def test_generator_attention_is_the_joint_softmax():
    w = gen.MsdaWorkload("t", N=1, M=2, D=2, shapes=((3, 4), (2, 2)), K=3)
    inp = gen.msda_inputs(w, seed=5)
    attn = inp["attn"].double().numpy()
    for q in range(w.queries):
        for h in range(w.M):
            z = inp["logits"][0, q, h].tolist()
            expect = scalar.normalize_weights(z)
            assert np.allclose(attn[0, q, h], expect, atol=1e-7)
    assert np.allclose(attn.sum(axis=(-1, -2)), 1.0, atol=1e-6)


# --------------------------------------------------------------------------
# Brute force: the C loop nests against the pure-Python twin
# --------------------------------------------------------------------------

@pytest.mark.parametrize("case", range(8))
def test_c_oracle_matches_python_twin(case):
    rng = np.random.default_rng(100 + case)
    Ho = Wo = 0
    while Ho <= 0 or Wo <= 0:             # redraw until the output is not empty
        kh, kw = int(rng.integers(1, 4)), int(rng.integers(1, 4))
        stride, dil = int(rng.integers(1, 3)), int(rng.integers(1, 3))
        pad = int(rng.integers(0, 3))
        G = int(rng.integers(1, 3))
        D = int(rng.integers(1, 3))
        N, H, W = 1, int(rng.integers(2, 6)), int(rng.integers(2, 6))
        Ho = scalar.out_size(H, kh, stride, pad, dil)
        Wo = scalar.out_size(W, kw, stride, pad, dil)
    C, K = G * D, kh * kw
    softmax_flag = case % 2
    x = rng.uniform(-1, 1, (N, H, W, C))
    off = rng.normal(0, 1.5, (N, Ho, Wo, G, K, 2))
    m = rng.normal(0, 1, (N, Ho, Wo, G, K))
    out = oracle.dcn_forward_ref(x, off, m, kh, kw, stride, pad, dil, softmax_flag)
    twin = np.array(scalar.dcn_forward_py(x.tolist(), off.tolist(), m.tolist(), kh, kw,
                                          stride, pad, dil, softmax_flag))
    assert np.allclose(out, twin, atol=1e-13, rtol=0)


def test_msda_c_oracle_matches_python_twin():
    shapes = [(3, 5), (2, 2)]
    starts = gen.level_start_index(shapes)
    N, M, D, K, Lq = 1, 2, 2, 2, 3
    S = sum(h * w for h, w in shapes)
    value = RNG.uniform(-1, 1, (N, S, M, D))
    loc = RNG.uniform(-0.2, 1.2, (N, Lq, M, 2, K, 2))
    attn = RNG.uniform(0, 1, (N, Lq, M, 2, K))
    out = oracle.msda_forward_ref(value, shapes, starts, loc, attn)
    for q in range(Lq):
        for h in range(M):
            for c in range(D):
                samples = []
                for l, (hh, ww) in enumerate(shapes):
                    grid = [[value[0, starts[l] + r * ww + cc, h, c] for cc in range(ww)]
                            for r in range(hh)]
                    samples.append([scalar.bilinear_normalized(grid, *loc[0, q, h, l, k])
                                    for k in range(K)])
                expect = scalar.aggregate(samples, attn[0, q, h].tolist())
                assert out[0, q, h * D + c] == pytest.approx(expect, abs=1e-13)


def test_sampling_location_helper():
    # point branch, valid ratio 1: s = p + dp / (W, H); (x, y) order
    s = scalar.sampling_location([0.5, 0.25], [3.0, -2.0], (150, 100))
    assert s == pytest.approx([0.5 + 3 / 150, 0.25 - 2 / 100])
    # and the generator places loc the same way (ref shared by heads/levels)
    w = gen.MsdaWorkload("t", N=1, M=1, D=1, shapes=((4, 8),), K=1, offset_sigma=0.0)
    inp = gen.msda_inputs(w, seed=3)
    loc = inp["loc"].double().numpy()
    assert np.all((loc >= 0) & (loc <= 1))           # zero offsets: loc = reference
