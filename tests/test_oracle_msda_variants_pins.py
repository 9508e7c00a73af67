"""Pins of the oracle's MSDA reference-point variants and value masking (no GPU).

The location loop of the C oracle is checked against closed forms the pages
fix: a box with zero offsets samples its centre, an offset of K points reaches
the box edge, a point with valid ratio 1 reduces to s = p + dp / (W, H), an
offset of one pixel moves the sample one pixel in that level, every image and
level takes its own ratio, and a reference on the valid-image edge lands half
a pixel inside the padding, so that a read there mixes the last valid value
with a masked zero.  Planted mistakes in the loop must fail one of these.  Masking is
checked against torch masked_fill followed by grid_sample (library routines).
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import gen
import oracle
from oracle import scalar

RNG = np.random.default_rng(41)


def location(ref, off, shape_hw, K, ratio=None):
    """One location of oracle.msda_locations_ref: a single image, query, head,
    level and point (the point index does not enter the formula, so the
    offset is placed at point 0 of K)."""
    rd = len(ref)
    offsets = np.zeros((1, 1, 1, 1, K, 2))
    offsets[0, 0, 0, 0, 0] = off
    vr = None if ratio is None else np.array(ratio, dtype=np.float64).reshape(1, 1, 2)
    loc = oracle.msda_locations_ref([shape_hw], np.array(ref, dtype=np.float64).reshape(1, 1, rd),
                                    offsets, vr)
    return loc[0, 0, 0, 0, 0].tolist()


def test_box_reference_closed_forms():
    ref = [0.4, 0.7, 0.2, 0.1]
    r = (0.8, 0.5)
    K = 4
    assert location(ref, [0.0, 0.0], (32, 64), K, r) == \
        pytest.approx([0.4 * 0.8, 0.7 * 0.5], abs=1e-15)
    # an offset of K points moves half the box size: the box's right / bottom edge
    s = location(ref, [K, K], (32, 64), K, r)
    assert s == pytest.approx([(0.4 + 0.1) * 0.8, (0.7 + 0.05) * 0.5], abs=1e-15)
    # box offsets do not depend on the level size
    assert location(ref, [1.0, -2.0], (9, 7), K, r) == \
        pytest.approx(location(ref, [1.0, -2.0], (5, 300), K, r), abs=0)


def test_point_reference_with_ratio_one_is_the_point_formula():
    for _ in range(20):
        ref = RNG.uniform(0, 1, 2).tolist()
        off = RNG.normal(0, 3, 2).tolist()
        hw = (int(RNG.integers(1, 200)), int(RNG.integers(1, 200)))
        assert location(ref, off, hw, 4) == \
            pytest.approx(scalar.sampling_location(ref, off, (hw[1], hw[0])), abs=1e-15)
        assert location(ref, off, hw, 4, (1.0, 1.0)) == location(ref, off, hw, 4)


def test_point_offset_of_one_pixel_moves_one_pixel():
    # dp = (1, 0) moves the sample one pixel right in that level's pixel grid,
    # dp = (0, 1) one pixel down, whatever the ratio (it scales the reference only)
    H, W = 25, 38
    ref = [0.3, 0.6]
    r = (0.75, 0.9)
    base = location(ref, [0.0, 0.0], (H, W), 4, r)
    right = location(ref, [1.0, 0.0], (H, W), 4, r)
    down = location(ref, [0.0, 1.0], (H, W), 4, r)
    assert (right[0] - base[0]) * W == pytest.approx(1.0, abs=1e-12)
    assert right[1] == base[1]
    assert (down[1] - base[1]) * H == pytest.approx(1.0, abs=1e-12)
    assert down[0] == base[0]
    assert base == pytest.approx([0.3 * 0.75, 0.6 * 0.9], abs=1e-15)


def test_each_image_and_level_uses_its_own_ratio():
    # two images, two levels: a zero offset lands on reference x ratio of
    # exactly that image and level, per axis
    N, L = 2, 2
    ref = np.array([[[0.5, 0.5]], [[0.25, 0.75]]])
    vr = np.array([[[1.0, 0.5], [0.8, 0.6]], [[0.7, 0.9], [0.4, 0.3]]])
    loc = oracle.msda_locations_ref([(4, 6), (2, 3)], ref, np.zeros((N, 1, 1, L, 1, 2)), vr)
    for n in range(N):
        for l in range(L):
            assert loc[n, 0, 0, l, 0].tolist() == pytest.approx(
                [ref[n, 0, 0] * vr[n, l, 0], ref[n, 0, 1] * vr[n, l, 1]], abs=1e-15)


def test_valid_edge_mixes_the_last_valid_value_with_a_masked_zero():
    H, W, Wv = 3, 8, 6                     # 6 valid columns, 2 padded
    value = np.zeros((1, H * W, 1, 1))
    value[0, :, 0, 0] = 1.0 + np.arange(H * W)
    mask = np.zeros((1, H * W), dtype=bool)
    mask[0, [y * W + x for y in range(H) for x in range(Wv, W)]] = True
    vr = np.array([[[Wv / W, 1.0]]])
    ref = np.array([[[1.0, 1.5 / H]]])     # the valid right edge, on row 1's centre
    off = np.zeros((1, 1, 1, 1, 1, 2))
    loc = oracle.msda_locations_ref([(H, W)], ref, off, vr)
    assert loc[0, 0, 0, 0, 0, 0] * W - 0.5 == pytest.approx(Wv - 0.5)
    out = oracle.msda_forward_ref(oracle.mask_value_ref(value, mask), [(H, W)], [0], loc,
                                  np.ones((1, 1, 1, 1, 1)))
    last_valid = value[0, 1 * W + Wv - 1, 0, 0]
    assert out[0, 0, 0] == pytest.approx(last_valid / 2.0, abs=1e-12)


def test_masked_values_match_masked_fill_and_grid_sample():
    w = gen.MsdaWorkload("pin", N=2, M=2, D=3, shapes=((5, 7), (3, 4)), K=3, Lq=6)
    inp = gen.msda_inputs(w, seed=2)
    mask = RNG.uniform(0, 1, (w.N, w.S)) < 0.3
    got = oracle.msda_forward_ref(oracle.mask_value_ref(inp["value"], mask),
                                  inp["spatial_shapes"], inp["level_start"], inp["loc"],
                                  inp["attn"])
    v = inp["value"].double().masked_fill(torch.tensor(mask)[:, :, None, None], 0.0)
    starts = gen.level_start_index(w.shapes)
    ref = torch.zeros(w.N, w.M, w.D, w.queries, dtype=torch.float64)
    loc = inp["loc"].double()
    attn = inp["attn"].double()
    for l, (h, wd) in enumerate(w.shapes):
        lvl = v[:, starts[l]:starts[l] + h * wd].permute(0, 2, 3, 1).reshape(w.N * w.M, w.D, h, wd)
        grid = (2 * loc[:, :, :, l] - 1).permute(0, 2, 1, 3, 4).reshape(w.N * w.M, w.queries, w.K, 2)
        s = F.grid_sample(lvl, grid, mode="bilinear", padding_mode="zeros", align_corners=False)
        a = attn[:, :, :, l].permute(0, 2, 1, 3).reshape(w.N * w.M, 1, w.queries, w.K)
        ref += (s * a).sum(-1).reshape(w.N, w.M, w.D, w.queries)
    ref = ref.permute(0, 3, 1, 2).reshape(w.N, w.queries, w.M * w.D).numpy()
    assert np.allclose(got, ref, rtol=0, atol=1e-12)


def test_locations_of_every_index_follow_the_formula():
    # the loop nest indexes every (n, q, m, l, k) with its own offset and the
    # reference of its (n, q): compared element by element with numpy broadcasting
    N, Lq, M, L, K = 2, 3, 2, 2, 3
    shapes = [(6, 9), (3, 5)]
    wh = np.array([[w, h] for h, w in shapes], dtype=np.float64)          # [L, 2]
    for rd in (2, 4):
        ref = RNG.uniform(0, 1, (N, Lq, rd))
        off = RNG.normal(0, 2, (N, Lq, M, L, K, 2))
        vr = RNG.uniform(0.5, 1, (N, L, 2))
        loc = oracle.msda_locations_ref(shapes, ref, off, vr)
        r = vr[:, None, None, :, None, :]
        centre = ref[:, :, None, None, None, :2] * r
        if rd == 2:
            expect = centre + off / wh[None, None, None, :, None, :]
        else:
            expect = centre + off / K * ref[:, :, None, None, None, 2:] * r / 2
        assert np.allclose(loc, expect, rtol=0, atol=1e-15)


# planted mistakes in the C location loop: each must fail one of the pins above
LOCATION_MUTANTS = {
    "point centre not scaled by the ratio": ("u = ref[0] * ratio_x + dx / level_w;",
                                             "u = ref[0] + dx / level_w;"),
    "box centre not scaled by the ratio": ("u = ref[0] * ratio_x + (dx / (double)K)",
                                           "u = ref[0] + (dx / (double)K)"),
    "box half size missing": ("* ref[2] * ratio_x / 2.0;", "* ref[2] * ratio_x;"),
    "box sizes swapped": ("* ref[2] * ratio_x / 2.0;", "* ref[3] * ratio_x / 2.0;"),
    "point offset over the height": ("u = ref[0] * ratio_x + dx / level_w;",
                                     "u = ref[0] * ratio_x + dx / level_h;"),
    "ratio of the wrong axis": ("double ratio_y = valid_ratios ? valid_ratios[(n * L + l) * 2 + 1]",
                                "double ratio_y = valid_ratios ? valid_ratios[(n * L + l) * 2]"),
    "ratio of the wrong image": ("double ratio_x = valid_ratios ? valid_ratios[(n * L + l) * 2]",
                                 "double ratio_x = valid_ratios ? valid_ratios[l * 2]"),
    "box offset not divided by K": ("(dy / (double)K) * ref[3]", "dy * ref[3]"),
}

LOCATION_PINS = [test_box_reference_closed_forms,
                 test_point_reference_with_ratio_one_is_the_point_formula,
                 test_point_offset_of_one_pixel_moves_one_pixel,
                 test_each_image_and_level_uses_its_own_ratio,
                 test_valid_edge_mixes_the_last_valid_value_with_a_masked_zero,
                 test_locations_of_every_index_follow_the_formula]


def test_real_location_loop_passes_its_pins():
    for pin in LOCATION_PINS:
        pin()


@pytest.mark.parametrize("name", sorted(LOCATION_MUTANTS))
def test_planted_location_mistakes_are_caught(name, tmp_path, monkeypatch):
    import ctypes

    from oracle import build as oracle_build
    original, planted = LOCATION_MUTANTS[name]
    src = open(oracle_build.SRC).read()
    assert src.count(original) >= 1, f"mutation site not found: {original}"
    mutant_src = tmp_path / "mutant.c"
    mutant_src.write_text(src.replace(original, planted, 1))
    lib_path = oracle_build.compile_oracle(str(mutant_src), str(tmp_path / "libmutant.so"),
                                           extra_flags=("-Wno-error",))
    monkeypatch.setattr(oracle, "_lib", oracle.bind(ctypes.CDLL(lib_path)))
    caught = 0
    for pin in LOCATION_PINS:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught > 0, f"no location pin caught the mutant '{name}'"
