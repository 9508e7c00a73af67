"""Pins of the oracle's MSDA reference-point variants and value masking (no GPU).

The location mapping is checked against closed forms the pages fix: a box
with zero offsets samples its centre, an offset of K points reaches the box
edge, a point with valid ratio 1 reduces to the plain point helper, and a
reference on the valid-image edge lands half a pixel inside the padding, so
that a read there mixes the last valid value with a masked zero.  Masking is
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


def test_box_reference_closed_forms():
    ref = [0.4, 0.7, 0.2, 0.1]
    r = (0.8, 0.5)
    K = 4
    assert scalar.sampling_location_ref(ref, [0.0, 0.0], (64, 32), K, r) == \
        pytest.approx([0.4 * 0.8, 0.7 * 0.5], abs=1e-15)
    # an offset of K points moves half the box size: the box's right / bottom edge
    s = scalar.sampling_location_ref(ref, [K, K], (64, 32), K, r)
    assert s == pytest.approx([(0.4 + 0.1) * 0.8, (0.7 + 0.05) * 0.5], abs=1e-15)
    # box offsets do not depend on the level size
    assert scalar.sampling_location_ref(ref, [1.0, -2.0], (7, 9), K, r) == \
        pytest.approx(scalar.sampling_location_ref(ref, [1.0, -2.0], (300, 5), K, r), abs=0)


def test_point_reference_with_ratio_one_is_the_point_helper():
    for _ in range(20):
        ref = RNG.uniform(0, 1, 2).tolist()
        off = RNG.normal(0, 3, 2).tolist()
        wh = (int(RNG.integers(1, 200)), int(RNG.integers(1, 200)))
        assert scalar.sampling_location_ref(ref, off, wh, 4) == \
            pytest.approx(scalar.sampling_location(ref, off, wh), abs=1e-15)


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


def test_vectorised_locations_follow_the_helper():
    N, Lq, M, L, K = 2, 3, 2, 2, 3
    shapes = [(6, 9), (3, 5)]
    for rd in (2, 4):
        ref = RNG.uniform(0, 1, (N, Lq, rd))
        off = RNG.normal(0, 2, (N, Lq, M, L, K, 2))
        vr = RNG.uniform(0.5, 1, (N, L, 2))
        loc = oracle.msda_locations_ref(shapes, ref, off, vr)
        n, q, m, l, k = 1, 2, 1, 1, 2
        wh = (shapes[l][1], shapes[l][0])
        assert loc[n, q, m, l, k].tolist() == pytest.approx(
            scalar.sampling_location_ref(ref[n, q], off[n, q, m, l, k], wh, K, vr[n, l]),
            abs=1e-15)
        if rd == 2:   # written out: r * p + offset / size
            assert loc[n, q, m, l, k, 0] == pytest.approx(
                ref[n, q, 0] * vr[n, l, 0] + off[n, q, m, l, k, 0] / wh[0], abs=1e-15)
        else:         # r * (c + offset / K * size / 2)
            assert loc[n, q, m, l, k, 1] == pytest.approx(
                vr[n, l, 1] * (ref[n, q, 1] + off[n, q, m, l, k, 1] / K * ref[n, q, 3] / 2),
                abs=1e-15)


# planted mistakes in the location helper: each must fail one of the pins above
def _m_centre_unscaled(reference, offset, shape_wh, points, valid_ratio=(1.0, 1.0)):
    out = []
    for axis in range(2):
        shift = (offset[axis] / points * reference[axis + 2] * valid_ratio[axis] / 2.0
                 if len(reference) == 4 else offset[axis] / shape_wh[axis])
        out.append(reference[axis] + shift)
    return out


def _m_box_half_missing(reference, offset, shape_wh, points, valid_ratio=(1.0, 1.0)):
    out = []
    for axis in range(2):
        shift = (offset[axis] / points * reference[axis + 2] * valid_ratio[axis]
                 if len(reference) == 4 else offset[axis] / shape_wh[axis])
        out.append(reference[axis] * valid_ratio[axis] + shift)
    return out


def _m_box_sizes_swapped(reference, offset, shape_wh, points, valid_ratio=(1.0, 1.0)):
    out = []
    for axis in range(2):
        shift = (offset[axis] / points * reference[3 - axis] * valid_ratio[axis] / 2.0
                 if len(reference) == 4 else offset[axis] / shape_wh[axis])
        out.append(reference[axis] * valid_ratio[axis] + shift)
    return out


def _m_point_shape_swapped(reference, offset, shape_wh, points, valid_ratio=(1.0, 1.0)):
    out = []
    for axis in range(2):
        shift = (offset[axis] / points * reference[axis + 2] * valid_ratio[axis] / 2.0
                 if len(reference) == 4 else offset[axis] / shape_wh[1 - axis])
        out.append(reference[axis] * valid_ratio[axis] + shift)
    return out


@pytest.mark.parametrize("mutant", [_m_centre_unscaled, _m_box_half_missing,
                                    _m_box_sizes_swapped, _m_point_shape_swapped])
def test_planted_location_mistakes_are_caught(mutant, monkeypatch):
    monkeypatch.setattr(scalar, "sampling_location_ref", mutant)
    pins = [test_box_reference_closed_forms, test_point_reference_with_ratio_one_is_the_point_helper,
            test_valid_edge_mixes_the_last_valid_value_with_a_masked_zero,
            test_vectorised_locations_follow_the_helper]
    caught = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught > 0
