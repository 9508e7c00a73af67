"""The oracle's pins catch plausible mistakes (no GPU).

Each mutant is a copy of the C oracle with one planted mistake: a dropped
term, a wrong sign, index or bound, a transposed operand.  It is compiled into
a temporary library, swapped in for the real one, and the pin battery of
test_oracle_pins is run against it: every mutant must fail at least one pin.
Mistakes planted in the backward functions face the battery of
test_oracle_backward_pins (adjoint identity, finite differences).
The real oracle source is never modified.
"""
import ctypes
import inspect
import os

import pytest

import oracle
from oracle import build as oracle_build
from tests import test_oracle_backward_pins as bwd
from tests import test_oracle_dynconv_pins as dyn
from tests import test_oracle_pins as pins
from tests.conftest import read_golden

MUTANTS = {
    "corner weight x swapped": ("double wx = (i == 0) ? (1.0 - a) : a;",
                                "double wx = (i == 0) ? a : (1.0 - a);"),
    "row weight dropped": ("total += wx * wy * map[idx];", "total += wx * map[idx];"),
    "dx and dy swapped": ("+ off[2 * k];", "+ off[2 * k + 1];"),
    "tap order transposed": ("long k = ix * kh + iy;", "long k = iy * kw + ix;"),
    "upper x bound off by one": ("xx < (double)W", "xx <= (double)W"),
    "truncation instead of floor": ("double x0 = floor(px);", "double x0 = (double)(long)px;"),
    "group channel offset": ("const double *xg = x + n * H * W * C + g * D;",
                             "const double *xg = x + n * H * W * C + g;"),
    "group offsets ignored": ("long site = ((n * Ho + oy) * Wo + ox) * G + g;",
                              "long site = ((n * Ho + oy) * Wo + ox) * G;"),
    "softmax not normalised": ("m[k] = m[k] / sum;", "m[k] = m[k];"),
    "softmax flag inverted": ("if (softmax_flag) {", "if (!softmax_flag) {"),
    "pad sign": ("(double)(ox * stride - pad + ix * dil)", "(double)(ox * stride + pad + ix * dil)"),
    "dilation ignored in y": ("(double)(oy * stride - pad + iy * dil)", "(double)(oy * stride - pad + iy)"),
    "msda half-pixel shift dropped": ("double x = u * (double)W - 0.5;", "double x = u * (double)W;"),
    "msda tent weight sign": ("(1.0 - fabs(y - row))", "(1.0 + fabs(y - row))"),
    "msda shapes read as (W, H)": ("long Hl = (long)shapes[2 * l];", "long Hl = (long)shapes[2 * l + 1];"),
    "msda level start ignored": ("(n * S + (long)level_start[l]) * M", "(n * S) * M"),
    "msda attention weight dropped": ("acc += attn[t] * sample_level(", "acc += 1.0 * sample_level("),
    "msda head stride": ("+ h) * D;", ") * D;"),
}

# mistakes planted in the backward functions, caught by the backward pins
MUTANTS_BWD = {
    "dcn d/dx drops (1-b)": ("gdx += go[c] * m[k] * ((1 - b) * (v01 - v00)",
                             "gdx += go[c] * m[k] * ((v01 - v00)"),
    "dcn d/dy uses the x difference": ("gdy += go[c] * m[k] * ((1 - a) * (v10 - v00)",
                                       "gdy += go[c] * m[k] * ((1 - a) * (v01 - v00)"),
    "dcn grad_x corner swapped": ("corner_add(gxg, H, W, C, c, x0 + 1, y0, gm_c * a * (1 - b));",
                                  "corner_add(gxg, H, W, C, c, x0, y0 + 1, gm_c * a * (1 - b));"),
    "dcn grad_x misses m": ("double gm_c = go[c] * m[k];", "double gm_c = go[c];"),
    "dcn softmax jacobian sign": ("gmsk[k] = m[k] * (gm[k] - dot);", "gmsk[k] = m[k] * (gm[k] + dot);"),
    "dcn grad_mask of the sample": ("gmk += go[c] * sample;", "gmk += go[c] * v00;"),
    "msda grad_loc misses W": ("* ((1 - b) * (v01 - v00) + b * (v11 - v10)) * Wl;",
                               "* ((1 - b) * (v01 - v00) + b * (v11 - v10));"),
    "msda grad_value misses A": ("double ga = go * A;", "double ga = go;"),
    "msda grad_attn": ("grad_attn[t] += go * sample;", "grad_attn[t] += sample;"),
}

# mistakes planted in the dynamic local aggregation (ContMix core)
MUTANTS_DYN = {
    "dyn taps column-major": ("acc += A[ky * K + kx] * x[", "acc += A[kx * K + ky] * x["),
    "dyn window not centred": ("long sy = y + ky - r, sx = xx + kx - r;",
                               "long sy = y + ky - r, sx = xx + kx;"),
    "dyn softmax not normalised": ("A[t] = A[t] / sum;", "A[t] = A[t];"),
    "dyn group channel offset": ("* C + g * D + c];\n            }", "* C + c];\n            }"),
    "dyn lower bound off by one": ("if (sy < 0 || sy >= H || sx < 0 || sx >= W)",
                                   "if (sy < 0 || sy >= H || sx < 1 || sx >= W)"),
    "dyn weights of the wrong group": ("const double *wt = w + (((n * H + y) * W + xx) * G + g) * KK;",
                                       "const double *wt = w + (((n * H + y) * W + xx) * G) * KK;"),
}

PIN_TESTS_DYN = [
    (dyn.test_matches_unfold_formulation, [dict(case=c) for c in dyn.CASES[:3]]),
    (dyn.test_one_hot_weights_copy_a_shifted_map, [{}]),
    (dyn.test_equal_logits_give_the_zero_padded_box_mean, [dict(K=3)]),
]

PIN_TESTS_BWD = [
    (bwd.test_dcn_grad_x_is_the_adjoint, [dict(case=c) for c in bwd.DCN_CASES[:2]]),
    (bwd.test_dcn_offset_and_mask_gradients_match_finite_differences,
     [dict(case=c) for c in bwd.DCN_CASES[:2]]),
    (bwd.test_msda_grad_value_is_the_adjoint, [{}]),
    (bwd.test_msda_loc_and_attn_gradients_match_finite_differences, [{}]),
]

PIN_TESTS = [
    (pins.test_bilinear_worked_example, [{}]),
    (pins.test_spike_1d, [{}]),
    (pins.test_dcnv3_softmax_worked_example, [{}]),
    (pins.test_right_minus_left_unbounded, [{}]),
    (pins.test_msda_corner_quarter, [{}]),
    (pins.test_bilinear_weights_sum_and_convex_hull, [{}]),
    (pins.test_constant_map_softmax_and_unbounded, [{}]),
    (pins.test_edge_straddle_and_far_outside, [{}]),
    (pins.test_identity_zero_offsets_k1, [{}]),
    (pins.test_zero_offsets_match_grouped_conv,
     [dict(kh=3, kw=3, stride=1, pad=1, dil=1, H=7, W=9),
      dict(kh=3, kw=1, stride=2, pad=0, dil=3, H=9, W=4),
      dict(kh=2, kw=3, stride=1, pad=1, dil=1, H=5, W=5)]),
    (pins.test_integer_offsets_are_a_shifted_gather, [{}]),
    (pins.test_bilinear_matches_grid_sample, [{}]),
    (pins.test_groups_use_their_own_offsets_and_masks, [{}]),
    (pins.test_msda_matches_grid_sample, [{}]),
    (pins.test_msda_pixel_centres_read_the_value, [{}]),
    (pins.test_dcn_and_msda_bilinear_forms_agree, [{}]),
]


def _failures(battery=PIN_TESTS):
    failed = []
    for fn, param_sets in battery:
        for params in param_sets:
            kwargs = dict(params)
            if "golden" in inspect.signature(fn).parameters:
                kwargs["golden"] = read_golden
            try:
                fn(**kwargs)
            except (AssertionError, ValueError):
                failed.append(fn.__name__)
    return failed


def test_real_oracle_passes_the_battery():
    assert _failures() == []
    assert _failures(PIN_TESTS_BWD) == []
    assert _failures(PIN_TESTS_DYN) == []


def _install_mutant(original, planted, tmp_path, monkeypatch):
    src = open(oracle_build.SRC).read()
    assert src.count(original) >= 1, f"mutation site not found: {original}"
    mutant_src = tmp_path / "mutant.c"
    mutant_src.write_text(src.replace(original, planted, 1))
    lib_path = oracle_build.compile_oracle(str(mutant_src), str(tmp_path / "libmutant.so"),
                                           extra_flags=("-Wno-error",))
    monkeypatch.setattr(oracle, "_lib", oracle.bind(ctypes.CDLL(lib_path)))


@pytest.mark.parametrize("name", sorted(MUTANTS_BWD))
def test_backward_mutant_is_caught(name, tmp_path, monkeypatch):
    _install_mutant(*MUTANTS_BWD[name], tmp_path, monkeypatch)
    assert _failures(PIN_TESTS_BWD), f"no backward pin caught the mutant '{name}'"


@pytest.mark.parametrize("name", sorted(MUTANTS_DYN))
def test_dynconv_mutant_is_caught(name, tmp_path, monkeypatch):
    _install_mutant(*MUTANTS_DYN[name], tmp_path, monkeypatch)
    assert _failures(PIN_TESTS_DYN), f"no dynamic-kernel pin caught the mutant '{name}'"


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path, monkeypatch):
    original, planted = MUTANTS[name]
    src = open(oracle_build.SRC).read()
    assert src.count(original) >= 1, f"mutation site not found: {original}"
    mutant_src = tmp_path / "mutant.c"
    mutant_src.write_text(src.replace(original, planted, 1))
    lib_path = oracle_build.compile_oracle(str(mutant_src), str(tmp_path / "libmutant.so"),
                                           extra_flags=("-Wno-error",))
    monkeypatch.setattr(oracle, "_lib", oracle.bind(ctypes.CDLL(lib_path)))
    assert _failures(), f"no pin caught the mutant '{name}'"
