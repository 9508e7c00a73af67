"""Pins of the oracle's DCNv4 front end (merged offset / mask linear feeding
the sampling core; no GPU): the linear part against an explicit per-pixel
sum, the split of its outputs against the core's layouts, and special cases
that reduce to the core alone."""
import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(53)


def _problem(N=1, H=5, W=6, C=8, G=2, k=3):
    K = k * k
    x = RNG.uniform(-1, 1, (N, H, W, C))
    w = RNG.normal(0, 0.3, (G * K * 3, C))
    b = RNG.normal(0, 0.5, G * K * 3)
    return x, w, b


def test_linear_outputs_and_their_split():
    x, w, b = _problem()
    G, K = 2, 9
    _, off, mask = oracle.dcnv4_front_end_ref(x, w, b, 3, 3, 1, 1, G)
    n, y, xx = 0, 3, 4
    om = [sum(w[j, c] * x[n, y, xx, c] for c in range(x.shape[3])) + b[j] for j in range(G * K * 3)]
    for g in range(G):
        for k in range(K):
            assert off[n, y, xx, g, k, 0] == pytest.approx(om[(g * K + k) * 2], abs=1e-13)
            assert off[n, y, xx, g, k, 1] == pytest.approx(om[(g * K + k) * 2 + 1], abs=1e-13)
            assert mask[n, y, xx, g, k] == pytest.approx(om[G * K * 2 + g * K + k], abs=1e-13)


def test_zero_offset_rows_reduce_to_the_core_with_constant_masks():
    x, w, b = _problem(C=6, G=3)
    G, K = 3, 9
    w[:] = 0.0
    b[:G * K * 2] = 0.0                        # zero offsets
    out, off, mask = oracle.dcnv4_front_end_ref(x, w, b, 3, 3, 1, 1, G)
    assert np.all(off == 0.0)
    expect = oracle.dcn_forward_ref(x, np.zeros_like(off), np.broadcast_to(b[G * K * 2:].reshape(G, K), mask.shape),
                                    3, 3, 1, 1, 1, 0, groups=G)
    assert np.allclose(out, expect, rtol=0, atol=1e-13)


def test_output_is_the_core_on_the_linear_outputs():
    x, w, b = _problem(N=2, H=4, W=7, C=8, G=2)
    out, off, mask = oracle.dcnv4_front_end_ref(x, w, b, 3, 3, 1, 1, 2)
    assert np.array_equal(out, oracle.dcn_forward_ref(x, off, mask, 3, 3, 1, 1, 1, 0, groups=2))
