"""Structure of the seeded MSDA inputs (host only).

Encoder-style workloads (one query per cell of every level) reference each
query at its own cell centre, as the Deformable DETR page states for the
encoder; other query sets draw reference points uniformly.
"""
import dataclasses

import numpy as np
import pytest

import gen

SHAPES = ((4, 6), (2, 3), (1, 2))


def small(**kw):
    return gen.MsdaWorkload("t", N=2, M=2, D=4, shapes=SHAPES, K=2, **kw)


def test_centres_follow_the_value_row_order():
    c = gen.msda_centres(SHAPES)
    assert c.shape == (24 + 6 + 2, 2)
    assert np.allclose(c[0], [0.5 / 6, 0.5 / 4])
    assert np.allclose(c[1], [1.5 / 6, 0.5 / 4])          # next column of row 0
    assert np.allclose(c[6], [0.5 / 6, 1.5 / 4])          # row 1 of level 0
    assert np.allclose(c[24], [0.5 / 3, 0.5 / 2])         # first cell of level 1
    assert np.allclose(c[-1], [1.5 / 2, 0.5 / 1])         # last cell of level 2
    assert ((c > 0) & (c < 1)).all()


def offsets_of(w, inp, rng_seed):
    """The pixel offsets msda_inputs drew (the same stream in every mode)."""
    rng = np.random.default_rng(rng_seed)
    rng.uniform(-1.0, 1.0, size=(w.N, w.S, w.M, w.D))
    rng.uniform(0.0, 1.0, size=(w.N, w.queries, 2))
    return rng.normal(0.0, w.offset_sigma, size=(w.N, w.queries, w.M, w.L, w.K, 2))


def test_encoder_queries_sample_around_their_own_cell():
    w = small()
    inp = gen.msda_inputs(w, seed=3)
    size_wh = np.array([[wd, h] for h, wd in SHAPES], dtype=np.float64)
    ref = inp["loc"].numpy() - offsets_of(w, inp, 3) / size_wh[None, None, None, :, None, :]
    centres = gen.msda_centres(SHAPES)
    for n in range(w.N):
        for m in range(w.M):
            for lvl in range(w.L):
                for k in range(w.K):
                    assert np.allclose(ref[n, :, m, lvl, k], centres, atol=1e-6)


def test_uniform_mode_keeps_every_other_tensor():
    w = small()
    u = dataclasses.replace(w, ref_points="uniform")
    a, b = gen.msda_inputs(w, seed=5), gen.msda_inputs(u, seed=5)
    for key in ("value", "attn"):
        assert np.array_equal(a[key].numpy(), b[key].numpy())
    assert not np.allclose(a["loc"].numpy(), b["loc"].numpy())


def test_explicit_query_count_draws_uniform_references_and_cells_need_every_cell():
    w = small(Lq=5)
    assert gen.msda_inputs(w, seed=1)["loc"].shape[1] == 5
    with pytest.raises(ValueError):
        gen.msda_inputs(small(Lq=5, ref_points="cell"), seed=1)
    with pytest.raises(ValueError):
        gen.msda_inputs(small(ref_points="grid"), seed=1)
