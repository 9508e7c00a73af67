"""Pins of the oracle's backward (no GPU).

The gradients are checked against things other than the backward code:
- the adjoint identity: out is linear in x (in value), so
  <forward(x), g> = <x, grad_x(g)> exactly (up to float64 rounding);
- central finite differences of the forward oracle, for offsets, masks,
  DCNv3 logits, MSDA locations and weights (fractional parts kept away from
  integers, where bilinear interpolation has kinks);
- torch autograd through CPU float64 grid_sample (a library routine).
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import gen
import oracle

RNG = np.random.default_rng(77)


def _frac_offsets(shape, spread):
    """Offsets whose sampling points sit at least 0.1 px from integers."""
    base = RNG.integers(-spread, spread + 1, shape).astype(np.float64)
    frac = RNG.uniform(0.1, 0.9, shape)
    return base + frac


DCN_CASES = [
    # N, H, W, C, G, kh, kw, stride, pad, dil, softmax
    (1, 5, 6, 4, 2, 3, 3, 1, 1, 1, 0),
    (2, 6, 5, 6, 3, 3, 3, 1, 1, 1, 1),
    (1, 7, 8, 4, 1, 3, 3, 2, 1, 1, 0),
    (1, 6, 6, 2, 2, 2, 3, 1, 2, 2, 1),
]


def _dcn_problem(case):
    N, H, W, C, G, kh, kw, stride, pad, dil, sm = case
    Ho = oracle.out_size(H, kh, stride, pad, dil)
    Wo = oracle.out_size(W, kw, stride, pad, dil)
    K = kh * kw
    x = RNG.uniform(-1, 1, (N, H, W, C))
    off = _frac_offsets((N, Ho, Wo, G, K, 2), 3)
    mask = RNG.normal(0, 1, (N, Ho, Wo, G, K))
    g = RNG.normal(0, 1, (N, Ho, Wo, C))
    return x, off, mask, g, dict(kh=kh, kw=kw, stride=stride, pad=pad, dil=dil,
                                 softmax_flag=sm)


@pytest.mark.parametrize("case", DCN_CASES)
def test_dcn_grad_x_is_the_adjoint(case):
    x, off, mask, g, kw_ = _dcn_problem(case)
    out = oracle.dcn_forward_ref(x, off, mask, **kw_)
    gx, _, _ = oracle.dcn_backward_ref(x, off, mask, g, **kw_)
    lhs = float(np.sum(out * g))
    rhs = float(np.sum(x * gx))
    assert lhs == pytest.approx(rhs, rel=1e-12, abs=1e-12)
    # and per basis vector: grad_x of a one-hot upstream gradient is the
    # column of the (linear) forward map
    e = np.zeros_like(g)
    e.flat[RNG.integers(0, e.size)] = 1.0
    gx_e, _, _ = oracle.dcn_backward_ref(x, off, mask, e, **kw_)
    for _ in range(5):
        probe = np.zeros_like(x)
        probe.flat[RNG.integers(0, x.size)] = 1.0
        assert float(np.sum(oracle.dcn_forward_ref(probe, off, mask, **kw_) * e)) == \
            pytest.approx(float(np.sum(probe * gx_e)), abs=1e-13)


@pytest.mark.parametrize("case", DCN_CASES)
def test_dcn_offset_and_mask_gradients_match_finite_differences(case):
    x, off, mask, g, kw_ = _dcn_problem(case)
    _, goff, gmask = oracle.dcn_backward_ref(x, off, mask, g, **kw_)
    loss = lambda o, m: float(np.sum(oracle.dcn_forward_ref(x, o, m, **kw_) * g))
    h = 1e-6
    for _ in range(12):
        i = RNG.integers(0, off.size)
        p, q = off.copy(), off.copy()
        p.flat[i] += h
        q.flat[i] -= h
        fd = (loss(p, mask) - loss(q, mask)) / (2 * h)
        assert goff.flat[i] == pytest.approx(fd, rel=1e-5, abs=1e-7)
        j = RNG.integers(0, mask.size)
        p, q = mask.copy(), mask.copy()
        p.flat[j] += h
        q.flat[j] -= h
        fd = (loss(off, p) - loss(off, q)) / (2 * h)
        assert gmask.flat[j] == pytest.approx(fd, rel=1e-5, abs=1e-7)


def _dcn_torch(x, off, mask, kh, kw, stride, pad, dil, softmax_flag):
    """DCN as a sum over taps of grid_sample (float64 autograd graph)."""
    N, H, W, C = x.shape
    _, Ho, Wo, G, K, _ = off.shape
    D = C // G
    xt = x.permute(0, 3, 1, 2).reshape(N * G, D, H, W)
    m = torch.softmax(mask, dim=-1) if softmax_flag else mask
    oy = torch.arange(Ho, dtype=torch.float64)[:, None] * stride - pad
    ox = torch.arange(Wo, dtype=torch.float64)[None, :] * stride - pad
    out = 0
    for ix in range(kw):
        for iy in range(kh):
            k = ix * kh + iy
            px = ox + ix * dil + off[..., k, 0].permute(0, 3, 1, 2)   # N, G, Ho, Wo
            py = oy + iy * dil + off[..., k, 1].permute(0, 3, 1, 2)
            grid = torch.stack([(2 * px + 1) / W - 1, (2 * py + 1) / H - 1], -1)
            s = F.grid_sample(xt, grid.reshape(N * G, Ho, Wo, 2), mode="bilinear",
                              padding_mode="zeros", align_corners=False)   # N*G, D, Ho, Wo
            mk = m[..., k].permute(0, 3, 1, 2).reshape(N * G, 1, Ho, Wo)
            out = out + s * mk
    return out.reshape(N, G * D, Ho, Wo).permute(0, 2, 3, 1)


@pytest.mark.parametrize("case", DCN_CASES)
def test_dcn_backward_matches_autograd_through_grid_sample(case):
    x, off, mask, g, kw_ = _dcn_problem(case)
    xt = torch.tensor(x, requires_grad=True)
    ot = torch.tensor(off, requires_grad=True)
    mt = torch.tensor(mask, requires_grad=True)
    out = _dcn_torch(xt, ot, mt, **kw_)
    assert np.allclose(out.detach().numpy(), oracle.dcn_forward_ref(x, off, mask, **kw_),
                       atol=1e-13)
    out.backward(torch.tensor(g))
    gx, goff, gmask = oracle.dcn_backward_ref(x, off, mask, g, **kw_)
    assert np.allclose(gx, xt.grad.numpy(), atol=1e-12)
    assert np.allclose(goff, ot.grad.numpy(), atol=1e-12)
    assert np.allclose(gmask, mt.grad.numpy(), atol=1e-12)


def _msda_problem(seed=0):
    rng = np.random.default_rng(seed)
    shapes = [(5, 7), (3, 4), (2, 3)]
    starts = gen.level_start_index(shapes)
    N, M, D, K, Lq = 2, 2, 3, 2, 5
    S = sum(h * w for h, w in shapes)
    value = rng.uniform(-1, 1, (N, S, M, D))
    loc = np.zeros((N, Lq, M, len(shapes), K, 2))
    for l, (h, w) in enumerate(shapes):
        px = rng.integers(-2, w + 1, (N, Lq, M, K)) + rng.uniform(0.1, 0.9, (N, Lq, M, K))
        py = rng.integers(-2, h + 1, (N, Lq, M, K)) + rng.uniform(0.1, 0.9, (N, Lq, M, K))
        loc[:, :, :, l, :, 0] = (px + 0.5) / w
        loc[:, :, :, l, :, 1] = (py + 0.5) / h
    attn = rng.uniform(0, 1, (N, Lq, M, len(shapes), K))
    g = rng.normal(0, 1, (N, Lq, M * D))
    return value, shapes, starts, loc, attn, g


def test_msda_grad_value_is_the_adjoint():
    value, shapes, starts, loc, attn, g = _msda_problem(1)
    out = oracle.msda_forward_ref(value, shapes, starts, loc, attn)
    gv, _, _ = oracle.msda_backward_ref(value, shapes, starts, loc, attn, g)
    assert float(np.sum(out * g)) == pytest.approx(float(np.sum(value * gv)), rel=1e-12)


def test_msda_loc_and_attn_gradients_match_finite_differences():
    value, shapes, starts, loc, attn, g = _msda_problem(2)
    _, gl, ga = oracle.msda_backward_ref(value, shapes, starts, loc, attn, g)
    loss = lambda lo, at: float(np.sum(oracle.msda_forward_ref(value, shapes, starts, lo, at) * g))
    h = 1e-7
    for _ in range(12):
        i = RNG.integers(0, loc.size)
        p, q = loc.copy(), loc.copy()
        p.flat[i] += h
        q.flat[i] -= h
        assert gl.flat[i] == pytest.approx((loss(p, attn) - loss(q, attn)) / (2 * h),
                                           rel=1e-5, abs=1e-6)
        j = RNG.integers(0, attn.size)
        p, q = attn.copy(), attn.copy()
        p.flat[j] += h
        q.flat[j] -= h
        assert ga.flat[j] == pytest.approx((loss(loc, p) - loss(loc, q)) / (2 * h),
                                           rel=1e-5, abs=1e-6)


def test_msda_backward_matches_autograd_through_grid_sample():
    value, shapes, starts, loc, attn, g = _msda_problem(3)
    N, S, M, D = value.shape
    _, Lq, _, L, K, _ = loc.shape
    vt = torch.tensor(value, requires_grad=True)
    lt = torch.tensor(loc, requires_grad=True)
    at = torch.tensor(attn, requires_grad=True)
    out = torch.zeros(N, M, D, Lq, dtype=torch.float64)
    for l, (h, w) in enumerate(shapes):
        lvl = vt[:, starts[l]:starts[l] + h * w].permute(0, 2, 3, 1).reshape(N * M, D, h, w)
        grid = (2 * lt[:, :, :, l] - 1).permute(0, 2, 1, 3, 4).reshape(N * M, Lq, K, 2)
        s = F.grid_sample(lvl, grid, mode="bilinear", padding_mode="zeros",
                          align_corners=False)
        a = at[:, :, :, l].permute(0, 2, 1, 3).reshape(N * M, 1, Lq, K)
        out = out + (s * a).sum(-1).reshape(N, M, D, Lq)
    out = out.permute(0, 3, 1, 2).reshape(N, Lq, M * D)
    out.backward(torch.tensor(g))
    gv, gl, ga = oracle.msda_backward_ref(value, shapes, starts, loc, attn, g)
    assert np.allclose(gv, vt.grad.numpy(), atol=1e-12)
    assert np.allclose(gl, lt.grad.numpy(), atol=1e-10)
    assert np.allclose(ga, at.grad.numpy(), atol=1e-12)
