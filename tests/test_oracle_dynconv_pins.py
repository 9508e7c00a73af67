"""Pins of the oracle's dynamic local aggregation (the ContMix core; no GPU).

Checked against things other than the function itself:
- torch unfold (a library routine): the K x K zero-padded neighbourhoods of
  every location, multiplied by the location's softmaxed weights and summed,
  as the OverLoCK note's ContMix steps 4-5 describe;
- the DCN oracle (pinned on its own) with all offsets zero, the same window
  and its own tap order: the dynamic kernel is a zero-offset DCNv3 / DCNv4;
- closed forms: one-hot weights copy a shifted map, equal logits give the
  zero-padded box mean (torch avg_pool2d counting the padding), adding a
  constant to every logit changes nothing, and the output is linear in x.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

RNG = np.random.default_rng(31)

CASES = [
    # N, H, W, C, G, K, softmax
    (1, 5, 6, 4, 2, 3, 1),
    (2, 7, 4, 6, 3, 5, 1),
    (1, 6, 9, 8, 1, 7, 0),
    (1, 3, 3, 2, 2, 5, 1),      # window larger than the map
    (2, 4, 5, 3, 3, 1, 0),      # K = 1: a per-pixel, per-group scale
]


def _problem(case):
    N, H, W, C, G, K, sm = case
    x = RNG.uniform(-1, 1, (N, H, W, C))
    w = RNG.normal(0, 1, (N, H, W, G, K * K))
    return x, w


def _unfold_reference(x, w, K, softmax_flag):
    """ContMix steps 4-5 with library routines, float64."""
    N, H, W, C = x.shape
    G = w.shape[3]
    D = C // G
    xt = torch.tensor(x).permute(0, 3, 1, 2)                       # N, C, H, W
    A = torch.tensor(w)
    if softmax_flag:
        A = torch.softmax(A, dim=-1)
    out = torch.zeros(N, C, H * W, dtype=torch.float64)
    for g in range(G):
        patches = F.unfold(xt[:, g * D:(g + 1) * D], K, padding=K // 2)   # N, D*K*K, H*W
        patches = patches.view(N, D, K * K, H * W)
        a = A[:, :, :, g, :].reshape(N, H * W, K * K).transpose(1, 2)  # N, K*K, H*W
        out[:, g * D:(g + 1) * D] = (patches * a[:, None]).sum(2)
    return out.view(N, C, H, W).permute(0, 2, 3, 1).numpy()


@pytest.mark.parametrize("case", CASES)
def test_matches_unfold_formulation(case):
    x, w = _problem(case)
    K, sm = case[5], case[6]
    got = oracle.dynconv_forward_ref(x, w, K, sm)
    assert np.allclose(got, _unfold_reference(x, w, K, sm), rtol=0, atol=1e-13)


@pytest.mark.parametrize("case", CASES)
def test_is_a_zero_offset_dcn(case):
    x, w = _problem(case)
    N, H, W, C, G, K, sm = case
    # the DCN oracle numbers taps k = ix * kh + iy (x slowest): reorder
    w_dcn = w.reshape(N, H, W, G, K, K).transpose(0, 1, 2, 3, 5, 4).reshape(N, H, W, G, K * K)
    off = np.zeros((N, H, W, G, K * K, 2))
    ref = oracle.dcn_forward_ref(x, off, w_dcn, K, K, stride=1, pad=K // 2, dil=1,
                                 softmax_flag=sm)
    assert np.allclose(oracle.dynconv_forward_ref(x, w, K, sm), ref, rtol=0, atol=1e-13)


def test_one_hot_weights_copy_a_shifted_map():
    N, H, W, C, G, K = 1, 6, 7, 4, 2, 5
    x = RNG.uniform(-1, 1, (N, H, W, C))
    r = K // 2
    for ky, kx in [(0, 0), (2, 2), (4, 1), (1, 3)]:
        w = np.zeros((N, H, W, G, K * K))
        w[..., ky * K + kx] = 1.0
        got = oracle.dynconv_forward_ref(x, w, K, softmax_flag=0)
        expect = np.zeros_like(x)
        for y in range(H):
            for xx in range(W):
                sy, sx = y + ky - r, xx + kx - r
                if 0 <= sy < H and 0 <= sx < W:
                    expect[0, y, xx] = x[0, sy, sx]
        assert np.array_equal(got, expect), (ky, kx)


@pytest.mark.parametrize("K", [3, 5, 7])
def test_equal_logits_give_the_zero_padded_box_mean(K):
    N, H, W, C, G = 2, 6, 8, 6, 3
    x = RNG.uniform(-1, 1, (N, H, W, C))
    w = np.full((N, H, W, G, K * K), 0.37)
    got = oracle.dynconv_forward_ref(x, w, K, softmax_flag=1)
    box = F.avg_pool2d(torch.tensor(x).permute(0, 3, 1, 2), K, stride=1, padding=K // 2,
                       count_include_pad=True).permute(0, 2, 3, 1).numpy()
    assert np.allclose(got, box, rtol=0, atol=1e-14)


def test_softmax_ignores_a_common_logit_shift_and_is_linear_in_x():
    x, w = _problem((1, 5, 5, 4, 2, 3, 1))
    a = oracle.dynconv_forward_ref(x, w, 3, 1)
    b = oracle.dynconv_forward_ref(x, w + 7.5, 3, 1)
    assert np.allclose(a, b, rtol=0, atol=1e-13)
    x2 = RNG.uniform(-1, 1, x.shape)
    lhs = oracle.dynconv_forward_ref(2.0 * x - 3.0 * x2, w, 3, 1)
    rhs = 2.0 * a - 3.0 * oracle.dynconv_forward_ref(x2, w, 3, 1)
    assert np.allclose(lhs, rhs, rtol=0, atol=1e-13)


def test_rejects_even_windows():
    with pytest.raises(ValueError):
        oracle.dynconv_forward_ref(np.zeros((1, 3, 3, 2)), np.zeros((1, 3, 3, 1, 4)), 2)
