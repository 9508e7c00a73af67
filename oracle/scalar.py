"""Pure-Python scalar twin of the oracle's arithmetic (test infrastructure only).

Small, loop-by-loop restatements used (a) to check the C oracle on tiny
inputs by brute force and (b) to expose intermediate quantities (corner
weights, modulations) that the worked examples on the pages print.

Sources (page title, section):
  "InternImage: Deformable Convolutions at Scale" ch.2 (bilinear read),
      ch.3 (softmax over the K taps, worked example with K = 3).
  "DCNv4", "1. Remove Softmax" (modulation used as given).
  "Deformable DETR: Learn Where to Read", "A reference links resolutions
      without equating their pixels" (point reference to sampling location),
      "A learned location can fall between cells" (normalised to pixel-index
      coordinates), helper 3 (joint softmax over levels and points of one
      head, aggregation).
"""
import math


def corner_weights(px, py):
    """Bilinear corner weights for a fractional point (InternImage ch.2).

    Returns ((x0, y0), {(dx, dy): weight}) with the corner offsets dx, dy in
    {0, 1}; a = px - floor(px), b = py - floor(py).
    """
    x0 = math.floor(px)
    y0 = math.floor(py)
    a = px - x0
    b = py - y0
    return (x0, y0), {
        (0, 0): (1 - a) * (1 - b),
        (1, 0): a * (1 - b),
        (0, 1): (1 - a) * b,
        (1, 1): a * b,
    }


def bilinear_pixel(grid, px, py):
    """Read grid[row][col] at pixel-index point (px, py), zero outside."""
    height, width = len(grid), len(grid[0])
    (x0, y0), weights = corner_weights(px, py)
    value = 0.0
    for (dx, dy), w in weights.items():
        col, row = x0 + dx, y0 + dy
        if 0 <= row < height and 0 <= col < width:
            value += w * grid[row][col]
    return value


def bilinear_normalized(grid, u, v):
    """align_corners=False sample of grid at normalised (u, v), zero padding.

    Deformable DETR, "A learned location can fall between cells": the
    normalised point maps to the pixel-index point (u W - 1/2, v H - 1/2),
    which is then read with the pixel bilinear above (the page's tent weights
    over the four floor/ceil neighbours are the same four corner weights).
    """
    return bilinear_pixel(grid, u * len(grid[0]) - 0.5, v * len(grid) - 0.5)


def softmax(logits):
    """Stable softmax of a list (subtract the maximum first)."""
    top = max(logits)
    exps = [math.exp(z - top) for z in logits]
    s = sum(exps)
    return [e / s for e in exps]


def normalize_weights(logits):
    """Joint softmax of one head's [L][K] logits over all levels and points.

    One maximum and one sum over the whole L x K array (Deformable DETR,
    helper 3), never one softmax per level.
    """
    flat = [z for level in logits for z in level]
    top = max(flat)
    total = sum(math.exp(z - top) for z in flat)
    return [[math.exp(z - top) / total for z in level] for level in logits]


def aggregate(values, weights):
    """sum over levels and points of weight * sampled value, for one head."""
    total = 0.0
    for level_values, level_weights in zip(values, weights):
        for v, w in zip(level_values, level_weights):
            total += w * v
    return total


def sampling_location(reference, offset, shape_wh):
    """2-D point reference to a normalised sampling location, valid ratio 1.

    Deformable DETR, "A reference links resolutions without equating their
    pixels": s = p + dp / (W_l, H_l), componentwise, not clamped.
    `shape_wh` is (width, height).
    """
    return [p + d / size for p, d, size in zip(reference, offset, shape_wh)]


def out_size(n_in, k, stride, pad, dil):
    return (n_in + 2 * pad - dil * (k - 1) - 1) // stride + 1


def dcn_forward_py(x, offset, mask, kh, kw, stride, pad, dil, softmax_flag):
    """Brute-force DCNv3/DCNv4 forward over nested lists (tiny inputs only).

    x[n][y][x][c], offset[n][oy][ox][g][k][2], mask[n][oy][ox][g][k];
    returns out[n][oy][ox][c].  G is read from the mask, D = C / G.
    """
    N, H, W, C = len(x), len(x[0]), len(x[0][0]), len(x[0][0][0])
    G = len(mask[0][0][0])
    D = C // G
    Ho = out_size(H, kh, stride, pad, dil)
    Wo = out_size(W, kw, stride, pad, dil)
    out = [[[[0.0] * C for _ in range(Wo)] for _ in range(Ho)] for _ in range(N)]
    for n in range(N):
        for oy in range(Ho):
            for ox in range(Wo):
                for g in range(G):
                    z = mask[n][oy][ox][g]
                    m = softmax(z) if softmax_flag else list(z)
                    for c in range(D):
                        plane = [[x[n][yy][xx][g * D + c] for xx in range(W)]
                                 for yy in range(H)]
                        acc = 0.0
                        for ix in range(kw):
                            for iy in range(kh):
                                k = ix * kh + iy
                                dx, dy = offset[n][oy][ox][g][k]
                                px = ox * stride - pad + ix * dil + dx
                                py = oy * stride - pad + iy * dil + dy
                                acc += m[k] * bilinear_pixel(plane, px, py)
                        out[n][oy][ox][g * D + c] = acc
    return out
