"""Seeded synthetic inputs for the deformable sampling-aggregation workloads.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests.  It draws random numbers (numpy PCG64, float64), applies the
stated input recipe of each workload and rounds once to the workload dtype
(torch `.to()`, round to nearest even).  It holds none of the operator's
arithmetic: no bilinear read, no modulation softmax, no aggregation.

The multi-scale recipe does contain the two module-side steps that produce the
operator's inputs upstream of it: a 2-D reference point plus a pixel offset
divided by the level size gives the normalised location, and the attention
logits are normalised jointly over levels and points of a head.  They run here
in numpy on the float64 draws, before rounding.

Workload names state their sizes.  Shapes and distributions follow the
DCNv4 note (Table 10 / Fig. 1 stage shapes), InternImage ch.5 (the 56/28/14/7
stage hierarchy) and Deformable DETR (four feature levels, K points per level,
M heads).  The features are synthetic stand-ins for backbone activations: no
dataset or trained weights are used.
"""
from dataclasses import dataclass

import numpy as np
import torch

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
# integer codes of the C interface (dcn_dtype_t)
DTYPE_CODES = {"f32": 0, "f16": 1, "bf16": 2}


@dataclass(frozen=True)
class DcnWorkload:
    name: str
    N: int
    H: int
    W: int
    C: int
    G: int
    kh: int = 3
    kw: int = 3
    stride: int = 1
    pad: int = 1
    dil: int = 1
    dtype: str = "f16"
    offset_sigma: float = 2.0    # std of the pixel offsets
    softmax_flag: int = 0        # 1: mask holds logits, softmax over K (DCNv3)

    @property
    def D(self):
        return self.C // self.G

    @property
    def K(self):
        return self.kh * self.kw

    @property
    def Ho(self):
        return (self.H + 2 * self.pad - self.dil * (self.kh - 1) - 1) // self.stride + 1

    @property
    def Wo(self):
        return (self.W + 2 * self.pad - self.dil * (self.kw - 1) - 1) // self.stride + 1

    def taps(self):
        """sampled taps: one per (output pixel, group, kernel point)."""
        return self.N * self.Ho * self.Wo * self.G * self.K

    def pixels(self):
        return self.N * self.Ho * self.Wo

    def compulsory_bytes(self):
        """x, offsets, mask and out, each read or written once."""
        es = DTYPES[self.dtype].itemsize
        x = self.N * self.H * self.W * self.C
        om = self.pixels() * self.G * self.K * 3
        out = self.pixels() * self.C
        return (x + om + out) * es

    def backward_bytes(self):
        """x, offsets, masks and grad_out read once; grad_x, grad_offset and
        grad_mask written once (no accumulator traffic)."""
        es = DTYPES[self.dtype].itemsize
        x = self.N * self.H * self.W * self.C
        om = self.pixels() * self.G * self.K * 3
        out = self.pixels() * self.C
        return (2 * x + 2 * om + out) * es


@dataclass(frozen=True)
class DynWorkload:
    """Dynamic local aggregation (ContMix core): per-pixel K x K kernels."""
    name: str
    N: int
    H: int
    W: int
    C: int
    G: int
    K: int
    dtype: str = "f16"
    softmax_flag: int = 1

    @property
    def D(self):
        return self.C // self.G

    def taps(self):
        """weighted reads: one per (pixel, group, kernel tap)."""
        return self.N * self.H * self.W * self.G * self.K * self.K

    def pixels(self):
        return self.N * self.H * self.W

    def compulsory_bytes(self):
        """x, weights and out, each read or written once."""
        es = DTYPES[self.dtype].itemsize
        return (2 * self.pixels() * self.C + self.taps()) * es


@dataclass(frozen=True)
class FusedWorkload:
    """DCNv4 core fed by its merged offset / mask linear (stride 1)."""
    name: str
    N: int
    H: int
    W: int
    C: int
    G: int
    kh: int = 3
    kw: int = 3
    pad: int = 1
    dil: int = 1
    dtype: str = "f16"
    offset_sigma: float = 2.0

    @property
    def K(self):
        return self.kh * self.kw

    @property
    def J(self):
        return self.G * self.K * 3

    @property
    def D(self):
        return self.C // self.G

    def taps(self):
        return self.N * self.H * self.W * self.G * self.K

    def pixels(self):
        return self.N * self.H * self.W

    def compulsory_bytes(self):
        """x and out once, the linear's weights and bias once."""
        es = DTYPES[self.dtype].itemsize
        return (2 * self.pixels() * self.C + self.J * (self.C + 1)) * es


@dataclass(frozen=True)
class MsdaWorkload:
    name: str
    N: int
    M: int
    D: int
    shapes: tuple             # ((H_l, W_l), ...)
    K: int
    Lq: int = 0               # 0: one query per pixel of all levels (encoder style)
    dtype: str = "f32"
    offset_sigma: float = 2.0  # std of the pixel offsets at each level
    ref_dim: int = 0          # 2 / 4: reference points / boxes with valid ratios
    # reference points of msda_inputs: "cell" puts each encoder query at its
    # own cell centre (the query is that cell), "uniform" draws them ~U[0,1]^2;
    # "" means "cell" for encoder-style queries (Lq = 0), else "uniform"
    ref_points: str = ""

    @property
    def L(self):
        return len(self.shapes)

    @property
    def S(self):
        return sum(h * w for h, w in self.shapes)

    @property
    def queries(self):
        return self.Lq if self.Lq else self.S

    def taps(self):
        return self.N * self.queries * self.M * self.L * self.K

    def pixels(self):
        return self.N * self.queries

    def compulsory_bytes(self):
        """value, locations (or offsets), weights and out once; the reference
        variants add the references and the valid ratios."""
        es = DTYPES[self.dtype].itemsize
        value = self.N * self.S * self.M * self.D
        loc = self.taps() * 2
        w = self.taps()
        out = self.N * self.queries * self.M * self.D
        refs = self.N * self.queries * self.ref_dim + (self.N * self.L * 2 if self.ref_dim else 0)
        return (value + loc + w + out + refs) * es

    def backward_bytes(self):
        """value, locations, weights and grad_out read once; grad_value,
        grad_loc and grad_attn written once (no accumulator traffic)."""
        es = DTYPES[self.dtype].itemsize
        value = self.N * self.S * self.M * self.D
        lw = self.taps() * 3
        out = self.N * self.queries * self.M * self.D
        return (2 * value + 2 * lw + out) * es


WORKLOADS = {w.name: w for w in [
    # DCNv3: softmax over the 9 taps, fp32
    DcnWorkload("dcnv3_f32_1x14x14x64_g4", N=1, H=14, W=14, C=64, G=4, dtype="f32",
                offset_sigma=1.0, softmax_flag=1),
    # DCNv4 fp16 at the first-stage shape, batch 64 (the headline workload)
    DcnWorkload("dcnv4_f16_64x56x56x64_g4", N=64, H=56, W=56, C=64, G=4, dtype="f16"),
    # DCNv4 bf16 over the four stage shapes, G = C / 16
    DcnWorkload("dcnv4_bf16_64x56x56x64_g4", N=64, H=56, W=56, C=64, G=4, dtype="bf16"),
    DcnWorkload("dcnv4_bf16_64x28x28x128_g8", N=64, H=28, W=28, C=128, G=8, dtype="bf16"),
    DcnWorkload("dcnv4_bf16_64x14x14x256_g16", N=64, H=14, W=14, C=256, G=16, dtype="bf16"),
    DcnWorkload("dcnv4_bf16_64x7x7x512_g32", N=64, H=7, W=7, C=512, G=32, dtype="bf16"),
    # DCNv4 fp16 at dense-prediction resolution with heavy-tailed offsets
    DcnWorkload("dcnv4_f16_2x200x320x64_g4", N=2, H=200, W=320, C=64, G=4, dtype="f16",
                offset_sigma=8.0),
    # the headline shape through the fused front end (merged offset / mask
    # linear on the tensor cores feeding the sampler)
    FusedWorkload("dcnv4_fused_f16_64x56x56x64_g4", N=64, H=56, W=56, C=64, G=4),
    # ContMix core (dynamic K x K kernels, softmax) at the first-stage shape:
    # the 7 x 7 and 13 x 13 kernel sizes of the OverLoCK networks
    DynWorkload("contmix_f16_64x56x56x64_g4_k7", N=64, H=56, W=56, C=64, G=4, K=7),
    DynWorkload("contmix_f16_64x56x56x64_g4_k13", N=64, H=56, W=56, C=64, G=4, K=13),
    # MSDeformAttn, four levels, encoder-style queries: one query per cell of
    # every level, referenced at its own cell centre
    MsdaWorkload("msda_f32_2x4lvl_m8_d32_k4", N=2, M=8, D=32,
                 shapes=((100, 150), (50, 75), (25, 38), (13, 19)), K=4, dtype="f32"),
    # the same queries with reference points drawn uniformly over the image:
    # no two consecutive queries share a neighbourhood (a stress case for the
    # gather path)
    MsdaWorkload("msda_f32_2x4lvl_m8_d32_k4_uniformref", N=2, M=8, D=32,
                 shapes=((100, 150), (50, 75), (25, 38), (13, 19)), K=4, dtype="f32",
                 ref_points="uniform"),
    # the same levels as a decoder with 4-D box references, valid ratios and
    # 300 object queries per image
    MsdaWorkload("msda_f32_2x4lvl_m8_d32_k4_box300", N=2, M=8, D=32,
                 shapes=((100, 150), (50, 75), (25, 38), (13, 19)), K=4, Lq=300, dtype="f32",
                 ref_dim=4),
]}

HEADLINE = "dcnv4_f16_64x56x56x64_g4"


def _round(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DTYPES[dtype])


def dcn_inputs(w, seed=0):
    """x [N,H,W,C] ~ U[-1,1]; offset [N,Ho,Wo,G,K,2] ~ N(0, sigma) px as (dx, dy);
    mask [N,Ho,Wo,G,K] ~ N(0, 1) (unbounded m, or DCNv3 logits).  CPU tensors."""
    rng = np.random.default_rng(seed)
    x = rng.uniform(-1.0, 1.0, size=(w.N, w.H, w.W, w.C))
    offset = rng.normal(0.0, w.offset_sigma, size=(w.N, w.Ho, w.Wo, w.G, w.K, 2))
    mask = rng.normal(0.0, 1.0, size=(w.N, w.Ho, w.Wo, w.G, w.K))
    return {"x": _round(x, w.dtype), "offset": _round(offset, w.dtype),
            "mask": _round(mask, w.dtype)}


def dynconv_inputs(w, seed=0):
    """x [N,H,W,C] ~ U[-1,1]; weights [N,H,W,G,K*K] ~ N(0, 1) (the numbers a
    softmax turns into each location's kernel).  CPU tensors."""
    rng = np.random.default_rng(seed)
    x = rng.uniform(-1.0, 1.0, size=(w.N, w.H, w.W, w.C))
    weights = rng.normal(0.0, 1.0, size=(w.N, w.H, w.W, w.G, w.K * w.K))
    return {"x": _round(x, w.dtype), "weights": _round(weights, w.dtype)}


def level_start_index(shapes):
    """First value row of each level (levels concatenated row-major)."""
    starts, s = [], 0
    for h, wd in shapes:
        starts.append(s)
        s += h * wd
    return starts


def msda_centres(shapes):
    """Normalised centres (x, y) = ((j + 1/2) / W_l, (i + 1/2) / H_l) of every
    cell of every level, in the row order of the concatenated value tensor."""
    parts = []
    for h, wd in shapes:
        cx, cy = np.meshgrid((np.arange(wd) + 0.5) / wd, (np.arange(h) + 0.5) / h, indexing="xy")
        parts.append(np.stack([cx, cy], axis=-1).reshape(-1, 2))
    return np.concatenate(parts, axis=0)


def msda_inputs(w, seed=0):
    """value [N,S,M,D] ~ U[-1,1]; one reference point per (n, q) shared by heads,
    levels and points: for encoder-style queries (one per cell, Lq = 0) the
    centre of the query's own cell, normalised by its level ("Deformable
    DETR": in the encoder a source cell centre is the reference), otherwise
    ~ U[0,1]^2 (w.ref_points overrides); pixel offsets ~ N(0, sigma) per
    (m, l, k) divided by (W_l, H_l); logits ~ N(0,1) normalised jointly over
    (l, k) per head."""
    rng = np.random.default_rng(seed)
    Lq = w.queries
    value = rng.uniform(-1.0, 1.0, size=(w.N, w.S, w.M, w.D))
    ref = rng.uniform(0.0, 1.0, size=(w.N, Lq, 2))   # drawn in every mode: same stream
    mode = w.ref_points or ("cell" if not w.Lq else "uniform")
    if mode == "cell":
        if Lq != w.S:
            raise ValueError("cell-centre references need one query per cell (Lq = 0)")
        ref = np.broadcast_to(msda_centres(w.shapes)[None], (w.N, Lq, 2))
    elif mode != "uniform":
        raise ValueError(f"unknown reference-point mode {mode!r}")
    dp = rng.normal(0.0, w.offset_sigma, size=(w.N, Lq, w.M, w.L, w.K, 2))
    logits = rng.normal(0.0, 1.0, size=(w.N, Lq, w.M, w.L, w.K))
    size_wh = np.array([[wd, h] for h, wd in w.shapes], dtype=np.float64)  # [L, 2]
    loc = ref[:, :, None, None, None, :] + dp / size_wh[None, None, None, :, None, :]
    flat = logits.reshape(w.N, Lq, w.M, w.L * w.K)
    e = np.exp(flat - flat.max(axis=-1, keepdims=True))
    attn = (e / e.sum(axis=-1, keepdims=True)).reshape(logits.shape)
    return {
        "value": _round(value, w.dtype),
        "spatial_shapes": torch.tensor(w.shapes, dtype=torch.int64),
        "level_start": torch.tensor(level_start_index(w.shapes), dtype=torch.int64),
        "loc": _round(loc, w.dtype),
        "attn": _round(attn, w.dtype),
        "logits": logits,
    }


def grad_out(shape, dtype, seed=0):
    """Upstream gradient for a backward pass: N(0, 1) of the output's shape,
    rounded to the dtype (a CPU tensor).  Drawn from its own stream, so the
    forward inputs of the same seed are unchanged."""
    rng = np.random.default_rng([seed, 0x6772])
    return _round(rng.normal(0.0, 1.0, size=tuple(shape)), dtype)


def front_end_inputs(w, seed=0):
    """x ~U[-1,1]; w_om ~N(0, s^2) with s chosen so that the linear's offsets
    have std offset_sigma px and its masks std 1 (x has variance 1/3 per
    channel); b_om ~N(0, 0.25).  CPU tensors."""
    rng = np.random.default_rng(seed)
    x = rng.uniform(-1.0, 1.0, size=(w.N, w.H, w.W, w.C))
    n_off = w.G * w.K * 2
    s_off = np.sqrt(3.0 * w.offset_sigma ** 2 / w.C)
    s_mask = np.sqrt(3.0 / w.C)
    w_om = np.concatenate([rng.normal(0.0, s_off, size=(n_off, w.C)),
                           rng.normal(0.0, s_mask, size=(w.J - n_off, w.C))], axis=0)
    b_om = rng.normal(0.0, 0.5, size=(w.J,))
    return {"x": _round(x, w.dtype), "w_om": _round(w_om, w.dtype), "b_om": _round(b_om, w.dtype)}


def msda_ref_inputs(w, seed=0):
    """Inputs of the reference-point variants (ref_dim 2 or 4): value as
    msda_inputs; valid ratios ~U[0.75, 1] per (n, level, axis) (right / bottom
    padding); points ~U[0,1]^2 in valid-image units, or boxes with centre
    ~U[0,1]^2 and size ~U[0.05, 0.3]; offsets ~N(0, sigma) (pixels for points,
    units of box size * K / 2 for boxes, so sigma / K box half-sizes); weights
    normalised jointly over (l, k); a padding mask [N, S] of the value rows
    beyond each level's valid extent."""
    rng = np.random.default_rng(seed)
    Lq = w.queries
    value = rng.uniform(-1.0, 1.0, size=(w.N, w.S, w.M, w.D))
    vr = rng.uniform(0.75, 1.0, size=(w.N, w.L, 2))
    if w.ref_dim == 4:
        ref = np.concatenate([rng.uniform(0.0, 1.0, size=(w.N, Lq, 2)),
                              rng.uniform(0.05, 0.3, size=(w.N, Lq, 2))], axis=-1)
        sigma = 1.0
    else:
        ref = rng.uniform(0.0, 1.0, size=(w.N, Lq, 2))
        sigma = w.offset_sigma
    off = rng.normal(0.0, sigma, size=(w.N, Lq, w.M, w.L, w.K, 2))
    logits = rng.normal(0.0, 1.0, size=(w.N, Lq, w.M, w.L, w.K))
    flat = logits.reshape(w.N, Lq, w.M, w.L * w.K)
    e = np.exp(flat - flat.max(axis=-1, keepdims=True))
    attn = (e / e.sum(axis=-1, keepdims=True)).reshape(logits.shape)
    mask = np.zeros((w.N, w.S), dtype=bool)
    starts = level_start_index(w.shapes)
    for n in range(w.N):
        for l, (h, wd) in enumerate(w.shapes):
            hv = int(np.ceil(vr[n, l, 1] * h))
            wv = int(np.ceil(vr[n, l, 0] * wd))
            m = np.ones((h, wd), dtype=bool)
            m[:hv, :wv] = False
            mask[n, starts[l]:starts[l] + h * wd] = m.reshape(-1)
    return {
        "value": _round(value, w.dtype),
        "spatial_shapes": torch.tensor(w.shapes, dtype=torch.int64),
        "level_start": torch.tensor(starts, dtype=torch.int64),
        "reference": _round(ref, w.dtype),
        "valid_ratios": _round(vr, w.dtype),
        "offsets": _round(off, w.dtype),
        "attn": _round(attn, w.dtype),
        "mask": torch.from_numpy(mask),
    }


def scaled(w, **changes):
    """A copy of workload `w` with some fields replaced (e.g. a smaller batch)."""
    fields = dict(w.__dict__)
    fields.update(changes)
    return type(w)(**fields)
