"""The band kernel's launch plan, from the library on the host, and a model of
the kernel's index arithmetic checked under that plan (no GPU).

`dcn_forward_plan` returns the launch shape that `dcn_forward_algo` uses
(rows per step, offset margin, ring rows, sampler warps, steps in flight,
runs per row, shared memory). The model below restates, in numpy, what the
band kernel computes from those numbers: the steps of each CTA's range of
output rows, the band of input rows of each step, the ring slots the
producer's bulk copies fill, the slots it may overwrite while earlier steps
are in flight, and every shared-memory and global address the samplers form
for seeded offsets. It checks that
- every copy stays inside x, the ring and its stage buffer, and fits in an
  mbarrier transaction count;
- no copy overwrites a ring slot that a step still in flight reads;
- every band row a step reads sits in the slot the step addresses;
- every shared read of a corner lies in the ring, every global fallback read
  in x, every offset or mask read in its stage buffer;
- every output item is stored exactly once.
The model is written from the kernel's source (dcn_band.cuh, abi_dcn_fwd.cu)
and shares no code with it.
"""
import ctypes

import numpy as np
import pytest

import deformable_attention_sampling_b200 as dcnb

F16 = dcnb.DTYPE_CODES["f16"]
F32 = dcnb.DTYPE_CODES["f32"]
ES = 2                      # 16-bit data
DESC_INTS = 8               # ints per step descriptor
TX_LIMIT = 1 << 20          # mbarrier transaction count


def out_size(n, k, s, p, d):
    return (n + 2 * p - d * (k - 1) - 1) // s + 1


def plan_of(N, H, W, C, G, k, stride, pad, dil, dtype=F16):
    return dcnb.dcn_forward_plan(N, H, W, C, G, k, k, stride, pad, dil, 0, dtype)


# ------------------------------------------------------------ plan values


def test_plan_of_the_64x56x56x64_forward():
    p = plan_of(64, 56, 56, 64, 4, 3, 1, 1, 1)
    assert p == {"algo": dcnb.DCN_ALGO_BAND, "rows_per_step": 2, "margin": 6, "ring_rows": 18,
                 "sampler_warps": 16, "steps_in_flight": 2, "runs_per_row": 7,
                 "smem_bytes": 18 * 56 * 64 * 2 + 2 * 24192 + 2 * 16 + 2 * DESC_INTS * 4}


def test_plan_takes_the_gather_kernel_where_the_band_does_not_apply():
    assert plan_of(64, 56, 56, 64, 4, 3, 1, 1, 1, dtype=F32)["algo"] == dcnb.DCN_ALGO_GATHER
    assert plan_of(2, 20, 20, 64, 2, 3, 1, 1, 1)["algo"] == dcnb.DCN_ALGO_GATHER   # D = 32
    # 40 KB rows: the band does not fit in shared memory
    assert plan_of(2, 200, 320, 64, 4, 3, 1, 1, 1)["algo"] == dcnb.DCN_ALGO_GATHER
    # offset and mask rows of a multiple of 16 bytes only (odd Wo at G = 4)
    assert plan_of(2, 13, 13, 64, 4, 3, 1, 1, 1)["algo"] == dcnb.DCN_ALGO_GATHER
    with pytest.raises(dcnb.DcnError) as e:
        dcnb.dcn_forward_plan(64, 56, 56, 64, 4, 3, 3, 1, 1, 1, 0, F32, algo=dcnb.DCN_ALGO_BAND)
    assert e.value.status == dcnb.DCN_ERR_UNSUPPORTED


def test_plan_argument_errors_match_the_forward_call():
    lib = dcnb.library()
    plan = (ctypes.c_int * 8)(*([-7] * 8))
    bad = [
        (-1, 8, 8, 64, 4, 3, 3, 1, 1, 1, 0, F16, 0),     # N < 0
        (1, 8, 8, 64, 5, 3, 3, 1, 1, 1, 0, F16, 0),      # C % G != 0
        (1, 8, 8, 64, 4, 3, 3, 1, 1, 1, 2, F16, 0),      # softmax flag
        (1, 8, 8, 64, 4, 3, 3, 1, 1, 1, 0, 9, 0),        # dtype
        (1, 8, 8, 64, 4, 3, 3, 1, 1, 1, 0, F16, 7),      # algo
        (1, 2, 2, 64, 4, 5, 5, 1, 0, 1, 0, F16, 0),      # Ho <= 0
    ]
    for args in bad:
        assert lib.dcn_forward_plan(*args, plan) == dcnb.DCN_ERR_INVALID_ARG, args
        assert list(plan) == [-7] * 8, "plan written on an error"
    assert lib.dcn_forward_plan(1, 8, 8, 64, 4, 3, 3, 1, 1, 1, 0, F16, 0, None) == \
        dcnb.DCN_ERR_INVALID_ARG
    assert lib.dcn_forward_plan(1, 1 << 17, 8, 64, 4, 3, 3, 1, 1, 1, 0, F16, 0, plan) == \
        dcnb.DCN_ERR_UNSUPPORTED
    p = dcnb.dcn_forward_plan(0, 56, 56, 64, 4, 3, 3, 1, 1, 1, 0, F16)
    assert p["algo"] == 0 and p["rows_per_step"] == 2      # N = 0 launches nothing


def test_debug_library_plans_the_same():
    args = (8, 28, 28, 128, 8, 3, 3, 1, 1, 1, 0, F16)
    assert dcnb.dcn_forward_plan(*args) == dcnb.dcn_forward_plan(*args, lib=dcnb.debug_library())


# ------------------------------------------------------- model of the kernel


class Layout:
    """Shared-memory layout and row sizes of one band launch, from the shape
    and the library's plan."""

    def __init__(self, N, H, W, C, G, k, stride, pad, dil, plan):
        self.N, self.H, self.W, self.C, self.G = N, H, W, C, G
        self.kh = self.kw = k
        self.K = k * k
        self.stride, self.pad, self.dil = stride, pad, dil
        self.Ho, self.Wo = out_size(H, k, stride, pad, dil), out_size(W, k, stride, pad, dil)
        self.th, self.margin = plan["rows_per_step"], plan["margin"]
        self.RB, self.NS = plan["ring_rows"], plan["steps_in_flight"]
        self.rpr, self.nc = plan["runs_per_row"], plan["sampler_warps"]
        self.row_bytes = W * C * ES
        self.pix_bytes = C * ES
        self.off_row = self.Wo * G * self.K * 2 * ES
        self.mask_row = self.Wo * G * self.K * ES
        self.stage = (self.th * (self.off_row + self.mask_row) + 127) // 128 * 128
        self.ring_bytes = self.RB * self.row_bytes
        self.smem = self.ring_bytes + self.NS * (self.stage + 16 + DESC_INTS * 4)
        self.rows_total = N * self.Ho
        self.x_bytes = N * H * self.row_bytes


def steps_of(L, r0, r1):
    """(n, o, nrows) of the steps of a CTA's rows [r0, r1): up to th rows of
    one image each."""
    cur = r0
    while cur < r1:
        n, o = divmod(cur, L.Ho)
        nrows = min(L.th, L.Ho - o, r1 - cur)
        yield n, o, nrows
        cur += nrows


def simulate(L, grid, sigma, rng):
    """Run the producer and the samplers of every CTA of a launch of `grid`
    CTAs; return a list of violations (empty when every check holds)."""
    errors = []
    stored = np.zeros((L.N, L.Ho, L.Wo * L.G), dtype=np.int64)
    row_items = L.Wo * L.G
    for b in range(grid):
        r0 = L.rows_total * b // grid
        r1 = L.rows_total * (b + 1) // grid
        prev_n, prev_ylo, prev_yhi, prev_vlo = -1, 0, -1, 0
        next_v, done = 0, -1
        descs, slots = {}, {}
        for step, (n, o, nrows) in enumerate(steps_of(L, r0, r1)):
            # ---------------------------------------------------- producer
            y_lo = max(0, o * L.stride - L.pad - L.margin)
            y_hi = min(L.H - 1, (o + nrows - 1) * L.stride - L.pad + (L.kh - 1) * L.dil + L.margin)
            if y_lo > y_hi:
                errors.append(("empty band", b, step))
                continue
            if n == prev_n and prev_ylo <= y_lo <= prev_yhi + 1:
                v_lo = prev_vlo + (y_lo - prev_ylo)          # the band continues
                first_new = max(y_lo, prev_yhi + 1)
            else:
                v_lo, first_new = next_v, y_lo                # a fresh band
            v_hi = v_lo + (y_hi - y_lo)
            v_first_new = v_lo + (first_new - y_lo)
            # release the stage buffer of step - NS and the steps whose rows
            # the new copies overwrite
            while done < step - 1:
                t = done + 1
                must = t <= step - L.NS or (first_new <= y_hi and descs[t]["v_lo"] <= v_hi - L.RB)
                if not must:
                    break
                done = t
            written = {v % L.RB for v in range(v_first_new, v_hi + 1)}
            for t in range(done + 1, step):
                d = descs[t]
                used = {(d["v_lo"] + i) % L.RB for i in range(d["y_hi"] - d["y_lo"] + 1)}
                if used & written:
                    errors.append(("slot overwritten while a step reads it", b, step, t))
            if {(v_lo + i) % L.RB for i in range(first_new - y_lo)} & written:
                errors.append(("the band's own rows overwritten", b, step))
            new_rows = max(0, y_hi - first_new + 1)
            if new_rows:
                src = (n * L.H + first_new) * L.row_bytes
                if src < 0 or src + new_rows * L.row_bytes > L.x_bytes:
                    errors.append(("x copy out of bounds", b, step))
                slot, left, y = v_first_new % L.RB, new_rows, first_new
                while left > 0:
                    cnt = min(left, L.RB - slot)
                    if (slot + cnt) * L.row_bytes > L.ring_bytes:
                        errors.append(("ring copy out of bounds", b, step))
                    for i in range(cnt):
                        slots[slot + i] = (n, y + i)
                    y, left, slot = y + cnt, left - cnt, 0
            if L.th * L.off_row + nrows * L.mask_row > L.stage:
                errors.append(("stage buffer overflow", b, step))
            if (n * L.Ho + o + nrows) * L.off_row > L.N * L.Ho * L.off_row:
                errors.append(("offset copy out of bounds", b, step))
            if new_rows * L.row_bytes + nrows * (L.off_row + L.mask_row) >= TX_LIMIT:
                errors.append(("transaction count too large", b, step))
            descs[step] = dict(y_lo=y_lo, y_hi=y_hi, v_lo=v_lo)
            span, slot_lo = y_hi - y_lo, v_lo % L.RB
            for y in range(y_lo, y_hi + 1):
                if slots.get((slot_lo + y - y_lo) % L.RB) != (n, y):
                    errors.append(("a slot holds the wrong row", b, step, y))
            prev_n, prev_ylo, prev_yhi, prev_vlo = n, y_lo, y_hi, v_lo
            next_v = max(next_v, v_hi + 1)

            # ---------------------------------------------------- samplers
            runs = nrows * L.rpr
            r = np.arange(runs)
            row_local, run_in_row = r // L.rpr, r % L.rpr
            item = run_in_row[:, None] * 32 + np.arange(32)[None, :]      # [runs, lane]
            active = item < row_items
            item = np.where(active, item, row_items - 1)
            lane = np.broadcast_to(np.arange(32), item.shape)
            oy = o + row_local[:, None] + 0 * item
            ox, g = item // L.G, item % L.G
            np.add.at(stored[n], (oy[active], item[active]), 1)
            # offsets and masks read from the stage buffer
            off_end = row_local[:, None] * L.off_row + (item + 1) * L.K * 2 * ES
            mask_end = L.th * L.off_row + row_local[:, None] * L.mask_row + (item + 1) * L.K * ES
            if (off_end > L.th * L.off_row).any() or (mask_end > L.stage).any():
                errors.append(("offset or mask read outside the stage", b, step))
            rot = (lane >> 2) & 1
            hb0, hb1 = rot * 16, (rot ^ 1) * 16
            for ix in range(L.kw):
                for iy in range(L.kh):
                    dx = np.floor(rng.normal(0.0, sigma, item.shape)).astype(np.int64)
                    dy = np.floor(rng.normal(0.0, sigma, item.shape)).astype(np.int64)
                    x0 = ox * L.stride - L.pad + ix * L.dil + dx
                    y0 = oy * L.stride - L.pad + iy * L.dil + dy
                    vx = [(x0 + j >= 0) & (x0 + j < L.W) for j in (0, 1)]
                    vy = [(y0 + j >= 0) & (y0 + j < L.H) for j in (0, 1)]
                    r0_ = y0 - y_lo
                    inb = [(r0_ + j >= 0) & (r0_ + j <= span) for j in (0, 1)]
                    fb = (vy[0] & ~inb[0]) | (vy[1] & ~inb[1])
                    for j in (0, 1):
                        s_ = slot_lo + np.clip(r0_ + j, 0, span)
                        s_ = np.where(s_ >= L.RB, s_ - L.RB, s_)
                        for i in (0, 1):
                            c = np.where(vx[i], x0 + i, 0) * L.pix_bytes
                            for hb in (hb0, hb1):
                                ad = s_ * L.row_bytes + c + g * 32 + hb
                                if ((ad < 0) | (ad + 16 > L.ring_bytes)).any():
                                    errors.append(("shared read outside the ring", b, step))
                            # the global fallback for taps that leave the band
                            gy = np.where(vy[j], y0 + j, 0)
                            gx = np.where(vx[i], x0 + i, 0)
                            ga = (n * L.H + gy) * L.row_bytes + gx * L.pix_bytes + g * 32
                            bad = fb & ((ga < 0) | (ga + 32 > L.x_bytes))
                            if bad.any():
                                errors.append(("global fallback read outside x", b, step))
            if len(errors) > 20:
                return errors
    if not (stored == 1).all():
        errors.append(("outputs not stored exactly once", int((stored != 1).sum())))
    return errors


# N, H, W, C, G, k, stride, pad, dil, offset sigma (px)
MODEL_CASES = [
    (3, 9, 6, 64, 4, 3, 1, 1, 1, 3.0),        # four rows per step, ragged last step
    (2, 7, 7, 512, 32, 3, 1, 1, 1, 2.0),      # 32 groups: 7 runs per row
    (2, 14, 14, 256, 16, 3, 1, 1, 1, 2.0),
    (2, 28, 28, 128, 8, 3, 1, 1, 1, 2.0),
    (2, 33, 16, 64, 4, 1, 1, 0, 1, 5.0),      # 1x1 window, taps far outside the band
    (1, 5, 40, 64, 4, 3, 1, 1, 1, 2.0),       # fewer rows than the band
    (3, 5, 40, 64, 4, 3, 1, 1, 1, 2.0),       # ring of 2H rows, bands that span images
    (4, 6, 16, 64, 4, 3, 1, 1, 1, 2.0),
    (5, 3, 24, 64, 4, 3, 1, 1, 1, 1.0),       # one step per image, ring of 2H rows
    (2, 24, 24, 64, 4, 3, 2, 1, 1, 2.0),      # stride 2
    (2, 20, 12, 64, 4, 3, 1, 2, 2, 2.0),      # dilation 2
    (1, 40, 100, 64, 4, 3, 1, 1, 1, 2.0),     # smaller margin (2 rows)
    (4, 17, 24, 128, 8, 3, 1, 1, 1, 8.0),     # heavy offsets
]


@pytest.mark.parametrize("case", MODEL_CASES, ids=lambda c: "x".join(map(str, c[:9])))
def test_band_kernel_model_under_the_library_plan(case):
    *shape, sigma = case
    N, H, W, C, G, k, stride, pad, dil = shape
    plan = plan_of(N, H, W, C, G, k, stride, pad, dil)
    assert plan["algo"] == dcnb.DCN_ALGO_BAND, plan
    L = Layout(N, H, W, C, G, k, stride, pad, dil, plan)
    assert L.smem == plan["smem_bytes"]
    assert L.smem <= 227 * 1024
    rng = np.random.default_rng(sum(shape))
    for grid in sorted({1, 3, min(L.rows_total, 148), L.rows_total}):
        errors = simulate(L, grid, sigma, rng)
        assert not errors, (grid, errors[:5])


def test_band_kernel_model_on_the_64x56x56x64_launch():
    """The whole 148-CTA launch of the N = 64, 56x56, C = 64, G = 4 forward
    (3584 output rows, 24 or 25 per CTA)."""
    plan = plan_of(64, 56, 56, 64, 4, 3, 1, 1, 1)
    L = Layout(64, 56, 56, 64, 4, 3, 1, 1, 1, plan)
    errors = simulate(L, 148, 2.0, np.random.default_rng(7))
    assert not errors, errors[:5]
