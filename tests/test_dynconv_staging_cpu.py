"""A model of how the tensor-core ContMix kernel stages its weights (no GPU).

Each CTA of `dynconv_mma_kernel` (dynconv_mma.cuh) covers 8 output rows x 32
columns of one group; warp w owns output row w. Per kernel row ky, the
numbers of the warp's 32 locations are copied with 8-byte `cp.async` into one
slot per location. Each slot holds the 8-byte units from the one holding the
row's first number, the last unit clipped to the row's end.
- At K = 13 (four units) four lanes take one location each, one unit per lane.
- At K = 7 each lane copies its own location's units.
Each thread then reads its own location's numbers from its slot, starting at
byte (address of the first number) mod 8.

The model restates that index arithmetic in plain Python, for maps whose edges cut
tiles, every group count the kernel serves and both compiled kernel sizes. It
checks that
- every unit of every in-map location is copied exactly once;
- the units cover the row's bytes with no gap;
- every copy stays inside its slot and inside the weights tensor;
- nothing is copied for a location outside the map;
- the bytes a thread reads hold its own location's row.
Planted mistakes in the mapping must fail it. The model is written from the
kernel's source and shares no code with it.
"""
import pytest

ES = 2                      # 16-bit weights
ROWS, COLS = 8, 32          # output rows (warps) and columns of a CTA


def row_units(K):
    """8-byte units a kernel row of K numbers can span, from the unit of its
    first number (the first number starts at an even byte offset 0..6)."""
    return (2 * K + 6 + 7) // 8


def slot_units(K):
    """Units of a location's slot: row_units rounded up to an odd count."""
    return row_units(K) | 1


def copies(K, G, W, H, n, ty, tx, g, ky, warp, base, mapping="kernel"):
    """(col, unit, src, nbytes, dst) of every copy warp `warp` issues for
    kernel row ky of tile (n, ty, tx, g); byte addresses (src from the
    tensor's start `base`, dst from the start of the warp's first slot)."""
    y0, x0 = ty * ROWS, tx * COLS
    w_col = G * K * K
    w_row = W * w_col
    wt = (((n * H + y0) * W + x0) * G + g) * K * K
    row_w = base + ES * (wt + warp * w_row)
    su = slot_units(K)
    nuc = row_units(K)
    out = []

    def emit(col, unit):
        if not (y0 + warp < H and x0 + col < W):
            return
        first = row_w + ES * (col * w_col + ky * K)
        last = first + ES * K
        u8 = (first & ~7) + 8 * unit
        if u8 < last:
            out.append((col, unit, u8, min(8, last - u8), col * su * 8 + 8 * unit))

    if mapping == "kernel":
        if nuc >= 4:                               # four (or eight) lanes per location
            upl = 4 if nuc <= 4 else 8
            for p in range(upl):
                for lane in range(32):
                    f = p * 32 + lane
                    emit(f // upl, f % upl)
        else:                                      # a lane per location
            for lane in range(32):
                for unit in range(nuc + 1):
                    emit(lane, unit)
    elif mapping == "three_lanes":                 # planted: too few lanes per location
        for p in range(3):
            for lane in range(32):
                f = p * 32 + lane
                emit(f // 3, f % 3)
    elif mapping == "unit_shift":                  # planted: units one off
        for p in range(4):
            for lane in range(32):
                f = p * 32 + lane
                emit(f // 4, f % 4 + 1)
    return out


def check_tile(K, G, W, H, n, ty, tx, g, base):
    errors = []
    total = base + ES * 2 * H * W * G * K * K   # two images of weights
    su = slot_units(K)
    y0, x0 = ty * ROWS, tx * COLS
    w_col = G * K * K
    for warp in range(ROWS):
        row_w = base + ES * ((((n * H + y0) * W + x0) * G + g) * K * K + warp * W * w_col)
        for ky in range(K):
            cs = copies(K, G, W, H, n, ty, tx, g, ky, warp, base)
            seen = {}
            for col, unit, src, nb, dst in cs:
                if (col, unit) in seen:
                    errors.append(("unit copied twice", warp, ky, col, unit))
                seen[(col, unit)] = (src, nb, dst)
                if not (y0 + warp < H and x0 + col < W):
                    errors.append(("copy for a location outside the map", warp, col))
                if dst < col * su * 8 or dst + 8 > (col + 1) * su * 8:
                    errors.append(("copy outside its slot", warp, ky, col, unit))
                if src < base or src + nb > total or src % 8 != 0:
                    errors.append(("source outside the tensor or unaligned", warp, ky, col))
            for col in range(COLS):
                if not (y0 + warp < H and x0 + col < W):
                    continue
                first = row_w + ES * (col * w_col + ky * K)
                last = first + ES * K
                have = sorted(v for (c, u), v in seen.items() if c == col)
                # the units tile [first & ~7, last) without a gap
                pos = first & ~7
                for src, nb, _ in have:
                    if src != pos:
                        errors.append(("gap or overlap in a row's units", warp, ky, col))
                        break
                    pos = src + nb
                if pos != last:
                    errors.append(("row not fully copied", warp, ky, col, pos - last))
                # the reader: bytes [o, o + 2K) of its slot, o = first mod 8
                o = first & 7
                slot = {(dst - col * su * 8) // 8: (src, nb) for src, nb, dst in have}
                for b in range(o, o + ES * K):
                    u, r = divmod(b, 8)
                    if u not in slot or r >= slot[u][1] or slot[u][0] + r != first - o + b:
                        errors.append(("a read byte is not the row's", warp, ky, col, b))
                        break
                if o + ES * K > su * 8:
                    errors.append(("the row does not fit its slot", warp, ky, col))
    return errors


CASES = [
    # H, W, G, K: maps whose right and bottom edges cut a tile, every group count
    (10, 40, 4, 13), (10, 40, 4, 7), (9, 33, 2, 13), (9, 33, 2, 7), (8, 32, 1, 13),
    (11, 70, 1, 7), (3, 5, 4, 13),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_weight_staging_model(case):
    H, W, G, K = case
    errors = []
    for base in (0, 16, 4096):
        for n in (0, 1):
            for ty in range((H + ROWS - 1) // ROWS):
                for tx in range((W + COLS - 1) // COLS):
                    for g in range(G):
                        errors += check_tile(K, G, W, H, n, ty, tx, g, base)
                        if len(errors) > 10:
                            break
    assert not errors, errors[:5]


@pytest.mark.parametrize("mapping", ["three_lanes", "unit_shift"])
def test_planted_mapping_mistakes_fail(mapping, monkeypatch):
    real = copies

    def wrong(*a, **k):
        return real(*a, mapping=mapping)
    monkeypatch.setitem(globals(), "copies", wrong)
    errors = check_tile(13, 4, 40, 10, 0, 0, 0, 1, 0)
    assert errors, mapping


def test_units_per_row():
    # a 13-number row spans at most four 8-byte units, a 7-number row three;
    # the slots hold five and three
    assert (row_units(13), slot_units(13)) == (4, 5)
    assert (row_units(7), slot_units(7)) == (3, 3)
    for K in (7, 13):
        for o in range(0, 8, 2):
            assert (o + ES * K + 7) // 8 <= row_units(K)
