"""Host-side work split of the decode-attention kernel (integer arithmetic,
no GPU).

Every (batch, KV head) unit has tpu tiles.  Unit u occupies positions
[u*(tpu+wb), (u+1)*(tpu+wb)) of a weighted line: the first wb positions stand
for the fixed cost of starting a unit, tile k sits at u*(tpu+wb) + wb + k.
CTA i of C owns the tiles whose positions fall in [i*W/C, (i+1)*W/C),
W = units*(tpu+wb).  The host and the kernel (csrc/kvq_internal.h) use the
two formulas below; these checks show that every tile is owned exactly once,
that ownership ranges are contiguous and agree with the per-tile owner
formula, that the CTAs touching a unit are exactly [first, last], and that
their number never exceeds floor(C / units) + 2, the bound the workspace is
sized by.  With wb = 0 it is the plain even split.
"""
import pytest


def first_tile_at(p, units, tpu, wb):
    span = tpu + wb
    u = p // span
    if u >= units:
        return units * tpu
    o = p - u * span
    return u * tpu + (0 if o <= wb else o - wb)


def cta_of_tile(t, tpu, wb, W, C):
    pos = t + (t // tpu + 1) * wb
    return ((pos + 1) * C + W - 1) // W - 1


@pytest.mark.parametrize("wb", [0, 1, 2, 3, 4, 7])
@pytest.mark.parametrize("units", [1, 2, 3, 7, 64, 128])
@pytest.mark.parametrize("tpu", [1, 2, 3, 5, 129, 513])
def test_weighted_split_covers_and_bounds(units, tpu, wb):
    T = units * tpu
    W = units * (tpu + wb)
    for C in sorted({1, 2, 3, 7, 64, 148, 296, 1000, T, max(1, T - 1)}):
        if C > T:
            continue
        owner = [None] * T
        touching = {}
        for i in range(C):
            tb = first_tile_at(W * i // C, units, tpu, wb)
            te = first_tile_at(W * (i + 1) // C, units, tpu, wb)
            assert tb <= te
            for t in range(tb, te):
                assert owner[t] is None
                owner[t] = i
                assert cta_of_tile(t, tpu, wb, W, C) == i
            seg = tb
            while seg < te:
                u = seg // tpu
                touching.setdefault(u, []).append(i)
                seg = min(te, (u + 1) * tpu)
        assert None not in owner
        for u in range(units):
            first = cta_of_tile(u * tpu, tpu, wb, W, C)
            last = cta_of_tile(u * tpu + tpu - 1, tpu, wb, W, C)
            assert touching[u] == list(range(first, last + 1))
            assert last - first + 1 <= C // units + 2


def test_unit_start_weight_shortens_two_unit_ranges():
    """Each CTA's tiles plus the unit-start positions inside its range add up
    to its share of the weighted line, so a CTA that crosses into a new unit
    owns wb fewer tiles than a CTA of the same share that crosses none."""
    units, tpu, wb, C = 64, 129, 3, 296
    span = tpu + wb
    W = units * span
    crossing, plain = [], []
    for i in range(C):
        p0, p1 = W * i // C, W * (i + 1) // C
        tb = first_tile_at(p0, units, tpu, wb)
        te = first_tile_at(p1, units, tpu, wb)
        virtual = sum(1 for p in range(p0, p1) if p % span < wb)
        assert (te - tb) + virtual == p1 - p0
        n_units = len({t // tpu for t in range(tb, te)})
        if n_units == 2:
            crossing.append((te - tb, p1 - p0))
        elif virtual == 0:
            plain.append((te - tb, p1 - p0))
    assert crossing and plain
    for share in {s for _, s in crossing} & {s for _, s in plain}:
        assert max(n for n, s in crossing if s == share) == share - wb
        assert min(n for n, s in plain if s == share) == share
