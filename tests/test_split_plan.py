"""Host-side work split of the decode-attention kernel.

The kernel cuts every (batch, KV head) unit into tpu tiles, flattens the
units' tiles and gives CTA i the tiles [i*T/C, (i+1)*T/C).  The host and the
kernel both locate the CTA owning tile t as ((t+1)*C + T - 1)/T - 1 and size
the per-unit record slots as last - first + 1.  These checks (pure integer
arithmetic, no GPU) show that every tile is owned exactly once, that the
CTAs touching a unit are exactly [first, last], and that the slot count
never exceeds floor(C / units) + 2, the bound the workspace is sized by.
"""
import pytest


def cta_of_tile(t, T, C):
    return ((t + 1) * C + T - 1) // T - 1


@pytest.mark.parametrize("units", [1, 2, 3, 7, 64, 128])
@pytest.mark.parametrize("tpu", [1, 2, 3, 5, 129, 513])
def test_even_split_covers_and_bounds(units, tpu):
    T = units * tpu
    for C in sorted({1, 2, 3, 7, 64, 148, 296, 1000, T, max(1, T - 1)}):
        if C > T:
            continue
        owner = [None] * T
        touching = {}
        for i in range(C):
            tb, te = T * i // C, T * (i + 1) // C
            for t in range(tb, te):
                assert owner[t] is None
                owner[t] = i
                assert cta_of_tile(t, T, C) == i
            seg = tb
            while seg < te:
                u = seg // tpu
                touching.setdefault(u, []).append(i)
                seg = min(te, (u + 1) * tpu)
        assert None not in owner
        for u in range(units):
            first = cta_of_tile(u * tpu, T, C)
            last = cta_of_tile(u * tpu + tpu - 1, T, C)
            assert touching[u] == list(range(first, last + 1))
            assert last - first + 1 <= C // units + 2
