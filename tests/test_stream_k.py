"""The stream-K partition arithmetic of the decode and prefill kernels, checked
by brute force on the CPU (test infrastructure).

Both kernels flatten their work into units (decode: (item, 64-key tile);
prefill: (128-row tile, 128-key block)) and give CTA c of C the units
[c W / C, (c + 1) W / C).  A CTA walks its range item by item; an item cut by
a range boundary is finished by the last of its CTAs, and each CTA stores its
partial record in slot c - (first CTA of the item).  Checked here: the
closed-form owner of a unit, ((t + 1) C - 1) / W, is the CTA whose range holds
it; every unit is visited exactly once; a segment is a whole item exactly when
one CTA holds the item; slots stay below the part count the workspace is sized
for.
"""

import pytest


def owner(t, W, C):
    return ((t + 1) * C - 1) // W


def ranges(W, C):
    return [(c * W // C, (c + 1) * W // C) for c in range(C)]


@pytest.mark.parametrize("W,C", [(1, 1), (7, 7), (8192, 148), (130, 130), (131, 130), (16384, 148), (149, 148),
                                 (10, 3), (1000, 148), (5 * 148 + 1, 148)])
def test_owner_formula_is_the_cta_holding_the_unit(W, C):
    for c, (lo, hi) in enumerate(ranges(W, C)):
        assert hi > lo  # W >= C: no CTA is idle
        for t in range(lo, hi):
            assert owner(t, W, C) == c


def _walk(sizes, C):
    """Split the items (unit counts `sizes`) over C CTAs; yield (cta, item, lo, hi, parts, slot)."""
    starts = [0]
    for n in sizes:
        starts.append(starts[-1] + n)
    W = starts[-1]
    for c, (f, f_end) in enumerate(ranges(W, C)):
        while f < f_end:
            it = max(i for i in range(len(sizes)) if starts[i] <= f)
            lo = f - starts[it]
            hi = min(sizes[it], lo + (f_end - f))
            first = owner(starts[it], W, C)
            last = owner(starts[it] + sizes[it] - 1, W, C)
            yield c, it, lo, hi, last - first + 1, c - first
            f += hi - lo


def _check_cover(sizes, C, max_parts):
    seen = set()
    for c, it, lo, hi, parts, slot in _walk(sizes, C):
        assert hi > lo
        for u in range(lo, hi):
            assert (it, u) not in seen
            seen.add((it, u))
        assert 0 <= slot < parts <= max_parts, (it, parts, max_parts)
        assert (lo == 0 and hi == sizes[it]) == (parts == 1)
    assert len(seen) == sum(sizes)


@pytest.mark.parametrize("S,N,Hq,Hkv,L", [(32, 3, 12, 2, 8192), (16, 2, 16, 8, 1024), (1, 3, 12, 2, 4097),
                                          (1, 5, 8, 1, 300), (4, 8, 16, 8, 65536 // 16)])
def test_decode_items_split_over_the_ctas(S, N, Hq, Hkv, L):
    R = N * (Hq // Hkv)
    n_rg = -(-R // 32)
    nt = -(-L // 64)
    items = S * Hkv * n_rg
    W = items * nt
    C = min(W, 148)
    whole = items <= 148 and nt <= -(-W // C) + 12  # the planner's whole-item rule
    if whole:
        C = items
    # the workspace holds, per item, as many records as the most CTAs any item touches
    touching = [0] * items
    for lo, hi in ranges(W, C):
        for it in range(lo // nt, (hi - 1) // nt + 1):
            touching[it] += 1
    assert not whole or max(touching) == 1  # one CTA per item: nothing to merge
    _check_cover([nt] * items, C, max(touching))


@pytest.mark.parametrize("T,L0,G,Hkv,N", [(512, 16384, 2, 8, 4), (100, 300, 2, 2, 2), (1, 77, 2, 4, 2),
                                          (257, 129, 1, 2, 1), (130, 4096, 2, 8, 2), (1000, 0, 8, 2, 3),
                                          (64, 0, 1, 8, 3), (90, 500, 2, 2, 2), (64, 8192, 6, 2, 3),
                                          (300, 1000, 5, 2, 2), (9, 40, 128, 1, 1)])
def test_prefill_tiles_split_over_the_ctas(T, L0, G, Hkv, N):
    tm = 128 // G  # chunk tokens per 128-row tile (G heads each; 128 mod G rows unused)
    n_tb = -(-T // tm)
    # key blocks a tile needs: up to the last key its last row sees (causal)
    nbs = [-(-(L0 + tb * tm + min(tm, T - tb * tm)) // 128) for tb in range(n_tb)]
    sizes = nbs * (Hkv * N)  # tiles ordered (agent, KV head) major, chunk tile minor
    W = sum(sizes)
    C = min(W, 148)
    # the planner's bound on the CTAs sharing a tile: the longest tile over the fewest blocks per CTA, plus one
    max_parts = -(-max(nbs) // (W // C)) + 1
    _check_cover(sizes, C, max_parts)
