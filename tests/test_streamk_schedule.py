"""The stream-K schedule of the GEMMs, checked on the CPU for the library's own choices.

For each shape, the library reports how many output tiles it shares out as pieces
(lora_testing_gemm_streamk); the rest of the schedule follows from the tile shape of the
weight's format.  This test walks every CTA pair's work units the way the kernels do
(whole tiles first, then an equal share of the remaining tiles' fills laid end to end)
and checks the invariants the kernels and the fixup kernel rely on: every fill of every
tile is computed exactly once; a tile computed whole has no piece; each pair writes at
most two slots (its first piece to slot 2p, its last to 2p + 1); and the fixup, reading
the pair boundaries alone, gathers exactly the pieces of every cut tile, in pair order,
with one owner per cut tile.
"""
import pytest

import qlora_linear_b200 as q

PAIRS = 74


def cdiv(a, b):
    return (a + b - 1) // b


def tile_shape(M, Nout, Kred, r, quantized):
    rows, bk = (512, 64) if quantized else (256, 128)
    tiles = cdiv(M, rows) * cdiv(Nout, 256)
    fills = cdiv(Kred, bk) + ((cdiv(r, 64) if quantized else 1) if r > 0 else 0)
    return tiles, fills


def walk(p, ntiles, L, dp_tiles):
    """Work units of pair p: (tile, first fill, end fill, slot or -1)."""
    units = []
    for k in range(dp_tiles // PAIRS):
        units.append((p + k * PAIRS, 0, L, -1))
    F = (ntiles - dp_tiles) * L
    g0, g1 = p * F // PAIRS, (p + 1) * F // PAIRS
    g = g0
    while g < g1:
        tr, f0 = divmod(g, L)
        f1 = min(L, f0 + (g1 - g))
        slot = -1 if (f0 == 0 and f1 == L) else (2 * p if g == g0 else 2 * p + 1)
        units.append((dp_tiles + tr, f0, f1, slot))
        g += f1 - f0
    return units


def fixup_plan(ntiles, L, dp_tiles):
    """Cut tile -> slots in the order the fixup adds them, from the boundaries alone."""
    F = (ntiles - dp_tiles) * L
    plan = {}
    for p in range(1, PAIRS):
        b = p * F // PAIRS
        if b % L == 0:
            continue
        ts = (b // L) * L
        if (p - 1) * F // PAIRS > ts:
            continue
        t = dp_tiles + b // L
        assert t not in plan, "two owners for one cut tile"
        slots = []
        for qq in range(p - 1, PAIRS):
            gq = qq * F // PAIRS
            if gq >= ts + L:
                break
            slots.append(2 * qq if gq >= ts else 2 * qq + 1)
        plan[t] = slots
    return plan


SHAPES = [
    # M, Nout, Kred, r, fmt
    (512, 8192, 8192, 16, q.LORA_W_BLOCK4),
    (512, 28672, 8192, 16, q.LORA_W_BLOCK4),
    (512, 8192, 28672, 128, q.LORA_W_BLOCK4),
    (8192, 4096, 14336, 16, q.LORA_W_BLOCK4),
    (4096, 8192, 8192, 64, q.LORA_W_INT8),
    (513, 1024, 8192, 64, q.LORA_W_FP8_E4M3),
    (300, 2048, 8256, 16, q.LORA_W_BLOCK4),
    (1100, 2048, 6400, 16, q.LORA_W_BLOCK4),
    (512, 28672, 8192, 16, q.LORA_W_BF16),
    (300, 2048, 8192, 32, q.LORA_W_BF16),
    (250, 2048, 19200, 8, q.LORA_W_BF16),
    (300, 4104, 8192, 16, q.LORA_W_BF16),
    (100, 1024, 65536, 8, q.LORA_W_BF16),
    (2000, 3072, 12288, 48, q.LORA_W_BF16),
]


@pytest.mark.parametrize("M,Nout,Kred,r,fmt", SHAPES)
def test_streamk_walk_covers_every_fill_once(M, Nout, Kred, r, fmt):
    quantized = fmt != q.LORA_W_BF16
    ntiles, L = tile_shape(M, Nout, Kred, r, quantized)
    shared = q.lora_testing_gemm_streamk(M, Nout, Kred, r, fmt)
    if shared == 0:
        pytest.skip("whole tiles for this shape")
    dp_tiles = ntiles - shared
    assert 0 <= dp_tiles < ntiles and dp_tiles % PAIRS == 0
    assert shared * L >= 4 * PAIRS  # every pair's range holds four fills or more (the kernels need one)

    cover = {t: [] for t in range(ntiles)}
    for p in range(PAIRS):
        units = walk(p, ntiles, L, dp_tiles)
        slots = [u[3] for u in units if u[3] >= 0]
        assert len(slots) == len(set(slots)) <= 2
        assert all(s in (2 * p, 2 * p + 1) for s in slots)
        for t, f0, f1, s in units:
            assert 0 <= t < ntiles and 0 <= f0 < f1 <= L
            cover[t].append((f0, f1, s, p))

    plan = fixup_plan(ntiles, L, dp_tiles)
    for t, pieces in cover.items():
        pieces.sort()
        pos = 0
        for f0, f1, _, _ in pieces:
            assert f0 == pos
            pos = f1
        assert pos == L
        if len(pieces) == 1 and pieces[0][2] == -1:
            assert t not in plan
        else:
            assert all(s >= 0 for _, _, s, _ in pieces)
            assert plan.get(t) == [s for _, _, s, _ in sorted(pieces, key=lambda x: x[3])]
    assert set(plan) == {t for t, pcs in cover.items() if not (len(pcs) == 1 and pcs[0][2] == -1)}


def test_some_shapes_take_streamk():
    taken = [s for s in SHAPES if q.lora_testing_gemm_streamk(*s) > 0]
    assert len(taken) >= 10
