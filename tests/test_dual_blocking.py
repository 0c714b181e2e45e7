"""The blockings of the one-pass kernel over an activation (dY for dY·B and dYᵀ·XA, X for
X·Aᵀ or for dA), checked on the CPU for the library's own choices.  The kernel's grid is
a × b blocks of row_tiles × 64 rows by col_tiles × 256 columns; every block writes the
fp32 partials of its rows and columns, and the finalize kernels add a (or b) partials per
output row.  So the blocks must tile the activation with none empty (an empty block
would leave its partials unwritten), fit one wave of the GPU, and keep the T accumulator
of a block within its 16 row tiles of shared memory."""
import itertools

import pytest

import qlora_linear_b200 as q
from synth import CONFIGS

SMS = 148


def cdiv(a, b):
    return (a + b - 1) // b


def shapes():
    out = set()
    for name in ("c0", "c1", "c2", "c3", "c4"):
        for c in CONFIGS[name]:
            out.add((c.M, c.N, c.r))   # dY [M, N]
            out.add((c.M, c.K, c.r))   # X [M, K]
    for M, C, r in itertools.product([64, 100, 300, 2000, 4000, 6000, 8100, 65536, 131072],
                                     [64, 264, 1088, 2112, 4160, 14336], [8, 16]):
        out.add((M, C, r))
    return sorted(out)


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_blockings_tile_the_activation_without_empty_blocks(mode):
    used = 0
    for M, C, r in shapes():
        ok, (a, b, rt, ct) = q.lora_testing_dual_blocking(M, C, r, mode)
        if r > 16:
            assert ok == 0
        if not ok:
            continue
        used += 1
        ntr, ntc = cdiv(M, 64), cdiv(C, 256)
        assert 1 <= rt <= 16 and 1 <= ct <= ntc, (M, C, r, a, b, rt, ct)
        assert a == cdiv(ntr, rt) and b == cdiv(ntc, ct), (M, C, r, a, b, rt, ct)
        assert a * b <= SMS
        # the last row block and the last column block still hold a tile
        assert (a - 1) * rt < ntr and (b - 1) * ct < ntc
    assert used >= 20


def test_blocking_is_used_where_it_pays_only():
    # the tiny configuration keeps the cp.async passes; the large ones stream
    assert q.lora_testing_dual_blocking(256, 512, 8, 0)[0] == 0
    assert q.lora_testing_dual_blocking(16384, 14336, 16, 0)[0] == 1
    assert q.lora_testing_dual_blocking(16384, 4096, 16, 1)[0] == 1
    assert q.lora_testing_dual_blocking(16384, 4096, 16, 2)[0] == 1
    assert q.lora_testing_dual_blocking(16384, 4096, 32, 0)[0] == 0
    assert q.lora_testing_dual_blocking(16384, 4096, 16, 3) == (-1, (0, 0, 0, 0))
