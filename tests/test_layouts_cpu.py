"""Host-side weight layouts the kernels rely on (no GPU): the paired q/k row order that puts every rotate-half
pair of RoPE in one 32-row block, and the 16-row gate/up interleave of the fused SwiGLU weight."""
import numpy as np
import pytest

from invariant_deterministic_full_b200 import model


@pytest.mark.parametrize("d", [64, 128])
def test_paired_rows_is_a_permutation_keeping_rope_pairs_together(d):
    r = model.paired_rows(d)
    assert sorted(r.tolist()) == list(range(d))
    half = d // 2
    for i in range(half):  # element i and its rotate-half partner i + d/2: same 32-row block, rows k and k + 16
        a, b = r[i], r[i + half]
        assert a // 32 == b // 32 and b == a + 16 and a % 32 < 16


def test_pair_heads_moves_rows_within_each_head():
    d, H, n = 64, 8, 3
    w = np.arange(n * d * H, dtype=np.float32).reshape(n * d, H)
    p = model.pair_heads(w, d)
    r = model.paired_rows(d)
    for h in range(n):
        for i in range(d):
            assert np.array_equal(p[h * d + r[i]], w[h * d + i])


def test_interleave_gu_granules():
    F, H, g = 64, 4, model.GU_INTERLEAVE
    wg = np.arange(F * H, dtype=np.float32).reshape(F, H)
    wu = -wg - 1
    out = model.interleave_gu(wg, wu)
    assert out.shape == (2 * F, H)
    for blk in range(F // g):
        assert np.array_equal(out[2 * g * blk:2 * g * blk + g], wg[g * blk:g * blk + g])
        assert np.array_equal(out[2 * g * blk + g:2 * g * (blk + 1)], wu[g * blk:g * blk + g])
