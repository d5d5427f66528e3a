"""Host-side pieces of the block-sparse path: the pair count behind its FLOP figure and the
benchmark's layout generator.

The pair count (accounting.block_sparse_pairs, closed-form per block row) is checked against
enumeration from the set definitions (visible_set, written in the oracle pins from the mask
definitions) on every mask kind with Nq != Nk both ways, small blocks and both layout forms.
"""

import numpy as np
import pytest

import synth
from exact_io_aware_82_b200 import accounting as acc

from .test_oracle_pins import visible_set

CASES = [(m, w, s) for m, w, s in ((0, 0, 0), (1, 0, 0), (2, 3, 2), (2, 1, 0), (2, 7, 9), (3, 2, 1),
                                   (3, 0, 3))]


@pytest.mark.parametrize("mask,w,s", CASES)
def test_block_sparse_pairs_by_enumeration(mask, w, s):
    rng = np.random.default_rng(mask * 100 + w * 10 + s)
    for Nq, Nk, blk in ((10, 13, 3), (13, 10, 4), (9, 9, 2), (1, 7, 3), (7, 1, 2)):
        Hq = 3
        for heads in (1, Hq):
            bm = (rng.random((heads, -(-Nq // blk), -(-Nk // blk))) < 0.5).astype(np.uint8)
            want = 0
            for h in range(Hq):
                layout = bm[0 if heads == 1 else h]
                for i in range(Nq):
                    want += sum(1 for j in visible_set(i + Nk - Nq, Nk, mask, w, s)
                                if layout[i // blk, j // blk])
            got = acc.block_sparse_pairs(bm, Nq, Nk, mask, w, s, Hq=Hq, block=blk)
            assert got == want, (Nq, Nk, blk, heads, got, want)


def test_every_block_selected_counts_the_dense_pairs():
    for mask, w, s in CASES:
        for Nq, Nk in ((300, 300), (200, 450), (450, 200)):
            bm = np.ones((1, -(-Nq // 128), -(-Nk // 128)), np.uint8)
            assert acc.block_sparse_pairs(bm, Nq, Nk, mask, w, s, Hq=2) == \
                2 * acc.visible_pairs(Nq, Nk, mask, w, s)


def test_bigbird_layout():
    bm = synth.block_layout_bigbird(11, 256, 256, 3)
    assert bm.shape == (1, 256, 256) and bm.dtype == np.uint8
    assert np.array_equal(bm, synth.block_layout_bigbird(11, 256, 256, 3))  # seeded
    assert np.all(bm[0, 0] == 1) and np.all(bm[0, :, 0] == 1)
    for qt in range(256):
        assert np.all(bm[0, qt, max(0, qt - 1):qt + 2] == 1)
        assert 3 <= bm[0, qt].sum() <= 7 or qt == 0
    # about (3 band + 1 global column + 3 random) / 256 of the blocks, plus the global row
    assert 0.02 < bm.mean() < 0.035
