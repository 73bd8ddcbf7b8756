"""Host-side model of the paged prefill kernel's per-CTA ranges (no GPU).

A CTA serves query rows [row0, row0 + 128) of one sequence (history hist, q_len
current tokens, a block-table row of `stride` entries of block_size positions). It is
active iff row0 < q_len; it loads 128-key sub-tiles 0 .. n_sub - 1 with
n_sub = ceil(key_end / 128), key_end = hist + min(row0 + 128, q_len), and row r masks
keys at or past its own limit hist + row0 + r + 1. This model restates those rules and
checks that every key a valid row may see is inside a loaded sub-tile, that no loaded
sub-tile reads past the sequence's positions or its table row, and that the kernel's
descriptor check (hist + q_len <= stride * block_size) is what keeps table reads in range.
"""

import random

import pytest

TILE = 128


def _check_cta(hist, q_len, row0, block_size, stride):
    assert row0 < q_len
    key_end = hist + min(row0 + TILE, q_len)
    n_sub = -(-key_end // TILE)
    for r in range(TILE):
        row = row0 + r
        if row >= q_len:
            continue                                  # not stored
        lim = hist + row + 1
        assert lim <= n_sub * TILE                    # every visible key is loaded
        assert lim <= hist + q_len                    # and exists in the sequence
    for j in range(n_sub):
        lb = (j * TILE) // block_size
        assert lb < stride                            # table reads stay in the row
        assert j * TILE < hist + q_len                # no sub-tile wholly past the sequence


@pytest.mark.parametrize("block_size", [128, 256, 384, 512])
def test_loaded_sub_tiles_cover_exactly_what_rows_see(block_size):
    rng = random.Random(block_size)
    for _ in range(400):
        hist, q_len = rng.randint(0, 5000), rng.randint(1, 1500)
        stride = -(-(hist + q_len) // block_size) + rng.randint(0, 2)
        assert hist + q_len <= stride * block_size    # the kernel's descriptor check
        for row0 in range(0, q_len, TILE):
            _check_cta(hist, q_len, row0, block_size, stride)
