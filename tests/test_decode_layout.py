"""Properties of the shared-memory word layout of the warp-MMA decode kernel (CPU).

The kernel stores a warp's 32 rows x CW packed words (CW = 16, or 8 for 16 tokens) at
row * CW + (w ^ swizzle(row)) and reads, per fragment, word w of 8 consecutive rows.  The
swizzle is restated here from mma_decode_block.cuh (word_slot) and checked for the three
properties the kernel relies on: a permutation of each row's words, 16-byte groups kept
whole (cp.async writes 4 words at once), and the 8 rows of a fragment read in 8 different
banks.
"""
import pytest


def word_slot(row: int, w: int, cw: int) -> int:
    if cw == 16:
        return row * cw + (w ^ (4 * ((row >> 1) & 3)))
    return row * cw + (w ^ (4 * ((row >> 2) & 1)))


@pytest.mark.parametrize("cw", [16, 8])
def test_swizzle_is_a_permutation_of_each_row(cw):
    for row in range(32):
        slots = sorted(word_slot(row, w, cw) - row * cw for w in range(cw))
        assert slots == list(range(cw))


@pytest.mark.parametrize("cw", [16, 8])
def test_swizzle_keeps_16_byte_groups(cw):
    for row in range(32):
        for q in range(cw // 4):
            base = word_slot(row, 4 * q, cw)
            assert base % 4 == 0
            assert [word_slot(row, 4 * q + i, cw) for i in range(4)] == [base + i for i in range(4)]


@pytest.mark.parametrize("cw", [16, 8])
def test_fragment_rows_hit_distinct_banks(cw):
    # rows 16 rt + gq + 8 h for gq = 0..7 are read together (one word w per lane group)
    for rt in range(2):
        for h in range(2):
            for w in range(cw):
                banks = {word_slot(16 * rt + gq + 8 * h, w, cw) % 32 for gq in range(8)}
                assert len(banks) == 8
