"""The packed weight layout of the synthetic-backbone projections (include/oda_backbone.h),
checked on the CPU: the header's formula must place every element of a matrix exactly once
inside the matrix's own storage, keep each 8-column chunk (16 bytes) contiguous, keep a tile's
K chunk of 512 columns in one 16 KiB block, and put the 8 rows of an ldmatrix read at one column
in 8 distinct 16-byte slots of a 128-byte bank window.  The GPU test compares the pack kernel
with the same formula bit for bit."""
import numpy as np
import pytest

from helpers import packed_index


@pytest.mark.parametrize("rows,cols", [(16, 512), (32, 1024), (48, 1536), (4096, 2048), (2048, 6144)])
def test_packed_index_is_a_bijection_with_contiguous_chunks(rows, cols):
    idx = packed_index(rows, cols)
    flat = np.sort(idx.reshape(-1))
    assert np.array_equal(flat, np.arange(rows * cols))
    # each 8-column chunk of a row stays contiguous and 16-byte aligned
    ch = idx.reshape(rows, cols // 8, 8)
    assert np.all(np.diff(ch, axis=2) == 1)
    assert np.all(ch[:, :, 0] % 8 == 0)
    # the 16 rows x 512 columns of a (tile, K chunk) form one contiguous 8192-element block
    blk = idx.reshape(rows // 16, 16, cols // 512, 512).transpose(0, 2, 1, 3).reshape(-1, 16 * 512)
    assert np.all(blk.max(axis=1) - blk.min(axis=1) == 16 * 512 - 1)
    assert np.all(blk.min(axis=1) % 8192 == 0)


def test_packed_rows_of_one_column_hit_distinct_bank_slots():
    idx = packed_index(16, 512)
    for col in range(0, 512, 8):
        for r0 in (0, 8):
            slots = {(int(idx[r, col]) * 2 % 128) // 16 for r in range(r0, r0 + 8)}
            assert len(slots) == 8, (col, r0)
