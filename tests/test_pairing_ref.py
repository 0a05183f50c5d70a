"""The tests' restatement of the tile-pairing schedule, on CPU: hand-worked
tables and the validity of its tables on random rows."""
import numpy as np

from pairing_ref import check_table, pair_head, pair_query_blocks
from parity import random_csr


def test_pairing_reference_pairs_identical_rows():
    """Blocks with identical kept sets pair up; order by lower block; leftovers ascending."""
    rows = [[0, 3], [0, 4], [0, 5], [0, 5], [0, 4], [0, 3], [0, 6]]
    assert pair_head(rows) == [(0, 5), (1, 4), (2, 3), (6, -1)]
    # every block keeps the same set: ties go to the nearest, lower block first
    assert pair_head([[0, 1]] * 6) == [(0, 1), (2, 3), (4, 5)]
    rp = np.array([0, 2, 4, 6, 8, 10, 12, 14], np.int32)
    ci = np.array([x for r in rows for x in r], np.int32)
    t = pair_query_blocks(rp, ci, 1, 7, 64, 4)
    check_table(t, 7, 64)
    assert t.tolist() == [[[0, 5], [1, 4], [2, 3], [6, -1]]]
    t128 = pair_query_blocks(rp, ci, 1, 7, 128, 7)
    check_table(t128, 7, 128)


def test_pairing_reference_on_random_rows_is_a_valid_table():
    for nb, keep in ((1, 1), (5, 2), (40, 6), (301, 9)):
        rp, ci = random_csr(2, nb, keep, seed=nb, forced=min(1, keep))
        check_table(pair_query_blocks(rp, ci, 2, nb, 64, (nb + 1) // 2), nb, 64)
