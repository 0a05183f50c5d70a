"""Plain restatement of rt_pair_query_blocks's schedule, for the tests.

The pairing is not part of the method (any table that lists each query
block once gives the same attention output); it is a deterministic heuristic
that the GPU must reproduce exactly, so the tests compare its table entry by
entry with this one.  The steps follow the rule stated in
include/rettention.h:
  1. for each query block i, the `cands` best partners j with
     |i - j| <= `window`, by (overlap desc, |i - j| asc, j asc), where overlap
     is the number of key blocks both rows keep;
  2. `rounds` rounds: every unpaired block picks its first unpaired
     candidate; two blocks that pick each other become a pair;
  3. tiles: the pairs by their lower block, then the unpaired blocks two by
     two in ascending order (-1 for an odd last half).
Block size 128: tile t = (t, -1).  Row entries outside [0, n_blocks) are
ignored and a row is cut to n_blocks entries, as the kernel does.
"""
import numpy as np

CANDS, ROUNDS, WINDOW = 8, 8, 224


def _rows(row_ptr, col_idx, h, nb):
    rows = []
    for i in range(nb):
        s, e = int(row_ptr[h * nb + i]), int(row_ptr[h * nb + i + 1])
        n = max(0, min(e - s, nb))
        rows.append([int(x) for x in col_idx[s:s + n] if 0 <= int(x) < nb])
    return rows


def pair_head(rows, cands=CANDS, rounds=ROUNDS, window=WINDOW):
    """Tiles (a, b) of one head from its kept rows (lists of key blocks)."""
    nb = len(rows)
    sets = [set(r) for r in rows]
    cand = []
    for i in range(nb):
        keys = []
        for j in range(max(0, i - window), min(nb - 1, i + window) + 1):
            if j != i:
                ov = len(sets[i] & sets[j])
                keys.append((-ov, abs(i - j), j))
        keys.sort()
        cand.append([j for _, _, j in keys[:cands]])
    partner = [-1] * nb
    for _ in range(rounds):
        choice = []
        for i in range(nb):
            pick = -1
            if partner[i] < 0:
                pick = next((j for j in cand[i] if partner[j] < 0), -1)
            choice.append(pick)
        for i in range(nb):
            j = choice[i]
            if j > i and choice[j] == i:
                partner[i], partner[j] = j, i
    tiles = [(i, partner[i]) for i in range(nb) if partner[i] > i]
    alone = [i for i in range(nb) if partner[i] < 0]
    tiles += [(alone[t], alone[t + 1] if t + 1 < len(alone) else -1) for t in range(0, len(alone), 2)]
    return tiles


def pair_query_blocks(row_ptr, col_idx, bh, nb, bs, n_tiles):
    """int32 [bh, n_tiles, 2] table, as rt_pair_query_blocks writes it."""
    out = np.full((bh, n_tiles, 2), -1, np.int32)
    if bs != 64:
        t = np.arange(n_tiles)
        out[:, :, 0] = np.where(t < nb, t, -1)
        return out
    for h in range(bh):
        tiles = pair_head(_rows(row_ptr, col_idx, h, nb))
        assert len(tiles) == n_tiles
        out[h] = np.array(tiles, np.int32).reshape(n_tiles, 2)
    return out


def check_table(table, nb, bs):
    """Every query block of every head in exactly one tile half; -1 elsewhere."""
    bh, n_tiles, _ = table.shape
    for h in range(bh):
        got = table[h].reshape(-1)
        blocks = sorted(int(x) for x in got if x >= 0)
        assert blocks == list(range(nb)), f"head {h}: blocks {blocks[:8]}..."
        if bs != 64:
            assert (table[h, :, 1] == -1).all()
