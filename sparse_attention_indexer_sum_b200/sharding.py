"""Sharing one long prefill out over ranks by query rows.

Every row of the stack is independent once its keys are there: row t's indexer
scores keys 0..t, its top-k and attention read only its own scores and index set.
So W ranks can each run `ic_layer_stack_rows` on their own rows. They need all
of the keys (k_idx, kv) and no communication, and each gathers only if a
consumer needs every row.

The work is causal: row t's indexer scores t + 1 keys, so contiguous ranges
would give the last rank the most work. The zig-zag plan cuts the L rows into 2W
equal chunks; rank r takes chunks r and 2W - 1 - r, one early and one late,
which evens out the causal pairs.
"""
from __future__ import annotations


def zigzag_row_ranges(L: int, world: int, rank: int) -> list:
    """[(row0, rows), ...] of `rank`: chunk rank and chunk 2 * world - 1 - rank of
    the 2 * world near-equal chunks of [0, L) (empty chunks left out)."""
    if world < 1 or not 0 <= rank < world or L < 0:
        raise ValueError("need world >= 1, 0 <= rank < world, L >= 0")
    n = 2 * world
    bounds = [L * i // n for i in range(n + 1)]
    out = []
    for c in (rank, n - 1 - rank):
        r0, r1 = bounds[c], bounds[c + 1]
        if r1 > r0:
            out.append((r0, r1 - r0))
    return out


def causal_pairs(row0: int, rows: int) -> int:
    """(query, key) pairs the indexer scores for rows [row0, row0 + rows):
    sum over t of (t + 1)."""
    return rows * (2 * row0 + rows + 1) // 2
