"""Host-side partition of one indexer layer over the ranks of a job.

The indexer needs no exchange between GPUs: every query row's top-k depends
only on its own query, the shared keys and its causal prefix ("PaperTrace
2.2.2 MISA, LISA and ResMiSA", section 2.3 "distributed execution": replicate
the light indexer so every device computes the same token sets without
communicating scores).  So one layer is split by query rows (prefill) or by
sequences (decode); every rank holds the whole key cache and calls the library
on its own rows, and each output row stays on the rank that computed it.

Prefill work is causal: row t scores t + 1 keys.  Cutting the rows into
2 * world equal chunks and giving rank r chunks r and 2 * world - 1 - r (a
zigzag) pairs a short prefix with a long one, so every rank scores the same
number of (query, key) pairs up to one row's length.

Pure host arithmetic on sizes; nothing here touches a GPU or the method's
arithmetic.
"""
from __future__ import annotations

from typing import List, Tuple


def _bounds(n: int, parts: int) -> List[int]:
    """parts + 1 cut points splitting range(n) into near-equal chunks."""
    return [(i * n) // parts for i in range(parts + 1)]


def prefill_row_ranges(n_q: int, world: int, rank: int) -> List[Tuple[int, int]]:
    """Query rows of one prefill sequence that `rank` computes, as (start, count)
    ranges in row order: chunk `rank` and chunk `2 * world - 1 - rank` of
    2 * world near-equal chunks.  Empty ranges are dropped."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if world == 1:
        return [(0, n_q)] if n_q > 0 else []
    cut = _bounds(n_q, 2 * world)
    out = []
    for c in (rank, 2 * world - 1 - rank):
        if cut[c + 1] > cut[c]:
            out.append((cut[c], cut[c + 1] - cut[c]))
    return out


def decode_seq_range(batch: int, world: int, rank: int) -> Tuple[int, int]:
    """Sequences (start, count) of a decode batch that `rank` computes."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    cut = _bounds(batch, world)
    return cut[rank], cut[rank + 1] - cut[rank]


def causal_pairs(ranges: List[Tuple[int, int]], pos0: int, k_len: int) -> int:
    """(query, key) pairs the rows of `ranges` score: row i sits at pos0 + i and
    scores min(pos0 + i + 1, k_len) keys."""
    total = 0
    for start, count in ranges:
        for i in range(start, start + count):
            total += max(0, min(pos0 + i + 1, k_len))
    return total
