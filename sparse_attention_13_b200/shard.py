"""Causally balanced query sharding of one sequence across ranks.

Query rows are independent once every rank holds the per-layer caches (the
indexer keys and the latent rows), so one long prefill can be split by query
rows with no data-path collective.  Row t costs about t indexer pairs and
min(t, k) attention rows, so contiguous equal slices would leave the last rank
with most of the work.  The zig-zag split cuts [0, L) into 2G equal chunks and
gives rank r chunks r and 2G - 1 - r: one early (cheap) and one late (costly)
chunk, which evens out the sum of t over ranks.  Each chunk runs as a chunked
prefill (start_pos = the chunk's first row, Lq = its length).
"""
from __future__ import annotations


def chunk_bounds(L: int, n_chunks: int) -> list[tuple[int, int]]:
    """[start, end) of n_chunks near-equal contiguous chunks of [0, L)."""
    if L < 1 or n_chunks < 1:
        raise ValueError("L and n_chunks must be positive")
    cuts = [c * L // n_chunks for c in range(n_chunks + 1)]
    return [(cuts[c], cuts[c + 1]) for c in range(n_chunks)]


def zigzag_chunks(L: int, world: int, rank: int) -> list[tuple[int, int]]:
    """The (start_pos, Lq) chunks of query rows that `rank` of `world` owns:
    chunks rank and 2*world - 1 - rank of 2*world, empty ones dropped."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    b = chunk_bounds(L, 2 * world)
    mine = [b[rank], b[2 * world - 1 - rank]]
    return [(s, e - s) for (s, e) in mine if e > s]


def indexer_pairs(start: int, n: int) -> int:
    """Causal (t, s) pairs the rows start .. start + n - 1 score: sum of t."""
    return n * start + n * (n - 1) // 2


def attention_rows(start: int, n: int, k: int) -> int:
    """Selected (t, r) entries of those rows: sum of min(t, k)."""
    lo = min(max(k - start, 0), n)          # rows with t < k
    return indexer_pairs(start, lo) + (n - lo) * k
