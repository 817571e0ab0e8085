"""Relabelling of physical blocks, for the invariance tests: the pages' block
table lets a sequence's blocks sit anywhere in the pool, so moving every block
to a new physical id (and rewriting the tables and slots to match) must leave
every sequence's logical content, and hence the attention output, unchanged.
Cache layout: [block][kv head][16][d]; slot = block * 16 + offset."""
from __future__ import annotations

import numpy as np

BLOCK_TOKENS = 16


def permute_pool(perm: np.ndarray, tables: np.ndarray, slots: np.ndarray, *caches):
    """Relabel physical blocks: block i moves to perm[i].  Returns the new
    tables, slots and caches; the logical content of every sequence is
    unchanged."""
    perm = np.asarray(perm, dtype=np.int64)
    t2 = np.where(tables >= 0, perm[np.clip(tables, 0, None)], tables).astype(np.int32)
    s2 = np.where(slots >= 0, perm[np.clip(slots, 0, None) // BLOCK_TOKENS] * BLOCK_TOKENS
                  + np.clip(slots, 0, None) % BLOCK_TOKENS, slots).astype(np.int64)
    out = []
    for c in caches:
        c2 = np.empty_like(c)
        c2[perm] = c
        out.append(c2)
    return (t2, s2, *out)
