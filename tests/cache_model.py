"""Host model of the row cache's replacement policy (test helper).

Direct-mapped, slot = row mod slots, tag = row + 1.  Per call, over the batch's distinct rows
of one table: a row whose slot holds it is a hit and pins the slot; each other slot is written
by the smallest distinct row that maps to it, unless a hit pinned it; rows outside the table
never enter the cache.  This mirrors the policy documented for engram_stage_rows_cached.
"""
from __future__ import annotations

import numpy as np


class CacheModel:
    def __init__(self, n_tables: int, slots: int, rows):
        self.slots = slots
        self.rows = list(rows)
        self.tags = [np.zeros(slots, dtype=np.int64) for _ in range(n_tables)]

    def step(self, idx: np.ndarray):
        """idx: [n_tok, H] row ids of one call.  Returns the hits per table."""
        hits = []
        for h, tags in enumerate(self.tags):
            distinct = np.unique(idx[:, h])
            slot = distinct % self.slots
            hit = tags[slot] == distinct + 1
            pinned = set(slot[hit].tolist())
            winners = {}
            for r, s, is_hit in zip(distinct.tolist(), slot.tolist(), hit.tolist()):
                if is_hit or s in pinned or r >= self.rows[h]:
                    continue
                if s not in winners or r < winners[s]:
                    winners[s] = r
            for s, r in winners.items():
                tags[s] = r + 1
            hits.append(int(hit.sum()))
        return hits
