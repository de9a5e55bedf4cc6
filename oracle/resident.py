"""Resident-page reuse for the streamed working set -- CPU oracle.

Test infrastructure only.

The KVMem reproduction (lcz.me/topic/1972, recall section) keeps a per-request GPU
working set of 128-token blocks and refreshes it from host RAM as the retrieval query
moves; the Adaptive KV Streaming announcement (wqu.guru, problem statement) streams the
bounded working set over PCIe.  A block that is already on the GPU need not cross PCIe
again.  The pages do not say how device slots are reused; the reading used here (the
plainest deterministic one):

* per unit (one layer and KV head) a fixed pool of `n_slots` device slots; each slot holds
  one logical block or is empty, and each block sits in at most one slot;
* a selected block that is resident keeps its slot (a hit);
* the free slots are the empty ones and the ones holding a block that is not selected;
* the selected blocks that are not resident (the misses), in ascending block order, take
  the free slots in ascending slot order; a block evicted this way is no longer resident;
* only misses are copied; the decode page list gives, for every selected block in the
  selection's order, the slot that holds it.
"""
from __future__ import annotations

import numpy as np


def resident_update(selected, slot_of_block, block_of_slot):
    """One update of a unit's slot pool.

    selected: ascending logical block ids (int); slot_of_block: int array [n_blocks], -1 when
    not resident; block_of_slot: int array [n_slots], -1 when empty (both updated in place).
    Returns (page_slots [len(selected)], copies [(block, slot), ...] in ascending block
    order).  Needs n_slots >= len(selected).
    """
    selected = [int(b) for b in selected]
    assert selected == sorted(set(selected)), "selection must be ascending and unique"
    assert len(block_of_slot) >= len(selected), "not enough slots"
    chosen = set(selected)
    misses = [b for b in selected if slot_of_block[b] < 0]
    free = [s for s in range(len(block_of_slot)) if block_of_slot[s] < 0 or int(block_of_slot[s]) not in chosen]
    copies = []
    for b, s in zip(misses, free):
        old = int(block_of_slot[s])
        if old >= 0:
            slot_of_block[old] = -1
        block_of_slot[s] = b
        slot_of_block[b] = s
        copies.append((b, s))
    page_slots = np.array([slot_of_block[b] for b in selected], dtype=np.int64)
    return page_slots, copies
