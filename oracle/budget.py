"""Global block order and greedy memory-budget fill (oracle).

Test infrastructure: see the package docstring.

Follows: Review, Fig. 2 caption (the residual blocks of all weights of all layers
sit in one universal stack on storage; blocks are loaded when memory grows and
offloaded when it shrinks); Rebuttal A1.B (each weight's blocks are loaded and
offloaded in a presorted order); README "Evaluation" (``--max_memory_MB`` sets the
budget the loaded blocks must fit).

The pages do not print the sorting algorithm (Algorithm 1 of the paper).  Stand-in
reading: matrix w has an importance weight a_w (seeded, from ``workloads``); block
(w, i) (i = 0, 1, ... in the weight's own decomposition order) gets the key
(i + 1) * a_w; the global order sorts keys ascending, ties broken by matrix index.
The key grows with i for a fixed w, so the order keeps every weight's blocks in
prefix order, as a per-weight stack requires.  Parity unpinned for the key itself;
the prefix property and the budget fill are pinned by the tests.
"""
from __future__ import annotations

import numpy as np

MIB = 1 << 20


def global_order(weights: np.ndarray, blocks_per_matrix) -> list:
    """[(matrix, block)] sorted by key (block + 1) * weight, ties by matrix index."""
    weights = np.asarray(weights, dtype=np.float64)
    counts = np.broadcast_to(np.asarray(blocks_per_matrix), weights.shape)
    entries = []
    for w, (a, cnt) in enumerate(zip(weights, counts)):
        for i in range(int(cnt)):
            entries.append(((i + 1) * float(a), w, i))
    entries.sort(key=lambda e: (e[0], e[1], e[2]))
    return [(w, i) for (_, w, i) in entries]


def budget_fill(order, block_bytes_per_matrix, budget_mib: float) -> np.ndarray:
    """Per-matrix loaded block counts: the longest prefix of ``order`` whose
    cumulative record bytes stay within ``budget_mib`` MiB.

    Reading: the pages' "MB" for block sizes is MiB (the 7.56 MB block of an 8B
    model equals 7.5625 MiB; see pack.block_bytes), so budgets are MiB as well.
    """
    sizes = np.asarray(block_bytes_per_matrix, dtype=np.int64)
    n = np.zeros(sizes.shape[0], dtype=np.int64)
    limit = int(budget_mib * MIB)
    used = 0
    for (w, i) in order:
        if used + int(sizes[w]) > limit:
            break
        assert n[w] == i, "order must keep each matrix's blocks in prefix order"
        used += int(sizes[w])
        n[w] += 1
    return n
