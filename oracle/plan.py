"""Plan-side quantities by definition: pages, page lists, pair counts.

Test infrastructure only (see the package docstring).  Source: the KPage
abstract ("KPage: block-sparse attention for partially occupied 3D blocks",
zhuanzhiai.com, abstract paragraph): K/V are handled as 16-row pages that
hold at least one valid row, and its accounting sets the physical query-key
pair capacity of the tiles against the useful (allowed) pairs.

Definitions (readings stated where the pages are silent):

* A K page is 16 consecutive K/V slots; page ``p`` covers slots
  ``[16p, 16p + 16)`` (the last page may be short).  It is *valid* when at
  least one of its slots is not padded.  A Q block is 64 consecutive query
  slots.
* The canonical page list of (head, Q block) is the ascending list of pages
  ``p`` such that some query slot of the block may attend some slot of ``p``.
* The transposed list of (head, page) is the ascending list of Q blocks whose
  canonical list holds ``p``.
* Useful pairs U = number of allowed (query slot, key slot) pairs, summed over
  batch and heads.
* BSA-style physical pairs: 64 x 64 for every (Q block, K block of 64 slots)
  pair holding at least one allowed pair.
"""

from __future__ import annotations

import numpy as np

from .attention import token_mask


def page_valid_masks(group):
    """uint16 mask per 16-slot page: bit r set iff slot 16p + r exists and is not padded."""
    g = np.asarray(group)
    n_pages = -(-g.size // 16)
    padded = np.full(n_pages * 16, -1, dtype=np.int64)
    padded[:g.size] = g
    bits = (padded.reshape(n_pages, 16) >= 0).astype(np.uint32)
    return (bits << np.arange(16, dtype=np.uint32)).sum(axis=1).astype(np.uint16)


def canonical_pages(q_group, kv_group, A, qblock):
    """Ascending pages p with an allowed pair between Q block ``qblock`` and page p."""
    rows = np.arange(64 * qblock, min(64 * qblock + 64, len(q_group)))
    mask = token_mask(q_group, kv_group, A, rows)
    cols = np.nonzero(mask.any(axis=0))[0]
    return np.unique(cols // 16).astype(np.int32)


def transposed_qblocks(q_group, kv_group, A, page):
    """Ascending Q blocks whose canonical list holds ``page``."""
    n_qb = -(-len(q_group) // 64)
    keys = np.arange(16 * page, min(16 * page + 16, len(kv_group)))
    out = []
    for qb in range(n_qb):
        rows = np.arange(64 * qb, min(64 * qb + 64, len(q_group)))
        m = token_mask(q_group, kv_group, A, rows)
        if m[:, keys].any():
            out.append(qb)
    return np.asarray(out, dtype=np.int32)


def useful_pairs_bruteforce(q_group, kv_group, A):
    """Count of allowed (i, j) for one head from the explicit token mask."""
    return int(token_mask(q_group, kv_group, A).sum())


def useful_pairs_closed_form(q_group, kv_group, row_ptr, kv_groups, n_q_groups, n_kv_groups, heads, batch=1):
    """sum over heads and listed (a, b) of n_q(a) * n_k(b), duplicates counted once."""
    nq = np.bincount(q_group[q_group >= 0], minlength=n_q_groups).astype(np.int64)
    nk = np.bincount(kv_group[kv_group >= 0], minlength=n_kv_groups).astype(np.int64)
    total = 0
    for h in range(heads):
        for a in range(n_q_groups):
            r = h * n_q_groups + a
            b = np.unique(kv_groups[row_ptr[r]:row_ptr[r + 1]])
            total += int(nq[a] * nk[b].sum())
    return total * batch


def bsa_physical_pairs(q_group, kv_group, A):
    """64 x 64 times the number of (Q block, K block) pairs with any allowed pair (one head)."""
    n_qb = -(-len(q_group) // 64)
    n_kb = -(-len(kv_group) // 64)
    count = 0
    for qb in range(n_qb):
        rows = np.arange(64 * qb, min(64 * qb + 64, len(q_group)))
        m = token_mask(q_group, kv_group, A, rows).any(axis=0)
        mp = np.zeros(n_kb * 64, dtype=bool)
        mp[:m.size] = m
        count += int(mp.reshape(n_kb, 64).any(axis=1).sum())
    return 64 * 64 * count
