"""Masked softmax attention and its gradients, float64, by definition.

Test infrastructure only (see the package docstring).  Source of the
definition: the KPage abstract ("KPage: block-sparse attention for partially
occupied 3D blocks", zhuanzhiai.com, abstract paragraph) — the scheme keeps
"exact masking" and preserves the original sparse graph in forward and
backward, so its output is ordinary softmax attention restricted to the
token pairs the graph allows.  The softmax-attention formulas are the
textbook ones that the FlashAttention teasers on the same pages refer to
("scifaro.com related/2411.10958", FlashAttention I/O-aware entry).

Notation: ``S = scale * Q K^T`` with disallowed entries at -inf,
``P = softmax_rows(S)``, ``O = P V``, ``LSE_i = log sum_j exp(S_ij)`` (natural
log).  Backward with upstream ``dO``: ``dV = P^T dO``, ``dP = dO V^T``,
``Delta_i = sum_j P_ij dP_ij``, ``dS = P * (dP - Delta)``,
``dQ = scale * dS K``, ``dK = scale * dS^T Q``.

Readings where the pages are silent: a valid query with no allowed key has
O = 0, LSE = -inf and dQ = 0 (the FlashAttention convention); padded slots are
never queries or keys.
"""

from __future__ import annotations

import numpy as np


def allowed_groups(row_ptr, kv_groups, n_q_groups, n_kv_groups, head):
    """Boolean [n_q_groups, n_kv_groups]: A_h[a, b] = key group b listed for query group a."""
    A = np.zeros((n_q_groups, n_kv_groups), dtype=bool)
    for a in range(n_q_groups):
        r = head * n_q_groups + a
        A[a, kv_groups[row_ptr[r]:row_ptr[r + 1]]] = True
    return A


def token_mask(q_group, kv_group, A, rows=None):
    """M[i, j] = q_group[i] >= 0 and kv_group[j] >= 0 and A[q_group[i], kv_group[j]].

    ``rows`` selects query slots (default: all).  Returns bool [len(rows), S_kv].
    """
    gq = np.asarray(q_group if rows is None else q_group[rows])
    gk = np.asarray(kv_group)
    qv = gq >= 0
    kv = gk >= 0
    M = A[np.where(qv, gq, 0)][:, np.where(kv, gk, 0)]
    return M & qv[:, None] & kv[None, :]


def _probs(q, k, mask, scale):
    """Row-normalised P (zeros on empty rows) and LSE (-inf on empty rows)."""
    s = scale * (q @ k.T)
    s = np.where(mask, s, -np.inf)
    nonempty = mask.any(axis=1)
    m = np.where(nonempty, np.max(np.where(mask, s, -np.inf), axis=1, initial=-np.inf), 0.0)
    e = np.where(mask, np.exp(s - m[:, None]), 0.0)
    l = e.sum(axis=1)
    p = np.where(nonempty[:, None], e / np.where(nonempty, l, 1.0)[:, None], 0.0)
    lse = np.where(nonempty, m + np.log(np.where(nonempty, l, 1.0)), -np.inf)
    return p, lse


def forward(q, k, v, mask, scale):
    """O [Sq, D] and LSE [Sq] for one (batch, head); inputs float64 [S, D]."""
    p, lse = _probs(q, k, mask, scale)
    return p @ v, lse


def backward(q, k, v, do, mask, scale):
    """dQ, dK, dV for one (batch, head) with loss gradient dO, all float64."""
    p, _ = _probs(q, k, mask, scale)
    dv = p.T @ do
    dp = do @ v.T
    delta = np.sum(p * dp, axis=1)
    ds = p * (dp - delta[:, None])
    dq = scale * (ds @ k)
    dk = scale * (ds.T @ q)
    return dq, dk, dv


def forward_rows(q, k, v, q_group, kv_group, A, rows, scale):
    """O and LSE for the query slots ``rows`` only (full rows, exact)."""
    rows = np.asarray(rows)
    mask = token_mask(q_group, kv_group, A, rows)
    cols = np.nonzero(mask.any(axis=0))[0]
    o = np.zeros((rows.size, q.shape[1]))
    lse = np.full(rows.size, -np.inf)
    if cols.size:
        o, lse = forward(q[rows], k[cols], v[cols], mask[:, cols], scale)
    return o, lse


def dq_rows(q, k, v, do, q_group, kv_group, A, rows, scale):
    """dQ for the query slots ``rows`` (each row's softmax over its full key set)."""
    rows = np.asarray(rows)
    mask = token_mask(q_group, kv_group, A, rows)
    cols = np.nonzero(mask.any(axis=0))[0]
    if cols.size == 0:
        return np.zeros((rows.size, q.shape[1]))
    p, _ = _probs(q[rows], k[cols], mask[:, cols], scale)
    dp = do[rows] @ v[cols].T
    delta = np.sum(p * dp, axis=1)
    ds = p * (dp - delta[:, None])
    return scale * (ds @ k[cols])


def dkdv_keys(q, k, v, do, q_group, kv_group, A, keys, scale, row_chunk=2048):
    """dK and dV for the key slots ``keys``.

    Every query that attends one of ``keys`` contributes; its probabilities
    and Delta are recomputed over that query's full key set.
    """
    keys = np.asarray(keys)
    D = q.shape[1]
    dk = np.zeros((keys.size, D))
    dv = np.zeros((keys.size, D))
    # queries attending any of the keys: those whose group lists a group of these keys
    kg = kv_group[keys]
    kg = np.unique(kg[kg >= 0])
    if kg.size == 0:
        return dk, dv
    qg_ok = A[:, kg].any(axis=1)
    qv = q_group >= 0
    rows = np.nonzero(qv & qg_ok[np.where(qv, q_group, 0)])[0]
    for r0 in range(0, rows.size, row_chunk):
        rr = rows[r0:r0 + row_chunk]
        mask = token_mask(q_group, kv_group, A, rr)
        cols = np.nonzero(mask.any(axis=0))[0]
        p, _ = _probs(q[rr], k[cols], mask[:, cols], scale)
        dp = do[rr] @ v[cols].T
        delta = np.sum(p * dp, axis=1)
        ds = p * (dp - delta[:, None])
        pos = np.searchsorted(cols, keys)
        hit = (pos < cols.size) & (cols[np.minimum(pos, cols.size - 1)] == keys)
        kp = pos[hit]
        dk[hit] += scale * (ds[:, kp].T @ q[rr])
        dv[hit] += p[:, kp].T @ do[rr]
    return dk, dv
