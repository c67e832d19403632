"""Pins of the CPU fp64 oracle against things other than itself.

Each test fixes the oracle with an independent fact: a hand-derived closed
form (``tests/golden``), dense attention from ``torch`` when the graph is
full, single-key and zero-query closed forms, central finite differences, and
brute-force counts.  A plausible slip in the oracle (a dropped scale, a
transposed mask, the wrong log base, a padded row leaking) fails one of them.
"""

import math
import os

import numpy as np
import pytest
import torch

import oracle
from workloads import configs as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f64(t):
    return t.to(torch.float64).numpy()


def _load_golden(name):
    env = {"e": math.e, "log": math.log, "inf": math.inf}
    spec = {}
    graph = {}
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, rest = line.split(None, 1)
            if key == "graph":
                a, b = rest.split(":")
                graph[int(a)] = [int(x) for x in b.split()]
            elif key in ("scale",):
                spec[key] = float(rest)
            elif key in ("q_group", "kv_group"):
                spec[key] = np.array([int(x) for x in rest.split()], dtype=np.int32)
            else:
                spec[key] = np.array([[float(eval(x, {"__builtins__": {}}, env)) for x in row.split()]
                                      for row in rest.split(";")])
    spec["graph"] = graph
    return spec


def test_golden_closed_form():
    g = _load_golden("closed_form_masked.txt")
    nq, nk = 2, 2
    A = np.zeros((nq, nk), bool)
    for a, bs in g["graph"].items():
        A[a, bs] = True
    mask = oracle.token_mask(g["q_group"], g["kv_group"], A)
    o, lse = oracle.forward(g["q"], g["k"], g["v"], mask, g["scale"])
    np.testing.assert_allclose(o, g["O"], rtol=0, atol=1e-14)
    np.testing.assert_array_equal(np.isinf(lse), np.isinf(g["LSE"].ravel()))
    fin = np.isfinite(lse)
    np.testing.assert_allclose(lse[fin], g["LSE"].ravel()[fin], rtol=0, atol=1e-14)
    dq, dk, dv = oracle.backward(g["q"], g["k"], g["v"], g["do"], mask, g["scale"])
    np.testing.assert_allclose(dq, g["dQ"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dk, g["dK"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dv, g["dV"], rtol=0, atol=1e-14)


def _head_inputs(p, t, h):
    return (_f64(t["q"][0, h]), _f64(t["k"][0, h]), _f64(t["v"][0, h]), _f64(t["do"][0, h]))


def test_full_graph_is_dense_attention():
    """tiny's clamped 3x3x3 window covers all 2x2x3 tiles: the graph is full."""
    p = W.make_problem("tiny")
    t = W.make_tensors(p)
    for h in range(p.heads):
        A = oracle.allowed_groups(p.row_ptr, p.kv_groups, p.n_q_groups, p.n_kv_groups, h)
        assert A.all()
        q, k, v, do = _head_inputs(p, t, h)
        mask = oracle.token_mask(p.q_group, p.kv_group, A)
        o, lse = oracle.forward(q, k, v, mask, p.scale)
        dq, dk, dv = oracle.backward(q, k, v, do, mask, p.scale)

        vq = np.nonzero(p.q_group >= 0)[0]
        vk = np.nonzero(p.kv_group >= 0)[0]
        tq = torch.tensor(q[vq], requires_grad=True)
        tk = torch.tensor(k[vk], requires_grad=True)
        tv = torch.tensor(v[vk], requires_grad=True)
        ref = torch.nn.functional.scaled_dot_product_attention(tq[None], tk[None], tv[None], scale=p.scale)[0]
        ref.backward(torch.tensor(do[vq]))
        ref_lse = torch.logsumexp(p.scale * (tq @ tk.T), dim=1)
        np.testing.assert_allclose(o[vq], ref.detach().numpy(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[vq], ref_lse.detach().numpy(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(dq[vq], tq.grad.numpy(), rtol=0, atol=1e-11)
        np.testing.assert_allclose(dk[vk], tk.grad.numpy(), rtol=0, atol=1e-11)
        np.testing.assert_allclose(dv[vk], tv.grad.numpy(), rtol=0, atol=1e-11)
        # padded slots: no output, no gradient
        pq = p.q_group < 0
        pk = p.kv_group < 0
        assert np.all(o[pq] == 0) and np.all(np.isneginf(lse[pq])) and np.all(dq[pq] == 0)
        assert np.all(dk[pk] == 0) and np.all(dv[pk] == 0)


def test_single_allowed_key():
    """A query group that may attend exactly one key: O = v_j, LSE = s_ij, dQ = 0, dK_j = 0."""
    rng = np.random.default_rng(7)
    qg = np.array([0, 0, 1, 1, 1, -1, 0], np.int32)
    kg = np.array([1, 1, -1, 0, 1, 1], np.int32)  # key 3 is the only member of group 0
    A = np.array([[True, False], [False, True]])
    D = 8
    q, k, v, do = (rng.standard_normal((n, D)) for n in (7, 6, 6, 7))
    scale = 0.37
    mask = oracle.token_mask(qg, kg, A)
    o, lse = oracle.forward(q, k, v, mask, scale)
    dq, dk, dv = oracle.backward(q, k, v, do, mask, scale)
    rows = np.nonzero(qg == 0)[0]
    np.testing.assert_allclose(o[rows], np.repeat(v[3][None], rows.size, 0), rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse[rows], scale * (q[rows] @ k[3]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(dq[rows], 0.0, atol=1e-15)
    np.testing.assert_allclose(dk[3], 0.0, atol=1e-15)
    np.testing.assert_allclose(dv[3], do[rows].sum(axis=0), rtol=0, atol=1e-14)


def test_zero_query_is_mean_of_allowed_values():
    p = W.make_problem("tiny_svg2")
    t = W.make_tensors(p)
    for h in range(p.heads):
        A = oracle.allowed_groups(p.row_ptr, p.kv_groups, p.n_q_groups, p.n_kv_groups, h)
        _, k, v, _ = _head_inputs(p, t, h)
        q = np.zeros((p.q_slots, p.head_dim))
        mask = oracle.token_mask(p.q_group, p.kv_group, A)
        o, lse = oracle.forward(q, k, v, mask, p.scale)
        for i in range(p.q_slots):
            cols = np.nonzero(mask[i])[0]
            if cols.size == 0:
                assert np.all(o[i] == 0) and np.isneginf(lse[i])
                continue
            np.testing.assert_allclose(o[i], v[cols].mean(axis=0), rtol=0, atol=1e-13)
            assert abs(lse[i] - math.log(cols.size)) < 1e-13


def test_rows_sum_to_one_and_empty_rows():
    p = W.make_problem("tiny_empty")
    t = W.make_tensors(p)
    for h in range(p.heads):
        A = oracle.allowed_groups(p.row_ptr, p.kv_groups, p.n_q_groups, p.n_kv_groups, h)
        q, k, _, _ = _head_inputs(p, t, h)
        v = np.ones((p.kv_slots, 3))
        mask = oracle.token_mask(p.q_group, p.kv_group, A)
        o, lse = oracle.forward(q, k, v, mask, p.scale)
        nonempty = mask.any(axis=1)
        np.testing.assert_allclose(o[nonempty], 1.0, rtol=0, atol=1e-13)
        assert np.all(o[~nonempty] == 0) and np.all(np.isneginf(lse[~nonempty]))
        # query tile 0 attends nothing in this workload
        assert not nonempty[p.q_group == 0].any()


def _loss(q, k, v, do, mask, scale, rows):
    o, _ = oracle.forward(q, k, v, mask, scale)
    return float(np.sum(do[rows] * o[rows]))


@pytest.mark.parametrize("name", ["tiny", "tiny_vsa", "tiny_svg2", "tiny_empty", "tiny_onekey"])
def test_gradients_match_central_differences(name):
    """L = sum over valid rows of dO * O; analytic grads vs central differences (h = 1e-5)."""
    p = W.make_problem(name)
    t = W.make_tensors(p)
    h = p.heads - 1
    A = oracle.allowed_groups(p.row_ptr, p.kv_groups, p.n_q_groups, p.n_kv_groups, h)
    q, k, v, do = _head_inputs(p, t, h)
    # keep magnitudes O(1) on padded rows too so the step size is meaningful everywhere
    q = np.where(p.q_group[:, None] >= 0, q, 0.5)
    k = np.where(p.kv_group[:, None] >= 0, k, 0.5)
    v = np.where(p.kv_group[:, None] >= 0, v, 0.5)
    mask = oracle.token_mask(p.q_group, p.kv_group, A)
    rows = np.nonzero(p.q_group >= 0)[0]
    dq, dk, dv = oracle.backward(q, k, v, do, mask, p.scale)
    grads = {"q": dq, "k": dk, "v": dv}
    base = {"q": q, "k": k, "v": v}
    rng = np.random.default_rng(99)
    eps = 1e-5
    gscale = max(np.abs(dq).max(), np.abs(dk).max(), np.abs(dv).max())

    def L(**kw):
        args = dict(base)
        args.update(kw)
        return _loss(args["q"], args["k"], args["v"], do, mask, p.scale, rows)

    for nm in ("q", "k", "v"):
        x = base[nm]
        idx = [tuple(rng.integers(0, s) for s in x.shape) for _ in range(40)]
        # always include entries on padded slots: their gradient must be exactly 0
        grp = p.q_group if nm == "q" else p.kv_group
        pads = np.nonzero(grp < 0)[0]
        if pads.size:
            idx += [(int(pads[0]), 0), (int(pads[-1]), x.shape[1] - 1)]
        for ix in idx:
            xp = x.copy()
            xm = x.copy()
            xp[ix] += eps
            xm[ix] -= eps
            fd = (L(**{nm: xp}) - L(**{nm: xm})) / (2 * eps)
            assert abs(fd - grads[nm][ix]) <= 1e-6 * max(abs(grads[nm][ix]), gscale), (nm, ix, fd, grads[nm][ix])
        for _ in range(8):
            d = rng.standard_normal(x.shape)
            fd = (L(**{nm: x + eps * d}) - L(**{nm: x - eps * d})) / (2 * eps)
            an = float(np.sum(grads[nm] * d))
            assert abs(fd - an) <= 1e-6 * max(abs(an), gscale), (nm, fd, an)


@pytest.mark.parametrize("name", ["tiny_vsa", "tiny_svg2", "tiny_empty", "tiny_onekey"])
def test_sampled_forms_equal_full_forms(name):
    p = W.make_problem(name)
    t = W.make_tensors(p)
    for h in range(p.heads):
        A = oracle.allowed_groups(p.row_ptr, p.kv_groups, p.n_q_groups, p.n_kv_groups, h)
        q, k, v, do = _head_inputs(p, t, h)
        mask = oracle.token_mask(p.q_group, p.kv_group, A)
        o, lse = oracle.forward(q, k, v, mask, p.scale)
        dq, dk, dv = oracle.backward(q, k, v, do, mask, p.scale)
        rows = np.arange(0, p.q_slots, 3)
        o2, lse2 = oracle.forward_rows(q, k, v, p.q_group, p.kv_group, A, rows, p.scale)
        np.testing.assert_allclose(o2, o[rows], rtol=0, atol=1e-13)
        np.testing.assert_array_equal(np.isinf(lse2), np.isinf(lse[rows]))
        fin = np.isfinite(lse2)
        np.testing.assert_allclose(lse2[fin], lse[rows][fin], rtol=0, atol=1e-13)
        np.testing.assert_allclose(oracle.dq_rows(q, k, v, do, p.q_group, p.kv_group, A, rows, p.scale),
                                   dq[rows], rtol=0, atol=1e-12)
        keys = np.arange(1, p.kv_slots, 2)
        dk2, dv2 = oracle.dkdv_keys(q, k, v, do, p.q_group, p.kv_group, A, keys, p.scale, row_chunk=37)
        np.testing.assert_allclose(dk2, dk[keys], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dv2, dv[keys], rtol=0, atol=1e-12)


def test_page_valid_masks_by_hand():
    g = np.full(37, -1, np.int32)
    g[[0, 3, 15, 16, 31, 32, 36]] = 5
    m = oracle.page_valid_masks(g)
    assert m.tolist() == [(1 << 0) | (1 << 3) | (1 << 15), (1 << 0) | (1 << 15), (1 << 0) | (1 << 4)]


@pytest.mark.parametrize("name", ["tiny", "tiny_vsa", "tiny_svg2", "tiny_empty", "tiny_onekey"])
def test_pair_counts_and_pages(name):
    p = W.make_problem(name)
    total_brute = 0
    for h in range(p.heads):
        A = oracle.allowed_groups(p.row_ptr, p.kv_groups, p.n_q_groups, p.n_kv_groups, h)
        mask = oracle.token_mask(p.q_group, p.kv_group, A)
        total_brute += oracle.useful_pairs_bruteforce(p.q_group, p.kv_group, A)
        # canonical page lists vs a group-based derivation written here
        kv_pages_of_group = {}
        for j, g in enumerate(p.kv_group):
            if g >= 0:
                kv_pages_of_group.setdefault(int(g), set()).add(j // 16)
        n_qb = -(-p.q_slots // 64)
        for qb in range(n_qb):
            groups = {int(g) for g in p.q_group[64 * qb:64 * qb + 64] if g >= 0}
            expect = set()
            for a in groups:
                for b in np.nonzero(A[a])[0]:
                    expect |= kv_pages_of_group.get(int(b), set())
            got = oracle.canonical_pages(p.q_group, p.kv_group, A, qb)
            assert got.tolist() == sorted(expect)
            # and from the explicit mask, page by page
            blk = mask[64 * qb:64 * qb + 64]
            by_mask = [pg for pg in range(-(-p.kv_slots // 16)) if blk[:, 16 * pg:16 * pg + 16].any()]
            assert got.tolist() == by_mask
        for pg in range(-(-p.kv_slots // 16)):
            tq = oracle.transposed_qblocks(p.q_group, p.kv_group, A, pg)
            exp = [qb for qb in range(n_qb) if pg in oracle.canonical_pages(p.q_group, p.kv_group, A, qb)]
            assert tq.tolist() == exp
    closed = oracle.useful_pairs_closed_form(p.q_group, p.kv_group, p.row_ptr, p.kv_groups,
                                             p.n_q_groups, p.n_kv_groups, p.heads)
    assert closed == total_brute


def test_tiny_counts_by_hand():
    """tiny: full graph over 300 valid tokens and 12 occupied 64-slot blocks, 2 heads."""
    p = W.make_problem("tiny")
    A = oracle.allowed_groups(p.row_ptr, p.kv_groups, p.n_q_groups, p.n_kv_groups, 0)
    assert oracle.useful_pairs_bruteforce(p.q_group, p.kv_group, A) == 300 * 300
    assert oracle.bsa_physical_pairs(p.q_group, p.kv_group, A) == 64 * 64 * 12 * 12
    valid_pages = np.nonzero(oracle.page_valid_masks(p.kv_group))[0]
    for qb in range(12):
        assert oracle.canonical_pages(p.q_group, p.kv_group, A, qb).tolist() == valid_pages.tolist()


def _axis_sum(n_valid, window):
    """sum over query tiles a of v(a) * sum over window(a) of v(b), one axis."""
    n = len(n_valid)
    total = 0
    for a in range(n):
        if n <= window:
            win = range(n)
        else:
            s = min(max(a - window // 2, 0), n - window)
            win = range(s, s + window)
        total += n_valid[a] * sum(n_valid[b] for b in win)
    return total


@pytest.mark.parametrize("name,grid,window,heads", [
    ("full", (16, 32, 32), (3, 3, 3), 16),
    ("partial", (21, 45, 80), (3, 5, 5), 40),
])
def test_sta_useful_pairs_separable_closed_form(name, grid, window, heads):
    """For an STA window the count factorises over the three axes."""
    p = W.make_problem(name)
    per_axis = []
    for extent, w in zip(grid, window):
        n = -(-extent // 4)
        nv = [min(4, extent - 4 * i) for i in range(n)]
        per_axis.append(_axis_sum(nv, w))
    expect = heads * per_axis[0] * per_axis[1] * per_axis[2]
    got = oracle.useful_pairs_closed_form(p.q_group, p.kv_group, p.row_ptr, p.kv_groups,
                                          p.n_q_groups, p.n_kv_groups, p.heads)
    assert got == expect
    if name == "full":
        assert got == 16 * 256 * 64 * 27 * 64


def test_sparse_counts_by_hand():
    """A sparse three-block case counted by hand (BSA block pairs, useful pairs, page lists).

    Query slots (3 blocks of 64): block 0 = group 0 except slot 60 = group 2;
    block 1 = group 1; block 2 padded except slot 130 = group 2.
    Key slots (3 blocks of 64): block 0 = group 0; block 1 padded except
    slot 100 = group 1; block 2 = group 2.
    Graph: q0 -> {k1}, q1 -> {} (attends nothing), q2 -> {k0, k2}.

    Block pairs with an allowed pair: Q block 0 reaches K blocks 1 (via q0 ->
    slot 100) and 0, 2 (via slot 60 -> k0, k2); Q block 1 none; Q block 2
    reaches K blocks 0 and 2: five pairs.  Counting every pair of blocks that
    merely hold valid slots would give 9, counting allowed group pairs 3.
    Useful pairs: 63 * 1 (q0 -> k1) + 2 * (64 + 64) (q2 -> k0, k2) = 319.
    """
    qg = np.zeros(192, np.int32)
    qg[60] = 2
    qg[64:128] = 1
    qg[128:] = -1
    qg[130] = 2
    kg = np.zeros(192, np.int32)
    kg[64:128] = -1
    kg[100] = 1
    kg[128:] = 2
    row_ptr = np.array([0, 1, 1, 3], np.int64)
    cols = np.array([1, 0, 2], np.int32)
    A = oracle.allowed_groups(row_ptr, cols, 3, 3, 0)
    assert oracle.bsa_physical_pairs(qg, kg, A) == 5 * 64 * 64
    assert oracle.useful_pairs_bruteforce(qg, kg, A) == 319
    assert oracle.useful_pairs_closed_form(qg, kg, row_ptr, cols, 3, 3, 1) == 319
    assert oracle.canonical_pages(qg, kg, A, 0).tolist() == [0, 1, 2, 3, 6, 8, 9, 10, 11]
    assert oracle.canonical_pages(qg, kg, A, 1).tolist() == []
    assert oracle.canonical_pages(qg, kg, A, 2).tolist() == [0, 1, 2, 3, 8, 9, 10, 11]
    assert oracle.transposed_qblocks(qg, kg, A, 6).tolist() == [0]
    assert oracle.transposed_qblocks(qg, kg, A, 4).tolist() == []
    assert oracle.transposed_qblocks(qg, kg, A, 9).tolist() == [0, 2]
