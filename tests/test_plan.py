"""Planner (C-ABI, host side) against the oracle: canonical page lists and
their transposes bit for bit, useful-pair counts exactly, and the coverage
invariant of both work lists (every allowed pair computed by exactly one
owned row of exactly one work item, and nothing else)."""

import numpy as np
import pytest

import block_sparse_attention_bwd_b200 as sp
import oracle
from workloads import configs as W

TINY = ["tiny", "tiny_vsa", "tiny_svg2", "tiny_empty", "tiny_d128", "tiny_onekey", "tiny_hedge"]


def _allowed(p, h):
    return oracle.allowed_groups(p.row_ptr, p.kv_groups, p.n_q_groups, p.n_kv_groups, h)


@pytest.mark.parametrize("name", TINY)
def test_page_lists_bit_exact_tiny(name):
    p = W.make_problem(name)
    pl = sp.Plan.from_problem(p)
    for h in range(p.heads):
        A = _allowed(p, h)
        for qb in range(-(-p.q_slots // 64)):
            got = pl.pages(h, qb)
            exp = oracle.canonical_pages(p.q_group, p.kv_group, A, qb)
            assert got.dtype == np.int32 and np.array_equal(got, exp), (h, qb)
        for pg in range(-(-p.kv_slots // 16)):
            assert np.array_equal(pl.qblocks(h, pg), oracle.transposed_qblocks(p.q_group, p.kv_group, A, pg)), (h, pg)


@pytest.mark.parametrize("name", TINY)
def test_pair_counts_tiny(name):
    p = W.make_problem(name)
    for batch in (1, 2):
        pl = sp.Plan.from_problem(p, batch=batch)
        st = pl.stats()
        brute = sum(oracle.useful_pairs_bruteforce(p.q_group, p.kv_group, _allowed(p, h)) for h in range(p.heads))
        assert st["useful_pairs"] == brute * batch
        bsa = sum(oracle.bsa_physical_pairs(p.q_group, p.kv_group, _allowed(p, h)) for h in range(p.heads))
        assert st["bsa_pairs"] == bsa * batch
        assert st["physical_pairs_fwd"] >= st["useful_pairs"]
        assert st["physical_pairs_dkdv"] >= st["useful_pairs"]


def pref_slots(ref):
    """The 16 slots of a page reference: a page p >= 0 covers 16p .. 16p+15;
    a negative value is a strided page with base slot b = ~ref, rows
    b + 16j + r for j, r in 0..3."""
    ref = int(ref)
    if ref >= 0:
        return np.arange(16, dtype=np.int64) + 16 * ref
    b = ~ref
    return np.array([b + 16 * (r // 4) + r % 4 for r in range(16)], dtype=np.int64)


def _codes(w):
    words = w[12:28].astype(np.int64) & 0xFFFFFFFF
    return np.array([(words[r // 8] >> (4 * (r % 8))) & 0xF for r in range(128)])


def _covered(p, pl, which, head_filter=None, row_filter=None):
    """Pairs (own slot, column slot) per head produced by the work list, with multiplicity."""
    work, pages, masks = pl.work(which)
    own_group = p.q_group if which == 0 else p.kv_group
    col_slots = p.kv_slots if which == 0 else p.q_slots
    pairs = {}
    owned = {}
    bits16 = np.arange(16, dtype=np.uint64)
    for w in work:
        bh = int(w[0])
        if bh >= p.heads:
            continue  # batch copies repeat the same lists
        h = bh
        if head_filter is not None and h not in head_filter:
            continue
        n_own, e0, e1 = int(w[1]), int(w[2]), int(w[3])
        assert 1 <= n_own <= 8 and 0 <= e0 <= e1 <= pages.size and masks.shape == (pages.size, 2)
        assert np.all(w[29:32] == 0) and int(w[28]) in (0, 1)
        route = int(w[28]) == 1
        codes = _codes(w)
        pg = pages[e0:e1].astype(np.int64)
        mk = masks[e0:e1].astype(np.uint64)  # [entries, 2]
        first = np.array([pref_slots(x)[0] for x in pg], dtype=np.int64)
        # half of every entry: 0 for the 128-row route; entries 4i, 4i+1 of
        # the 64-row route serve rows 0..63, entries 4i+2, 4i+3 rows 64..127
        ehalf = (np.arange(e1 - e0) % 4) // 2 if route else np.zeros(e1 - e0, np.int64)
        if route:
            assert which == 0 and n_own == 8 and (e1 - e0) % 4 == 0
            for hf in (0, 1):
                live = (ehalf == hf) & ((mk[:, 0] | mk[:, 1]) != 0)
                assert np.all(np.diff(first[live]) > 0), "each half's entries in ascending slot order"
        else:
            assert np.all(np.diff(first) > 0), "column entries must be in ascending slot order"
        col_slot = np.stack([pref_slots(x) for x in pg]) if pg.size else np.zeros((0, 16), np.int64)
        for r in range(128):
            c = int(codes[r])
            if c == 15:
                continue
            assert r < 16 * n_own
            slot = int(pref_slots(w[4 + r // 16])[r % 16])
            assert slot < own_group.size
            if row_filter is not None and slot not in row_filter:
                continue
            owned[(h, slot)] = owned.get((h, slot), 0) + 1
            if c == 14:
                assert own_group[slot] == -1
                continue
            assert c < 8 and own_group[slot] >= 0
            bits = ((mk[:, c // 4, None] >> (np.uint64(16 * (c % 4)) + bits16)) & np.uint64(1)).astype(bool)
            if route:
                # a row of half r // 64 sees only its half's entries, and the
                # other half's entries carry no bit of its segment (so that a
                # kernel running every entry against all rows stays exact)
                assert not bits[ehalf != r // 64].any()
            cols = col_slot[bits]
            assert np.all(cols < col_slots)
            for col in cols.tolist():
                pairs[(h, slot, col)] = pairs.get((h, slot, col), 0) + 1
    return pairs, owned


def _split_pages(pl, which):
    """Work items that repeat a page another item also owns rows of."""
    work, _, _ = pl.work(which)
    seen, shared = {}, 0
    for w in work:
        for r in w[4:4 + int(w[1])].tolist():
            seen[(int(w[0]), r)] = seen.get((int(w[0]), r), 0) + 1
    return sum(1 for v in seen.values() if v > 1)


@pytest.mark.parametrize("name", TINY)
@pytest.mark.parametrize("which", [0, 1])
@pytest.mark.parametrize("pack", ["best", "split", "route64"])
def test_coverage_invariant_tiny(name, which, pack, monkeypatch):
    """Every allowed pair exactly once, on exactly one owned row; with the
    group-split packing forced, pages shared by several work items (each
    owning the rows of its group) are covered exactly once as well; with the
    64-row route forced, each half of a tile over its own list."""
    p = W.make_problem(name)
    if pack != "best":
        monkeypatch.setenv("SPATTN_PLAN_PACK", pack)
    pl = sp.Plan.from_problem(p)
    monkeypatch.delenv("SPATTN_PLAN_PACK", raising=False)
    if pack == "split" and name == "tiny_svg2":
        assert _split_pages(pl, which) > 0  # the clustered layout does split pages
    if pack == "route64":
        routed = pl.work(which)[0][:, 28]
        assert np.all(routed == 1) if which == 0 else np.all(routed == 0)
    pairs, owned = _covered(p, pl, which)
    assert all(v == 1 for v in pairs.values()), "a pair is computed by two owned rows"
    own_group = p.q_group if which == 0 else p.kv_group
    valid_pages = oracle.page_valid_masks(own_group) != 0
    for h in range(p.heads):
        M = oracle.token_mask(p.q_group, p.kv_group, _allowed(p, h))
        if which == 1:
            M = M.T
        got = np.zeros_like(M)
        for (hh, i, j) in pairs:
            if hh == h:
                got[i, j] = True
        assert np.array_equal(got, M)
        for slot in range(own_group.size):
            # every valid slot is owned exactly once; a padded slot at most once
            # (the padded rows a strided owned page leaves out are filled instead)
            n = owned.get((h, slot), 0)
            if own_group[slot] >= 0:
                assert n == 1, (h, slot)
            else:
                assert n <= (1 if valid_pages[slot // 16] else 0), (h, slot)


@pytest.mark.parametrize("name", ["full", "partial", "vsa", "svg2"])
def test_page_lists_and_counts_large_sampled(name):
    p = W.make_problem(name)
    pl = sp.Plan.from_problem(p)
    st = pl.stats()
    assert st["useful_pairs"] == oracle.useful_pairs_closed_form(
        p.q_group, p.kv_group, p.row_ptr, p.kv_groups, p.n_q_groups, p.n_kv_groups, p.heads)
    rng = np.random.default_rng(17)
    n_qb = -(-p.q_slots // 64)
    for _ in range(12):
        h = int(rng.integers(p.heads))
        qb = int(rng.integers(n_qb))
        A = _allowed(p, h)
        assert np.array_equal(pl.pages(h, qb), oracle.canonical_pages(p.q_group, p.kv_group, A, qb)), (h, qb)
    # coverage restricted to a few query rows / key rows of one head
    h = int(rng.integers(p.heads))
    A = _allowed(p, h)
    rows = set(rng.integers(0, p.q_slots, size=6).tolist())
    pairs, owned = _covered(p, pl, 0, head_filter={h}, row_filter=rows)
    M = oracle.token_mask(p.q_group, p.kv_group, A, np.array(sorted(rows)))
    for k, i in enumerate(sorted(rows)):
        got = sorted(j for (hh, ii, j) in pairs if ii == i)
        assert got == np.nonzero(M[k])[0].tolist()
    keys = set(rng.integers(0, p.kv_slots, size=4).tolist())
    pairs, owned = _covered(p, pl, 1, head_filter={h}, row_filter=keys)
    Mt = oracle.token_mask(p.q_group, p.kv_group, A)[:, sorted(keys)].T if p.q_slots <= 20000 else None
    for k, j in enumerate(sorted(keys)):
        got = sorted(i for (hh, jj, i) in pairs if jj == j)
        if Mt is not None:
            exp = np.nonzero(Mt[k])[0].tolist()
        else:
            g = p.kv_group[j]
            exp = [] if g < 0 else np.nonzero((p.q_group >= 0) & A[np.where(p.q_group >= 0, p.q_group, 0), g])[0].tolist()
        assert got == exp


@pytest.mark.parametrize("name", ["vsa", "partial"])
def test_route64_large_sampled(name, monkeypatch):
    """The 64-row route forced on a full-size layout: every query-owned item
    is routed with whole 4-entry steps, the physical-pair count is 64 rows x
    16 columns per entry, and sampled query rows of one head see exactly
    their allowed keys (through their own half's entries only)."""
    p = W.make_problem(name)
    monkeypatch.setenv("SPATTN_PLAN_PACK", "route64")
    pl = sp.Plan.from_problem(p)
    monkeypatch.delenv("SPATTN_PLAN_PACK")
    work, pages, _ = pl.work(0)
    assert (work[:, 28] == 1).all() and ((work[:, 3] - work[:, 2]) % 4 == 0).all()
    st = pl.stats()
    assert st["physical_pairs_fwd"] == 64 * 16 * int((work[:, 3] - work[:, 2]).sum())
    assert st["physical_pairs_fwd"] >= st["useful_pairs"]
    rng = np.random.default_rng(23)
    h = int(rng.integers(p.heads))
    A = _allowed(p, h)
    rows = set(rng.integers(0, p.q_slots, size=6).tolist())
    pairs, _ = _covered(p, pl, 0, head_filter={h}, row_filter=rows)
    assert all(v == 1 for v in pairs.values())
    M = oracle.token_mask(p.q_group, p.kv_group, A, np.array(sorted(rows)))
    for k, i in enumerate(sorted(rows)):
        assert sorted(j for (hh, ii, j) in pairs if ii == i) == np.nonzero(M[k])[0].tolist()


@pytest.mark.parametrize("name,batch", [("partial", 1), ("tiny_gqa", 2), ("tiny_bgraph", 2), ("tiny_vsa", 1)])
def test_plan_dedup_of_identical_heads(name, batch, monkeypatch):
    """Heads with the same graph rows are planned once and copied: the
    plan equals, word for word, the plan that builds every head."""
    p = W.make_problem(name)
    plans = []
    for dedup in ("1", "0"):
        monkeypatch.setenv("SPATTN_PLAN_DEDUP", dedup)
        pl = sp.Plan.from_problem(p, batch=batch)
        plans.append(([np.array(x, copy=True) for w in (0, 1) for x in pl.work(w)]
                      + [np.array(pl.entry_heads(w), copy=True) for w in (0, 1)], pl.stats()))
    monkeypatch.delenv("SPATTN_PLAN_DEDUP")
    (a, sa), (b, sb) = plans
    assert all(np.array_equal(x, y) for x, y in zip(a, b))
    for k in ("useful_pairs", "physical_pairs_fwd", "physical_pairs_dkdv", "n_work_fwd", "n_work_dkdv"):
        assert sa[k] == sb[k], k


@pytest.mark.parametrize("name", ["partial", "svg2"])
def test_plan_independent_of_thread_count(name, monkeypatch):
    p = W.with_heads(W.make_problem(name), 5)
    plans = []
    for threads in ("1", "7"):
        monkeypatch.setenv("SPATTN_PLAN_THREADS", threads)
        plans.append(sp.Plan.from_problem(p))
    for which in (0, 1):
        a, b = plans[0].work(which), plans[1].work(which)
        for x, y in zip(a, b):
            assert np.array_equal(x, y)
    sa, sb = plans[0].stats(), plans[1].stats()
    for k in ("useful_pairs", "physical_pairs_fwd", "physical_pairs_dkdv", "n_work_fwd", "n_entries_dkdv"):
        assert sa[k] == sb[k], k


def test_strided_pages_are_formed_where_rows_share_a_group():
    """tiny_hedge's H-edge tiles: four pages with valid rows 0..3 each become
    one strided owned page, and their key pages one strided column entry."""
    p = W.make_problem("tiny_hedge")
    pl = sp.Plan.from_problem(p)
    for which in (0, 1):
        work, pages, _ = pl.work(which)
        assert (pages < 0).any(), which
        owned = work[:, 4:12][np.arange(8)[None, :] < work[:, 1:2]]
        assert (owned < 0).any(), which
        for ref in np.concatenate([pages[pages < 0], owned[owned < 0]]):
            slots = pref_slots(ref)
            assert (p.kv_group[slots] >= 0).all() if which == 0 and ref in pages else True
            assert slots.max() < p.q_slots


def test_strided_pages_stay_inside_the_tensor():
    """Key rows 12..15 of every page valid, 62 slots: a strided page over the
    4-row group 12..15 of pages 0..3 would reach slots 60..63, past the end of
    the tensor, so none may cover a slot >= 62."""
    kg = np.full(62, -1, np.int32)
    for j in range(4):
        kg[16 * j + 12:16 * j + 16] = 0
    kg = kg[:62]
    qg = np.zeros(16, np.int32)
    pl = sp.Plan(qg, kg, 1, 1, np.array([0, 1], np.int64), np.array([0], np.int32), batch=1, heads=1, head_dim=64)
    for which in (0, 1):
        work, pages, _ = pl.work(which)
        refs = list(pages) + list(work[:, 4:12][np.arange(8)[None, :] < work[:, 1:2]])
        for ref in refs:
            assert pref_slots(ref).max() < 62 or int(ref) >= 0, ref
    # the allowed pairs are still covered exactly once
    pairs, _ = _covered(W.Problem("ragged", 1, 1, 64, qg, kg, 1, 1, np.array([0, 1], np.int64),
                                  np.array([0], np.int32), 0), pl, 0)
    assert sorted(j for (_, _, j) in pairs) == sorted(np.nonzero(kg >= 0)[0].tolist() * 16)


def _covered_heads(p, pl, which, batch):
    """{(owned bh, owned slot, column bh, column slot): count} over all work
    items, with the column head of key-owned entries resolved through the
    entry head offsets (grouped-query attention)."""
    work, pages, masks = pl.work(which)
    eh = pl.entry_heads(which)
    H, Hkv = p.heads, p.n_kv_heads
    g = H // Hkv
    out = {}
    bits16 = np.arange(16, dtype=np.uint64)
    for w in work:
        bh = int(w[0])
        codes = _codes(w)
        e0, e1 = int(w[2]), int(w[3])
        col_slot = [pref_slots(x) for x in pages[e0:e1]]
        for r in range(128):
            c = int(codes[r])
            if c >= 14:
                continue
            slot = int(pref_slots(w[4 + r // 16])[r % 16])
            for e in range(e0, e1):
                m = (int(masks[e, c // 4]) >> (16 * (c % 4))) & 0xFFFF
                if not m:
                    continue
                cbh = bh if which == 0 else (bh // Hkv) * H + (bh % Hkv) * g + int(eh[e])
                if which == 0:
                    cbh = (bh // H) * Hkv + (bh % H) // g
                for bit in range(16):
                    if (m >> bit) & 1:
                        key = (bh, slot, cbh, int(col_slot[e - e0][bit]))
                        out[key] = out.get(key, 0) + 1
    return out


@pytest.mark.parametrize("name", ["tiny_gqa", "tiny_mqa", "tiny_bgraph"])
def test_coverage_grouped_heads_and_batch_graphs(name):
    """Grouped-query attention and per-batch graphs: the query-owned list
    computes, for every (batch, query head), exactly the pairs of that head's
    graph against its K/V head; the key-owned list computes, for every
    (batch, K/V head), the pairs of all query heads of its group, each once."""
    p = W.make_problem(name)
    pl = sp.Plan.from_problem(p)
    B, H, Hkv = p.batch, p.heads, p.n_kv_heads
    g = H // Hkv
    expect_q, expect_k = set(), set()
    for b in range(B):
        for h in range(H):
            A = _allowed(p, p.graph_head(b, h))
            M = oracle.token_mask(p.q_group, p.kv_group, A)
            hk = h // g
            for i, j in zip(*np.nonzero(M)):
                expect_q.add((b * H + h, int(i), b * Hkv + hk, int(j)))
                expect_k.add((b * Hkv + hk, int(j), b * H + h, int(i)))
    got_q = _covered_heads(p, pl, 0, B)
    got_k = _covered_heads(p, pl, 1, B)
    assert all(v == 1 for v in got_q.values()) and all(v == 1 for v in got_k.values())
    assert set(got_q) == expect_q
    assert set(got_k) == expect_k
    st = pl.stats()
    assert st["useful_pairs"] == len(expect_q)
