"""Device-side planner (spattn_plan_set_graph_device) on the GPU.

The re-planned work lists must equal, bit for bit, what the host planner
builds for the same graph with slot-order tiles (SPATTN_PLAN_PACK=slot), up to
the order of the work items; the pair counts must match; the forward and
backward passes on the re-planned lists must match the oracle; and a
malformed graph must be rejected without touching the plan.
"""

import dataclasses

import numpy as np
import pytest
import torch

import block_sparse_attention_bwd_b200 as sp
import oracle
from workloads import configs as W

pytestmark = pytest.mark.gpu


def _items(plan, which):
    """{(bh, owned refs, row codes): [(page ref, mask, head offset), ...]} of a work list."""
    work, pages, masks = plan.work(which)
    heads = plan.entry_heads(which)
    out = {}
    for w in work:
        n = int(w[1])
        key = (int(w[0]), tuple(int(x) for x in w[4:4 + n]), tuple(int(x) for x in w[12:28]))
        lst = list(zip(pages[w[2]:w[3]].tolist(), map(tuple, masks[w[2]:w[3]].tolist()), heads[w[2]:w[3]].tolist()))
        assert key not in out
        out[key] = lst
    return out


def _graph_variant(p, seed):
    """The same layout with another graph: each query group's list redrawn
    (same lengths), from a seeded generator."""
    rng = np.random.default_rng(seed)
    rows = []
    for r in range(p.graph_batches * p.heads * p.n_q_groups):
        n = int(p.row_ptr[r + 1] - p.row_ptr[r])
        rows.append(np.sort(rng.choice(p.n_kv_groups, size=min(n, p.n_kv_groups), replace=False)).tolist())
    row_ptr = np.zeros(len(rows) + 1, np.int64)
    row_ptr[1:] = np.cumsum([len(x) for x in rows])
    cols = np.concatenate([np.asarray(x, np.int32) for x in rows]) if rows else np.zeros(0, np.int32)
    return row_ptr, cols.astype(np.int32)


def _host_slot_plan(p, row_ptr, cols, monkeypatch, batch=None):
    monkeypatch.setenv("SPATTN_PLAN_PACK", "slot")
    pl = sp.Plan(p.q_group, p.kv_group, p.n_q_groups, p.n_kv_groups, row_ptr, cols,
                 batch=p.batch if batch is None else batch, heads=p.heads, head_dim=p.head_dim, scale=p.scale,
                 kv_heads=p.kv_heads, graph_batches=p.graph_batches)
    monkeypatch.delenv("SPATTN_PLAN_PACK")
    return pl


def _replan(pl, row_ptr, cols):
    pl.set_graph_device(torch.from_numpy(row_ptr).cuda(), torch.from_numpy(cols).cuda())


@pytest.mark.parametrize("name", ["tiny_vsa", "tiny_svg2", "tiny_hedge", "tiny_empty"])
def test_device_replan_bit_exact_tiny(name, monkeypatch):
    p = W.make_problem(name)
    pl = sp.Plan.from_problem(p)
    row_ptr, cols = _graph_variant(p, 91)
    _replan(pl, row_ptr, cols)
    ref = _host_slot_plan(p, row_ptr, cols, monkeypatch)
    for which in (0, 1):
        assert _items(pl, which) == _items(ref, which), which
    a, b = pl.stats(), ref.stats()
    for k in ("useful_pairs", "physical_pairs_fwd", "physical_pairs_dkdv", "n_work_fwd", "n_work_dkdv",
              "n_entries_fwd", "n_entries_dkdv", "bsa_pairs"):
        assert a[k] == b[k], k
    # the canonical lists follow the new graph too
    A = oracle.allowed_groups(row_ptr, cols, p.n_q_groups, p.n_kv_groups, 0)
    assert np.array_equal(pl.pages(0, 0), oracle.canonical_pages(p.q_group, p.kv_group, A, 0))


@pytest.mark.parametrize("name", ["tiny_vsa", "tiny_hedge"])
def test_device_replan_parity_tiny(name):
    from test_gpu_parity import check_tiny, run_gpu

    p = W.make_problem(name)
    pl = sp.Plan.from_problem(p)
    row_ptr, cols = _graph_variant(p, 7)
    _replan(pl, row_ptr, cols)
    q = W.Problem(p.name, p.batch, p.heads, p.head_dim, p.q_group, p.kv_group, p.n_q_groups, p.n_kv_groups, row_ptr,
                  cols, p.seed_base)
    t, out, _ = run_gpu(q, pl=pl)
    check_tiny(q, t, out, 1)


def test_device_replan_of_a_routed_plan(monkeypatch):
    """A host plan whose query-owned items take the 64-row route, re-planned
    on the device: the new items are 128-row (route word 0, the kernel form
    without the route), and the forward and backward match the oracle."""
    from test_gpu_parity import check_tiny, run_gpu

    p = W.make_problem("tiny_vsa")
    monkeypatch.setenv("SPATTN_PLAN_PACK", "route64")
    pl = sp.Plan.from_problem(p)
    monkeypatch.delenv("SPATTN_PLAN_PACK")
    assert (pl.work(0)[0][:, 28] == 1).all()
    row_ptr, cols = _graph_variant(p, 13)
    _replan(pl, row_ptr, cols)
    assert (pl.work(0)[0][:, 28] == 0).all()
    assert _items(pl, 0) == _items(_host_slot_plan(p, row_ptr, cols, monkeypatch), 0)
    q = W.Problem(p.name, p.batch, p.heads, p.head_dim, p.q_group, p.kv_group, p.n_q_groups, p.n_kv_groups, row_ptr,
                  cols, p.seed_base)
    t, out, _ = run_gpu(q, pl=pl)
    check_tiny(q, t, out, 1)


@pytest.mark.parametrize("name,batch", [("tiny_gqa", 2), ("tiny_mqa", 1), ("tiny_bgraph", 2)])
def test_device_replan_grouped_heads_and_batch_graphs(name, batch, monkeypatch):
    """Grouped-query attention (key-owned entries carry their query-head
    offset) and one graph per batch entry: the re-planned lists equal the
    host's slot-order plan of the same graph, entry heads included, and the
    passes on them match the oracle."""
    from test_gpu_parity import check_tiny, run_gpu

    p = W.make_problem(name)
    pl = sp.Plan.from_problem(p, batch=batch)
    row_ptr, cols = _graph_variant(p, 23)
    _replan(pl, row_ptr, cols)
    ref = _host_slot_plan(p, row_ptr, cols, monkeypatch, batch=batch)
    for which in (0, 1):
        assert _items(pl, which) == _items(ref, which), which
    a, b = pl.stats(), ref.stats()
    for k in ("useful_pairs", "physical_pairs_fwd", "physical_pairs_dkdv", "n_work_fwd", "n_work_dkdv",
              "n_entries_fwd", "n_entries_dkdv"):
        assert a[k] == b[k], k
    q = dataclasses.replace(p, row_ptr=row_ptr, kv_groups=cols)
    t, out, _ = run_gpu(q, batch, pl=pl)
    check_tiny(q, t, out, batch)


@pytest.mark.parametrize("name,batch", [("tiny_vsa", 1), ("tiny_gqa", 2)])
def test_device_replan_to_a_denser_graph(name, batch, monkeypatch):
    """A dense graph re-planned over a sparse plan: every list grows past
    the sizes the plan was built with (device buffers and per-entry arrays
    must follow), and the passes on the new lists match the oracle."""
    from test_gpu_parity import check_tiny, run_gpu

    p = W.make_problem(name)
    pl = sp.Plan.from_problem(p, batch=batch)
    before = pl.stats()
    rows = p.graph_batches * p.heads * p.n_q_groups
    row_ptr = np.arange(rows + 1, dtype=np.int64) * p.n_kv_groups
    cols = np.tile(np.arange(p.n_kv_groups, dtype=np.int32), rows)
    _replan(pl, row_ptr, cols)
    after = pl.stats()
    assert after["n_entries_fwd"] > before["n_entries_fwd"] and after["n_entries_dkdv"] > before["n_entries_dkdv"]
    ref = _host_slot_plan(p, row_ptr, cols, monkeypatch, batch=batch)
    for which in (0, 1):
        assert _items(pl, which) == _items(ref, which), which
    q = dataclasses.replace(p, row_ptr=row_ptr, kv_groups=cols)
    t, out, _ = run_gpu(q, batch, pl=pl)
    check_tiny(q, t, out, batch)


def test_device_replan_rejects_bad_graph():
    p = W.make_problem("tiny_vsa")
    t = {k: v.cuda() for k, v in W.make_tensors(p).items()}
    pl = sp.Plan.from_problem(p)
    o0, l0 = sp.spattn_fwd(t["q"], t["k"], t["v"], pl)
    o0, l0 = o0.clone(), l0.clone()
    row_ptr, cols = _graph_variant(p, 3)
    bad = cols.copy()
    bad[5] = p.n_kv_groups  # out of range
    with pytest.raises(sp.SpattnError) as e:
        _replan(pl, row_ptr, bad)
    assert e.value.status == sp.SPATTN_ERR_INVALID_ARG
    bad_ptr = row_ptr.copy()
    bad_ptr[3], bad_ptr[4] = bad_ptr[4], bad_ptr[3] + 100  # not monotone / beyond nnz
    with pytest.raises(sp.SpattnError):
        _replan(pl, bad_ptr, cols)
    o, l = sp.spattn_fwd(t["q"], t["k"], t["v"], pl)
    sp.spattn_check(pl)
    assert torch.equal(o, o0) and torch.equal(l, l0)


def test_device_replan_vsa_full_size(monkeypatch):
    """The VSA-style workload at full size: a new draw of every head's lists,
    re-planned on the device, equals the host's slot-order plan of that draw;
    sampled query blocks of the new graph match the oracle."""
    p = W.make_problem("vsa")
    pl = sp.Plan.from_problem(p)
    rng = np.random.default_rng(4242)
    row_ptr, cols = W.vsa_graph(-(-p.q_slots // 64), p.heads, 32, rng)
    d_rp, d_cols = torch.from_numpy(row_ptr).cuda(), torch.from_numpy(cols).cuda()
    pl.set_graph_device(d_rp, d_cols)
    torch.cuda.synchronize()
    ref = _host_slot_plan(p, row_ptr, cols, monkeypatch)
    for which in (0, 1):
        assert _items(pl, which) == _items(ref, which), which
    a, b = pl.stats(), ref.stats()
    assert a["useful_pairs"] == b["useful_pairs"]
    assert a["physical_pairs_fwd"] == b["physical_pairs_fwd"] and a["physical_pairs_dkdv"] == b["physical_pairs_dkdv"]
    # numerics on the re-planned lists, two query blocks
    t = W.make_tensors(p)
    dev = {k: v.cuda() for k, v in t.items()}
    o, lse = sp.spattn_fwd(dev["q"], dev["k"], dev["v"], pl)
    sp.spattn_check(pl)
    for h, qb in ((0, 0), (17, 1000)):
        A = oracle.allowed_groups(row_ptr, cols, p.n_q_groups, p.n_kv_groups, h)
        rows = np.arange(64 * qb, 64 * qb + 64)
        rows = rows[p.q_group[rows] >= 0]
        f = lambda x: x[0, h].to(torch.float64).numpy()  # noqa: E731
        o_ref, lse_ref = oracle.forward_rows(f(t["q"]), f(t["k"]), f(t["v"]), p.q_group, p.kv_group, A, rows, p.scale)
        og = o[0, h].cpu().double().numpy()[rows]
        assert np.linalg.norm(og - o_ref) / np.linalg.norm(o_ref) <= 5e-3
        assert np.abs(lse[0, h].cpu().double().numpy()[rows] - lse_ref).max() <= 1e-3
