"""CUDA path (through the C ABI) against the fp64 oracle, element by element.

Tolerances (over valid rows, the bf16 outputs against fp64 on the same bf16
inputs): O max-abs <= 1e-2 and relative L2 <= 5e-3; LSE abs <= 1e-3;
dQ, dK, dV relative L2 <= 1e-2.  Padded and attention-free rows must be
exact: O = 0, LSE = -inf, dQ = 0, dK = dV = 0.  The backward consumes the
GPU's own O and LSE.

Every tolerance is applied per (batch, head) for the tiny workloads and per
sampled unit (one head and one 64-slot block) for the large ones, so that an
error confined to one head or one block is not diluted by the others; the
pooled figures are checked as well.

Tiny workloads are compared in full; the large ones are run at full size in
the launch configuration the benchmark uses and compared on sampled units
(whole Q blocks for O / LSE / dQ, whole 64-slot key blocks for dK / dV),
stratified over interior, T-edge, H-edge and corner blocks.
"""

import numpy as np
import pytest
import torch

import block_sparse_attention_bwd_b200 as sp
import oracle
from workloads import configs as W

pytestmark = pytest.mark.gpu

TOL = dict(o_abs=1e-2, o_rel=5e-3, lse_abs=1e-3, grad_rel=1e-2)


def rel_l2(a, b):
    den = float(np.linalg.norm(b))
    num = float(np.linalg.norm(a - b))
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return num / den


def _allowed(p, h):
    return oracle.allowed_groups(p.row_ptr, p.kv_groups, p.n_q_groups, p.n_kv_groups, h)


def run_gpu(p, batch=None, t=None, pl=None):
    t = W.make_tensors(p, batch=batch) if t is None else t
    dev = {k: v.cuda() for k, v in t.items()}
    pl = sp.Plan.from_problem(p, batch=batch) if pl is None else pl
    o, lse = sp.spattn_fwd(dev["q"], dev["k"], dev["v"], pl)
    dq, dk, dv = sp.spattn_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], pl)
    sp.spattn_check(pl)
    out = {"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv}
    return t, {k: v.cpu() for k, v in out.items()}, pl


def _f64(x):
    return x.to(torch.float64).numpy()


def check_padded(p, out):
    pq = torch.from_numpy(p.q_group < 0)
    pk = torch.from_numpy(p.kv_group < 0)
    if bool(pq.any()):
        assert torch.all(out["o"][:, :, pq] == 0)
        assert torch.all(torch.isneginf(out["lse"][:, :, pq]))
        assert torch.all(out["dq"][:, :, pq] == 0)
    if bool(pk.any()):
        assert torch.all(out["dk"][:, :, pk] == 0)
        assert torch.all(out["dv"][:, :, pk] == 0)
    for k, v in out.items():
        if k != "lse":
            assert torch.isfinite(v.float()).all(), k


def check_tiny(p, t, out, batch):
    """Full comparison of every (batch, head).  Under grouped-query attention
    a query head h reads K/V head h // (heads / kv_heads), and dK, dV of a
    K/V head are the sums over its query heads; with one graph per batch
    entry, (b, h) uses the graph of graph head b * heads + h."""
    check_padded(p, out)
    vq = p.q_group >= 0
    vk = p.kv_group >= 0
    H, Hkv = p.heads, p.n_kv_heads
    grp = H // Hkv
    pooled = {k: ([], []) for k in ("o", "dq", "dk", "dv")}
    kv_ref = {}
    for b in range(batch):
        for h in range(H):
            hk = h // grp
            A = _allowed(p, p.graph_head(b, h))
            q, do = _f64(t["q"][b, h]), _f64(t["do"][b, h])
            k, v = _f64(t["k"][b, hk]), _f64(t["v"][b, hk])
            M = oracle.token_mask(p.q_group, p.kv_group, A)
            o_ref, lse_ref = oracle.forward(q, k, v, M, p.scale)
            dq_ref, dk_ref, dv_ref = oracle.backward(q, k, v, do, M, p.scale)
            nonempty = M.any(axis=1)
            lse_gpu = out["lse"][b, h].numpy().astype(np.float64)
            assert np.array_equal(np.isneginf(lse_gpu), ~nonempty), (b, h)
            assert np.all(np.abs(lse_gpu[nonempty] - lse_ref[nonempty]) <= TOL["lse_abs"]), (b, h)
            o_g = _f64(out["o"][b, h])
            assert np.abs(o_g[vq] - o_ref[vq]).max() <= TOL["o_abs"], (b, h)
            assert rel_l2(o_g[vq], o_ref[vq]) <= TOL["o_rel"], (b, h, rel_l2(o_g[vq], o_ref[vq]))
            pooled["o"][0].append(o_g[vq]); pooled["o"][1].append(o_ref[vq])
            dq_g = _f64(out["dq"][b, h])
            assert rel_l2(dq_g[vq], dq_ref[vq]) <= TOL["grad_rel"], ("dq", b, h, rel_l2(dq_g[vq], dq_ref[vq]))
            pooled["dq"][0].append(dq_g[vq]); pooled["dq"][1].append(dq_ref[vq])
            # attention-free valid rows are exact zeros
            assert np.all(o_g[~nonempty] == 0)
            assert np.all(dq_g[~nonempty] == 0)
            acc = kv_ref.setdefault((b, hk), [0.0, 0.0, np.zeros(p.kv_slots, bool)])
            acc[0] = acc[0] + dk_ref
            acc[1] = acc[1] + dv_ref
            acc[2] |= M.any(axis=0)
    for (b, hk), (dk_ref, dv_ref, reached) in kv_ref.items():
        for name, ref in (("dk", dk_ref), ("dv", dv_ref)):
            g = _f64(out[name][b, hk])
            assert rel_l2(g[vk], ref[vk]) <= TOL["grad_rel"], (name, b, hk, rel_l2(g[vk], ref[vk]))
            pooled[name][0].append(g[vk]); pooled[name][1].append(ref[vk])
            # keys no query head of the group attends get exact zero gradients
            assert np.all(g[~reached] == 0), (name, b, hk)
    g = {k: (np.concatenate(a), np.concatenate(r)) for k, (a, r) in pooled.items() if a}
    assert rel_l2(*g["o"]) <= TOL["o_rel"], rel_l2(*g["o"])
    for k in ("dq", "dk", "dv"):
        assert rel_l2(*g[k]) <= TOL["grad_rel"], (k, rel_l2(*g[k]))


@pytest.mark.parametrize("name,batch", [(n, 1) for n in ["tiny"] + list(W.EXTRA_TINY) if n != "tiny_bgraph"]
                         + [("tiny_svg2", 2), ("tiny_gqa", 2), ("tiny_bgraph", 2)])
def test_tiny_full_parity(name, batch):
    p = W.make_problem(name)
    t, out, _ = run_gpu(p, batch=batch)
    check_tiny(p, t, out, batch)


@pytest.mark.parametrize("batch", [1, 2])
def test_tiny_split_packing_parity(batch, monkeypatch):
    """Clustered layout with the group-split packing forced: pages shared by
    two work items (each owning the rows of its cluster) in both passes."""
    p = W.make_problem("tiny_svg2")
    monkeypatch.setenv("SPATTN_PLAN_PACK", "split")
    pl = sp.Plan.from_problem(p, batch=batch)
    monkeypatch.delenv("SPATTN_PLAN_PACK")
    t, out, _ = run_gpu(p, batch, pl=pl)
    check_tiny(p, t, out, batch)


@pytest.mark.parametrize("name,batch", [(n, 1) for n in ["tiny", "tiny_vsa", "tiny_svg2", "tiny_hedge", "tiny_onekey",
                                                          "tiny_nokeys", "tiny_d128", "tiny_gqa"]]
                         + [("tiny_vsa", 2), ("tiny_bgraph", 2)])
def test_tiny_route64_parity(name, batch, monkeypatch):
    """The 64-row route forced on every query-owned item (two M = 64 halves
    per tile, each over its own column list; dQ runs the same list over all
    128 rows), forward and backward against the oracle."""
    p = W.make_problem(name)
    monkeypatch.setenv("SPATTN_PLAN_PACK", "route64")
    pl = sp.Plan.from_problem(p, batch=batch)
    monkeypatch.delenv("SPATTN_PLAN_PACK")
    assert (pl.work(0)[0][:, 28] == 1).all()
    t, out, _ = run_gpu(p, batch, pl=pl)
    check_tiny(p, t, out, batch)


def test_empty_column_lists_are_exercised():
    """tiny_nokeys head 1 attends nothing: its work items have empty column
    lists (no steps); the outputs are exact zeros and LSE = -inf there."""
    p = W.make_problem("tiny_nokeys")
    pl = sp.Plan.from_problem(p)
    for which in (0, 1):
        work, _, _ = pl.work(which)
        empty = work[:, 3] == work[:, 2]
        assert empty.any() and (work[empty, 0] == 1).all()
    t, out, _ = run_gpu(p, pl=pl)
    check_tiny(p, t, out, 1)
    valid_q = torch.from_numpy(p.q_group >= 0)
    assert torch.isneginf(out["lse"][0, 1, valid_q]).all()
    assert (out["dk"][0, 1] == 0).all() and (out["dv"][0, 1] == 0).all()


@pytest.mark.parametrize("name", ["tiny_svg2", "tiny_vsa", "tiny_empty"])
def test_repeat_parity(name):
    """The same launch repeated 20 times, each result against the oracle.

    tiny_svg2's key tiles hold more than four groups and are split into
    several work items that share the tile (the split-tile path); tiny_vsa
    and tiny_empty exercise partial last steps and rows without keys.  A
    race between warps of a CTA would show up as a run that differs."""
    p = W.make_problem(name)
    t = W.make_tensors(p)
    pl = sp.Plan.from_problem(p)
    first = None
    for _ in range(20):
        _, out, _ = run_gpu(p, t=t, pl=pl)
        if first is None:
            check_tiny(p, t, out, 1)
            first = out
        else:
            for k in out:
                if not torch.equal(out[k], first[k]):
                    check_tiny(p, t, out, 1)  # a differing run must still be correct
                    raise AssertionError(f"{name}: {k} differs between identical launches")


# Stratified sample units of the 21x45x80 STA layouts (6 x 12 x 20 tiles of
# 4x4x4): interior, T-edge (t = 5), H-edge (h = 11), the T x H corner
# (5, 11, 19), the origin (0, 0, 0) and an interior tile next to both edges.
STA_PARTIAL_TILES = [(2, 5, 7), (5, 5, 9), (2, 11, 3), (5, 11, 19), (0, 0, 0), (3, 6, 10), (4, 10, 19), (5, 0, 0)]


def _sample_units(p, rng):
    """(head, Q block) and (head, 64-slot key block) units, stratified for STA layouts."""
    n_qb = -(-p.q_slots // 64)
    n_kb = -(-p.kv_slots // 64)
    if p.name in ("partial", "vsa"):
        nh, nw = 12, 20
        blocks = [(a * nh + b) * nw + c for (a, b, c) in STA_PARTIAL_TILES]
        kblocks = list(blocks)
    elif p.name == "full":
        blocks = [0, 37, 128, 255, 100, 201]
        kblocks = [0, 255, 31, 224, 100, 137]
    else:
        blocks = rng.choice(n_qb, size=6, replace=False).tolist()
        blocks[-1] = n_qb - 1
        kblocks = rng.choice(n_kb, size=6, replace=False).tolist()
        kblocks[-1] = n_kb - 1
    qunits = [(int(rng.integers(p.heads)), int(b)) for b in blocks]
    kunits = [(int(rng.integers(p.heads)), int(b)) for b in kblocks]
    return qunits, kunits


@pytest.mark.parametrize("name", ["full", "partial", "vsa", "svg2"])
def test_large_sampled_parity(name):
    p = W.make_problem(name)
    t, out, pl = run_gpu(p)
    check_padded(p, out)
    rng = np.random.default_rng(1234)
    qunits, kunits = _sample_units(p, rng)
    o_g, o_r, dq_g, dq_r = [], [], [], []
    for h, qb in qunits:
        A = _allowed(p, h)
        rows = np.arange(64 * qb, min(64 * qb + 64, p.q_slots))
        rows = rows[p.q_group[rows] >= 0]
        if rows.size == 0:
            continue
        q, k, v, do = (_f64(t[n][0, h]) for n in ("q", "k", "v", "do"))
        o_ref, lse_ref = oracle.forward_rows(q, k, v, p.q_group, p.kv_group, A, rows, p.scale)
        dq_ref = oracle.dq_rows(q, k, v, do, p.q_group, p.kv_group, A, rows, p.scale)
        lse_gpu = out["lse"][0, h].numpy()[rows].astype(np.float64)
        assert np.all(np.abs(lse_gpu - lse_ref) <= TOL["lse_abs"]), (h, qb, np.abs(lse_gpu - lse_ref).max())
        og = _f64(out["o"][0, h])[rows]
        dqg = _f64(out["dq"][0, h])[rows]
        assert np.abs(og - o_ref).max() <= TOL["o_abs"], (h, qb)
        assert rel_l2(og, o_ref) <= TOL["o_rel"], (h, qb, rel_l2(og, o_ref))
        assert rel_l2(dqg, dq_ref) <= TOL["grad_rel"], (h, qb, rel_l2(dqg, dq_ref))
        o_g.append(og); o_r.append(o_ref)
        dq_g.append(dqg); dq_r.append(dq_ref)
    assert rel_l2(np.concatenate(o_g), np.concatenate(o_r)) <= TOL["o_rel"]
    assert rel_l2(np.concatenate(dq_g), np.concatenate(dq_r)) <= TOL["grad_rel"]
    dk_g, dk_r, dv_g, dv_r = [], [], [], []
    for h, kb in kunits:
        A = _allowed(p, h)
        keys = np.arange(64 * kb, min(64 * kb + 64, p.kv_slots))
        keys = keys[p.kv_group[keys] >= 0]
        if keys.size == 0:
            continue
        q, k, v, do = (_f64(t[n][0, h]) for n in ("q", "k", "v", "do"))
        dk_ref, dv_ref = oracle.dkdv_keys(q, k, v, do, p.q_group, p.kv_group, A, keys, p.scale)
        dkg = _f64(out["dk"][0, h])[keys]
        dvg = _f64(out["dv"][0, h])[keys]
        assert rel_l2(dkg, dk_ref) <= TOL["grad_rel"], (h, kb, rel_l2(dkg, dk_ref))
        assert rel_l2(dvg, dv_ref) <= TOL["grad_rel"], (h, kb, rel_l2(dvg, dv_ref))
        dk_g.append(dkg); dk_r.append(dk_ref)
        dv_g.append(dvg); dv_r.append(dv_ref)
    assert len(dk_g) >= 6
    assert rel_l2(np.concatenate(dk_g), np.concatenate(dk_r)) <= TOL["grad_rel"]
    assert rel_l2(np.concatenate(dv_g), np.concatenate(dv_r)) <= TOL["grad_rel"]


def test_repeat_calls_are_deterministic():
    p = W.make_problem("tiny_svg2")
    t = W.make_tensors(p)
    dev = {k: v.cuda() for k, v in t.items()}
    pl = sp.Plan.from_problem(p)
    outs = []
    for _ in range(2):
        o, lse = sp.spattn_fwd(dev["q"], dev["k"], dev["v"], pl)
        g = sp.spattn_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], pl)
        outs.append([o.clone(), lse.clone(), *[x.clone() for x in g]])
    sp.spattn_check(pl)
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_rejects_misaligned_pointer():
    p = W.make_problem("tiny")
    t = W.make_tensors(p)
    pl = sp.Plan.from_problem(p)
    q = t["q"].cuda()
    lib = sp.load_library()
    import ctypes
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    st = lib.spattn_fwd(ctypes.c_void_p(q.data_ptr() + 2), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(q.data_ptr()),
                        pl.handle, ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()), None)
    assert st == 1
