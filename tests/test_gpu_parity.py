"""CUDA path (through the C ABI) against the fp64 oracle, element by element.

Tolerances (over valid rows, the bf16 outputs against fp64 on the same bf16
inputs): O max-abs <= 1e-2 and relative L2 <= 5e-3; LSE abs <= 1e-3;
dQ, dK, dV relative L2 <= 1e-2.  Padded and attention-free rows must be
exact: O = 0, LSE = -inf, dQ = 0, dK = dV = 0.  The backward consumes the
GPU's own O and LSE.

Tiny workloads are compared in full; the large ones are run at full size in
the launch configuration the benchmark uses and compared on sampled units
(whole Q blocks for O / LSE / dQ, whole 64-slot key blocks for dK / dV),
stratified over interior, T-edge, H-edge and corner blocks.
"""

import math

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
    return float(np.linalg.norm(a - b)) / max(den, 1e-30)


def _allowed(p, h):
    return oracle.allowed_groups(p.row_ptr, p.kv_groups, p.n_q_groups, p.n_kv_groups, h)


def run_gpu(p, batch=None):
    t = W.make_tensors(p, batch=batch)
    dev = {k: v.cuda() for k, v in t.items()}
    pl = sp.Plan.from_problem(p, batch=batch)
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


@pytest.mark.parametrize("name,batch", [(n, 1) for n in ["tiny"] + list(W.EXTRA_TINY)] + [("tiny_svg2", 2)])
def test_tiny_full_parity(name, batch):
    p = W.make_problem(name)
    t, out, _ = run_gpu(p, batch=batch)
    check_padded(p, out)
    vq = p.q_group >= 0
    vk = p.kv_group >= 0
    acc = {k: ([], []) for k in ("o", "lse", "dq", "dk", "dv")}
    for b in range(batch):
        for h in range(p.heads):
            A = _allowed(p, h)
            q, k, v, do = (_f64(t[n][b, h]) for n in ("q", "k", "v", "do"))
            M = oracle.token_mask(p.q_group, p.kv_group, A)
            o_ref, lse_ref = oracle.forward(q, k, v, M, p.scale)
            dq_ref, dk_ref, dv_ref = oracle.backward(q, k, v, do, M, p.scale)
            nonempty = M.any(axis=1)
            lse_gpu = out["lse"][b, h].numpy().astype(np.float64)
            assert np.array_equal(np.isneginf(lse_gpu), ~nonempty)
            assert np.all(np.abs(lse_gpu[nonempty] - lse_ref[nonempty]) <= TOL["lse_abs"])
            acc["o"][0].append(_f64(out["o"][b, h])[vq]); acc["o"][1].append(o_ref[vq])
            acc["dq"][0].append(_f64(out["dq"][b, h])[vq]); acc["dq"][1].append(dq_ref[vq])
            acc["dk"][0].append(_f64(out["dk"][b, h])[vk]); acc["dk"][1].append(dk_ref[vk])
            acc["dv"][0].append(_f64(out["dv"][b, h])[vk]); acc["dv"][1].append(dv_ref[vk])
            # attention-free valid rows are exact zeros
            assert np.all(_f64(out["o"][b, h])[~nonempty] == 0)
            assert np.all(_f64(out["dq"][b, h])[~nonempty] == 0)
    g = {k: (np.concatenate(a), np.concatenate(r)) for k, (a, r) in acc.items() if a}
    assert np.abs(g["o"][0] - g["o"][1]).max() <= TOL["o_abs"]
    assert rel_l2(*g["o"]) <= TOL["o_rel"], rel_l2(*g["o"])
    for k in ("dq", "dk", "dv"):
        assert rel_l2(*g[k]) <= TOL["grad_rel"], (k, rel_l2(*g[k]))


def _sample_units(p, rng):
    """(head, Q block) and (head, 64-slot key block) units, stratified for STA layouts."""
    n_qb = -(-p.q_slots // 64)
    n_kb = -(-p.kv_slots // 64)
    blocks = []
    if p.name in ("partial", "vsa"):
        nt, nh, nw = 6, 12, 20
        for (a, b, c) in [(2, 5, 7), (5, 5, 9), (2, 11, 3), (5, 11, 19), (0, 0, 0), (3, 6, 10)]:
            blocks.append((a * nh + b) * nw + c)
    elif p.name == "full":
        blocks = [0, 37, 128, 255, 100, 201]
    else:
        blocks = rng.choice(n_qb, size=6, replace=False).tolist()
        blocks[-1] = n_qb - 1
    qunits = [(int(rng.integers(p.heads)), int(b)) for b in blocks]
    kblocks = blocks[:3]
    if p.name == "svg2":
        kblocks = rng.choice(n_kb, size=3, replace=False).tolist()
        kblocks[-1] = n_kb - 1
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
        assert np.all(np.abs(lse_gpu - lse_ref) <= TOL["lse_abs"]), np.abs(lse_gpu - lse_ref).max()
        o_g.append(_f64(out["o"][0, h])[rows]); o_r.append(o_ref)
        dq_g.append(_f64(out["dq"][0, h])[rows]); dq_r.append(dq_ref)
    o_g, o_r = np.concatenate(o_g), np.concatenate(o_r)
    assert np.abs(o_g - o_r).max() <= TOL["o_abs"]
    assert rel_l2(o_g, o_r) <= TOL["o_rel"], rel_l2(o_g, o_r)
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
        dk_g.append(_f64(out["dk"][0, h])[keys]); dk_r.append(dk_ref)
        dv_g.append(_f64(out["dv"][0, h])[keys]); dv_r.append(dv_ref)
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
