"""FP8 forward (spattn_quantize_fp8, spattn_fwd_fp8) against the fp64 oracle.

The quantiser is integer work (one byte per element) and must match the
oracle's E4M3 quantiser bit for bit, codes and descale factors.  The forward
is compared with the oracle's attention of the oracle-dequantised Q and K
(v in bf16 as in the bf16 path), with the bf16 forward's tolerances: the
kernel's S accumulates exact E4M3 x E4M3 products in fp32 and P, V, O are
handled exactly as in spattn_fwd, so the error budget is the same
(O max-abs <= 1e-2, relative L2 <= 5e-3, LSE abs <= 1e-3 per (batch, head)
or per sampled unit; padded rows exact).
"""

import dataclasses

import numpy as np
import pytest
import torch

import block_sparse_attention_bwd_b200 as sp
import oracle
from oracle import fp8
from workloads import configs as W

pytestmark = pytest.mark.gpu

TOL = dict(o_abs=1e-2, o_rel=5e-3, lse_abs=1e-3)


def rel_l2(a, b):
    den = float(np.linalg.norm(b))
    num = float(np.linalg.norm(a - b))
    return (0.0 if num == 0.0 else float("inf")) if den == 0.0 else num / den


def _d128(name):
    return dataclasses.replace(W.make_problem(name), head_dim=128)


def _oracle_quant(x):
    """Oracle codes and descale of a [B, H, S, D] bf16 tensor (per (b, h) slice)."""
    B, H, S, D = x.shape
    c, d = fp8.quantize_e4m3(x.float().numpy().reshape(B * H, S, D))
    return c.reshape(B, H, S, D), d.reshape(B, H)


def _check_quant(x):
    x8, ds = sp.quantize_fp8(x.cuda())
    c_ref, d_ref = _oracle_quant(x)
    assert np.array_equal(x8.cpu().numpy(), c_ref)
    assert np.array_equal(ds.cpu().numpy().view(np.uint32), d_ref.view(np.uint32))
    return c_ref, d_ref


def test_quantize_bit_exact_wide_range():
    g = torch.Generator().manual_seed(5)
    x = torch.randn(2, 3, 200, 128, generator=g)
    x[0, 1] *= torch.logspace(-6, 2, 200).unsqueeze(1)  # subnormal codes and a wide spread in one slice
    x[1, 0] = 0.0                                       # an all-zero slice: descale 1, codes 0
    x[1, 2, 7, 3] = 3.0e4                               # one large outlier
    _check_quant(x.to(torch.bfloat16))
    _check_quant(torch.randn(1, 2, 40, 64, generator=g).to(torch.bfloat16))


@pytest.mark.parametrize("name,batch,route", [("tiny_d128", 1, ""), ("tiny_vsa", 1, ""), ("tiny_hedge", 1, ""),
                                              ("tiny_svg2", 2, ""), ("tiny_gqa", 2, ""), ("tiny_empty", 1, ""),
                                              ("tiny_bgraph", 2, ""), ("tiny_vsa", 1, "route64"),
                                              ("tiny_svg2", 2, "route64")])
def test_fwd_fp8_tiny_parity(name, batch, route, monkeypatch):
    p = _d128(name) if name != "tiny_d128" else W.make_problem(name)
    t = W.make_tensors(p, batch=batch)
    if route:
        monkeypatch.setenv("SPATTN_PLAN_PACK", route)  # the 64-row route forced on every query-owned item
    pl = sp.Plan.from_problem(p, batch=batch)
    monkeypatch.delenv("SPATTN_PLAN_PACK", raising=False)
    assert (pl.work(0)[0][:, 28] == 1).all() or not route
    q8c, qd = _check_quant(t["q"])
    k8c, kd = _check_quant(t["k"])
    q8, qds = sp.quantize_fp8(t["q"].cuda())
    k8, kds = sp.quantize_fp8(t["k"].cuda())
    o, lse = sp.spattn_fwd_fp8(q8, k8, qds, kds, t["v"].cuda(), pl)
    sp.spattn_check(pl)
    o, lse = o.cpu(), lse.cpu()
    q_hat = fp8.e4m3_decode(q8c) * qd[..., None, None]
    k_hat = fp8.e4m3_decode(k8c) * kd[..., None, None]
    vq = p.q_group >= 0
    pq = torch.from_numpy(~vq)
    if bool(pq.any()):
        assert torch.all(o[:, :, pq] == 0) and torch.all(torch.isneginf(lse[:, :, pq]))
    grp = p.heads // p.n_kv_heads
    for b in range(batch):
        for h in range(p.heads):
            hk = h // grp
            A = oracle.allowed_groups(p.row_ptr, p.kv_groups, p.n_q_groups, p.n_kv_groups, p.graph_head(b, h))
            M = oracle.token_mask(p.q_group, p.kv_group, A)
            o_ref, lse_ref = oracle.forward(q_hat[b, h], k_hat[b, hk], t["v"][b, hk].to(torch.float64).numpy(), M,
                                            p.scale)
            nonempty = M.any(axis=1)
            lg = lse[b, h].numpy().astype(np.float64)
            assert np.array_equal(np.isneginf(lg), ~nonempty), (b, h)
            assert np.all(np.abs(lg[nonempty] - lse_ref[nonempty]) <= TOL["lse_abs"]), (b, h)
            og = o[b, h].to(torch.float64).numpy()
            assert np.abs(og[vq] - o_ref[vq]).max() <= TOL["o_abs"], (b, h)
            assert rel_l2(og[vq], o_ref[vq]) <= TOL["o_rel"], (b, h, rel_l2(og[vq], o_ref[vq]))
            assert np.all(og[~nonempty] == 0)


def test_fwd_fp8_large_sampled_partial():
    """The partial-block workload at full size (the benchmark's launch
    configuration): codes of two heads bit-exact, O / LSE of sampled query
    blocks (interior, T-edge, H-edge, corner) per unit."""
    p = W.make_problem("partial")
    t = W.make_tensors(p)
    pl = sp.Plan.from_problem(p)
    q8, qds = sp.quantize_fp8(t["q"].cuda())
    k8, kds = sp.quantize_fp8(t["k"].cuda())
    o, lse = sp.spattn_fwd_fp8(q8, k8, qds, kds, t["v"].cuda(), pl)
    sp.spattn_check(pl)
    blocks = (0, 19, 11 * 20 + 3, 5 * 240 + 11 * 20 + 19)  # interior-ish, W-edge, H-edge, T/H corner
    for h in (0, 23):
        qc, qd = fp8.quantize_e4m3(t["q"][0, h].float().numpy()[None])
        kc, kd = fp8.quantize_e4m3(t["k"][0, h].float().numpy()[None])
        assert np.array_equal(q8[0, h].cpu().numpy(), qc[0]) and np.array_equal(k8[0, h].cpu().numpy(), kc[0])
        assert qds[0, h].item() == float(qd[0]) and kds[0, h].item() == float(kd[0])
        q_hat = fp8.dequantize_e4m3(qc, qd)[0]
        k_hat = fp8.dequantize_e4m3(kc, kd)[0]
        A = oracle.allowed_groups(p.row_ptr, p.kv_groups, p.n_q_groups, p.n_kv_groups, h)
        v = t["v"][0, h].to(torch.float64).numpy()
        for qb in blocks:
            rows = np.arange(64 * qb, 64 * qb + 64)
            rows = rows[p.q_group[rows] >= 0]
            o_ref, lse_ref = oracle.forward_rows(q_hat, k_hat, v, p.q_group, p.kv_group, A, rows, p.scale)
            og = o[0, h].cpu().to(torch.float64).numpy()[rows]
            lg = lse[0, h].cpu().numpy().astype(np.float64)[rows]
            assert np.abs(og - o_ref).max() <= TOL["o_abs"], (h, qb)
            assert rel_l2(og, o_ref) <= TOL["o_rel"], (h, qb, rel_l2(og, o_ref))
            assert np.abs(lg - lse_ref).max() <= TOL["lse_abs"], (h, qb)


def test_fwd_fp8_rejects_head_dim_64():
    p = W.make_problem("tiny")  # D = 64
    t = W.make_tensors(p)
    pl = sp.Plan.from_problem(p)
    q8, qds = sp.quantize_fp8(t["q"].cuda())
    k8, kds = sp.quantize_fp8(t["k"].cuda())
    with pytest.raises(sp.SpattnError) as e:
        sp.spattn_fwd_fp8(q8, k8, qds, kds, t["v"].cuda(), pl)
    assert e.value.status == sp.SPATTN_ERR_UNSUPPORTED
