"""Failure detection on the GPU without a fault: a device-side wait that can
never complete ends by its deadline, the host reads SPATTN_ERR_TIMEOUT, and
the context stays usable for the next fwd/bwd."""

import pytest
import torch

import block_sparse_attention_bwd_b200 as sp
from workloads import configs as W

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    p = W.make_problem("tiny_d128")
    t = {k: v.cuda() for k, v in W.make_tensors(p).items()}
    pl = sp.Plan.from_problem(p)
    o_ref, lse_ref = sp.spattn_fwd(t["q"], t["k"], t["v"], pl)
    sp.spattn_check(pl)
    # ~1 ms at B200 clocks: warp 0 times out, warp 1 follows the abort flag
    assert sp.spattn_wait_selftest(pl, 2_000_000) == sp.SPATTN_ERR_TIMEOUT
    # the error word was cleared by that check
    sp.spattn_check(pl)
    # the context is intact: the same inputs give the same results
    o, lse = sp.spattn_fwd(t["q"], t["k"], t["v"], pl)
    g = sp.spattn_bwd(t["q"], t["k"], t["v"], o, lse, t["do"], pl)
    sp.spattn_check(pl)
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
    assert all(torch.isfinite(x.float()).all() for x in g)
