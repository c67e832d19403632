"""The C-ABI library loads, exports every declared entry point, and rejects
bad arguments with the documented status codes (host-side checks only)."""

import ctypes
import os
import re

import numpy as np
import pytest

import block_sparse_attention_bwd_b200 as sp
from workloads import configs as W

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "spattn.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(spattn_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(sp.LIB_PATH)
    names = declared_functions()
    assert "spattn_plan" in names and "spattn_fwd" in names and "spattn_bwd" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(sp.ENTRY_POINTS)


def _plan(p, **over):
    kw = dict(batch=p.batch, heads=p.heads, head_dim=p.head_dim, scale=p.scale)
    kw.update(over)
    return sp.Plan(p.q_group, p.kv_group, p.n_q_groups, p.n_kv_groups, p.row_ptr, p.kv_groups, **kw)


def test_plan_builds_on_host():
    p = W.make_problem("tiny")
    pl = _plan(p)
    st = pl.stats()
    assert st["useful_pairs"] == 2 * 300 * 300
    pl.close()


@pytest.mark.parametrize("over,code", [
    (dict(head_dim=96), 2),
    (dict(head_dim=32), 2),
    (dict(batch=0), 1),
    (dict(heads=0), 1),
])
def test_plan_rejects_bad_sizes(over, code):
    p = W.make_problem("tiny")
    with pytest.raises(sp.SpattnError) as e:
        _plan(p, **over)
    assert e.value.status == code


def test_plan_rejects_bad_groups_and_graph():
    p = W.make_problem("tiny_onekey")
    bad = p.q_group.copy()
    bad[3] = p.n_q_groups  # out of range
    with pytest.raises(sp.SpattnError) as e:
        sp.Plan(bad, p.kv_group, p.n_q_groups, p.n_kv_groups, p.row_ptr, p.kv_groups, batch=1, heads=1, head_dim=64)
    assert e.value.status == 1
    bad = p.kv_group.copy()
    bad[0] = -2
    with pytest.raises(sp.SpattnError):
        sp.Plan(p.q_group, bad, p.n_q_groups, p.n_kv_groups, p.row_ptr, p.kv_groups, batch=1, heads=1, head_dim=64)
    cols = p.kv_groups.copy()
    cols[0] = 7
    with pytest.raises(sp.SpattnError):
        sp.Plan(p.q_group, p.kv_group, p.n_q_groups, p.n_kv_groups, p.row_ptr, cols, batch=1, heads=1, head_dim=64)
    rp = p.row_ptr.copy()
    rp[1] = rp[2] + 1  # decreasing
    with pytest.raises(sp.SpattnError):
        sp.Plan(p.q_group, p.kv_group, p.n_q_groups, p.n_kv_groups, rp, p.kv_groups, batch=1, heads=1, head_dim=64)


def test_null_arguments_are_rejected():
    lib = sp.load_library()
    assert lib.spattn_plan(None, None, None) == 1
    h = ctypes.c_void_p()
    assert lib.spattn_plan(None, None, ctypes.byref(h)) == 1
    assert lib.spattn_fwd(None, None, None, None, None, None, None) == 1
    assert lib.spattn_bwd(None, None, None, None, None, None, None, None, None, None, None) == 1
    assert lib.spattn_check(None, None) == 1
    assert lib.spattn_plan_stats(None, None) == 1
    lib.spattn_plan_destroy(None)
    assert lib.spattn_status_string(5) == b"device-side wait timed out"


def test_inspection_rejects_out_of_range():
    p = W.make_problem("tiny")
    pl = _plan(p)
    with pytest.raises(sp.SpattnError):
        pl.pages(p.heads, 0)
    with pytest.raises(sp.SpattnError):
        pl.pages(0, 12)
    with pytest.raises(sp.SpattnError):
        pl.qblocks(0, 10 ** 6)
    with pytest.raises(sp.SpattnError):
        pl.work(2)


def test_wait_selftest_argument_checks_on_host():
    lib = sp.load_library()
    assert lib.spattn_wait_selftest(None, 1_000_000, None) == 1
    p = W.make_problem("tiny")
    pl = _plan(p)
    # deadline outside 10^4 .. 2*10^9 cycles
    assert lib.spattn_wait_selftest(pl.handle, 10, None) == 1
    assert lib.spattn_wait_selftest(pl.handle, 3_000_000_000, None) == 1
    # a plan built without a GPU cannot launch anything
    if not sp_device_available():
        assert lib.spattn_wait_selftest(pl.handle, 1_000_000, None) == 4
    pl.close()


def sp_device_available():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def test_device_replan_needs_a_device_and_arguments():
    """spattn_plan_set_graph_device: argument checks on the host, and a plan
    built without a device answers SPATTN_ERR_CUDA."""
    p = W.make_problem("tiny")
    pl = _plan(p)
    lib = sp.load_library()
    one = ctypes.c_void_p(16)
    assert lib.spattn_plan_set_graph_device(None, one, one, 0, None) == sp.SPATTN_ERR_INVALID_ARG
    assert lib.spattn_plan_set_graph_device(pl.handle, None, one, 0, None) == sp.SPATTN_ERR_INVALID_ARG
    assert lib.spattn_plan_set_graph_device(pl.handle, one, None, 5, None) == sp.SPATTN_ERR_INVALID_ARG
    assert lib.spattn_plan_set_graph_device(pl.handle, one, one, -1, None) == sp.SPATTN_ERR_INVALID_ARG
    import torch
    if not torch.cuda.is_available():
        assert lib.spattn_plan_set_graph_device(pl.handle, one, one, 0, None) == sp.SPATTN_ERR_CUDA
