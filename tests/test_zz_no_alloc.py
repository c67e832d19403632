"""spattn_bwd_noalloc: the backward pass that allocates nothing.

Callers that cannot allocate device memory when they run the backward pass
(another allocator owns the GPU, or a fixed memory budget) use this entry
point; its scratch is a static device array inside the library.  These tests
call it through the C ABI twice in a row, the second time with a different
dO, and compare each result with spattn_bwd on the same inputs.  Both paths
run the same deterministic, atomic-free kernels, so the outputs must be
bit-identical; the second call would differ if it read the first call's
Delta from the shared scratch instead of rewriting it.  Sizes beyond the
static scratch must be rejected before anything is launched.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_bwd_b200 as sp
from workloads import configs as W

pytestmark = pytest.mark.gpu

SCRATCH_ROWS = 1 << 22


@pytest.mark.parametrize("name", ["tiny_svg2", "tiny_d128", "tiny_vsa"])
def test_noalloc_matches_bwd_on_two_calls(name):
    p = W.make_problem(name)
    t = {k: v.cuda() for k, v in W.make_tensors(p).items()}
    plan = sp.Plan.from_problem(p)
    o, lse = sp.spattn_fwd(t["q"], t["k"], t["v"], plan)
    # a second loss gradient: another seeded draw, same shape (padded rows keep the sentinel)
    do2 = torch.flip(t["do"], dims=[3]).contiguous() * 0.5
    lib = sp.load_library()
    stream = torch.cuda.current_stream()
    for do in (t["do"], do2):
        ref = sp.spattn_bwd(t["q"], t["k"], t["v"], o, lse, do, plan)
        sp.spattn_check(plan)
        # pre-fill with a value the pass must overwrite everywhere
        out = [torch.full_like(r, 7.0) for r in ref]
        st = lib.spattn_bwd_noalloc(*(ctypes.c_void_p(x.data_ptr()) for x in (t["q"], t["k"], t["v"], o, lse, do)),
                                    plan.handle, *(ctypes.c_void_p(x.data_ptr()) for x in out),
                                    ctypes.c_void_p(stream.cuda_stream))
        assert st == 0, sp.STATUS_NAMES.get(st, st)
        sp.spattn_check(plan)
        for got, want in zip(out, ref):
            assert torch.equal(got, want)
    # the two calls really saw different gradients
    assert not torch.equal(sp.spattn_bwd(t["q"], t["k"], t["v"], o, lse, do2, plan)[0],
                           sp.spattn_bwd(t["q"], t["k"], t["v"], o, lse, t["do"], plan)[0])


def test_noalloc_rejects_rows_beyond_scratch():
    q_slots = SCRATCH_ROWS + 1
    qg = np.full(q_slots, -1, np.int32)
    qg[:16] = 0
    kg = np.zeros(16, np.int32)
    plan = sp.Plan(qg, kg, 1, 1, np.array([0, 1], np.int64), np.array([0], np.int32), batch=1, heads=1, head_dim=64)
    small = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    ptr = ctypes.c_void_p(small.data_ptr())
    lib = sp.load_library()
    st = lib.spattn_bwd_noalloc(ptr, ptr, ptr, ptr, ptr, ptr, plan.handle, ptr, ptr, ptr, None)
    assert st == 2  # SPATTN_ERR_UNSUPPORTED, nothing launched
    torch.cuda.synchronize()
