"""CPU fp64 oracle for exact block-sparse attention — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (the C-ABI library and its Python binding) never calls it, and it
shares no code with that path: it is a plain, slow restatement of the
definition, written from the KPage abstract ("KPage: block-sparse attention
for partially occupied 3D blocks", zhuanzhiai.com, abstract paragraph), which
states that the method preserves the original sparse graph exactly in forward
and backward execution.  The exact result it must reach is therefore masked
softmax attention over the explicit token-level mask and its analytic
gradients, which is what this package computes, in float64, with NumPy.

Every function here is pinned by ``tests/test_oracle.py`` against something
other than itself (dense attention from ``torch`` on a full graph, closed
forms for single-key rows and zero queries, central finite differences,
brute-force counts).  ``oracle.fp8`` (the E4M3 codec and per-slice quantiser
of the FP8 forward) is pinned by ``tests/test_oracle_fp8.py`` against
hand-computed codes of the format and a brute-force nearest-value search.
"""

from .attention import (  # noqa: F401
    allowed_groups,
    token_mask,
    forward,
    backward,
    forward_rows,
    dq_rows,
    dkdv_keys,
)
from .plan import (  # noqa: F401
    page_valid_masks,
    canonical_pages,
    transposed_qblocks,
    useful_pairs_bruteforce,
    useful_pairs_closed_form,
    bsa_physical_pairs,
)
from . import fp8  # noqa: F401,E402
