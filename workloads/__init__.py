"""Seeded synthetic workloads for exact block-sparse attention.

This package only *builds inputs*: token layouts (which slot holds which
token group, or a padded row), sparse group graphs (which key groups each
query group may attend, per head) and the bf16 tensors Q, K, V, dO.  It holds
none of the attention arithmetic, so both the CPU oracle and the CUDA path can
consume the same inputs without sharing any of the method's code.
"""

from .configs import (  # noqa: F401
    CONFIG_NAMES,
    EXTRA_TINY,
    Problem,
    make_problem,
    make_tensors,
    with_heads,
    sta_layout,
    sta_graph,
    vsa_graph,
    cluster_layout,
    cluster_graph,
)
