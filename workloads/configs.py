"""Seeded synthetic inputs: layouts, sparse group graphs and bf16 tensors.

Definitions used throughout (they mirror the problem statement of the KPage
abstract, "KPage: block-sparse attention for partially occupied 3D blocks",
zhuanzhiai.com, abstract paragraph: a sparse graph over logical blocks of a
3D video token layout whose edge blocks are only partly occupied):

* A *slot* is one row of Q (or K/V).  ``q_group[i]`` is the query group of
  slot ``i`` (``-1`` marks a padded slot that is never a query);
  ``kv_group[j]`` likewise for keys.
* The sparse *graph* is a CSR over (head, query group): row
  ``h * n_q_groups + a`` lists the key groups that query group ``a`` may attend
  in head ``h``.  The same graph serves every batch index.
* Query slot ``i`` may attend key slot ``j`` in head ``h`` iff both are valid
  and ``kv_group[j]`` is listed for ``q_group[i]``.

Layouts
-------
STA-style layouts reorder a T x H x W latent grid *tile-major* into 4x4x4
tiles: tiles are row-major over (tile_t, tile_h, tile_w) and, inside a tile,
slots are row-major over (dt, dh, dw) with dw fastest.  Each tile is one
64-slot logical block and one group; grid points outside T x H x W leave
padded slots, so edge tiles are partially occupied.

Cluster layouts (independent Q/K partitions) split N tokens into contiguous
clusters whose sizes are ``1 + Multinomial(N - C, uniform)``; the seeded token
permutation of the source only relabels i.i.d. inputs, so slots are generated
directly in cluster order.

Graph readings
--------------
* "clamped" window: along an axis with ``n`` tiles and window ``w``, take all
  tiles when ``n <= w``; otherwise the window starts at
  ``clamp(c - w // 2, 0, n - w)``, i.e. it is shifted inward, not truncated.
* VSA-style: per head and per query tile (tile-major order), the own tile plus
  ``k - 1`` other tiles drawn uniformly without replacement.
* cluster graph: per head, each query cluster draws ``k`` key clusters
  uniformly without replacement.

Tensors
-------
Q, K, V, dO are fp32 ``randn`` from a seeded ``torch.Generator`` rounded to
bf16 (round-to-nearest-even), shape [B, H, S, D].  Padded slots hold the
finite sentinel 1000.0 (exact in bf16) so that any leak of a padded row into a
result is visible.
"""

from __future__ import annotations

import dataclasses
import itertools
import math
from typing import Dict, Iterable, Optional, Sequence, Tuple

import numpy as np

PAD_SENTINEL = 1000.0

CONFIG_NAMES = ("tiny", "full", "partial", "vsa", "svg2")
EXTRA_TINY = ("tiny_vsa", "tiny_svg2", "tiny_empty", "tiny_d128", "tiny_onekey", "tiny_nokeys", "tiny_hedge",
              "tiny_gqa", "tiny_mqa", "tiny_bgraph")


@dataclasses.dataclass
class Problem:
    name: str
    batch: int
    heads: int
    head_dim: int
    q_group: np.ndarray  # int32 [q_slots]
    kv_group: np.ndarray  # int32 [kv_slots]
    n_q_groups: int
    n_kv_groups: int
    row_ptr: np.ndarray  # int64 [heads * n_q_groups + 1]
    kv_groups: np.ndarray  # int32 [nnz]
    seed_base: int
    description: str = ""
    kv_heads: int = 0        # K/V heads (grouped-query attention); 0 = heads
    graph_batches: int = 1   # 1: one graph for every batch entry; batch: one graph per entry

    @property
    def n_kv_heads(self) -> int:
        return self.heads if self.kv_heads == 0 else self.kv_heads

    def graph_head(self, b: int, h: int) -> int:
        """Row block of the graph that (batch entry b, query head h) uses."""
        return (b * self.heads + h) if self.graph_batches > 1 else h

    @property
    def q_slots(self) -> int:
        return int(self.q_group.shape[0])

    @property
    def kv_slots(self) -> int:
        return int(self.kv_group.shape[0])

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    def graph_row(self, head: int, q_grp: int) -> np.ndarray:
        r = head * self.n_q_groups + q_grp
        return self.kv_groups[self.row_ptr[r]:self.row_ptr[r + 1]]


# ----------------------------------------------------------------------------
# layouts
# ----------------------------------------------------------------------------

def sta_layout(grid: Sequence[int], tile: Sequence[int] = (4, 4, 4)) -> Tuple[np.ndarray, Tuple[int, int, int]]:
    """Tile-major slot layout of a T x H x W grid; returns (group, tiles_per_axis)."""
    T, H, W = grid
    tt, th, tw = tile
    nt, nh, nw = -(-T // tt), -(-H // th), -(-W // tw)
    per = tt * th * tw
    group = np.full(nt * nh * nw * per, -1, dtype=np.int32)
    ti, hi, wi, dt, dh, dw = np.meshgrid(
        np.arange(nt), np.arange(nh), np.arange(nw),
        np.arange(tt), np.arange(th), np.arange(tw), indexing="ij")
    tile_idx = (ti * nh + hi) * nw + wi
    slot = tile_idx * per + (dt * th + dh) * tw + dw
    valid = (ti * tt + dt < T) & (hi * th + dh < H) & (wi * tw + dw < W)
    group[slot[valid]] = tile_idx[valid]
    return group, (nt, nh, nw)


def cluster_layout(n_tokens: int, n_clusters: int, rng: np.random.Generator) -> np.ndarray:
    """Contiguous clusters with sizes 1 + Multinomial(N - C, uniform)."""
    sizes = 1 + rng.multinomial(n_tokens - n_clusters, np.full(n_clusters, 1.0 / n_clusters))
    return np.repeat(np.arange(n_clusters, dtype=np.int32), sizes)


# ----------------------------------------------------------------------------
# graphs
# ----------------------------------------------------------------------------

def _clamped_window(n: int, w: int, c: int) -> range:
    if n <= w:
        return range(n)
    s = min(max(c - w // 2, 0), n - w)
    return range(s, s + w)


def _csr(rows: Iterable[Sequence[int]]) -> Tuple[np.ndarray, np.ndarray]:
    rows = [np.asarray(sorted(r), dtype=np.int32) for r in rows]
    row_ptr = np.zeros(len(rows) + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum([len(r) for r in rows])
    cols = np.concatenate(rows) if rows else np.zeros(0, np.int32)
    return row_ptr, cols.astype(np.int32)


def sta_graph(tiles: Sequence[int], window: Sequence[int], heads: int) -> Tuple[np.ndarray, np.ndarray]:
    """Clamped sliding-tile window graph, identical for every head."""
    nt, nh, nw = tiles
    one_head = []
    for a, b, c in itertools.product(range(nt), range(nh), range(nw)):
        one_head.append([(x * nh + y) * nw + z
                         for x in _clamped_window(nt, window[0], a)
                         for y in _clamped_window(nh, window[1], b)
                         for z in _clamped_window(nw, window[2], c)])
    return _csr(one_head * heads)


def vsa_graph(n_tiles: int, heads: int, k: int, rng: np.random.Generator) -> Tuple[np.ndarray, np.ndarray]:
    """Own tile plus k-1 other tiles drawn without replacement, per head and tile."""
    rows = []
    for _h in range(heads):
        for a in range(n_tiles):
            other = rng.choice(n_tiles - 1, size=k - 1, replace=False)
            other = np.where(other >= a, other + 1, other)
            rows.append([a] + other.tolist())
    return _csr(rows)


def cluster_graph(n_q: int, n_k: int, heads: int, k: int, rng: np.random.Generator) -> Tuple[np.ndarray, np.ndarray]:
    rows = []
    for _h in range(heads):
        for _a in range(n_q):
            rows.append(rng.choice(n_k, size=k, replace=False).tolist())
    return _csr(rows)


# ----------------------------------------------------------------------------
# problems
# ----------------------------------------------------------------------------

def _sta_problem(name, idx, grid, window, heads, d, description):
    group, tiles = sta_layout(grid)
    n = tiles[0] * tiles[1] * tiles[2]
    row_ptr, cols = sta_graph(tiles, window, heads)
    return Problem(name, 1, heads, d, group, group.copy(), n, n, row_ptr, cols, 1000 * idx, description)


def make_problem(name: str) -> Problem:
    """Build the layout and graph of a named workload (no tensors)."""
    if name == "tiny":
        return _sta_problem(name, 1, (5, 6, 10), (3, 3, 3), 2, 64,
                            "tiny STA 5x6x10 in 4x4x4 tiles, clamped 3x3x3 window, H=2, D=64")
    if name == "full":
        return _sta_problem(name, 2, (16, 32, 32), (3, 3, 3), 16, 128,
                            "full-occupancy STA 16x32x32, clamped 3x3x3 window, H=16, D=128")
    if name == "partial":
        return _sta_problem(name, 3, (21, 45, 80), (3, 5, 5), 40, 128,
                            "partial-block STA 21x45x80, clamped 3x5x5 window, H=40, D=128")
    if name == "vsa":
        group, tiles = sta_layout((21, 45, 80))
        n = tiles[0] * tiles[1] * tiles[2]
        rng = np.random.default_rng(4000 + 5)
        row_ptr, cols = vsa_graph(n, 40, 32, rng)
        return Problem(name, 1, 40, 128, group, group.copy(), n, n, row_ptr, cols, 4000,
                       "VSA-style top-32 tiles (own + 31 random) over 21x45x80, H=40, D=128")
    if name == "svg2":
        rng = np.random.default_rng(5000 + 5)
        qg = cluster_layout(75600, 100, rng)
        kg = cluster_layout(75600, 500, rng)
        row_ptr, cols = cluster_graph(100, 500, 40, 64, rng)
        return Problem(name, 1, 40, 128, qg, kg, 100, 500, row_ptr, cols, 5000,
                       "independent Q/K partitions: 100 Q / 500 K clusters, 64 K clusters per Q cluster, H=40, D=128")
    if name == "tiny_vsa":
        group, tiles = sta_layout((5, 6, 10))
        rng = np.random.default_rng(10005)
        row_ptr, cols = vsa_graph(12, 2, 4, rng)
        return Problem(name, 1, 2, 64, group, group.copy(), 12, 12, row_ptr, cols, 10000,
                       "tiny VSA-style: own + 3 random of 12 tiles")
    if name == "tiny_svg2":
        rng = np.random.default_rng(11005)
        qg = cluster_layout(300, 7, rng)
        kg = cluster_layout(300, 23, rng)
        row_ptr, cols = cluster_graph(7, 23, 2, 5, rng)
        return Problem(name, 1, 2, 64, qg, kg, 7, 23, row_ptr, cols, 11000,
                       "tiny clusters: 300 tokens, 7 Q / 23 K clusters, 5 K clusters per Q cluster")
    if name == "tiny_empty":
        group, tiles = sta_layout((5, 6, 10))
        rows = []
        for h, window in enumerate([(1, 1, 3), (1, 1, 1)]):
            rp, cols = sta_graph(tiles, window, 1)
            for a in range(12):
                rows.append([] if a == 0 else cols[rp[a]:rp[a + 1]].tolist())
        row_ptr, cols = _csr(rows)
        return Problem(name, 1, 2, 64, group, group.copy(), 12, 12, row_ptr, cols, 12000,
                       "tiny STA with query tile 0 attending nothing (empty rows)")
    if name == "tiny_d128":
        group, tiles = sta_layout((5, 6, 10))
        row_ptr, cols = sta_graph(tiles, (1, 2, 1), 2)
        return Problem(name, 1, 2, 128, group, group.copy(), 12, 12, row_ptr, cols, 13000,
                       "tiny STA, window 1x2x1, D=128")
    if name == "tiny_onekey":
        qg = np.zeros(40, np.int32)
        qg[20:] = 1
        qg[5] = -1
        kg = np.full(50, -1, np.int32)
        kg[7] = 0
        kg[16:] = 1
        row_ptr, cols = _csr([[0], [0, 1]])
        return Problem(name, 1, 1, 64, qg, kg, 2, 2, row_ptr, cols, 14000,
                       "ragged 40x50 slots; query group 0 attends a single key")
    if name == "tiny_nokeys":
        # head 0: a clamped 1x1x3 window; head 1: no query attends anything, so
        # every work item of that head has an empty column list (and every key
        # tile of that head receives no gradient)
        group, tiles = sta_layout((5, 6, 10))
        rp, cols = sta_graph(tiles, (1, 1, 3), 1)
        rows = [cols[rp[a]:rp[a + 1]].tolist() for a in range(12)] + [[] for _ in range(12)]
        row_ptr, cols = _csr(rows)
        return Problem(name, 1, 2, 64, group, group.copy(), 12, 12, row_ptr, cols, 15000,
                       "tiny STA; head 1 attends nothing (empty column lists)")
    if name == "tiny_hedge":
        # 4x5x12 grid: the tiles of the second tile row in H hold a single dh
        # row, so each of their four pages has 4 valid rows in the same 4-row
        # group (the case the strided pages compact); clamped 1x2x2 window
        group, tiles = sta_layout((4, 5, 12))
        row_ptr, cols = sta_graph(tiles, (1, 2, 2), 2)
        return Problem(name, 1, 2, 64, group, group.copy(), 6, 6, row_ptr, cols, 16000,
                       "tiny STA whose H-edge tiles keep one dh row (strided pages)")
    if name in ("tiny_gqa", "tiny_mqa"):
        # grouped-query attention: 4 query heads over 2 K/V heads (gqa) or 3
        # over 1 (mqa); every query head has its own VSA-style lists
        heads, kvh = (4, 2) if name == "tiny_gqa" else (3, 1)
        group, tiles = sta_layout((5, 6, 10))
        rng = np.random.default_rng(17005 if name == "tiny_gqa" else 18005)
        row_ptr, cols = vsa_graph(12, heads, 4, rng)
        return Problem(name, 1, heads, 64, group, group.copy(), 12, 12, row_ptr, cols,
                       17000 if name == "tiny_gqa" else 18000,
                       f"tiny VSA-style, {heads} query heads over {kvh} K/V head(s)", kv_heads=kvh)
    if name == "tiny_bgraph":
        # two batch entries with their own graphs (own tile + 3 random tiles
        # per query tile, drawn per batch entry and head)
        group, tiles = sta_layout((5, 6, 10))
        rng = np.random.default_rng(19005)
        row_ptr, cols = vsa_graph(12, 2 * 2, 4, rng)  # batch-major (b, h) graphs
        return Problem(name, 2, 2, 64, group, group.copy(), 12, 12, row_ptr, cols, 19000,
                       "tiny VSA-style, one graph per batch entry", graph_batches=2)
    raise KeyError(name)


def with_heads(problem: Problem, heads: int) -> Problem:
    """The same layout with the graph of the first ``heads`` heads only."""
    if not 1 <= heads <= problem.heads:
        raise ValueError(f"heads must be in [1, {problem.heads}]")
    end = problem.row_ptr[heads * problem.n_q_groups]
    return dataclasses.replace(problem, heads=heads, row_ptr=problem.row_ptr[:heads * problem.n_q_groups + 1].copy(),
                               kv_groups=problem.kv_groups[:end].copy())


def make_tensors(problem: Problem, names: Sequence[str] = ("q", "k", "v", "do"),
                 batch: Optional[int] = None) -> Dict[str, "torch.Tensor"]:
    """Seeded bf16 tensors [B, H, S, D] on the CPU; padded slots hold the sentinel."""
    import torch

    b = problem.batch if batch is None else batch
    seeds = {"q": 1, "k": 2, "v": 3, "do": 4}
    out = {}
    for nm in names:
        slots = problem.kv_slots if nm in ("k", "v") else problem.q_slots
        grp = problem.kv_group if nm in ("k", "v") else problem.q_group
        nh = problem.n_kv_heads if nm in ("k", "v") else problem.heads
        g = torch.Generator().manual_seed(problem.seed_base + seeds[nm])
        t = torch.randn((b, nh, slots, problem.head_dim), generator=g, dtype=torch.float32)
        t = t.to(torch.bfloat16)
        pad = torch.from_numpy(grp < 0)
        if bool(pad.any()):
            t[:, :, pad, :] = PAD_SENTINEL
        out[nm] = t
    return out
