// Host planner: valid pages, owned-tile packing, per-tile page lists with
// exact per-segment row masks, and the key-owned (transposed) work list.
//
// Source: the KPage abstract ("KPage: block-sparse attention for partially
// occupied 3D blocks", zhuanzhiai.com, abstract paragraph).  It packs valid
// 16-row K/V pages across logical-block boundaries into large tiles, routes
// Q blocks to tile shapes that cut query-side padding, and owns K/V pages in
// the backward pass so that the sparse graph is kept exactly.  Here both
// passes use one tile shape on the tensor core (128 rows x up to 128
// columns per step) and the planner decides what fills it:
//   * an owned tile is up to 8 valid 16-row pages of the owned side (whole
//     64-slot blocks, pages without a valid row left out), so partly
//     occupied blocks share a tile instead of padding it.  Which blocks
//     share a tile is decided per head: blocks whose column lists overlap
//     most are grouped (every row of a tile runs over the union of the
//     tile's lists), and the result is kept if it computes fewer physical
//     pairs than plain slot order;
//   * the work items of a head run longest column list first;
//   * the tile's column list is the sorted union of the other side's pages
//     reachable from the groups in the tile, each with one 16-bit row mask
//     per group ("segment") present in the tile, so masking stays exact
//     even when a tile or a page straddles groups;
//   * a tile with more than four groups is split into several work items
//     that each own the rows of at most four groups.
#include "plan.hpp"

#include <cuda_runtime.h>

#include <algorithm>
#include <chrono>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <functional>
#include <iterator>
#include <new>
#include <queue>
#include <thread>
#include <tuple>
#include <unordered_map>

namespace spattn {

bool strided_setting() {
  const char* env = std::getenv("SPATTN_PLAN_STRIDED");
  return !(env && env[0] == '0');
}

namespace {

int build_side(int64_t slots, const int32_t* grp, int32_t n_groups, Side& s) {
  s.slots = slots;
  s.n_groups = n_groups;
  s.n_pages = (slots + kPageRows - 1) / kPageRows;
  s.group.assign(grp, grp + slots);
  s.page_mask.assign(s.n_pages, 0);
  s.group_size.assign(n_groups, 0);
  std::vector<int64_t> count(n_groups, 0), last(n_groups, -1);
  for (int64_t i = 0; i < slots; ++i) {
    const int32_t g = grp[i];
    if (g < -1 || g >= n_groups) return SPATTN_ERR_INVALID_ARG;
    if (g < 0) continue;
    const int64_t p = i / kPageRows;
    s.page_mask[p] |= static_cast<uint16_t>(1u << (i % kPageRows));
    s.group_size[g] += 1;
    if (last[g] != p) {
      last[g] = p;
      count[g] += 1;
    }
  }
  s.gp_ptr.assign(n_groups + 1, 0);
  for (int32_t g = 0; g < n_groups; ++g) s.gp_ptr[g + 1] = s.gp_ptr[g] + count[g];
  s.gp_page.assign(s.gp_ptr[n_groups], 0);
  s.gp_mask.assign(s.gp_ptr[n_groups], 0);
  std::vector<int64_t> fill(s.gp_ptr.begin(), s.gp_ptr.end() - 1);
  std::fill(last.begin(), last.end(), -1);
  for (int64_t i = 0; i < slots; ++i) {
    const int32_t g = grp[i];
    if (g < 0) continue;
    const int64_t p = i / kPageRows;
    if (last[g] != p) {
      last[g] = p;
      s.gp_page[fill[g]] = static_cast<int32_t>(p);
      fill[g] += 1;
    }
    s.gp_mask[fill[g] - 1] |= static_cast<uint16_t>(1u << (i % kPageRows));
  }
  return SPATTN_OK;
}

int build_fwd_adjacency(const spattn_graph* g, int32_t heads, int32_t n_q, int32_t n_k, Adjacency& a) {
  const int64_t rows = static_cast<int64_t>(heads) * n_q;
  if (g->row_ptr[0] != 0) return SPATTN_ERR_INVALID_ARG;
  for (int64_t r = 0; r < rows; ++r)
    if (g->row_ptr[r + 1] < g->row_ptr[r]) return SPATTN_ERR_INVALID_ARG;
  a.n_src = n_q;
  a.ptr.assign(rows + 1, 0);
  a.dst.clear();
  a.dst.reserve(g->row_ptr[rows]);
  std::vector<int32_t> tmp;
  for (int64_t r = 0; r < rows; ++r) {
    tmp.assign(g->kv_groups + g->row_ptr[r], g->kv_groups + g->row_ptr[r + 1]);
    for (int32_t b : tmp)
      if (b < 0 || b >= n_k) return SPATTN_ERR_INVALID_ARG;
    std::sort(tmp.begin(), tmp.end());
    tmp.erase(std::unique(tmp.begin(), tmp.end()), tmp.end());
    a.dst.insert(a.dst.end(), tmp.begin(), tmp.end());
    a.ptr[r + 1] = static_cast<int64_t>(a.dst.size());
  }
  return SPATTN_OK;
}

void build_bwd_adjacency(const Adjacency& f, int32_t heads, int32_t n_q, int32_t n_k, Adjacency& b) {
  b.n_src = n_k;
  b.ptr.assign(static_cast<int64_t>(heads) * n_k + 1, 0);
  for (int32_t h = 0; h < heads; ++h)
    for (int32_t a = 0; a < n_q; ++a) {
      const int64_t r = static_cast<int64_t>(h) * n_q + a;
      for (int64_t e = f.ptr[r]; e < f.ptr[r + 1]; ++e) b.ptr[static_cast<int64_t>(h) * n_k + f.dst[e] + 1] += 1;
    }
  for (size_t i = 1; i < b.ptr.size(); ++i) b.ptr[i] += b.ptr[i - 1];
  b.dst.assign(b.ptr.back(), 0);
  std::vector<int64_t> fill(b.ptr.begin(), b.ptr.end() - 1);
  for (int32_t h = 0; h < heads; ++h)
    for (int32_t a = 0; a < n_q; ++a) {
      const int64_t r = static_cast<int64_t>(h) * n_q + a;
      for (int64_t e = f.ptr[r]; e < f.ptr[r + 1]; ++e) {
        const int64_t d = static_cast<int64_t>(h) * n_k + f.dst[e];
        b.dst[fill[d]++] = a;  // a ascending -> rows stay sorted
      }
    }
}

// The 4-row group k that holds every set bit of a 16-bit row mask, or -1
// (an empty mask, or rows in more than one group).
int sub_group(uint32_t m) {
  for (int k = 0; k < 4; ++k)
    if (m != 0u && (m & ~(0xFu << (4 * k))) == 0u) return k;
  return -1;
}

// Strided pages are used unless SPATTN_PLAN_STRIDED=0 (for comparisons).
bool strided_enabled() { return strided_setting(); }

// A 64-slot block of the owned side: references to its valid pages (one
// strided page when all four pages are valid and their valid rows share a
// 4-row group k; the block's other rows are then padded) and its groups.
struct OwnBlock {
  int32_t pages[kBlockRows / kPageRows];
  int npg = 0;
  int strided_group = -1;  // k of the strided page, else -1
  std::vector<int32_t> groups;  // distinct, ascending
  int32_t only = -1;       // >= 0: the unit owns only the rows of this group
};

// The owned units of a side: its 64-slot blocks.  With split_groups, a block
// whose rows belong to several groups becomes one unit per group (the block's
// pages that hold rows of the group, owning only those rows), so that a tile
// can run over one group's list only; a page shared by two units is then
// computed by two work items that own disjoint rows.
std::vector<OwnBlock> owned_blocks(const Side& s, bool split_groups = false) {
  const int per = kBlockRows / kPageRows;
  const bool strided = strided_enabled();
  std::vector<OwnBlock> out;
  const int64_t n_blocks = (s.n_pages + per - 1) / per;
  for (int64_t blk = 0; blk < n_blocks; ++blk) {
    OwnBlock b;
    for (int i = 0; i < per; ++i) {
      const int64_t p = blk * per + i;
      if (p < s.n_pages && s.page_mask[p]) b.pages[b.npg++] = static_cast<int32_t>(p);
    }
    if (b.npg == 0) continue;
    if (strided && b.npg == per) {
      const int k = sub_group(s.page_mask[b.pages[0]]);
      bool same = k >= 0;
      for (int i = 1; i < per && same; ++i) same = sub_group(s.page_mask[b.pages[i]]) == k;
      const int64_t p0 = blk * per;
      if (same && 16 * (p0 + 3) + 4 * k + 4 <= s.slots) {
        b.pages[0] = ~static_cast<int32_t>(16 * p0 + 4 * k);
        b.npg = 1;
        b.strided_group = k;
      }
    }
    const int64_t r1 = std::min<int64_t>((blk + 1) * per * kPageRows, s.slots);
    for (int64_t i = blk * per * kPageRows; i < r1; ++i)
      if (s.group[i] >= 0) b.groups.push_back(s.group[i]);
    std::sort(b.groups.begin(), b.groups.end());
    b.groups.erase(std::unique(b.groups.begin(), b.groups.end()), b.groups.end());
    if (split_groups && b.strided_group < 0 && b.groups.size() > 1) {
      for (int32_t g : b.groups) {
        OwnBlock u;
        u.groups = {g};
        u.only = g;
        for (int i = 0; i < b.npg; ++i) {
          const int64_t p0 = static_cast<int64_t>(b.pages[i]) * kPageRows;
          bool has = false;
          for (int64_t x = p0; x < std::min<int64_t>(p0 + kPageRows, s.slots) && !has; ++x) has = s.group[x] == g;
          if (has) u.pages[u.npg++] = b.pages[i];
        }
        out.push_back(std::move(u));
      }
      continue;
    }
    out.push_back(std::move(b));
  }
  return out;
}

// Smallest group with a row on regular page p (-1 if none): the unit of that
// group owns the page's padded rows when the page is split between units.
int32_t first_group_of_page(const Side& s, int32_t p) {
  int32_t m = -1;
  const int64_t p0 = static_cast<int64_t>(p) * kPageRows;
  for (int64_t x = p0; x < std::min<int64_t>(p0 + kPageRows, s.slots); ++x)
    if (s.group[x] >= 0 && (m < 0 || s.group[x] < m)) m = s.group[x];
  return m;
}

// Owned tiles in slot order: whole blocks appended while the tile holds at
// most 8 pages.
std::vector<std::vector<int32_t>> pack_slot_order(const std::vector<OwnBlock>& blocks) {
  std::vector<std::vector<int32_t>> tiles;
  std::vector<int32_t> cur;
  for (const auto& b : blocks) {
    if (cur.size() + b.npg > static_cast<size_t>(kTilePages)) {
      tiles.push_back(cur);
      cur.clear();
    }
    cur.insert(cur.end(), b.pages, b.pages + b.npg);
  }
  if (!cur.empty()) tiles.push_back(cur);
  return tiles;
}

size_t union_size(const std::vector<int32_t>& a, const std::vector<int32_t>& b) {
  size_t n = 0, i = 0, j = 0;
  while (i < a.size() && j < b.size()) {
    if (a[i] == b[j]) { ++i; ++j; }
    else if (a[i] < b[j]) ++i;
    else ++j;
    ++n;
  }
  return n + (a.size() - i) + (b.size() - j);
}

// Owned tiles grouped by the similarity of what their rows attend (the
// query-side routing of the KPage abstract, B200 form): every row of a tile
// runs over the union of the tile's column lists, so blocks whose column
// lists overlap most are packed together.  Greedy agglomeration: the pair of
// clusters with the largest overlap (column groups they share, weighted by
// the pages of each group) merges first, while the merged cluster holds at
// most 8 pages and at most 8 groups (one work item).  Clusters left with room
// are then filled in slot order under the same limits.
//
// A merge saves the same pairs (the overlap) whatever the sizes of the two
// clusters, but a 4-page block merged with a 1-page edge block leaves a tile
// that nothing larger than 3 pages can fill.  With two_phase, the first
// round merges only clusters of like size (both at least one full block of
// 4 pages, or both smaller), and a second round then merges freely.
std::vector<std::vector<int32_t>> pack_similar(const Side& col, const Adjacency& adj,
                                               const std::vector<int64_t>& src_heads,
                                               const std::vector<OwnBlock>& blocks, bool two_phase,
                                               std::vector<std::vector<int32_t>>* only_out = nullptr) {
  const int32_t nb = static_cast<int32_t>(blocks.size());
  const int32_t ng = col.n_groups;
  const int64_t n_codes = static_cast<int64_t>(ng) * static_cast<int64_t>(src_heads.size());
  // a block's signature: (head offset j, column group) pairs as j * ng + group
  std::vector<std::vector<int32_t>> sig(nb);
  for (int32_t b = 0; b < nb; ++b) {
    for (size_t j = 0; j < src_heads.size(); ++j)
      for (int32_t g : blocks[b].groups) {
        const int64_t r = src_heads[j] * adj.n_src + g;
        for (int64_t e = adj.ptr[r]; e < adj.ptr[r + 1]; ++e)
          sig[b].push_back(static_cast<int32_t>(j * ng + adj.dst[e]));
      }
    std::sort(sig[b].begin(), sig[b].end());
    sig[b].erase(std::unique(sig[b].begin(), sig[b].end()), sig[b].end());
  }
  auto wt = [&](int32_t code) {
    const int32_t g = code % ng;
    return col.gp_ptr[g + 1] - col.gp_ptr[g];
  };
  // signature code -> blocks whose signature holds it
  std::vector<int64_t> ip(static_cast<size_t>(n_codes) + 1, 0);
  for (int32_t b = 0; b < nb; ++b)
    for (int32_t g : sig[b]) ip[g + 1] += 1;
  for (int64_t g = 0; g < n_codes; ++g) ip[g + 1] += ip[g];
  std::vector<int32_t> iv(ip.back());
  {
    std::vector<int64_t> fill(ip.begin(), ip.end() - 1);
    for (int32_t b = 0; b < nb; ++b)
      for (int32_t g : sig[b]) iv[fill[g]++] = b;
  }
  std::vector<int32_t> parent(nb), npg(nb);
  std::vector<std::vector<int32_t>> groups(nb), members(nb);
  for (int32_t b = 0; b < nb; ++b) {
    parent[b] = b;
    npg[b] = blocks[b].npg;
    groups[b] = blocks[b].groups;
    members[b] = {b};
  }
  auto find = [&](int32_t x) {
    while (parent[x] != x) x = parent[x] = parent[parent[x]];
    return x;
  };
  constexpr int kFullBlock = kBlockRows / kPageRows;
  bool like_sizes = two_phase;  // first round of the two-phase grouping
  auto fits = [&](int32_t a, int32_t b) {
    if (like_sizes && (npg[a] >= kFullBlock) != (npg[b] >= kFullBlock)) return false;
    return npg[a] + npg[b] <= kTilePages && union_size(groups[a], groups[b]) <= static_cast<size_t>(kMaxSegments);
  };
  auto overlap = [&](int32_t a, int32_t b) {
    int64_t w = 0;
    size_t i = 0, j = 0;
    while (i < sig[a].size() && j < sig[b].size()) {
      if (sig[a][i] == sig[b][j]) { w += wt(sig[a][i]); ++i; ++j; }
      else if (sig[a][i] < sig[b][j]) ++i;
      else ++j;
    }
    return w;
  };
  // (overlap, -distance in slot order, a, b): ties go to nearby blocks
  using Cand = std::tuple<int64_t, int32_t, int32_t, int32_t>;
  std::priority_queue<Cand> heap;
  std::vector<int64_t> cnt(nb, 0);
  std::vector<int32_t> touched;
  // Candidates of cluster a: clusters sharing a column group.  The counts are
  // exact before any merge and upper bounds after; every popped candidate is
  // re-evaluated exactly.
  auto push_candidates = [&](int32_t a, bool only_greater) {
    touched.clear();
    for (int32_t g : sig[a])
      for (int64_t x = ip[g]; x < ip[g + 1]; ++x) {
        const int32_t r = find(iv[x]);
        if (r == a || (only_greater && r < a)) continue;
        if (cnt[r] == 0) touched.push_back(r);
        cnt[r] += wt(g);
      }
    for (int32_t r : touched) {
      if (cnt[r] > 0 && fits(a, r)) heap.emplace(cnt[r], -std::abs(r - a), std::min(a, r), std::max(a, r));
      cnt[r] = 0;
    }
  };
  for (int round = 0; round < (two_phase ? 2 : 1); ++round) {
    if (round == 1) {
      like_sizes = false;
      for (int32_t b = 0; b < nb; ++b)
        if (parent[b] == b && npg[b] < kTilePages) push_candidates(b, true);
    } else {
      for (int32_t b = 0; b < nb; ++b) push_candidates(b, true);
    }
    while (!heap.empty()) {
      const auto [w, nd, a, b] = heap.top();
      heap.pop();
      if (parent[a] != a || parent[b] != b || !fits(a, b)) continue;
      const int64_t exact = overlap(a, b);
      if (exact != w) {
        if (exact > 0) heap.emplace(exact, nd, a, b);
        continue;
      }
      // merge b into a
      parent[b] = a;
      npg[a] += npg[b];
      std::vector<int32_t> u;
      std::set_union(groups[a].begin(), groups[a].end(), groups[b].begin(), groups[b].end(), std::back_inserter(u));
      groups[a].swap(u);
      u.clear();
      std::set_union(sig[a].begin(), sig[a].end(), sig[b].begin(), sig[b].end(), std::back_inserter(u));
      sig[a].swap(u);
      std::vector<int32_t>().swap(sig[b]);
      members[a].insert(members[a].end(), members[b].begin(), members[b].end());
      std::vector<int32_t>().swap(members[b]);
      if (npg[a] < kTilePages) push_candidates(a, false);
    }
  }
  // fill: clusters left with room, in slot order of their first block (a
  // cluster's root is its lowest block index)
  std::vector<int32_t> heads_of_tiles;
  int32_t cur = -1;
  for (int32_t r = 0; r < nb; ++r) {
    if (parent[r] != r) continue;
    if (cur >= 0 && fits(cur, r)) {
      npg[cur] += npg[r];
      std::vector<int32_t> u;
      std::set_union(groups[cur].begin(), groups[cur].end(), groups[r].begin(), groups[r].end(),
                     std::back_inserter(u));
      groups[cur].swap(u);
      members[cur].insert(members[cur].end(), members[r].begin(), members[r].end());
      continue;
    }
    cur = r;
    heads_of_tiles.push_back(r);
  }
  std::vector<std::vector<int32_t>> tiles;
  tiles.reserve(heads_of_tiles.size());
  if (only_out) only_out->clear();
  for (int32_t r : heads_of_tiles) {
    std::vector<std::pair<int32_t, int32_t>> pg;  // (page reference, owned group or -1)
    for (int32_t b : members[r])
      for (int i = 0; i < blocks[b].npg; ++i) pg.emplace_back(blocks[b].pages[i], blocks[b].only);
    std::sort(pg.begin(), pg.end());
    std::vector<int32_t> pages, only;
    for (const auto& x : pg) {
      pages.push_back(x.first);
      only.push_back(x.second);
    }
    tiles.push_back(std::move(pages));
    if (only_out) only_out->push_back(std::move(only));
  }
  return tiles;
}

// Column entries of one list, in slot order, from the masks accumulated in
// `acc` for the (head offset, page) keys of `touched` (sorted); the keys' acc
// words are cleared on the way.  Up to four consecutive pages whose attended
// rows (over all segments) lie in one 4-row group k, at least two of them in
// the list, become one strided entry: the four groups then cost one 16-column
// page instead of one page each.
void append_entries(const Side& col, bool strided, std::vector<uint64_t>& acc, const std::vector<int64_t>& touched,
                    std::vector<int32_t>& pages, std::vector<uint64_t>& masks, std::vector<uint16_t>& heads) {
  const int64_t npc = col.n_pages;
  auto fold = [&](int64_t c) {
    const uint64_t m = acc[2 * c] | acc[2 * c + 1];
    return static_cast<uint32_t>((m | (m >> 16) | (m >> 32) | (m >> 48)) & 0xFFFFu);
  };
  size_t i = 0;
  while (i < touched.size()) {
    const int64_t c = touched[i];
    const int32_t p = static_cast<int32_t>(c % npc);
    const uint16_t jh = static_cast<uint16_t>(c / npc);
    const int k = strided ? sub_group(fold(c)) : -1;
    // (the bound keeps p + 3 inside the side, so c + 3 stays in head jh)
    if (k >= 0 && 16 * (static_cast<int64_t>(p) + 3) + 4 * k + 4 <= col.slots) {
      size_t j = i;
      bool same = true;
      while (j < touched.size() && touched[j] <= c + 3) {
        if (sub_group(fold(touched[j])) != k) {
          same = false;
          break;
        }
        ++j;
      }
      if (same && j - i >= 2) {
        uint64_t m[kMaskWords] = {0, 0};
        for (size_t x = i; x < j; ++x) {
          const int jj = static_cast<int>(touched[x] - c);
          for (int sg = 0; sg < kMaxSegments; ++sg)
            m[sg / 4] |= ((acc[2 * touched[x] + sg / 4] >> (16 * (sg % 4) + 4 * k)) & 0xFull)
                         << (16 * (sg % 4) + 4 * jj);
          acc[2 * touched[x]] = acc[2 * touched[x] + 1] = 0;
        }
        pages.push_back(~static_cast<int32_t>(16 * p + 4 * k));
        masks.push_back(m[0]);
        masks.push_back(m[1]);
        heads.push_back(jh);
        i = j;
        continue;
      }
    }
    pages.push_back(p);
    masks.push_back(acc[2 * c]);
    masks.push_back(acc[2 * c + 1]);
    heads.push_back(jh);
    acc[2 * c] = acc[2 * c + 1] = 0;
    ++i;
  }
}

// Work items of one unit for one pass (work words use bh = the unit, batch
// 0).  A unit is one owned head (w[0] before batch replication) whose
// columns come from the adjacency rows of the graph heads src_heads[j]: one
// for the query-owned pass, the query heads of a K/V head's group for the
// key-owned pass (entries carry j).
void build_head(const Side& own, const Side& col, const Adjacency& adj, int32_t unit,
                const std::vector<int64_t>& src_heads, const std::vector<std::vector<int32_t>>& tiles, WorkList& wl,
                std::vector<uint64_t>& acc, std::vector<int64_t>& touched,
                const std::vector<std::vector<int32_t>>* only = nullptr) {
  const int64_t npc = col.n_pages;
  const bool strided = strided_enabled();
  int32_t rg[kTilePages * kPageRows];
  for (size_t ti = 0; ti < tiles.size(); ++ti) {
    const auto& tile = tiles[ti];
    const int npg = static_cast<int>(tile.size());
    std::vector<int32_t> segs;
    for (int r = 0; r < kTilePages * kPageRows; ++r) {
      int32_t g = -2;  // row does not exist in this tile / tensor
      if (r < npg * kPageRows) {
        const int64_t slot = pref_slot(tile[r / kPageRows], r % kPageRows);
        if (slot < own.slots) g = own.group[slot];
        const int32_t og = only ? (*only)[ti][r / kPageRows] : -1;
        // a page split between units: this item owns the rows of its group,
        // and the padded rows if its group is the page's smallest
        if (og >= 0 && ((g >= 0 && g != og) || (g == -1 && og != first_group_of_page(own, tile[r / kPageRows]))))
          g = -2;
      }
      rg[r] = g;
      if (g >= 0 && std::find(segs.begin(), segs.end(), g) == segs.end()) segs.push_back(g);
    }
    const int n_items = std::max<int>(1, (static_cast<int>(segs.size()) + kMaxSegments - 1) / kMaxSegments);
    for (int it = 0; it < n_items; ++it) {
      const int s0 = it * kMaxSegments;
      const int s1 = std::min<int>(s0 + kMaxSegments, static_cast<int>(segs.size()));
      touched.clear();
      for (size_t j = 0; j < src_heads.size(); ++j)
        for (int s = s0; s < s1; ++s) {
          const int64_t r = src_heads[j] * adj.n_src + segs[s];
          for (int64_t e = adj.ptr[r]; e < adj.ptr[r + 1]; ++e) {
            const int32_t b = adj.dst[e];
            for (int64_t x = col.gp_ptr[b]; x < col.gp_ptr[b + 1]; ++x) {
              const int64_t c = static_cast<int64_t>(j) * npc + col.gp_page[x];  // (head offset, page)
              if (acc[2 * c] == 0 && acc[2 * c + 1] == 0) touched.push_back(c);
              const int sg = s - s0;
              acc[2 * c + sg / 4] |= static_cast<uint64_t>(col.gp_mask[x]) << (16 * (sg % 4));
            }
          }
        }
      std::sort(touched.begin(), touched.end());
      int32_t w[kWorkWords];
      std::memset(w, 0, sizeof(w));
      w[0] = unit;
      w[1] = npg;
      w[2] = static_cast<int32_t>(wl.pages.size());
      append_entries(col, strided, acc, touched, wl.pages, wl.masks, wl.heads);
      const size_t n_entries = wl.pages.size() - static_cast<size_t>(w[2]);
      w[3] = static_cast<int32_t>(wl.pages.size());
      for (int i = 0; i < npg; ++i) w[4 + i] = tile[i];
      for (int r = 0; r < kTilePages * kPageRows; ++r) {
        uint32_t code = kCodeNotOwned;
        if (rg[r] == -1) {
          code = (it == 0) ? kCodeNoSegment : kCodeNotOwned;
        } else if (rg[r] >= 0) {
          for (int s = s0; s < s1; ++s)
            if (segs[s] == rg[r]) code = static_cast<uint32_t>(s - s0);
        }
        reinterpret_cast<uint32_t*>(w)[12 + r / 8] |= code << (4 * (r % 8));
      }
      wl.physical_pairs += static_cast<int64_t>(kTilePages * kPageRows) * kPageRows * static_cast<int64_t>(n_entries);
      wl.work.insert(wl.work.end(), w, w + kWorkWords);
    }
  }
}

// Work items of the 64-row route (the KPage abstract's routing of Q blocks
// to a smaller tile shape, B200 form): two 64-slot blocks per item, rows
// 0..63 (owned pages 0..3) and 64..127 (owned pages 4..7), each half with
// its own column list.  The forward runs each half as M = 64 products, so a
// pair of blocks with unrelated lists (VSA-style selection) no longer pays
// for the union of both lists.  The lists are interleaved two entries at a
// time and padded to whole 4-entry steps with zero-mask entries (that repeat
// a page of the list, so every load stays inside the tensor).  Blocks are
// paired in slot order; a last odd block runs alone (its other half owns no
// row).  Returns false, leaving wl partly built, when a pair holds more than
// kMaxSegments groups.
bool build_head_halves(const Side& own, const Side& col, const Adjacency& adj, int32_t unit,
                       const std::vector<int64_t>& src_heads, const std::vector<OwnBlock>& blocks, WorkList& wl,
                       std::vector<uint64_t>& acc, std::vector<int64_t>& touched) {
  const int64_t npc = col.n_pages;
  const bool strided = strided_enabled();
  constexpr int kHalfPages = kTilePages / 2;
  std::vector<int32_t> hp[2];
  std::vector<uint64_t> hm[2];
  std::vector<uint16_t> hh[2];
  for (size_t bi = 0; bi < blocks.size(); bi += 2) {
    const OwnBlock* half[2] = {&blocks[bi], bi + 1 < blocks.size() ? &blocks[bi + 1] : nullptr};
    int32_t tile[kTilePages];
    int32_t rg[kTilePages * kPageRows];  // segment of each row, or -1 (owned padded row) / -2 (not owned)
    // Segments are numbered per half (those of half 0 first): a group with
    // rows in both halves gets one segment in each, so that the entries of
    // one half never carry bits of the other half's rows (a kernel that
    // ignores the route then still computes every pair once).
    std::vector<int32_t> segs;
    size_t seg0[3] = {0, 0, 0};  // half h owns segments seg0[h] .. seg0[h+1]-1
    for (int h = 0; h < 2; ++h) {
      const OwnBlock* b = half[h] ? half[h] : half[0];
      if (b->npg > kHalfPages) return false;
      for (int i = 0; i < kHalfPages; ++i) tile[kHalfPages * h + i] = i < b->npg ? b->pages[i] : b->pages[0];
      seg0[h] = segs.size();
      for (int r = 64 * h; r < 64 * h + 64; ++r) {
        int32_t g = -2;  // row not owned: a padding page, or beyond the tensor
        if (half[h] && (r - 64 * h) / kPageRows < half[h]->npg) {
          const int64_t slot = pref_slot(tile[r / kPageRows], r % kPageRows);
          if (slot < own.slots) g = own.group[slot];
        }
        if (g < 0) {
          rg[r] = g;
          continue;
        }
        const auto first = segs.begin() + static_cast<std::ptrdiff_t>(seg0[h]);
        const auto it = std::find(first, segs.end(), g);
        rg[r] = static_cast<int32_t>(it - segs.begin());
        if (it == segs.end()) segs.push_back(g);
      }
      seg0[h + 1] = segs.size();
    }
    if (segs.size() > static_cast<size_t>(kMaxSegments)) return false;
    for (int h = 0; h < 2; ++h) {
      touched.clear();
      for (size_t j = 0; j < src_heads.size(); ++j)
        for (int sg = static_cast<int>(seg0[h]); sg < static_cast<int>(seg0[h + 1]); ++sg) {
          const int64_t r = src_heads[j] * adj.n_src + segs[sg];
          for (int64_t e = adj.ptr[r]; e < adj.ptr[r + 1]; ++e) {
            const int32_t b = adj.dst[e];
            for (int64_t x = col.gp_ptr[b]; x < col.gp_ptr[b + 1]; ++x) {
              const int64_t c = static_cast<int64_t>(j) * npc + col.gp_page[x];
              if (acc[2 * c] == 0 && acc[2 * c + 1] == 0) touched.push_back(c);
              acc[2 * c + sg / 4] |= static_cast<uint64_t>(col.gp_mask[x]) << (16 * (sg % 4));
            }
          }
        }
      std::sort(touched.begin(), touched.end());
      hp[h].clear();
      hm[h].clear();
      hh[h].clear();
      append_entries(col, strided, acc, touched, hp[h], hm[h], hh[h]);
    }
    int32_t w[kWorkWords];
    std::memset(w, 0, sizeof(w));
    w[0] = unit;
    w[1] = kTilePages;
    w[2] = static_cast<int32_t>(wl.pages.size());
    const size_t n_steps = std::max((hp[0].size() + 1) / 2, (hp[1].size() + 1) / 2);
    for (size_t st = 0; st < n_steps; ++st)
      for (int h = 0; h < 2; ++h)
        for (size_t j = 0; j < 2; ++j) {
          const size_t idx = 2 * st + j;
          if (idx < hp[h].size()) {
            wl.pages.push_back(hp[h][idx]);
            wl.masks.push_back(hm[h][2 * idx]);
            wl.masks.push_back(hm[h][2 * idx + 1]);
            wl.heads.push_back(hh[h][idx]);
          } else {
            wl.pages.push_back(!hp[h].empty() ? hp[h][0] : hp[1 - h][0]);
            wl.masks.push_back(0);
            wl.masks.push_back(0);
            wl.heads.push_back(0);
          }
        }
    w[3] = static_cast<int32_t>(wl.pages.size());
    for (int i = 0; i < kTilePages; ++i) w[4 + i] = tile[i];
    for (int r = 0; r < kTilePages * kPageRows; ++r) {
      const uint32_t code = rg[r] >= 0 ? static_cast<uint32_t>(rg[r]) : (rg[r] == -1 ? kCodeNoSegment : kCodeNotOwned);
      reinterpret_cast<uint32_t*>(w)[12 + r / 8] |= code << (4 * (r % 8));
    }
    w[28] = 1;
    // each entry meets the 64 rows of its half
    wl.physical_pairs += static_cast<int64_t>(64) * kPageRows * static_cast<int64_t>(w[3] - w[2]);
    wl.work.insert(wl.work.end(), w, w + kWorkWords);
  }
  return true;
}

// Work item templates of the slot-order tiles (the device planner's items):
// the same rows, segments and row codes as build_head gives those tiles.
void make_templates(const Side& own, PassTemplates& t) {
  const auto tiles = pack_slot_order(owned_blocks(own));
  t.words.clear();
  t.segs.clear();
  t.seg_rows.clear();
  int32_t rg[kTilePages * kPageRows];
  for (const auto& tile : tiles) {
    const int npg = static_cast<int>(tile.size());
    std::vector<int32_t> segs;
    for (int r = 0; r < kTilePages * kPageRows; ++r) {
      int32_t g = -2;
      if (r < npg * kPageRows) {
        const int64_t slot = pref_slot(tile[r / kPageRows], r % kPageRows);
        if (slot < own.slots) g = own.group[slot];
      }
      rg[r] = g;
      if (g >= 0 && std::find(segs.begin(), segs.end(), g) == segs.end()) segs.push_back(g);
    }
    const int n_items = std::max<int>(1, (static_cast<int>(segs.size()) + kMaxSegments - 1) / kMaxSegments);
    for (int it = 0; it < n_items; ++it) {
      const int s0 = it * kMaxSegments;
      const int s1 = std::min<int>(s0 + kMaxSegments, static_cast<int>(segs.size()));
      int32_t w[kWorkWords];
      std::memset(w, 0, sizeof(w));
      w[1] = npg;
      for (int i = 0; i < npg; ++i) w[4 + i] = tile[i];
      int32_t rows[kMaxSegments] = {};
      for (int r = 0; r < kTilePages * kPageRows; ++r) {
        uint32_t code = kCodeNotOwned;
        if (rg[r] == -1) {
          code = (it == 0) ? kCodeNoSegment : kCodeNotOwned;
        } else if (rg[r] >= 0) {
          for (int s = s0; s < s1; ++s)
            if (segs[s] == rg[r]) code = static_cast<uint32_t>(s - s0);
        }
        if (code < static_cast<uint32_t>(kMaxSegments)) rows[code] += 1;
        reinterpret_cast<uint32_t*>(w)[12 + r / 8] |= code << (4 * (r % 8));
      }
      t.words.insert(t.words.end(), w, w + kWorkWords);
      for (int s = 0; s < kMaxSegments; ++s) {
        t.segs.push_back(s0 + s < s1 ? segs[s0 + s] : -1);
        t.seg_rows.push_back(rows[s]);
      }
    }
  }
  t.n = static_cast<int64_t>(t.words.size()) / kWorkWords;
}

// Items of one head, longest column list first: CTAs start in grid order,
// so the longest items start earliest and short ones fill in at the end.
void order_longest_first(WorkList& w) {
  const size_t n = w.work.size() / kWorkWords;
  std::vector<size_t> idx(n);
  for (size_t i = 0; i < n; ++i) idx[i] = i;
  std::stable_sort(idx.begin(), idx.end(), [&](size_t x, size_t y) {
    const int32_t* a = w.work.data() + x * kWorkWords;
    const int32_t* b = w.work.data() + y * kWorkWords;
    return (a[3] - a[2]) > (b[3] - b[2]);
  });
  std::vector<int32_t> out;
  out.reserve(w.work.size());
  for (size_t i : idx) out.insert(out.end(), w.work.begin() + i * kWorkWords, w.work.begin() + (i + 1) * kWorkWords);
  w.work.swap(out);
}

// Tile packing of a pass: 0 = best per head (default), 1 = slot order only,
// 2 = similarity grouping only, 3 = only the two-round grouping of
// group-split blocks, 4 = the 64-row route for the query-owned pass wherever
// a pair of blocks allows it (the key-owned pass as in 0).
// SPATTN_PLAN_PACK=slot|similar|split|route64 selects one (for comparisons
// and tests).
int packing_mode() {
  const char* env = std::getenv("SPATTN_PLAN_PACK");
  if (!env) return 0;
  if (std::strcmp(env, "slot") == 0) return 1;
  if (std::strcmp(env, "similar") == 0) return 2;
  if (std::strcmp(env, "split") == 0) return 3;
  if (std::strcmp(env, "route64") == 0) return 4;
  return 0;
}

// Modelled time of a query-owned work list (forward then dQ, which both run
// it), in forward steps of 128 rows x 64 columns.  A dQ step costs about
// 1.45 forward steps whatever the route (dQ computes every entry against all
// 128 rows).  A forward step of the 64-row route (2 x 64 rows x 32 columns)
// costs 0.89-0.94 of one (measured on B200 with the route forced: partial
// and VSA-style workloads): half the exponentials per row, but two M = 64
// score products at N = 32 take as much tensor time as one M = 128 product
// at N = 64.  So the route wins only where a tile's two blocks have
// disjoint lists of equal length, which the workloads measured here never
// give (the VSA-style union carries fewer steps than the padded halves).
constexpr double kDqStepCost = 1.45;
constexpr double kRoute64StepCost = 0.92;
double query_pass_cost(const WorkList& w) {
  double t = 0.0;
  for (size_t i = 0; i < w.work.size(); i += kWorkWords) {
    const int32_t* x = w.work.data() + i;
    t += static_cast<double>((x[3] - x[2] + 3) / 4) * ((x[28] ? kRoute64StepCost : 1.0) + kDqStepCost);
  }
  return t;
}

// Work list of one pass.  Unit u (0 <= u < n_units) owns tensor head u of the
// owned side (before batch replication) and takes its columns from the graph
// heads src_heads(u); with one graph for every batch entry the units are the
// heads of batch entry 0 and the items are repeated per batch entry with
// their owned head shifted by b * owned_heads (they share the entries).
int build_worklist(const Side& own, const Side& col, const Adjacency& adj, int32_t n_units, int32_t owned_heads,
                   int32_t batch_copies, const std::function<std::vector<int64_t>(int32_t)>& src_heads,
                   bool route64, WorkList& wl) {
  const auto blocks = owned_blocks(own);
  const auto split_blocks = owned_blocks(own, true);
  const auto slot_tiles = pack_slot_order(blocks);

  const int route_mode = packing_mode();
  const int mode = route_mode == 4 ? 0 : route_mode;  // tile packing of the 128-row route
  // Units are independent: each is built on its own into part[u] (worker t
  // takes units t, t + n, ...), then the parts are joined in unit order, so
  // the result does not depend on the number of threads.
  std::vector<WorkList> part(n_units);
  // Units whose column sources are the same graph rows get the same list
  // (every head of a layout whose heads share one graph, as the STA-style
  // windows do): it is built for the first such unit and copied, with the
  // owned head rewritten.  SPATTN_PLAN_DEDUP=0 builds every unit (the plans
  // are identical; tests compare them).
  std::vector<int32_t> same_as(n_units, -1);
  const char* dedup_env = std::getenv("SPATTN_PLAN_DEDUP");
  if (!(dedup_env && std::strcmp(dedup_env, "0") == 0)) {
    auto same_rows = [&](const std::vector<int64_t>& a, const std::vector<int64_t>& b) {
      if (a.size() != b.size()) return false;
      for (size_t j = 0; j < a.size(); ++j)
        for (int32_t g = 0; g < adj.n_src; ++g) {
          const int64_t ra = a[j] * adj.n_src + g, rb = b[j] * adj.n_src + g;
          const int64_t na = adj.ptr[ra + 1] - adj.ptr[ra];
          if (na != adj.ptr[rb + 1] - adj.ptr[rb] ||
              !std::equal(adj.dst.begin() + adj.ptr[ra], adj.dst.begin() + adj.ptr[ra + 1], adj.dst.begin() + adj.ptr[rb]))
            return false;
        }
      return true;
    };
    std::unordered_map<uint64_t, std::vector<int32_t>> seen;
    for (int32_t u = 0; u < n_units; ++u) {
      const std::vector<int64_t> src = src_heads(u);
      uint64_t h = 1469598103934665603ull;  // FNV-1a over the rows' lengths and entries
      auto mix = [&](uint64_t x) { h = (h ^ x) * 1099511628211ull; };
      mix(src.size());
      for (int64_t sh : src)
        for (int32_t g = 0; g < adj.n_src; ++g) {
          const int64_t r = sh * adj.n_src + g;
          mix(static_cast<uint64_t>(adj.ptr[r + 1] - adj.ptr[r]));
          for (int64_t e = adj.ptr[r]; e < adj.ptr[r + 1]; ++e) mix(static_cast<uint32_t>(adj.dst[e]));
        }
      auto& cand = seen[h];
      for (int32_t c : cand)
        if (same_rows(src_heads(c), src)) {
          same_as[u] = c;
          break;
        }
      if (same_as[u] < 0) cand.push_back(u);
    }
  }
  // all hardware threads, unless SPATTN_PLAN_THREADS (>= 1) asks for fewer or more
  int want = static_cast<int>(std::thread::hardware_concurrency());
  if (const char* env = std::getenv("SPATTN_PLAN_THREADS")) want = std::max(1, std::atoi(env));
  const int n_threads = std::max(1, std::min<int>(n_units, want));
  std::vector<char> failed(n_threads, 0);
  auto worker = [&](int t) {
    try {
      std::vector<int64_t> touched;
      std::vector<uint64_t> acc;
      for (int32_t u = t; u < n_units; u += n_threads) {
        if (same_as[u] >= 0) continue;
        const std::vector<int64_t> src = src_heads(u);
        acc.assign(static_cast<size_t>(col.n_pages) * src.size() * kMaskWords, 0);
        // Per unit, the packing with fewer physical pairs (then fewer items).
        if (mode == 0 || mode == 1) build_head(own, col, adj, u, src, slot_tiles, part[u], acc, touched);
        if (mode != 1) {
          // one-round grouping of whole blocks (modes 0, 2), and two-round
          // grouping of blocks split by group (modes 0, 3)
          for (int two = (mode == 3 ? 1 : 0); two < (mode == 2 ? 1 : 2); ++two) {
            WorkList sim;
            std::vector<std::vector<int32_t>> only;
            const auto tiles = pack_similar(col, adj, src, two == 1 ? split_blocks : blocks, two == 1, &only);
            build_head(own, col, adj, u, src, tiles, sim, acc, touched, &only);
            const bool forced = mode == 2 || mode == 3;
            const bool better = forced || sim.physical_pairs < part[u].physical_pairs ||
                                (sim.physical_pairs == part[u].physical_pairs && sim.work.size() < part[u].work.size());
            if (better) part[u] = std::move(sim);
          }
        }
        // the 64-row route, where the model gives it the shorter time
        if (route64 && (route_mode == 0 || route_mode == 4)) {
          WorkList hv;
          if (build_head_halves(own, col, adj, u, src, blocks, hv, acc, touched) &&
              (route_mode == 4 || query_pass_cost(hv) < query_pass_cost(part[u])))
            part[u] = std::move(hv);
        }
        order_longest_first(part[u]);
      }
    } catch (...) {
      failed[t] = 1;  // an allocation failed; reported below as OOM
    }
  };
  if (n_threads == 1) {
    worker(0);
  } else {
    // A thread that cannot be created (std::system_error, or bad_alloc for
    // the pool) leaves its share to the calling thread; threads already
    // started are always joined, so nothing escapes the C ABI.
    std::vector<std::thread> pool;
    int started = 0;
    try {
      pool.reserve(n_threads);
      for (; started < n_threads; ++started) pool.emplace_back(worker, started);
    } catch (...) {
    }
    for (int t = started; t < n_threads; ++t) worker(t);
    for (auto& th : pool) th.join();
  }
  for (char f : failed)
    if (f) return SPATTN_ERR_OOM;
  try {
    for (int32_t u = 0; u < n_units; ++u) {
      if (same_as[u] < 0) continue;
      part[u] = part[same_as[u]];
      for (size_t i = 0; i < part[u].work.size(); i += kWorkWords) part[u].work[i] = u;
    }
  } catch (...) {
    return SPATTN_ERR_OOM;
  }
  size_t n_entries = 0;
  for (const auto& pt : part) n_entries += pt.pages.size();
  if (n_entries > static_cast<size_t>(INT32_MAX)) return SPATTN_ERR_UNSUPPORTED;
  wl.work.clear();
  wl.pages.clear();
  wl.masks.clear();
  wl.heads.clear();
  wl.physical_pairs = 0;
  wl.pages.reserve(n_entries);
  wl.masks.reserve(n_entries * kMaskWords);
  wl.heads.reserve(n_entries);
  for (auto& pt : part) {
    const int32_t off = static_cast<int32_t>(wl.pages.size());  // entry ranges are per part
    for (size_t i = 0; i < pt.work.size(); i += kWorkWords) {
      pt.work[i + 2] += off;
      pt.work[i + 3] += off;
    }
    wl.work.insert(wl.work.end(), pt.work.begin(), pt.work.end());
    wl.pages.insert(wl.pages.end(), pt.pages.begin(), pt.pages.end());
    wl.masks.insert(wl.masks.end(), pt.masks.begin(), pt.masks.end());
    wl.heads.insert(wl.heads.end(), pt.heads.begin(), pt.heads.end());
    wl.physical_pairs += pt.physical_pairs;
    pt = WorkList();  // release the part's memory as soon as it is copied
  }
  const int64_t per_copy = static_cast<int64_t>(wl.work.size()) / kWorkWords;
  std::vector<int32_t> all;
  all.reserve(static_cast<size_t>(per_copy) * batch_copies * kWorkWords);
  for (int32_t b = 0; b < batch_copies; ++b)
    for (int64_t i = 0; i < per_copy; ++i) {
      const int32_t* w = wl.work.data() + i * kWorkWords;
      all.insert(all.end(), w, w + kWorkWords);
      all[all.size() - kWorkWords] = b * owned_heads + w[0];
    }
  wl.work.swap(all);
  wl.n_work = per_copy * batch_copies;
  wl.physical_pairs *= batch_copies;
  wl.route64 = false;
  for (size_t i = 28; i < wl.work.size(); i += kWorkWords) wl.route64 = wl.route64 || wl.work[i] != 0;
  return SPATTN_OK;
}


// Rows of one side that no work item writes, as (page, row mask) pairs:
// pages without a valid slot (all 16 rows), and the rows outside the 4-row
// group of the pages that a strided owned page stands for (padded rows).
void fill_list(const Side& s, std::vector<int32_t>& out) {
  out.clear();
  std::vector<uint16_t> fill(s.n_pages, 0);
  for (int64_t p = 0; p < s.n_pages; ++p)
    if (!s.page_mask[p]) fill[p] = 0xFFFFu;
  for (const auto& b : owned_blocks(s)) {
    if (b.strided_group < 0) continue;
    const int64_t p0 = (~b.pages[0]) / 16;
    for (int j = 0; j < 4; ++j) fill[p0 + j] = static_cast<uint16_t>(0xFFFFu & ~(0xFu << (4 * b.strided_group)));
  }
  for (int64_t p = 0; p < s.n_pages; ++p)
    if (fill[p]) {
      out.push_back(static_cast<int32_t>(p));
      out.push_back(fill[p]);
    }
}

template <typename T>
int upload(const std::vector<T>& host, T** dev, int64_t& bytes, int64_t* cap = nullptr) {
  const size_t n = std::max<size_t>(host.size(), 1) * sizeof(T);
  if (cudaMalloc(reinterpret_cast<void**>(dev), n) != cudaSuccess) return SPATTN_ERR_OOM;
  if (cap) *cap = static_cast<int64_t>(std::max<size_t>(host.size(), 1));
  bytes += static_cast<int64_t>(n);
  if (!host.empty() && cudaMemcpy(*dev, host.data(), host.size() * sizeof(T), cudaMemcpyHostToDevice) != cudaSuccess)
    return SPATTN_ERR_CUDA;
  return SPATTN_OK;
}

}  // namespace

// Canonical page list of (head, Q block) from the groups present in the block.
void canonical_pages(const spattn_plan_s& P, int32_t h, int64_t qb, std::vector<int32_t>& out) {
  out.clear();
  std::vector<int32_t> groups;
  const int64_t r0 = qb * kBlockRows, r1 = std::min<int64_t>(r0 + kBlockRows, P.q.slots);
  for (int64_t i = r0; i < r1; ++i) {
    const int32_t g = P.q.group[i];
    if (g >= 0 && std::find(groups.begin(), groups.end(), g) == groups.end()) groups.push_back(g);
  }
  for (int32_t a : groups) {
    const int64_t r = static_cast<int64_t>(h) * P.fwd_adj.n_src + a;
    for (int64_t e = P.fwd_adj.ptr[r]; e < P.fwd_adj.ptr[r + 1]; ++e) {
      const int32_t b = P.fwd_adj.dst[e];
      for (int64_t x = P.k.gp_ptr[b]; x < P.k.gp_ptr[b + 1]; ++x) out.push_back(P.k.gp_page[x]);
    }
  }
  std::sort(out.begin(), out.end());
  out.erase(std::unique(out.begin(), out.end()), out.end());
}

void transposed_qblocks(const spattn_plan_s& P, int32_t h, int64_t page, std::vector<int32_t>& out) {
  out.clear();
  std::vector<int32_t> groups;
  const int64_t r0 = page * kPageRows, r1 = std::min<int64_t>(r0 + kPageRows, P.k.slots);
  for (int64_t j = r0; j < r1; ++j) {
    const int32_t g = P.k.group[j];
    if (g >= 0 && std::find(groups.begin(), groups.end(), g) == groups.end()) groups.push_back(g);
  }
  const int per = kBlockRows / kPageRows;
  for (int32_t b : groups) {
    const int64_t r = static_cast<int64_t>(h) * P.bwd_adj.n_src + b;
    for (int64_t e = P.bwd_adj.ptr[r]; e < P.bwd_adj.ptr[r + 1]; ++e) {
      const int32_t a = P.bwd_adj.dst[e];
      for (int64_t x = P.q.gp_ptr[a]; x < P.q.gp_ptr[a + 1]; ++x) out.push_back(P.q.gp_page[x] / per);
    }
  }
  std::sort(out.begin(), out.end());
  out.erase(std::unique(out.begin(), out.end()), out.end());
}

int64_t bsa_pairs(const spattn_plan_s& P) {
  const int64_t n_qb = (P.q.slots + kBlockRows - 1) / kBlockRows;
  const int per = kBlockRows / kPageRows;
  std::vector<int32_t> pages;
  int64_t count = 0;
  for (int32_t h = 0; h < P.graph_batches * P.heads; ++h)
    for (int64_t qb = 0; qb < n_qb; ++qb) {
      canonical_pages(P, h, qb, pages);
      int64_t prev = -1;
      for (int32_t p : pages)
        if (p / per != prev) {
          prev = p / per;
          ++count;
        }
    }
  return count * kBlockRows * kBlockRows * (P.batch / P.graph_batches);
}

void free_device_planner(DevPlanner& d);

void free_plan_device(spattn_plan_s* P) {
  free_device_planner(P->dp);
  cudaFree(P->wk.d_heads);
  P->wk.d_heads = nullptr;
  cudaFree(P->wq.d_work);
  cudaFree(P->wq.d_pages);
  cudaFree(P->wq.d_masks);
  cudaFree(P->wk.d_work);
  cudaFree(P->wk.d_pages);
  cudaFree(P->wk.d_masks);
  cudaFree(P->d_q_fill);
  cudaFree(P->d_k_fill);
  cudaFree(P->d_err);
  cudaFree(P->d_sched);
  cudaFree(P->d_delta);
  for (auto& e : P->events) {
    cudaEventDestroy(e.start);
    cudaEventDestroy(e.stop);
  }
  P->events.clear();
  P->n_events = 0;
}

// After a device re-plan: bring the work lists and the graph back to the host
// copies that the inspection calls read (synchronises the device).
int refresh_host(spattn_plan_s* P) {
  if (!P->host_stale) return SPATTN_OK;
  if (cudaDeviceSynchronize() != cudaSuccess) return SPATTN_ERR_CUDA;
  for (WorkList* w : {&P->wq, &P->wk}) {
    w->work.resize(static_cast<size_t>(w->n_work) * kWorkWords);
    w->pages.resize(static_cast<size_t>(w->n_entries_dev));
    w->masks.resize(static_cast<size_t>(w->n_entries_dev) * kMaskWords);
    if ((!w->work.empty() && cudaMemcpy(w->work.data(), w->d_work, w->work.size() * sizeof(int32_t),
                                        cudaMemcpyDeviceToHost) != cudaSuccess) ||
        (!w->pages.empty() && cudaMemcpy(w->pages.data(), w->d_pages, w->pages.size() * sizeof(int32_t),
                                         cudaMemcpyDeviceToHost) != cudaSuccess) ||
        (!w->masks.empty() && cudaMemcpy(w->masks.data(), w->d_masks, w->masks.size() * sizeof(uint64_t),
                                         cudaMemcpyDeviceToHost) != cudaSuccess))
      return SPATTN_ERR_CUDA;
  }
  // entry head offsets: written by the device planner under grouped-query
  // attention, else all 0
  P->wk.heads.assign(static_cast<size_t>(P->wk.n_entries_dev), 0);
  if (P->kv_heads != P->heads && !P->wk.heads.empty() &&
      cudaMemcpy(P->wk.heads.data(), P->wk.d_heads, P->wk.heads.size() * sizeof(uint16_t), cudaMemcpyDeviceToHost) !=
          cudaSuccess)
    return SPATTN_ERR_CUDA;
  const int64_t rows = static_cast<int64_t>(P->graph_batches) * P->heads * P->q.n_groups;
  std::vector<int64_t> rp(rows + 1);
  std::vector<int32_t> dst(std::max<int64_t>(P->graph_nnz, 1));
  if (cudaMemcpy(rp.data(), P->dp.d_fwd_ptr, rp.size() * sizeof(int64_t), cudaMemcpyDeviceToHost) != cudaSuccess ||
      (P->graph_nnz > 0 && cudaMemcpy(dst.data(), P->dp.d_fwd_dst, P->graph_nnz * sizeof(int32_t),
                                      cudaMemcpyDeviceToHost) != cudaSuccess))
    return SPATTN_ERR_CUDA;
  spattn_graph g{rp.data(), dst.data()};
  const int32_t GH = P->graph_batches * P->heads;
  int st = build_fwd_adjacency(&g, GH, P->q.n_groups, P->k.n_groups, P->fwd_adj);
  if (st) return st;
  build_bwd_adjacency(P->fwd_adj, GH, P->q.n_groups, P->k.n_groups, P->bwd_adj);
  P->host_stale = false;
  return SPATTN_OK;
}

int build_plan(const spattn_layout* L, const spattn_graph* G, spattn_plan_s* P) {
  const auto t0 = std::chrono::steady_clock::now();
  if (!L || !G || !L->q_group || !L->kv_group || !G->row_ptr) return SPATTN_ERR_INVALID_ARG;
  if (L->batch < 1 || L->heads < 1 || L->q_slots < 1 || L->kv_slots < 1) return SPATTN_ERR_INVALID_ARG;
  if (L->n_q_groups < 0 || L->n_kv_groups < 0) return SPATTN_ERR_INVALID_ARG;
  if (L->head_dim != 64 && L->head_dim != 128) return SPATTN_ERR_UNSUPPORTED;
  if (L->q_slots >= (int64_t(1) << 31) - 64 || L->kv_slots >= (int64_t(1) << 31) - 64) return SPATTN_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(L->batch) * L->heads >= (int64_t(1) << 31)) return SPATTN_ERR_UNSUPPORTED;
  if (!std::isfinite(L->scale) || L->scale < 0.f) return SPATTN_ERR_INVALID_ARG;
  const int32_t kv_heads = L->kv_heads == 0 ? L->heads : L->kv_heads;
  if (kv_heads < 1 || L->heads % kv_heads != 0) return SPATTN_ERR_INVALID_ARG;
  if (L->heads / kv_heads > 65535) return SPATTN_ERR_UNSUPPORTED;
  const int32_t gb = L->graph_batches == 0 ? 1 : L->graph_batches;
  if (gb != 1 && gb != L->batch) return SPATTN_ERR_INVALID_ARG;
  const int32_t GH = gb * L->heads;  // graph heads: one graph per (graph batch, head)
  if (static_cast<int64_t>(GH) * std::max(L->n_q_groups, L->n_kv_groups) >= (int64_t(1) << 40))
    return SPATTN_ERR_UNSUPPORTED;
  if (G->row_ptr[static_cast<int64_t>(GH) * L->n_q_groups] > 0 && !G->kv_groups) return SPATTN_ERR_INVALID_ARG;

  P->batch = L->batch;
  P->heads = L->heads;
  P->kv_heads = kv_heads;
  P->graph_batches = gb;
  P->head_dim = L->head_dim;
  P->scale = L->scale != 0.f ? L->scale : 1.0f / std::sqrt(static_cast<float>(L->head_dim));
  // Without a usable CUDA device the plan is kept on the host only: the
  // inspection calls work, spattn_fwd / spattn_bwd return SPATTN_ERR_CUDA.
  int n_dev = 0;
  if (cudaGetDeviceCount(&n_dev) != cudaSuccess || n_dev == 0 || cudaGetDevice(&P->device) != cudaSuccess) {
    P->device = -1;
    cudaGetLastError();
  }

  int st = build_side(L->q_slots, L->q_group, L->n_q_groups, P->q);
  if (st) return st;
  st = build_side(L->kv_slots, L->kv_group, L->n_kv_groups, P->k);
  if (st) return st;
  st = build_fwd_adjacency(G, GH, L->n_q_groups, L->n_kv_groups, P->fwd_adj);
  if (st) return st;
  build_bwd_adjacency(P->fwd_adj, GH, L->n_q_groups, L->n_kv_groups, P->bwd_adj);

  int64_t useful = 0;
  for (int32_t h = 0; h < GH; ++h)
    for (int32_t a = 0; a < L->n_q_groups; ++a) {
      const int64_t r = static_cast<int64_t>(h) * L->n_q_groups + a;
      int64_t nk = 0;
      for (int64_t e = P->fwd_adj.ptr[r]; e < P->fwd_adj.ptr[r + 1]; ++e) nk += P->k.group_size[P->fwd_adj.dst[e]];
      useful += P->q.group_size[a] * nk;
    }
  const int32_t copies = L->batch / gb;  // batch entries that share each graph
  P->useful_pairs = useful * copies;

  // key-owned pass: unit = K/V head of a graph batch; its columns are the
  // transposed rows of the query heads of its group (head offset j).  It
  // only reads the layout and its own adjacency, so it runs on a thread of
  // its own while this thread builds the query-owned pass (after it, if no
  // thread can be created).
  const int32_t grp = L->heads / kv_heads;
  const int32_t H = L->heads;
  const int32_t n_kv_units = gb * kv_heads;
  int st_k = SPATTN_OK;
  auto key_pass = [&]() {
    try {
      st_k = build_worklist(P->k, P->q, P->bwd_adj, n_kv_units, kv_heads, copies,
                            [=](int32_t u) {
                              std::vector<int64_t> v(grp);
                              for (int32_t j = 0; j < grp; ++j)
                                v[j] = static_cast<int64_t>(u / kv_heads) * H + (u % kv_heads) * grp + j;
                              return v;
                            },
                            false, P->wk);
    } catch (...) {
      st_k = SPATTN_ERR_OOM;
    }
  };
  std::thread key_thread;
  bool key_threaded = false;
  try {
    key_thread = std::thread(key_pass);
    key_threaded = true;
  } catch (...) {
  }
  // query-owned pass: unit = graph head (its own graph rows)
  try {
    st = build_worklist(P->q, P->k, P->fwd_adj, GH, L->heads, copies,
                        [](int32_t u) { return std::vector<int64_t>{u}; }, true, P->wq);
  } catch (...) {
    st = SPATTN_ERR_OOM;
  }
  if (key_threaded) key_thread.join();
  else key_pass();
  if (st) return st;
  if (st_k) return st_k;

  fill_list(P->q, P->q_fill);
  fill_list(P->k, P->k_fill);
  make_templates(P->q, P->dp.tq);
  make_templates(P->k, P->dp.tk);

  P->plan_ms = std::chrono::duration<double, std::milli>(std::chrono::steady_clock::now() - t0).count();
  if (P->device < 0) return SPATTN_OK;

  int64_t bytes = 0;
  if ((st = upload(P->wk.heads, &P->wk.d_heads, bytes, &P->wk.cap_heads))) return st;
  for (WorkList* w : {&P->wq, &P->wk}) {
    if ((st = upload(w->work, &w->d_work, bytes, &w->cap_work))) return st;
    if ((st = upload(w->pages, &w->d_pages, bytes, &w->cap_pages))) return st;
    if ((st = upload(w->masks, &w->d_masks, bytes, &w->cap_masks))) return st;
  }
  if ((st = upload(P->q_fill, &P->d_q_fill, bytes))) return st;
  if ((st = upload(P->k_fill, &P->d_k_fill, bytes))) return st;
  if (cudaMalloc(reinterpret_cast<void**>(&P->d_err), sizeof(int)) != cudaSuccess) return SPATTN_ERR_OOM;
  if (cudaMalloc(reinterpret_cast<void**>(&P->d_sched), sizeof(int)) != cudaSuccess) return SPATTN_ERR_OOM;
  if (cudaMemset(P->d_err, 0, sizeof(int)) != cudaSuccess) return SPATTN_ERR_CUDA;
  const size_t delta_bytes = static_cast<size_t>(L->batch) * L->heads * L->q_slots * sizeof(float);
  if (cudaMalloc(reinterpret_cast<void**>(&P->d_delta), delta_bytes) != cudaSuccess) return SPATTN_ERR_OOM;
  P->device_bytes = bytes + static_cast<int64_t>(delta_bytes) + static_cast<int64_t>(sizeof(int));
  P->plan_ms = std::chrono::duration<double, std::milli>(std::chrono::steady_clock::now() - t0).count();
  return SPATTN_OK;
}

}  // namespace spattn
