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
//     64-slot blocks packed in slot order, pages without a valid row left
//     out), so partly occupied blocks share a tile instead of padding it;
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
#include <new>
#include <thread>

namespace spattn {

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

// Owned tiles: whole 64-slot blocks, valid pages only, packed in slot order
// while the tile holds at most 8 pages.
std::vector<std::vector<int32_t>> pack_tiles(const Side& s) {
  std::vector<std::vector<int32_t>> tiles;
  std::vector<int32_t> cur;
  const int64_t n_blocks = (s.slots + kBlockRows - 1) / kBlockRows;
  const int per = kBlockRows / kPageRows;
  for (int64_t blk = 0; blk < n_blocks; ++blk) {
    std::vector<int32_t> vp;
    for (int i = 0; i < per; ++i) {
      const int64_t p = blk * per + i;
      if (p < s.n_pages && s.page_mask[p]) vp.push_back(static_cast<int32_t>(p));
    }
    if (vp.empty()) continue;
    if (cur.size() + vp.size() > static_cast<size_t>(kTilePages)) {
      tiles.push_back(cur);
      cur.clear();
    }
    cur.insert(cur.end(), vp.begin(), vp.end());
  }
  if (!cur.empty()) tiles.push_back(cur);
  return tiles;
}

// Work items of one head for one pass; work words use bh = head (batch 0).
void build_head(const Side& own, const Side& col, const Adjacency& adj, int32_t h,
                const std::vector<std::vector<int32_t>>& tiles, WorkList& wl, std::vector<uint64_t>& acc,
                std::vector<int32_t>& touched) {
  int32_t rg[kTilePages * kPageRows];
  for (const auto& tile : tiles) {
    const int npg = static_cast<int>(tile.size());
    std::vector<int32_t> segs;
    for (int r = 0; r < kTilePages * kPageRows; ++r) {
      int32_t g = -2;  // row does not exist in this tile / tensor
      if (r < npg * kPageRows) {
        const int64_t slot = static_cast<int64_t>(tile[r / kPageRows]) * kPageRows + r % kPageRows;
        if (slot < own.slots) g = own.group[slot];
      }
      rg[r] = g;
      if (g >= 0 && std::find(segs.begin(), segs.end(), g) == segs.end()) segs.push_back(g);
    }
    const int n_items = std::max<int>(1, (static_cast<int>(segs.size()) + kMaxSegments - 1) / kMaxSegments);
    for (int it = 0; it < n_items; ++it) {
      const int s0 = it * kMaxSegments;
      const int s1 = std::min<int>(s0 + kMaxSegments, static_cast<int>(segs.size()));
      touched.clear();
      for (int s = s0; s < s1; ++s) {
        const int64_t r = static_cast<int64_t>(h) * adj.n_src + segs[s];
        for (int64_t e = adj.ptr[r]; e < adj.ptr[r + 1]; ++e) {
          const int32_t b = adj.dst[e];
          for (int64_t x = col.gp_ptr[b]; x < col.gp_ptr[b + 1]; ++x) {
            const int32_t p = col.gp_page[x];
            if (acc[p] == 0) touched.push_back(p);
            acc[p] |= static_cast<uint64_t>(col.gp_mask[x]) << (16 * (s - s0));
          }
        }
      }
      std::sort(touched.begin(), touched.end());
      int32_t w[kWorkWords];
      std::memset(w, 0, sizeof(w));
      w[0] = h;
      w[1] = npg;
      w[2] = static_cast<int32_t>(wl.pages.size());
      for (int32_t p : touched) {
        wl.pages.push_back(p);
        wl.masks.push_back(acc[p]);
        acc[p] = 0;
      }
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
      wl.physical_pairs += static_cast<int64_t>(kTilePages * kPageRows) * kPageRows * static_cast<int64_t>(touched.size());
      wl.work.insert(wl.work.end(), w, w + kWorkWords);
    }
  }
}

int build_worklist(const Side& own, const Side& col, const Adjacency& adj, int32_t heads, int32_t batch,
                   WorkList& wl) {
  const auto tiles = pack_tiles(own);
  // Heads are independent: each is built on its own into part[h] (worker t
  // takes heads t, t + n, ...), then the parts are joined in head order, so
  // the result does not depend on the number of threads.
  std::vector<WorkList> part(heads);
  // all hardware threads, unless SPATTN_PLAN_THREADS (>= 1) asks for fewer or more
  int want = static_cast<int>(std::thread::hardware_concurrency());
  if (const char* env = std::getenv("SPATTN_PLAN_THREADS")) want = std::max(1, std::atoi(env));
  const int n_threads = std::max(1, std::min<int>(heads, want));
  std::vector<char> failed(n_threads, 0);
  auto worker = [&](int t) {
    try {
      std::vector<uint64_t> acc(col.n_pages, 0);
      std::vector<int32_t> touched;
      for (int32_t h = t; h < heads; h += n_threads) build_head(own, col, adj, h, tiles, part[h], acc, touched);
    } catch (...) {
      failed[t] = 1;  // an allocation failed; reported below as OOM
    }
  };
  if (n_threads == 1) {
    worker(0);
  } else {
    std::vector<std::thread> pool;
    pool.reserve(n_threads);
    for (int t = 0; t < n_threads; ++t) pool.emplace_back(worker, t);
    for (auto& th : pool) th.join();
  }
  for (char f : failed)
    if (f) return SPATTN_ERR_OOM;
  size_t n_entries = 0;
  for (const auto& pt : part) n_entries += pt.pages.size();
  if (n_entries > static_cast<size_t>(INT32_MAX)) return SPATTN_ERR_UNSUPPORTED;
  wl.work.clear();
  wl.pages.clear();
  wl.masks.clear();
  wl.physical_pairs = 0;
  wl.pages.reserve(n_entries);
  wl.masks.reserve(n_entries);
  for (auto& pt : part) {
    const int32_t off = static_cast<int32_t>(wl.pages.size());  // entry ranges are per part
    for (size_t i = 0; i < pt.work.size(); i += kWorkWords) {
      pt.work[i + 2] += off;
      pt.work[i + 3] += off;
    }
    wl.work.insert(wl.work.end(), pt.work.begin(), pt.work.end());
    wl.pages.insert(wl.pages.end(), pt.pages.begin(), pt.pages.end());
    wl.masks.insert(wl.masks.end(), pt.masks.begin(), pt.masks.end());
    wl.physical_pairs += pt.physical_pairs;
    pt = WorkList();  // release the part's memory as soon as it is copied
  }
  const int64_t per_batch = static_cast<int64_t>(wl.work.size()) / kWorkWords;
  std::vector<int32_t> all;
  all.reserve(static_cast<size_t>(per_batch) * batch * kWorkWords);
  for (int32_t b = 0; b < batch; ++b)
    for (int64_t i = 0; i < per_batch; ++i) {
      const int32_t* w = wl.work.data() + i * kWorkWords;
      all.insert(all.end(), w, w + kWorkWords);
      all[all.size() - kWorkWords] = b * heads + w[0];
    }
  wl.work.swap(all);
  wl.n_work = per_batch * batch;
  return SPATTN_OK;
}

template <typename T>
int upload(const std::vector<T>& host, T** dev, int64_t& bytes) {
  const size_t n = std::max<size_t>(host.size(), 1) * sizeof(T);
  if (cudaMalloc(reinterpret_cast<void**>(dev), n) != cudaSuccess) return SPATTN_ERR_OOM;
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
  for (int32_t h = 0; h < P.heads; ++h)
    for (int64_t qb = 0; qb < n_qb; ++qb) {
      canonical_pages(P, h, qb, pages);
      int64_t prev = -1;
      for (int32_t p : pages)
        if (p / per != prev) {
          prev = p / per;
          ++count;
        }
    }
  return count * kBlockRows * kBlockRows * P.batch;
}

void free_plan_device(spattn_plan_s* P) {
  cudaFree(P->wq.d_work);
  cudaFree(P->wq.d_pages);
  cudaFree(P->wq.d_masks);
  cudaFree(P->wk.d_work);
  cudaFree(P->wk.d_pages);
  cudaFree(P->wk.d_masks);
  cudaFree(P->d_q_invalid);
  cudaFree(P->d_k_invalid);
  cudaFree(P->d_err);
  cudaFree(P->d_delta);
  for (auto& e : P->events) {
    cudaEventDestroy(e.start);
    cudaEventDestroy(e.stop);
  }
  P->events.clear();
  P->n_events = 0;
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
  if (G->row_ptr[static_cast<int64_t>(L->heads) * L->n_q_groups] > 0 && !G->kv_groups) return SPATTN_ERR_INVALID_ARG;

  P->batch = L->batch;
  P->heads = L->heads;
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
  st = build_fwd_adjacency(G, L->heads, L->n_q_groups, L->n_kv_groups, P->fwd_adj);
  if (st) return st;
  build_bwd_adjacency(P->fwd_adj, L->heads, L->n_q_groups, L->n_kv_groups, P->bwd_adj);

  int64_t useful = 0;
  for (int32_t h = 0; h < L->heads; ++h)
    for (int32_t a = 0; a < L->n_q_groups; ++a) {
      const int64_t r = static_cast<int64_t>(h) * L->n_q_groups + a;
      int64_t nk = 0;
      for (int64_t e = P->fwd_adj.ptr[r]; e < P->fwd_adj.ptr[r + 1]; ++e) nk += P->k.group_size[P->fwd_adj.dst[e]];
      useful += P->q.group_size[a] * nk;
    }
  P->useful_pairs = useful * L->batch;

  st = build_worklist(P->q, P->k, P->fwd_adj, L->heads, L->batch, P->wq);
  if (st) return st;
  st = build_worklist(P->k, P->q, P->bwd_adj, L->heads, L->batch, P->wk);
  if (st) return st;

  for (int64_t p = 0; p < P->q.n_pages; ++p)
    if (!P->q.page_mask[p]) P->q_invalid_pages.push_back(static_cast<int32_t>(p));
  for (int64_t p = 0; p < P->k.n_pages; ++p)
    if (!P->k.page_mask[p]) P->k_invalid_pages.push_back(static_cast<int32_t>(p));

  P->plan_ms = std::chrono::duration<double, std::milli>(std::chrono::steady_clock::now() - t0).count();
  if (P->device < 0) return SPATTN_OK;

  int64_t bytes = 0;
  if ((st = upload(P->wq.work, &P->wq.d_work, bytes))) return st;
  if ((st = upload(P->wq.pages, &P->wq.d_pages, bytes))) return st;
  if ((st = upload(P->wq.masks, &P->wq.d_masks, bytes))) return st;
  if ((st = upload(P->wk.work, &P->wk.d_work, bytes))) return st;
  if ((st = upload(P->wk.pages, &P->wk.d_pages, bytes))) return st;
  if ((st = upload(P->wk.masks, &P->wk.d_masks, bytes))) return st;
  if ((st = upload(P->q_invalid_pages, &P->d_q_invalid, bytes))) return st;
  if ((st = upload(P->k_invalid_pages, &P->d_k_invalid, bytes))) return st;
  if (cudaMalloc(reinterpret_cast<void**>(&P->d_err), sizeof(int)) != cudaSuccess) return SPATTN_ERR_OOM;
  if (cudaMemset(P->d_err, 0, sizeof(int)) != cudaSuccess) return SPATTN_ERR_CUDA;
  const size_t delta_bytes = static_cast<size_t>(L->batch) * L->heads * L->q_slots * sizeof(float);
  if (cudaMalloc(reinterpret_cast<void**>(&P->d_delta), delta_bytes) != cudaSuccess) return SPATTN_ERR_OOM;
  P->device_bytes = bytes + static_cast<int64_t>(delta_bytes) + static_cast<int64_t>(sizeof(int));
  P->plan_ms = std::chrono::duration<double, std::milli>(std::chrono::steady_clock::now() - t0).count();
  return SPATTN_OK;
}

}  // namespace spattn
