// Host planner internals: owned-tile packing, per-tile page lists and masks.
#pragma once

#include <stdint.h>

#include <string>
#include <vector>

#include <cuda_runtime.h>

#include "spattn.h"

namespace spattn {

constexpr int kPageRows = 16;     // rows per page (the unit packed into tiles)
constexpr int kBlockRows = 64;    // rows per logical Q block
constexpr int kTilePages = 8;     // pages per 128-row tile
constexpr int kMaxSegments = 8;   // distinct groups per work item (16-bit mask each)
constexpr int kMaskWords = 2;     // uint64 words per column entry: segment s at bits 16 (s % 4) of word s / 4
constexpr int kWorkWords = 32;    // int32 words per work item

// Page references (owned pages of a work item, column entries of its list):
// a value p >= 0 is the 16-row page of slots 16p .. 16p+15; a negative value
// is a strided page with base slot b = ~value (a multiple of 4), the four
// 4-row groups b + 16j .. b + 16j + 3 (j = 0..3), row r of it at
// b + 16 (r / 4) + r % 4.  A strided page gathers rows that sit in the same
// 4-row group of four consecutive pages, e.g. the single valid dh row of
// each dt slice of a tile cut by the grid's H edge.
inline int64_t pref_slot(int32_t ref, int r) {
  return ref >= 0 ? static_cast<int64_t>(ref) * 16 + r : static_cast<int64_t>(~ref) + 16 * (r >> 2) + (r & 3);
}
inline int64_t pref_first_slot(int32_t ref) { return ref >= 0 ? static_cast<int64_t>(ref) * 16 : ~ref; }

// Row codes in a work item (4 bits per tile row).
constexpr uint32_t kCodeNoSegment = 14;  // owned row without a group (padded): writes zeros
constexpr uint32_t kCodeNotOwned = 15;   // row written by another item (or beyond the tensor)

// One side (queries or keys) of the layout.
struct Side {
  int64_t slots = 0;
  int32_t n_groups = 0;
  int64_t n_pages = 0;
  std::vector<int32_t> group;       // [slots]
  std::vector<uint16_t> page_mask;  // [n_pages] valid-row bits
  // group -> (page, rows of that group in the page), pages ascending
  std::vector<int64_t> gp_ptr;      // [n_groups + 1]
  std::vector<int32_t> gp_page;
  std::vector<uint16_t> gp_mask;
  std::vector<int64_t> group_size;  // [n_groups]
};

// Adjacency of one direction for all heads: CSR over (head, source group).
struct Adjacency {
  int32_t n_src = 0;
  std::vector<int64_t> ptr;   // [heads * n_src + 1]
  std::vector<int32_t> dst;   // sorted, unique per row
};

// Work list of one pass (query-owned or key-owned), host and device copies.
struct WorkList {
  std::vector<int32_t> work;     // n_work * kWorkWords (all batches)
  std::vector<int32_t> pages;    // entries of one batch
  std::vector<uint64_t> masks;   // kMaskWords per entry
  // per entry: the query head of the entry within the item's K/V head group
  // (key-owned pass under grouped-query attention; 0 otherwise)
  std::vector<uint16_t> heads;
  uint16_t* d_heads = nullptr;
  int64_t n_work = 0;
  bool route64 = false;          // some item takes the 64-row route (word 28)
  int64_t physical_pairs = 0;    // one batch
  int32_t* d_work = nullptr;
  int32_t* d_pages = nullptr;
  uint64_t* d_masks = nullptr;
  // capacities of the device arrays (elements) and, after a device re-plan,
  // the number of entries on the device
  int64_t cap_work = 0, cap_pages = 0, cap_masks = 0, cap_heads = 0;
  int64_t n_entries_dev = -1;
};

// Work item templates of one pass for the device planner: the slot-order
// tiles of the layout split into items, without their column lists.
struct PassTemplates {
  std::vector<int32_t> words;     // n x kWorkWords (bh and entry range set on the device)
  std::vector<int32_t> segs;      // n x kMaxSegments group of each segment, -1 = none
  std::vector<int32_t> seg_rows;  // n x kMaxSegments owned rows of each segment
  int64_t n = 0;
  int32_t* d_words = nullptr;
  int32_t* d_segs = nullptr;
  int32_t* d_seg_rows = nullptr;
};

// Device state of spattn_plan_set_graph_device (allocated on first use).
struct DevPlanner {
  bool ready = false;
  PassTemplates tq, tk;  // query-owned, key-owned
  int64_t* d_q_gp_ptr = nullptr;
  int32_t* d_q_gp_page = nullptr;
  uint16_t* d_q_gp_mask = nullptr;
  int64_t* d_k_gp_ptr = nullptr;
  int32_t* d_k_gp_page = nullptr;
  uint16_t* d_k_gp_mask = nullptr;
  int64_t* d_fwd_ptr = nullptr;   // the graph (plan-owned copy)
  int32_t* d_fwd_dst = nullptr;
  int64_t fwd_cap = 0;
  int64_t* d_bwd_ptr = nullptr;   // its transpose
  int32_t* d_bwd_dst = nullptr;
  int64_t bwd_cap = 0;
  int64_t* d_cursor = nullptr;
  int64_t* d_counts = nullptr;
  unsigned long long* d_stats = nullptr;
};

bool strided_setting();

}  // namespace spattn

struct spattn_plan_s {
  int32_t batch = 0, heads = 0, head_dim = 0;
  int32_t kv_heads = 0;       // K/V heads (heads % kv_heads == 0)
  int32_t graph_batches = 1;  // 1: one graph for every batch entry; batch: one graph per entry
  float scale = 0.f;
  int device = 0;
  spattn::Side q, k;
  spattn::Adjacency fwd_adj;  // query group -> key groups
  spattn::Adjacency bwd_adj;  // key group -> query groups
  spattn::WorkList wq;        // query-owned tiles (forward, dQ)
  spattn::WorkList wk;        // key-owned tiles (dK/dV)
  // Rows that no work item writes, per side, as (page, 16-bit row mask)
  // pairs: every row of a page with no valid slot, and the padded rows that a
  // strided owned page leaves out.  The fill kernel writes zeros (and
  // LSE = -inf) there.
  std::vector<int32_t> q_fill, k_fill;
  int32_t* d_q_fill = nullptr;
  int32_t* d_k_fill = nullptr;
  int* d_err = nullptr;        // device error word
  int* d_sched = nullptr;      // work-item counter of the persistent dK/dV kernel
  float* d_delta = nullptr;    // [batch, heads, q_slots] rowsum(dO * O)
  spattn::DevPlanner dp;        // device planner state
  bool host_stale = false;      // the work lists / graph were rebuilt on the device
  int64_t graph_nnz = 0;        // entries of the graph the device lists follow
  int64_t useful_pairs = 0;
  int64_t bsa_pairs = -1;      // computed on first request
  int64_t device_bytes = 0;
  double plan_ms = 0.0;
  std::vector<int32_t> scratch;  // buffer behind spattn_plan_pages / spattn_plan_qblocks
  // per-kernel event record (spattn_profile)
  bool profiling = false;
  struct EventRec {
    int kernel;
    cudaEvent_t start, stop;
  };
  std::vector<EventRec> events;   // pool; the first n_events are in use
  size_t n_events = 0;
};
