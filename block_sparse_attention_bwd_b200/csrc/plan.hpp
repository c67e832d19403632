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
constexpr int kMaxSegments = 4;   // distinct groups per work item (16-bit mask each)
constexpr int kWorkWords = 32;    // int32 words per work item

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
  std::vector<uint64_t> masks;
  int64_t n_work = 0;
  int64_t physical_pairs = 0;    // one batch
  int32_t* d_work = nullptr;
  int32_t* d_pages = nullptr;
  uint64_t* d_masks = nullptr;
};

}  // namespace spattn

struct spattn_plan_s {
  int32_t batch = 0, heads = 0, head_dim = 0;
  float scale = 0.f;
  int device = 0;
  spattn::Side q, k;
  spattn::Adjacency fwd_adj;  // query group -> key groups
  spattn::Adjacency bwd_adj;  // key group -> query groups
  spattn::WorkList wq;        // query-owned tiles (forward, dQ)
  spattn::WorkList wk;        // key-owned tiles (dK/dV)
  // pages with no valid row, per side (filled with zeros / -inf)
  std::vector<int32_t> q_invalid_pages, k_invalid_pages;
  int32_t* d_q_invalid = nullptr;
  int32_t* d_k_invalid = nullptr;
  int* d_err = nullptr;        // device error word
  float* d_delta = nullptr;    // [batch, heads, q_slots] rowsum(dO * O)
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
