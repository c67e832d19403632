// Device-side planner: the column lists of both passes rebuilt on the GPU for
// a new sparse graph over the plan's layout (spattn_plan_set_graph_device).
//
// Dynamic graphs (VSA-style block selection, which the KPage abstract names
// among its layouts) change every call, and host planning of one graph of
// the 21x45x80 layout takes about a second.  Here only what depends on the
// graph is rebuilt, on the device:
//   * the owned tiles are the slot-order tiles of the layout (strided owned
//     pages included), computed once on the host: for each tile and group
//     split, a work item template (owned pages, row codes, the up-to-eight
//     groups of its segments, the owned rows of each segment);
//   * per (unit, template) one CTA gathers, for each segment group, the
//     pages of every column group the graph lists for it (the column side's
//     group -> page table), with the group's row mask on that page; sorts
//     them by (head offset, page) in shared memory; merges them into one
//     entry per (head offset, page) (eight 16-bit segment masks); and
//     compacts runs of pages whose attended rows share a 4-row group into
//     strided entries, exactly as the host planner does.  A unit is a graph
//     head in the query-owned pass and a (graph batch, K/V head) in the
//     key-owned pass, whose columns come from every query head of its group
//     (grouped-query attention; the entries carry the head offset);
//   * the key-owned pass walks the transposed graph (key group -> query
//     groups), built on the device with a counting sort;
//   * two passes (count, then fill) with a device prefix sum place the lists.
// Useful pairs are summed from the lists themselves: every allowed pair is
// computed by exactly one owned row, so sum over entries and segments of
// (owned rows of the segment) x (attended columns) is the useful count.
#include <algorithm>
#include <vector>

#include "kernels.cuh"
#include "plan.hpp"

namespace spattn {

constexpr int kListCap = 8192;      // gathered (page, segment) pairs per work item
constexpr int kListThreads = 256;

namespace {

enum : int { kDpOk = 0, kDpBadGraph = 1, kDpOverflow = 2 };

__device__ __forceinline__ int dp_sub_group(uint32_t m) {
  for (int k = 0; k < 4; ++k)
    if (m != 0u && (m & ~(0xFu << (4 * k))) == 0u) return k;
  return -1;
}

__device__ __forceinline__ uint32_t dp_fold(uint64_t lo, uint64_t hi) {
  const uint64_t m = lo | hi;
  return static_cast<uint32_t>((m | (m >> 16) | (m >> 32) | (m >> 48)) & 0xFFFFu);
}

// Row bounds of CSR row r, clamped to [0, nnz]; a bad row raises the flag.
__device__ __forceinline__ void dp_row(const int64_t* ptr, int64_t r, int64_t nnz, int64_t& a, int64_t& b, int* flag) {
  a = ptr[r];
  b = ptr[r + 1];
  if (a < 0 || b < a || b > nnz) {
    atomicCAS(flag, kDpOk, kDpBadGraph);
    a = b = 0;
  }
}

__global__ void dp_validate(const int64_t* __restrict__ ptr, const int32_t* __restrict__ dst, int64_t rows, int64_t nnz,
                            int32_t n_dst, int* flag) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t0 == 0 && (ptr[0] != 0 || ptr[rows] != nnz)) atomicCAS(flag, kDpOk, kDpBadGraph);
  for (int64_t r = t0; r < rows; r += stride)
    if (ptr[r + 1] < ptr[r]) atomicCAS(flag, kDpOk, kDpBadGraph);
  for (int64_t e = t0; e < nnz; e += stride)
    if (dst[e] < 0 || dst[e] >= n_dst) atomicCAS(flag, kDpOk, kDpBadGraph);
}

// Transposed graph, step 1: entries per (head, key group) (shifted by one for
// the exclusive scan).
__global__ void dp_t_count(const int64_t* __restrict__ ptr, const int32_t* __restrict__ dst, int32_t heads, int32_t n_q,
                           int32_t n_k, int64_t nnz, int64_t* __restrict__ cnt, int* flag) {
  const int64_t rows = static_cast<int64_t>(heads) * n_q;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; r < rows;
       r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t h = r / n_q;
    int64_t a, b;
    dp_row(ptr, r, nnz, a, b, flag);
    for (int64_t e = a; e < b; ++e) {
      const int32_t g = dst[e];
      if (g < 0 || g >= n_k) continue;
      atomicAdd(reinterpret_cast<unsigned long long*>(cnt + h * n_k + g + 1), 1ull);
    }
  }
}

// Transposed graph, step 2: scatter query groups into their key groups' rows.
// The order inside a row is arbitrary; the list builder sorts what it
// gathers, so the lists do not depend on it.
__global__ void dp_t_scatter(const int64_t* __restrict__ ptr, const int32_t* __restrict__ dst, int32_t heads,
                             int32_t n_q, int32_t n_k, int64_t nnz, const int64_t* __restrict__ tptr,
                             int64_t* __restrict__ cursor, int32_t* __restrict__ tdst, int* flag) {
  const int64_t rows = static_cast<int64_t>(heads) * n_q;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; r < rows;
       r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t h = r / n_q;
    const int32_t qa = static_cast<int32_t>(r % n_q);
    int64_t a, b;
    dp_row(ptr, r, nnz, a, b, flag);
    for (int64_t e = a; e < b; ++e) {
      const int32_t g = dst[e];
      if (g < 0 || g >= n_k) continue;
      const int64_t row = h * n_k + g;
      const int64_t pos = static_cast<int64_t>(atomicAdd(reinterpret_cast<unsigned long long*>(cursor + row), 1ull));
      tdst[tptr[row] + pos] = qa;
    }
  }
}

// In-place inclusive scan of n int64 values with one CTA of 1024 threads
// (chunked; the lists have at most a few million rows).
__global__ void __launch_bounds__(1024) dp_scan_inclusive(int64_t* __restrict__ v, int64_t n) {
  __shared__ int64_t part[1024];
  __shared__ int64_t carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int64_t per = 1024;
  for (int64_t base = 0; base < n; base += per) {
    const int64_t i = base + threadIdx.x;
    part[threadIdx.x] = i < n ? v[i] : 0;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {
      const int64_t add = threadIdx.x >= off ? part[threadIdx.x - off] : 0;
      __syncthreads();
      part[threadIdx.x] += add;
      __syncthreads();
    }
    if (i < n) v[i] = part[threadIdx.x] + carry;
    __syncthreads();
    if (threadIdx.x == 1023) carry += part[1023];
    __syncthreads();
  }
}

struct ListArgs {
  // templates of this pass
  const int32_t* words;     // n_tmpl x 32
  const int32_t* segs;      // n_tmpl x kMaxSegments (group id or -1)
  const int32_t* seg_rows;  // n_tmpl x kMaxSegments
  int64_t n_tmpl;
  // graph rows of the owned side's groups
  const int64_t* adj_ptr;
  const int32_t* adj_dst;
  int64_t adj_nnz;
  int32_t n_src, n_col_groups;
  // column side
  const int64_t* gp_ptr;
  const int32_t* gp_page;
  const uint16_t* gp_mask;
  int64_t col_slots;
  // units: grid y.  Unit u takes its columns from graph heads src(u, j),
  // j < src_n: u itself in the query-owned pass (a graph head), the query
  // heads of K/V head u % kv_heads of graph batch u / kv_heads in the
  // key-owned pass.  Its items are repeated for `copies` batch entries
  // (one graph for all of them), with work word 0 = copy * owned_heads + u.
  int32_t n_units, src_n, heads, kv_heads, owned_heads, copies;
  bool strided;
  // outputs
  int64_t* counts;          // [n_units * n_tmpl] entries; inclusive-scanned between the passes
  int32_t* out_work;        // [copies * n_units * n_tmpl * 32] (fill pass)
  int32_t* out_pages;
  uint64_t* out_masks;
  uint16_t* out_heads;      // entry head offsets j (key-owned pass under grouped-query attention) or null
  unsigned long long* stats;  // [0] useful pairs (one batch, query pass), [1 + pass] entries
  int pass;                   // 0 = query-owned, 1 = key-owned
  int* flag;
};

// One CTA per (template, unit): the column list of that work item.
template <bool FILL>
__global__ void __launch_bounds__(kListThreads) dp_list(ListArgs a) {
  extern __shared__ uint8_t dp_smem[];
  uint64_t* keys = reinterpret_cast<uint64_t*>(dp_smem);               // [kListCap]
  __shared__ int n_keys;
  const int64_t ti = blockIdx.x;
  const int32_t u = blockIdx.y;
  if (threadIdx.x == 0) n_keys = 0;
  __syncthreads();
  // gather (j << 44 | page << 20 | segment << 16 | row mask of the column
  // group on the page), j the head offset of the source graph head
  for (int j = 0; j < a.src_n; ++j) {
    const int64_t gh = a.pass == 0 ? static_cast<int64_t>(u)
                                   : static_cast<int64_t>(u / a.kv_heads) * a.heads + (u % a.kv_heads) * a.src_n + j;
    for (int s = 0; s < kMaxSegments; ++s) {
      const int32_t g = a.segs[ti * kMaxSegments + s];
      if (g < 0) continue;
      int64_t r0, r1;
      dp_row(a.adj_ptr, gh * a.n_src + g, a.adj_nnz, r0, r1, a.flag);
      for (int64_t e = r0 + threadIdx.x; e < r1; e += blockDim.x) {
        const int32_t b = a.adj_dst[e];
        if (b < 0 || b >= a.n_col_groups) continue;
        for (int64_t x = a.gp_ptr[b]; x < a.gp_ptr[b + 1]; ++x) {
          const int idx = atomicAdd(&n_keys, 1);
          if (idx < kListCap)
            keys[idx] = (static_cast<uint64_t>(j) << 44) | (static_cast<uint64_t>(a.gp_page[x]) << 20) |
                        (static_cast<uint64_t>(s) << 16) | a.gp_mask[x];
        }
      }
    }
  }
  __syncthreads();
  const int n = n_keys;
  if (n > kListCap) {
    if (threadIdx.x == 0) atomicCAS(a.flag, kDpOk, kDpOverflow);
    return;
  }
  // bitonic sort of the next power of two, padded with the largest key
  int np2 = 1;
  while (np2 < n) np2 <<= 1;
  for (int i = n + threadIdx.x; i < np2; i += blockDim.x) keys[i] = ~0ull;
  __syncthreads();
  for (int k = 2; k <= np2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < np2; i += blockDim.x) {
        const int l = i ^ j;
        if (l > i) {
          const uint64_t x = keys[i], y = keys[l];
          const bool up = (i & k) == 0;
          if ((x > y) == up) {
            keys[i] = y;
            keys[l] = x;
          }
        }
      }
      __syncthreads();
    }
  }
  if (threadIdx.x != 0) return;
  // Merge (one entry per (head offset, page), eight 16-bit segment masks in
  // two words) and strided compaction (the host planner's rule) in one pass
  // over the sorted keys.  The rule looks at the entries of pages p .. p+3 of
  // one head offset only, so a window of the next four merged entries
  // suffices.
  const int64_t slot = static_cast<int64_t>(u) * a.n_tmpl + ti;
  const int64_t off = FILL ? (slot == 0 ? 0 : a.counts[slot - 1]) : 0;
  int64_t cnt = 0;
  unsigned long long useful = 0;
  const int32_t* sr = a.seg_rows + ti * kMaxSegments;
  auto emit = [&](int32_t ref, int32_t j, uint64_t lo, uint64_t hi) {
    if (FILL) {
      a.out_pages[off + cnt] = ref;
      a.out_masks[2 * (off + cnt)] = lo;
      a.out_masks[2 * (off + cnt) + 1] = hi;
      if (a.out_heads) a.out_heads[off + cnt] = static_cast<uint16_t>(j);
    } else {
      for (int s = 0; s < kMaxSegments; ++s)
        useful += static_cast<unsigned long long>(sr[s]) * __popcll(((s < 4 ? lo : hi) >> (16 * (s & 3))) & 0xFFFFull);
    }
    ++cnt;
  };
  int64_t wp[4];  // (head offset << 24) | page
  uint64_t wlo[4], whi[4];
  int wn = 0, ki = 0;
  auto refill = [&]() {
    while (wn < 4 && ki < n) {
      const int64_t p = static_cast<int64_t>(keys[ki] >> 20);
      uint64_t mk[2] = {0, 0};
      for (; ki < n && static_cast<int64_t>(keys[ki] >> 20) == p; ++ki) {
        const int sg = static_cast<int>((keys[ki] >> 16) & 0xF);
        mk[sg >> 2] |= static_cast<uint64_t>(keys[ki] & 0xFFFFu) << (16 * (sg & 3));
      }
      wp[wn] = p;
      wlo[wn] = mk[0];
      whi[wn] = mk[1];
      ++wn;
    }
  };
  refill();
  while (wn > 0) {
    const int64_t jp = wp[0];
    const int32_t p = static_cast<int32_t>(jp & 0xFFFFFF), jh = static_cast<int32_t>(jp >> 24);
    const int k = a.strided ? dp_sub_group(dp_fold(wlo[0], whi[0])) : -1;
    int used = 1;
    if (k >= 0 && 16 * (static_cast<int64_t>(p) + 3) + 4 * k + 4 <= a.col_slots) {
      int j = 0;
      bool same = true;
      while (j < wn && wp[j] <= jp + 3) {  // p + 3 stays below 2^24: the same head offset
        if (dp_sub_group(dp_fold(wlo[j], whi[j])) != k) {
          same = false;
          break;
        }
        ++j;
      }
      if (same && j >= 2) {
        uint64_t mk[2] = {0, 0};
        for (int x = 0; x < j; ++x) {
          const int jj = static_cast<int>(wp[x] - jp);
          for (int sg = 0; sg < kMaxSegments; ++sg)
            mk[sg >> 2] |= (((sg < 4 ? wlo[x] : whi[x]) >> (16 * (sg & 3) + 4 * k)) & 0xFull)
                           << (16 * (sg & 3) + 4 * jj);
        }
        emit(~static_cast<int32_t>(16 * p + 4 * k), jh, mk[0], mk[1]);
        used = j;
      }
    }
    if (used == 1) emit(p, jh, wlo[0], whi[0]);
    for (int x = used; x < wn; ++x) {
      wp[x - used] = wp[x];
      wlo[x - used] = wlo[x];
      whi[x - used] = whi[x];
    }
    wn -= used;
    refill();
  }
  if (!FILL) {
    a.counts[slot] = cnt;
    if (a.pass == 0) atomicAdd(&a.stats[0], useful);
    atomicAdd(&a.stats[1 + a.pass], static_cast<unsigned long long>(cnt));
  } else {
    const int32_t* tw = a.words + ti * 32;
    for (int32_t b = 0; b < a.copies; ++b) {
      int32_t* w = a.out_work + ((static_cast<int64_t>(b) * a.n_units + u) * a.n_tmpl + ti) * 32;
      for (int x = 0; x < 32; ++x) w[x] = tw[x];
      w[0] = b * a.owned_heads + u;
      w[2] = static_cast<int32_t>(off);
      w[3] = static_cast<int32_t>(off + cnt);
    }
  }
}

template <typename T>
cudaError_t ensure(T** p, int64_t& cap, int64_t need) {
  if (*p && cap >= need) return cudaSuccess;
  cudaFree(*p);
  *p = nullptr;
  cap = 0;
  const int64_t n = std::max<int64_t>(need, 1);
  cudaError_t e = cudaMalloc(reinterpret_cast<void**>(p), static_cast<size_t>(n) * sizeof(T));
  if (e == cudaSuccess) cap = n;
  return e;
}

template <typename T>
cudaError_t upload_vec(T** p, const std::vector<T>& v) {
  cudaFree(*p);
  *p = nullptr;
  const size_t n = std::max<size_t>(v.size(), 1) * sizeof(T);
  cudaError_t e = cudaMalloc(reinterpret_cast<void**>(p), n);
  if (e == cudaSuccess && !v.empty()) e = cudaMemcpy(*p, v.data(), v.size() * sizeof(T), cudaMemcpyHostToDevice);
  return e;
}

}  // namespace

void free_device_planner(DevPlanner& d) {
  for (PassTemplates* t : {&d.tq, &d.tk}) {
    cudaFree(t->d_words);
    cudaFree(t->d_segs);
    cudaFree(t->d_seg_rows);
    t->d_words = t->d_segs = t->d_seg_rows = nullptr;
  }
  cudaFree(d.d_q_gp_ptr);
  cudaFree(d.d_q_gp_page);
  cudaFree(d.d_q_gp_mask);
  cudaFree(d.d_k_gp_ptr);
  cudaFree(d.d_k_gp_page);
  cudaFree(d.d_k_gp_mask);
  cudaFree(d.d_fwd_ptr);
  cudaFree(d.d_fwd_dst);
  cudaFree(d.d_bwd_ptr);
  cudaFree(d.d_bwd_dst);
  cudaFree(d.d_cursor);
  cudaFree(d.d_counts);
  cudaFree(d.d_stats);
  d = DevPlanner();
}

int device_replan(spattn_plan_s* P, const int64_t* row_ptr, const int32_t* kv_groups, int64_t nnz, cudaStream_t st) {
  DevPlanner& d = P->dp;
  const int32_t H = P->heads, nq = P->q.n_groups, nk = P->k.n_groups;
  const int32_t kvh = P->kv_heads, grp = H / kvh, gb = P->graph_batches, copies = P->batch / gb;
  const int32_t GH = gb * H;                   // graph heads (query-owned units)
  const int32_t units[2] = {GH, gb * kvh};     // units of the query- and key-owned passes
  const int64_t rows_f = static_cast<int64_t>(GH) * nq, rows_b = static_cast<int64_t>(GH) * nk;
  // keys hold a page in 24 bits
  if (P->q.n_pages >= (int64_t(1) << 24) || P->k.n_pages >= (int64_t(1) << 24)) return SPATTN_ERR_UNSUPPORTED;
  cudaError_t e = cudaSuccess;
  auto ck = [&](cudaError_t x) {
    if (e == cudaSuccess) e = x;
  };
  if (!d.ready) {
    ck(upload_vec(&d.tq.d_words, d.tq.words));
    ck(upload_vec(&d.tq.d_segs, d.tq.segs));
    ck(upload_vec(&d.tq.d_seg_rows, d.tq.seg_rows));
    ck(upload_vec(&d.tk.d_words, d.tk.words));
    ck(upload_vec(&d.tk.d_segs, d.tk.segs));
    ck(upload_vec(&d.tk.d_seg_rows, d.tk.seg_rows));
    ck(upload_vec(&d.d_q_gp_ptr, P->q.gp_ptr));
    ck(upload_vec(&d.d_q_gp_page, P->q.gp_page));
    ck(upload_vec(&d.d_q_gp_mask, P->q.gp_mask));
    ck(upload_vec(&d.d_k_gp_ptr, P->k.gp_ptr));
    ck(upload_vec(&d.d_k_gp_page, P->k.gp_page));
    ck(upload_vec(&d.d_k_gp_mask, P->k.gp_mask));
    ck(cudaMalloc(reinterpret_cast<void**>(&d.d_bwd_ptr), (rows_b + 1) * sizeof(int64_t)));
    ck(cudaMalloc(reinterpret_cast<void**>(&d.d_cursor), std::max<int64_t>(rows_b, 1) * sizeof(int64_t)));
    ck(cudaMalloc(reinterpret_cast<void**>(&d.d_fwd_ptr), (rows_f + 1) * sizeof(int64_t)));
    ck(cudaMalloc(reinterpret_cast<void**>(&d.d_stats), 4 * sizeof(unsigned long long) + sizeof(int)));
    const int64_t nc = std::max<int64_t>(static_cast<int64_t>(units[0]) * d.tq.n + static_cast<int64_t>(units[1]) * d.tk.n, 1);
    ck(cudaMalloc(reinterpret_cast<void**>(&d.d_counts), nc * sizeof(int64_t)));
    if (e != cudaSuccess) return SPATTN_ERR_OOM;
    cudaFuncSetAttribute(dp_list<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kListCap * 8);
    cudaFuncSetAttribute(dp_list<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kListCap * 8);
    d.ready = true;
  }
  // the plan keeps its own copy of the graph (inspection calls read it later)
  if (ensure(&d.d_fwd_dst, d.fwd_cap, nnz) != cudaSuccess) return SPATTN_ERR_OOM;
  if (ensure(&d.d_bwd_dst, d.bwd_cap, nnz) != cudaSuccess) return SPATTN_ERR_OOM;
  ck(cudaMemcpyAsync(d.d_fwd_ptr, row_ptr, (rows_f + 1) * sizeof(int64_t), cudaMemcpyDeviceToDevice, st));
  if (nnz > 0) ck(cudaMemcpyAsync(d.d_fwd_dst, kv_groups, nnz * sizeof(int32_t), cudaMemcpyDeviceToDevice, st));
  unsigned long long* stats = d.d_stats;  // [0] useful, [1] entries q, [2] entries k, [3] unused
  int* flag = reinterpret_cast<int*>(stats + 4);
  ck(cudaMemsetAsync(stats, 0, 4 * sizeof(unsigned long long) + sizeof(int), st));
  ck(cudaMemsetAsync(d.d_bwd_ptr, 0, (rows_b + 1) * sizeof(int64_t), st));
  ck(cudaMemsetAsync(d.d_cursor, 0, std::max<int64_t>(rows_b, 1) * sizeof(int64_t), st));
  if (e != cudaSuccess) return SPATTN_ERR_CUDA;
  const unsigned g1 = static_cast<unsigned>(std::min<int64_t>((std::max(rows_f, nnz) + 255) / 256, 148 * 8));
  dp_validate<<<g1, 256, 0, st>>>(d.d_fwd_ptr, d.d_fwd_dst, rows_f, nnz, nk, flag);
  dp_t_count<<<g1, 256, 0, st>>>(d.d_fwd_ptr, d.d_fwd_dst, GH, nq, nk, nnz, d.d_bwd_ptr, flag);
  dp_scan_inclusive<<<1, 1024, 0, st>>>(d.d_bwd_ptr + 1, rows_b);
  dp_t_scatter<<<g1, 256, 0, st>>>(d.d_fwd_ptr, d.d_fwd_dst, GH, nq, nk, nnz, d.d_bwd_ptr, d.d_cursor, d.d_bwd_dst, flag);
  const bool strided = strided_setting();
  auto args = [&](bool qpass) {
    ListArgs a;
    const PassTemplates& t = qpass ? d.tq : d.tk;
    a.words = t.d_words;
    a.segs = t.d_segs;
    a.seg_rows = t.d_seg_rows;
    a.n_tmpl = t.n;
    a.adj_ptr = qpass ? d.d_fwd_ptr : d.d_bwd_ptr;
    a.adj_dst = qpass ? d.d_fwd_dst : d.d_bwd_dst;
    a.adj_nnz = nnz;
    a.n_src = qpass ? nq : nk;
    a.n_col_groups = qpass ? nk : nq;
    a.gp_ptr = qpass ? d.d_k_gp_ptr : d.d_q_gp_ptr;
    a.gp_page = qpass ? d.d_k_gp_page : d.d_q_gp_page;
    a.gp_mask = qpass ? d.d_k_gp_mask : d.d_q_gp_mask;
    a.col_slots = qpass ? P->k.slots : P->q.slots;
    a.n_units = units[qpass ? 0 : 1];
    a.src_n = qpass ? 1 : grp;
    a.heads = H;
    a.kv_heads = kvh;
    a.owned_heads = qpass ? H : kvh;
    a.copies = copies;
    a.out_heads = nullptr;
    a.strided = strided;
    a.counts = d.d_counts;
    a.stats = stats;
    a.flag = flag;
    return a;
  };
  const size_t smem = kListCap * 8;
  ListArgs la[2] = {args(true), args(false)};
  const PassTemplates* tt[2] = {&d.tq, &d.tk};
  WorkList* wls[2] = {&P->wq, &P->wk};
  // count both passes, then check everything at one synchronisation before
  // any list of the plan is touched (a rejected graph leaves the plan as it was)
  for (int pass = 0; pass < 2; ++pass) {
    la[pass].pass = pass;
    la[pass].counts = d.d_counts + (pass == 0 ? 0 : static_cast<int64_t>(units[0]) * d.tq.n);
    if (tt[pass]->n > 0 && units[pass] > 0) {
      dp_list<false><<<dim3(static_cast<unsigned>(tt[pass]->n), static_cast<unsigned>(units[pass])), kListThreads, smem,
                       st>>>(la[pass]);
      dp_scan_inclusive<<<1, 1024, 0, st>>>(la[pass].counts, static_cast<int64_t>(units[pass]) * tt[pass]->n);
    }
  }
  if (cudaGetLastError() != cudaSuccess) return SPATTN_ERR_CUDA;
  unsigned long long hs[4];
  int hflag = 0;
  if (cudaMemcpyAsync(hs, stats, sizeof(hs), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyAsync(&hflag, flag, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return SPATTN_ERR_CUDA;
  if (hflag == kDpBadGraph) return SPATTN_ERR_INVALID_ARG;
  if (hflag == kDpOverflow) return SPATTN_ERR_UNSUPPORTED;
  const int64_t useful = static_cast<int64_t>(hs[0]) * copies;
  for (int pass = 0; pass < 2; ++pass) {
    const int64_t total = static_cast<int64_t>(hs[1 + pass]);
    if (total > static_cast<int64_t>(INT32_MAX)) return SPATTN_ERR_UNSUPPORTED;
    WorkList& wl = *wls[pass];
    const int64_t n_work = static_cast<int64_t>(copies) * units[pass] * tt[pass]->n;
    if (ensure(&wl.d_work, wl.cap_work, n_work * kWorkWords) != cudaSuccess ||
        ensure(&wl.d_pages, wl.cap_pages, total) != cudaSuccess ||
        ensure(&wl.d_masks, wl.cap_masks, total * kMaskWords) != cudaSuccess)
      return SPATTN_ERR_OOM;
    la[pass].out_work = wl.d_work;
    la[pass].out_pages = wl.d_pages;
    la[pass].out_masks = wl.d_masks;
    // head offsets of the key-owned entries under grouped-query attention
    if (pass == 1 && grp > 1) {
      if (ensure(&wl.d_heads, wl.cap_heads, total) != cudaSuccess) return SPATTN_ERR_OOM;
      la[pass].out_heads = wl.d_heads;
    }
    if (tt[pass]->n > 0 && units[pass] > 0)
      dp_list<true><<<dim3(static_cast<unsigned>(tt[pass]->n), static_cast<unsigned>(units[pass])), kListThreads, smem,
                      st>>>(la[pass]);
    if (cudaGetLastError() != cudaSuccess) return SPATTN_ERR_CUDA;
    wl.n_work = n_work;
    wl.route64 = false;  // the templates are 128-row items
    wl.n_entries_dev = total;
    wl.physical_pairs = static_cast<int64_t>(kTilePages * kPageRows) * kPageRows * total * copies;
  }
  P->useful_pairs = useful;
  P->bsa_pairs = -1;
  P->host_stale = true;
  P->graph_nnz = nnz;
  return SPATTN_OK;
}

}  // namespace spattn
