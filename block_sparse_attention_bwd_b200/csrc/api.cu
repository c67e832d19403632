// C ABI of libspattn (declared in include/spattn.h): argument checks, tensor
// maps, and the launch sequence of each pass.  No allocation happens here
// except in spattn_plan (the plan's device lists and workspace).
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>
#include <new>

#include "kernels.cuh"
#include "plan.hpp"

namespace spattn {
int build_plan(const spattn_layout* L, const spattn_graph* G, spattn_plan_s* P);
void free_plan_device(spattn_plan_s* P);
void canonical_pages(const spattn_plan_s& P, int32_t h, int64_t qb, std::vector<int32_t>& out);
void transposed_qblocks(const spattn_plan_s& P, int32_t h, int64_t page, std::vector<int32_t>& out);
int64_t bsa_pairs(const spattn_plan_s& P);
int refresh_host(spattn_plan_s* P);
int device_replan(spattn_plan_s* P, const int64_t* row_ptr, const int32_t* kv_groups, int64_t nnz, cudaStream_t st);

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Element types of the mapped tensors: bf16, or one-byte E4M3 codes (moved
// as bytes).  Every box row is 128 bytes (64 bf16 or 128 codes), the width of
// the 128-byte swizzle the MMA descriptors expect.
CUtensorMapDataType map_type(int eb) { return eb == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16; }

// [rows_per_bh, head_dim] matrices stacked over batch*heads; boxes of
// `box_rows` rows x one 128-byte chunk, 128-byte swizzle.  Rows past the end
// of a (batch, head) read as zeros.
bool make_map(CUtensorMap* m, const void* ptr, int head_dim, int64_t rows, int64_t bh, int box_rows, int eb = 2) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(bh)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * eb, static_cast<cuuint64_t>(head_dim) * eb * rows};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / eb), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, map_type(eb), 3, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4D view (64 columns, rows, head_dim / 64 chunks, bh): one 64-row box holds
// every chunk of those rows, chunk after chunk.  The chunk stride (128 B) is
// below the row stride; a tiled map only needs each stride to be a multiple
// of 16 bytes.
bool make_wide_map(CUtensorMap* m, const void* ptr, int head_dim, int64_t rows, int64_t bh, int box_rows,
                   int eb = 2) {
  auto fn = encode_fn();
  if (!fn) return false;
  const int nch = head_dim * eb / 128;
  const cuuint64_t row_bytes = static_cast<cuuint64_t>(head_dim) * eb;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(128 / eb), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(nch),
                        static_cast<cuuint64_t>(bh)};
  cuuint64_t strides[3] = {row_bytes, 128, row_bytes * rows};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / eb), static_cast<cuuint32_t>(box_rows), static_cast<cuuint32_t>(nch), 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, map_type(eb), 4, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 5D view of strided pages: (64 columns, 4 rows, 4 groups 16 rows apart,
// slot, batch*head).  The row and group dimensions overlap the slot
// dimension; every box the kernels request lies inside one (batch, head),
// because the planner only forms a strided page when all 16 of its slots
// exist.
bool make_strided_map(CUtensorMap* m, const void* ptr, int head_dim, int64_t rows, int64_t bh, int eb = 2) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t row_bytes = static_cast<cuuint64_t>(head_dim) * eb;
  cuuint64_t dims[5] = {static_cast<cuuint64_t>(head_dim), 4, 4, static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(bh)};
  cuuint64_t strides[4] = {row_bytes, 16 * row_bytes, row_bytes, row_bytes * static_cast<cuuint64_t>(rows)};
  cuuint32_t box[5] = {static_cast<cuuint32_t>(128 / eb), 4, 4, 1, 1};
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return fn(m, map_type(eb), 5, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_pages(TmaPages* t, const void* ptr, int head_dim, int64_t rows, int64_t bh, int eb = 2) {
  if (!make_strided_map(&t->m4s, ptr, head_dim, rows, bh, eb)) return false;
  if (!make_map(&t->m16, ptr, head_dim, rows, bh, 16, eb) || !make_map(&t->m32, ptr, head_dim, rows, bh, 32, eb) ||
      !make_map(&t->m64, ptr, head_dim, rows, bh, 64, eb))
    return false;
  if (!make_wide_map(&t->m128w, ptr, head_dim, rows, bh, 128, eb)) return false;
  if (head_dim * eb == 128) {  // one chunk per row
    t->m64w = t->m64;
    return true;
  }
  return make_wide_map(&t->m64w, ptr, head_dim, rows, bh, 64, eb);
}

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_plan_device(const spattn_plan_s* P) {
  if (P->device < 0) return SPATTN_ERR_CUDA;  // host-only plan (no device when it was built)
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SPATTN_ERR_CUDA;
  return dev == P->device ? SPATTN_OK : SPATTN_ERR_INVALID_ARG;
}

// Launch helper: runs `launch` and, while profiling, brackets it with events.
template <typename F>
cudaError_t timed(spattn_plan_s* P, int kernel, cudaStream_t s, F&& launch) {
  if (!P->profiling) return launch();
  if (P->n_events == P->events.size()) {
    spattn_plan_s::EventRec r{kernel, nullptr, nullptr};
    if (cudaEventCreate(&r.start) != cudaSuccess || cudaEventCreate(&r.stop) != cudaSuccess) return cudaErrorMemoryAllocation;
    P->events.push_back(r);
  }
  auto& r = P->events[P->n_events++];
  r.kernel = kernel;
  cudaError_t e = cudaEventRecord(r.start, s);
  if (e == cudaSuccess) e = launch();
  if (e == cudaSuccess) e = cudaEventRecord(r.stop, s);
  return e;
}

int64_t fill_launches(const std::vector<int32_t>& fill) { return fill.empty() ? 0 : 1; }

TileArgs tile_args(const spattn_plan_s* P, const WorkList& w, int64_t own_slots, int64_t col_slots) {
  TileArgs a;
  a.work = w.d_work;
  a.pages = w.d_pages;
  a.masks = w.d_masks;
  a.n_work = w.n_work;
  a.own_slots = own_slots;
  a.col_slots = col_slots;
  a.scale = P->scale;
  a.err = P->d_err;
  a.sched = P->d_sched;
  a.heads = P->heads;
  a.kv_heads = P->kv_heads;
  a.kv_group = P->heads / P->kv_heads;
  // entry head offsets exist only under grouped-query attention (else all 0)
  a.col_heads = P->kv_heads == P->heads ? nullptr : w.d_heads;
  a.route64 = w.route64;
  return a;
}

}  // namespace

// Entry points for other translation units of the library.
bool make_tensor_pages(TmaPages* t, const void* ptr, int head_dim, int64_t rows, int64_t bh) {
  return make_pages(t, ptr, head_dim, rows, bh);
}
TileArgs make_tile_args(const spattn_plan_s* P, const WorkList& w, int64_t own_slots, int64_t col_slots) {
  return tile_args(P, w, own_slots, col_slots);
}

}  // namespace spattn

using namespace spattn;

extern "C" {

int spattn_plan(const spattn_layout* layout, const spattn_graph* graph, spattn_plan_t* out) {
  if (!out) return SPATTN_ERR_INVALID_ARG;
  *out = nullptr;
  spattn_plan_s* P = nullptr;
  try {
    P = new spattn_plan_s();
    const int st = build_plan(layout, graph, P);
    if (st != SPATTN_OK) {
      free_plan_device(P);
      delete P;
      return st;
    }
  } catch (const std::bad_alloc&) {
    if (P) {
      free_plan_device(P);
      delete P;
    }
    return SPATTN_ERR_OOM;
  } catch (...) {
    // any other exception (e.g. std::system_error from the host runtime)
    if (P) {
      free_plan_device(P);
      delete P;
    }
    return SPATTN_ERR_OOM;
  }
  *out = P;
  return SPATTN_OK;
}

int spattn_fwd(const void* q, const void* k, const void* v, spattn_plan_t plan, void* o, float* lse, void* stream) {
  if (!plan) return SPATTN_ERR_INVALID_ARG;
  int st = check_plan_device(plan);
  if (st) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return SPATTN_ERR_INVALID_ARG;
  const int D = plan->head_dim;
  const int64_t bh = static_cast<int64_t>(plan->batch) * plan->heads;
  const int64_t bh_kv = static_cast<int64_t>(plan->batch) * plan->kv_heads;
  TmaPages tq, tk, tv;
  if (!make_pages(&tq, q, D, plan->q.slots, bh) || !make_pages(&tk, k, D, plan->k.slots, bh_kv) ||
      !make_pages(&tv, v, D, plan->k.slots, bh_kv))
    return SPATTN_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto* O = static_cast<__nv_bfloat16*>(o);
  cudaError_t e = timed(plan, SPATTN_K_FWD, s, [&] {
    return launch_fwd(D, tq, tk, tv, tile_args(plan, plan->wq, plan->q.slots, plan->k.slots), O, lse, s);
  });
  if (e == cudaSuccess && !plan->q_fill.empty())
    e = timed(plan, SPATTN_K_FILL, s, [&] {
      return launch_fill(D, plan->d_q_fill, static_cast<int64_t>(plan->q_fill.size() / 2), bh, plan->q.slots, O,
                         nullptr, lse, s);
    });
  return e == cudaSuccess ? SPATTN_OK : SPATTN_ERR_CUDA;
}

int spattn_quantize_fp8(const void* x, int64_t bh, int64_t rows, int head_dim, void* x8, float* descale,
                        void* stream) {
  if (bh < 0 || rows < 0 || (head_dim != 64 && head_dim != 128)) return SPATTN_ERR_INVALID_ARG;
  if (bh == 0) return SPATTN_OK;
  if (!aligned16(x) || !aligned16(x8) || !descale || (reinterpret_cast<uintptr_t>(descale) & 3u))
    return SPATTN_ERR_INVALID_ARG;
  const cudaError_t e = launch_quantize_e4m3(static_cast<const __nv_bfloat16*>(x), bh, rows * head_dim,
                                             static_cast<uint8_t*>(x8), descale, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SPATTN_OK : SPATTN_ERR_CUDA;
}

int spattn_fwd_fp8(const void* q8, const void* k8, const float* q_descale, const float* k_descale, const void* v,
                   spattn_plan_t plan, void* o, float* lse, void* stream) {
  if (!plan) return SPATTN_ERR_INVALID_ARG;
  int st = check_plan_device(plan);
  if (st) return st;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !q_descale ||
      !k_descale || (reinterpret_cast<uintptr_t>(q_descale) & 3u) || (reinterpret_cast<uintptr_t>(k_descale) & 3u))
    return SPATTN_ERR_INVALID_ARG;
  const int D = plan->head_dim;
  if (D != 128) return SPATTN_ERR_UNSUPPORTED;
  const int64_t bh = static_cast<int64_t>(plan->batch) * plan->heads;
  const int64_t bh_kv = static_cast<int64_t>(plan->batch) * plan->kv_heads;
  TmaPages tq, tk, tv;
  if (!make_pages(&tq, q8, D, plan->q.slots, bh, 1) || !make_pages(&tk, k8, D, plan->k.slots, bh_kv, 1) ||
      !make_pages(&tv, v, D, plan->k.slots, bh_kv))
    return SPATTN_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto* O = static_cast<__nv_bfloat16*>(o);
  cudaError_t e = timed(plan, SPATTN_K_FWD, s, [&] {
    return launch_fwd_e4m3(tq, tk, tv, tile_args(plan, plan->wq, plan->q.slots, plan->k.slots), q_descale, k_descale,
                           O, lse, s);
  });
  if (e == cudaSuccess && !plan->q_fill.empty())
    e = timed(plan, SPATTN_K_FILL, s, [&] {
      return launch_fill(D, plan->d_q_fill, static_cast<int64_t>(plan->q_fill.size() / 2), bh, plan->q.slots, O,
                         nullptr, lse, s);
    });
  return e == cudaSuccess ? SPATTN_OK : SPATTN_ERR_CUDA;
}

int spattn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* d_o,
               spattn_plan_t plan, void* dq, void* dk, void* dv, void* stream) {
  if (!plan) return SPATTN_ERR_INVALID_ARG;
  int st = check_plan_device(plan);
  if (st) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(d_o) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return SPATTN_ERR_INVALID_ARG;
  const int D = plan->head_dim;
  const int64_t bh = static_cast<int64_t>(plan->batch) * plan->heads;
  const int64_t bh_kv = static_cast<int64_t>(plan->batch) * plan->kv_heads;
  TmaPages tq, tk, tv, tdo;
  if (!make_pages(&tq, q, D, plan->q.slots, bh) || !make_pages(&tk, k, D, plan->k.slots, bh_kv) ||
      !make_pages(&tv, v, D, plan->k.slots, bh_kv) || !make_pages(&tdo, d_o, D, plan->q.slots, bh))
    return SPATTN_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto* dQ = static_cast<__nv_bfloat16*>(dq);
  auto* dK = static_cast<__nv_bfloat16*>(dk);
  auto* dV = static_cast<__nv_bfloat16*>(dv);
  cudaError_t e = timed(plan, SPATTN_K_DELTA, s, [&] {
    return launch_delta(D, static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(d_o), plan->d_delta,
                        bh * plan->q.slots, s);
  });
  if (e == cudaSuccess)
    e = timed(plan, SPATTN_K_DKDV, s, [&] {
      return launch_dkdv(D, tk, tv, tq, tdo, tile_args(plan, plan->wk, plan->k.slots, plan->q.slots), lse,
                         plan->d_delta, dK, dV, s);
    });
  if (e == cudaSuccess)
    e = timed(plan, SPATTN_K_DQ, s, [&] {
      return launch_dq(D, static_cast<const __nv_bfloat16*>(q), tdo, tk, tv, tile_args(plan, plan->wq, plan->q.slots, plan->k.slots), lse,
                       plan->d_delta, dQ, s);
    });
  if (e == cudaSuccess && !plan->k_fill.empty())
    e = timed(plan, SPATTN_K_FILL, s, [&] {
      return launch_fill(D, plan->d_k_fill, static_cast<int64_t>(plan->k_fill.size() / 2), bh_kv, plan->k.slots, dK,
                         dV, nullptr, s);
    });
  if (e == cudaSuccess && !plan->q_fill.empty())
    e = timed(plan, SPATTN_K_FILL, s, [&] {
      return launch_fill(D, plan->d_q_fill, static_cast<int64_t>(plan->q_fill.size() / 2), bh, plan->q.slots, dQ,
                         nullptr, nullptr, s);
    });
  return e == cudaSuccess ? SPATTN_OK : SPATTN_ERR_CUDA;
}

int spattn_wait_selftest(spattn_plan_t plan, int64_t deadline_cycles, void* stream) {
  if (!plan) return SPATTN_ERR_INVALID_ARG;
  if (deadline_cycles < 10000 || deadline_cycles > 2000000000ll) return SPATTN_ERR_INVALID_ARG;
  const int st = check_plan_device(plan);
  if (st) return st;
  return launch_wait_selftest(plan->d_err, deadline_cycles, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SPATTN_OK
             : SPATTN_ERR_CUDA;
}

int spattn_check(spattn_plan_t plan, void* stream) {
  if (!plan) return SPATTN_ERR_INVALID_ARG;
  if (plan->device < 0) return SPATTN_ERR_CUDA;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SPATTN_ERR_CUDA;
  int h = 0;
  if (cudaMemcpy(&h, plan->d_err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SPATTN_ERR_CUDA;
  if (h == 0) return SPATTN_OK;
  if (cudaMemset(plan->d_err, 0, sizeof(int)) != cudaSuccess) return SPATTN_ERR_CUDA;
  return h == 1 ? SPATTN_ERR_TIMEOUT : SPATTN_ERR_DEVICE;
}

int spattn_plan_set_graph_device(spattn_plan_t plan, const int64_t* row_ptr, const int32_t* kv_groups, int64_t nnz,
                                 void* stream) {
  if (!plan || !row_ptr || nnz < 0 || (nnz > 0 && !kv_groups)) return SPATTN_ERR_INVALID_ARG;
  const int st = check_plan_device(plan);
  if (st) return st;
  try {
    return device_replan(plan, row_ptr, kv_groups, nnz, static_cast<cudaStream_t>(stream));
  } catch (...) {
    return SPATTN_ERR_OOM;
  }
}

int spattn_plan_stats(spattn_plan_t plan, spattn_stats* s) {
  if (!plan || !s) return SPATTN_ERR_INVALID_ARG;
  {
    const int st = refresh_host(plan);
    if (st) return st;
  }
  if (plan->bsa_pairs < 0) plan->bsa_pairs = bsa_pairs(*plan);
  std::memset(s, 0, sizeof(*s));
  s->useful_pairs = plan->useful_pairs;
  s->physical_pairs_fwd = plan->wq.physical_pairs;
  s->physical_pairs_dq = plan->wq.physical_pairs;
  s->physical_pairs_dkdv = plan->wk.physical_pairs;
  s->bsa_pairs = plan->bsa_pairs;
  s->n_work_fwd = plan->wq.n_work;
  s->n_work_dkdv = plan->wk.n_work;
  s->n_entries_fwd = static_cast<int64_t>(plan->wq.pages.size());
  s->n_entries_dkdv = static_cast<int64_t>(plan->wk.pages.size());
  s->device_bytes = plan->device_bytes;
  s->launches_fwd = (plan->wq.n_work > 0) + fill_launches(plan->q_fill);
  s->launches_bwd = 1 + (plan->wk.n_work > 0) + (plan->wq.n_work > 0) + fill_launches(plan->k_fill) +
                    fill_launches(plan->q_fill);
  s->plan_ms = plan->plan_ms;
  return SPATTN_OK;
}

int spattn_profile(spattn_plan_t plan, int enable) {
  if (!plan) return SPATTN_ERR_INVALID_ARG;
  plan->profiling = enable != 0;
  plan->n_events = 0;
  return SPATTN_OK;
}

int spattn_profile_read(spattn_plan_t plan, spattn_kernel_times* out) {
  if (!plan || !out) return SPATTN_ERR_INVALID_ARG;
  std::memset(out, 0, sizeof(*out));
  int st = SPATTN_OK;
  for (size_t i = 0; i < plan->n_events; ++i) {
    auto& r = plan->events[i];
    float ms = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) {
      st = SPATTN_ERR_CUDA;
      continue;
    }
    out->ms[r.kernel] += ms;
    out->launches[r.kernel] += 1;
  }
  plan->n_events = 0;
  return st;
}

int spattn_plan_pages(spattn_plan_t plan, int32_t head, int64_t qblock, const int32_t** pages, int64_t* n) {
  if (plan) {
    const int st = refresh_host(plan);
    if (st) return st;
  }
  if (!plan || !pages || !n || head < 0 || head >= plan->graph_batches * plan->heads || qblock < 0 ||
      qblock >= (plan->q.slots + kBlockRows - 1) / kBlockRows)
    return SPATTN_ERR_INVALID_ARG;
  canonical_pages(*plan, head, qblock, plan->scratch);
  *pages = plan->scratch.data();
  *n = static_cast<int64_t>(plan->scratch.size());
  return SPATTN_OK;
}

int spattn_plan_qblocks(spattn_plan_t plan, int32_t head, int64_t page, const int32_t** qblocks, int64_t* n) {
  if (plan) {
    const int st = refresh_host(plan);
    if (st) return st;
  }
  if (!plan || !qblocks || !n || head < 0 || head >= plan->graph_batches * plan->heads || page < 0 ||
      page >= plan->k.n_pages)
    return SPATTN_ERR_INVALID_ARG;
  transposed_qblocks(*plan, head, page, plan->scratch);
  *qblocks = plan->scratch.data();
  *n = static_cast<int64_t>(plan->scratch.size());
  return SPATTN_OK;
}

int spattn_plan_work(spattn_plan_t plan, int32_t which, const int32_t** work, int64_t* n_work, const int32_t** pages,
                     const uint64_t** masks, int64_t* n_entries) {
  if (plan) {
    const int st = refresh_host(plan);
    if (st) return st;
  }
  if (!plan || !work || !n_work || !pages || !masks || !n_entries || (which != 0 && which != 1))
    return SPATTN_ERR_INVALID_ARG;
  const WorkList& w = which == 0 ? plan->wq : plan->wk;
  *work = w.work.data();
  *n_work = w.n_work;
  *pages = w.pages.data();
  *masks = w.masks.data();
  *n_entries = static_cast<int64_t>(w.pages.size());
  return SPATTN_OK;
}

int spattn_plan_entry_heads(spattn_plan_t plan, int32_t which, const uint16_t** heads, int64_t* n_entries) {
  if (!plan || !heads || !n_entries || (which != 0 && which != 1)) return SPATTN_ERR_INVALID_ARG;
  const int st = refresh_host(plan);
  if (st) return st;
  WorkList& w = which == 0 ? plan->wq : plan->wk;
  if (w.heads.size() != w.pages.size()) w.heads.assign(w.pages.size(), 0);  // lists rebuilt on the device
  *heads = w.heads.data();
  *n_entries = static_cast<int64_t>(w.heads.size());
  return SPATTN_OK;
}

void spattn_plan_destroy(spattn_plan_t plan) {
  if (!plan) return;
  free_plan_device(plan);
  delete plan;
}

const char* spattn_status_string(int status) {
  switch (status) {
    case SPATTN_OK: return "ok";
    case SPATTN_ERR_INVALID_ARG: return "invalid argument";
    case SPATTN_ERR_UNSUPPORTED: return "unsupported configuration";
    case SPATTN_ERR_OOM: return "out of memory";
    case SPATTN_ERR_CUDA: return "CUDA runtime error";
    case SPATTN_ERR_TIMEOUT: return "device-side wait timed out";
    case SPATTN_ERR_DEVICE: return "device rejected a work item";
    default: return "unknown status";
  }
}

}  // extern "C"
