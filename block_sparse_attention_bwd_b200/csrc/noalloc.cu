// spattn_bwd_noalloc: the backward pass with its scratch in a fixed,
// statically sized device array, for callers that cannot allocate device
// memory when they run the backward pass.
//
// The backward pass needs one scratch value per query row (Delta =
// rowsum(dO * O), fp32).  spattn_bwd takes it from a workspace that
// spattn_plan allocates with cudaMalloc for every plan.  Some callers cannot
// grant that: a host framework whose caching allocator reserves the whole GPU
// up front (so any allocation outside its pool fails or fragments it), or a
// service that runs many plans under a fixed device-memory budget and may not
// let each plan hold its own workspace.  This entry point allocates nothing:
// Delta lives in the array below, which every GPU that loads the library
// holds until the process exits.
#include <cudaTypedefs.h>

#include "kernels.cuh"
#include "plan.hpp"

namespace spattn {

// Largest batch * heads * q_slots the static scratch holds (16 MiB of fp32).
constexpr int64_t kNoAllocDeltaRows = int64_t(1) << 22;

namespace {

// File-scope scratch for Delta.  In host code this name is only a host-side
// stand-in, never a device address: kernels get the address that
// cudaGetSymbolAddress returns in the calling thread's current context.
static __device__ __align__(256) float g_delta_scratch[kNoAllocDeltaRows];

// Device address of the scratch in the current context.  It is looked up on
// every call (a table lookup that allocates nothing) rather than cached: a
// device reset, or a primary context that is released and created again,
// loads the module anew and may place the array elsewhere, and a cached
// address would then point at freed memory.  The first call in a context
// also loads the library's device code there.
int scratch_address(float** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_delta_scratch) != cudaSuccess || !p) {
    cudaGetLastError();
    return SPATTN_ERR_CUDA;
  }
  *out = static_cast<float*>(p);
  return SPATTN_OK;
}

}  // namespace

// Shared with api.cu: tensor maps and tile arguments.
bool make_tensor_pages(TmaPages* t, const void* ptr, int head_dim, int64_t rows, int64_t bh);
TileArgs make_tile_args(const spattn_plan_s* P, const WorkList& w, int64_t own_slots, int64_t col_slots);

}  // namespace spattn

using namespace spattn;

extern "C" int spattn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                  const void* d_o, spattn_plan_t plan, void* dq, void* dk, void* dv, void* stream) {
  if (!plan) return SPATTN_ERR_INVALID_ARG;
  if (plan->device < 0) return SPATTN_ERR_CUDA;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SPATTN_ERR_CUDA;
  if (dev != plan->device) return SPATTN_ERR_INVALID_ARG;
  const int64_t bh = static_cast<int64_t>(plan->batch) * plan->heads;
  if (bh * plan->q.slots > kNoAllocDeltaRows) return SPATTN_ERR_UNSUPPORTED;
  auto aligned = [](const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!aligned(q) || !aligned(k) || !aligned(v) || !aligned(o) || !aligned(lse) || !aligned(d_o) || !aligned(dq) ||
      !aligned(dk) || !aligned(dv))
    return SPATTN_ERR_INVALID_ARG;
  float* delta = nullptr;
  int st = scratch_address(&delta);
  if (st) return st;
  const int D = plan->head_dim;
  const int64_t bh_kv = static_cast<int64_t>(plan->batch) * plan->kv_heads;
  TmaPages tq, tk, tv, tdo;
  if (!make_tensor_pages(&tq, q, D, plan->q.slots, bh) || !make_tensor_pages(&tk, k, D, plan->k.slots, bh_kv) ||
      !make_tensor_pages(&tv, v, D, plan->k.slots, bh_kv) || !make_tensor_pages(&tdo, d_o, D, plan->q.slots, bh))
    return SPATTN_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto* dQ = static_cast<__nv_bfloat16*>(dq);
  auto* dK = static_cast<__nv_bfloat16*>(dk);
  auto* dV = static_cast<__nv_bfloat16*>(dv);
  // Delta is written for every row before the tile kernels read it, so the
  // scratch needs no clearing between calls.
  cudaError_t e = launch_delta(D, static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(d_o), delta,
                               bh * plan->q.slots, s);
  if (e == cudaSuccess)
    e = launch_dkdv(D, tk, tv, tq, tdo, make_tile_args(plan, plan->wk, plan->k.slots, plan->q.slots), lse, delta, dK,
                    dV, s);
  if (e == cudaSuccess)
    e = launch_dq(D, static_cast<const __nv_bfloat16*>(q), tdo, tk, tv, make_tile_args(plan, plan->wq, plan->q.slots, plan->k.slots), lse, delta, dQ, s);
  if (e == cudaSuccess && !plan->k_fill.empty())
    e = launch_fill(D, plan->d_k_fill, static_cast<int64_t>(plan->k_fill.size() / 2), bh_kv, plan->k.slots, dK, dV,
                    nullptr, s);
  if (e == cudaSuccess && !plan->q_fill.empty())
    e = launch_fill(D, plan->d_q_fill, static_cast<int64_t>(plan->q_fill.size() / 2), bh, plan->q.slots, dQ,
                    nullptr, nullptr, s);
  return e == cudaSuccess ? SPATTN_OK : SPATTN_ERR_CUDA;
}
