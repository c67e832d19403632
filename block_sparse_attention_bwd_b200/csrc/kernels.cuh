// Kernel launchers shared by the C ABI (api.cpp) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace spattn {

// Three TMA descriptors over the same [rows, head_dim] x (batch*heads) bf16
// tensor, with boxes of 16, 32 and 64 rows (64 columns, 128-byte swizzle).
// A run of consecutive 16-row pages is fetched with the fewest boxes: the TMA
// engine's cost is per request, so one 64-row box moves 4x the bytes of a
// page-sized box in about the same time.
struct TmaPages {
  CUtensorMap m16, m32, m64;
  // 64 rows x every 64-column chunk in one request (4D map: columns, rows,
  // chunk, batch*head); it lands chunk after chunk, 8 KB apart, which is the
  // layout of a 64-row stage.  Equal to m64 when head_dim is 64.
  CUtensorMap m64w;
  // The same 4D view with 128-row boxes: a whole 128-row stage or owned tile
  // (chunks 16 KB apart) in one request.
  CUtensorMap m128w;
  // Strided pages: a 5D view (64-column x, 4 rows, 4 groups 16 rows apart,
  // slot, batch*head) whose 64 x 4 x 4 box is the 16 rows of a strided page
  // (base slot b: rows b + 16j + r), one 64-column chunk per request; it lands
  // as a 16-row page of that chunk.
  CUtensorMap m4s;
};

// Everything one attention launch needs besides its tensor maps.
struct TileArgs {
  const int32_t* work = nullptr;    // n_work x 32 words (see spattn_plan_work)
  const int32_t* pages = nullptr;   // column page ids
  const uint64_t* masks = nullptr;  // 8 x 16-bit row masks per entry (two words)
  int64_t n_work = 0;
  int64_t own_slots = 0;            // rows per (batch, head) of the owned side
  int64_t col_slots = 0;            // rows per (batch, head) of the column side
  float scale = 0.f;                // softmax scale
  int* err = nullptr;               // device error word
  int* sched = nullptr;             // work-item counter of a persistent kernel (the launcher zeroes it)
  // Grouped-query attention: query head h reads K/V head h / kv_group
  // (heads = query heads, kv_heads = heads / kv_group).  For the key-owned
  // pass, entry e's column head is the item's first query head + col_heads[e].
  int heads = 1, kv_heads = 1, kv_group = 1;
  const uint16_t* col_heads = nullptr;
  // some query-owned item takes the 64-row route (the forward then runs the
  // kernel form that reads the route flag of each item)
  bool route64 = false;
};

// K1: O, LSE for every query-owned work item.
cudaError_t launch_fwd(int head_dim, const TmaPages& tq, const TmaPages& tk, const TmaPages& tv, const TileArgs& a,
                       __nv_bfloat16* o, float* lse, cudaStream_t st);

// K1 with E4M3 Q and K (head_dim 128): tq8 / tk8 map the one-byte codes (128
// per 128-byte row), S is scaled by q_descale[bh] * k_descale[kv_bh].
cudaError_t launch_fwd_e4m3(const TmaPages& tq8, const TmaPages& tk8, const TmaPages& tv, const TileArgs& a,
                            const float* q_descale, const float* k_descale, __nv_bfloat16* o, float* lse,
                            cudaStream_t st);

// Per-slice E4M3 quantisation of a [bh, rows, head_dim] bf16 tensor: amax of
// each slice, codes = e4m3(x * (448 / amax)), descale = amax / 448 (1 for an
// all-zero slice).  `descale` doubles as the amax scratch.
cudaError_t launch_quantize_e4m3(const __nv_bfloat16* x, int64_t bh, int64_t elems_per_bh, uint8_t* x8,
                                 float* descale, cudaStream_t st);

// K2: delta[row] = sum_d dO[row, d] * O[row, d] over rows = batch*heads*q_slots.
cudaError_t launch_delta(int head_dim, const __nv_bfloat16* o, const __nv_bfloat16* d_o, float* delta,
                         int64_t rows, cudaStream_t st);

// K3: dK, dV for every key-owned work item.
cudaError_t launch_dkdv(int head_dim, const TmaPages& tk, const TmaPages& tv, const TmaPages& tq, const TmaPages& tdo,
                        const TileArgs& a, const float* lse, const float* delta, __nv_bfloat16* dk,
                        __nv_bfloat16* dv, cudaStream_t st);

// K4: dQ for every query-owned work item (Q rows are read directly into TMEM).
cudaError_t launch_dq(int head_dim, const __nv_bfloat16* q, const TmaPages& tdo, const TmaPages& tk,
                      const TmaPages& tv, const TileArgs& a, const float* lse, const float* delta,
                      __nv_bfloat16* dq, cudaStream_t st);

// K5: zero the rows that no work item writes (and LSE = -inf).
// One CTA whose warp 0 waits, with the given deadline, on an mbarrier that
// nothing arrives at, and whose warp 1 waits on it with the tile kernels'
// deadline: warp 0 times out and records SPATTN_ERR_TIMEOUT's device code in
// `err`, warp 1 sees the CTA abort flag and gives up.  Both return.
cudaError_t launch_wait_selftest(int* err, long long deadline_cycles, cudaStream_t st);

// `fill` holds n (page, 16-bit row mask) pairs: the rows r of page p with bit r
// set are zeroed in t0 and t1 (if given) and get LSE = -inf (if given), for
// every (batch, head).
cudaError_t launch_fill(int head_dim, const int32_t* fill, int64_t n, int64_t bh, int64_t slots,
                        __nv_bfloat16* t0, __nv_bfloat16* t1, float* lse, cudaStream_t st);

}  // namespace spattn
