// Device-side helpers shared by the attention kernels: work-item decode,
// per-row masks of one 128-column step, smem layout constants.
#pragma once

#include "kernels.cuh"
#include "sm100.cuh"

namespace spattn {
namespace dev {

constexpr int kRows = 128;              // rows of an owned tile (TMEM lanes)
constexpr int kStepPages = 8;           // column pages per step
constexpr int kChunkBytes = 128 * 128;  // one 64-column chunk of a 128-row operand
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~static_cast<uintptr_t>(1023));
}

// Slot of row r (0..15) of a page reference: p >= 0 is the page of slots
// 16p .. 16p+15; a negative value is a strided page with base slot b = ~ref,
// the four 4-row groups b + 16j .. b + 16j + 3.
__device__ __forceinline__ int64_t pref_slot(int32_t ref, int r) {
  return ref >= 0 ? static_cast<int64_t>(ref) * 16 + r : static_cast<int64_t>(~ref) + 16 * (r >> 2) + (r & 3);
}

// Work item words (see spattn_plan_work in include/spattn.h).
struct Work {
  int bh, n_own, e0, e1;
  const int32_t* w;
  __device__ __forceinline__ int own_page(int i) const { return w[4 + i]; }
  __device__ __forceinline__ uint32_t row_code(int r) const {
    return (static_cast<uint32_t>(w[12 + (r >> 3)]) >> (4 * (r & 7))) & 0xFu;
  }
  // 64-row route (query-owned items only): rows 0..63 (own pages 0..3) and
  // 64..127 (own pages 4..7) each run over their own pages, two per half in
  // every 4-entry step (entries 0, 1 for rows 0..63, entries 2, 3 for the
  // rest).  The masks alone already make the item exact, so a kernel that
  // ignores the flag computes the same result over all 128 rows.
  __device__ __forceinline__ bool halves() const { return w[28] != 0; }
};

__device__ __forceinline__ Work load_work(const int32_t* work, int64_t idx) {
  Work x;
  x.w = work + idx * 32;
  x.bh = x.w[0];
  x.n_own = x.w[1];
  x.e0 = x.w[2];
  x.e1 = x.w[3];
  return x;
}

// The column-list masks of one step of NP pages for one row: each entry
// holds 16 bits per segment in two 64-bit words (segment s at bits
// 16 (s % 4) of word s / 4), and a row reads only the 16-bit half-word of its
// own segment.  `fetch` only issues the loads; the words are read by
// `bits`, an iteration later, so the load latency never stalls the row math
// that runs in between.
template <int NP>
struct StepMasks {
  uint32_t w[NP];
  // `seg` < 0 (a row without a segment) gives an all-zero mask.
  __device__ __forceinline__ void fetch(const uint64_t* __restrict__ masks, int first, int n, int seg) {
    const uint16_t* h = reinterpret_cast<const uint16_t*>(masks + 2 * static_cast<int64_t>(first)) + (seg < 0 ? 0 : seg);
#pragma unroll
    for (int j = 0; j < NP; ++j) {
      w[j] = 0u;
      if (j < n && seg >= 0) w[j] = __ldg(h + 8 * j);
    }
  }
  // Row mask of the step: bit c of word c/32 <=> column c may be attended.
  __device__ __forceinline__ void bits(uint32_t (&mw)[NP / 2]) const {
#pragma unroll
    for (int i = 0; i < NP / 2; ++i) mw[i] = w[2 * i] | (w[2 * i + 1] << 16);
  }
};

// Warp-collective TMA gather of n (<= 32) pages into a stage whose 64-column
// chunks are `chunk_bytes` apart; page j lands at rows 16j..16j+15 of every
// chunk.  Lane j < n holds page id `pid` of page j and the batch*head `bh` it
// is read from (a run never spans two heads).  Maximal runs of
// consecutive page ids are fetched with 64-, 32- and 16-row boxes by the
// run's first lane; a run that fills a whole 64-row stage (chunks 8 KB
// apart) or a whole 128-row stage or tile (chunks 16 KB apart) takes one
// request for all chunks.  Each TMA request costs the
// issuing thread time whatever its size, so fewer, larger boxes keep the
// producer off the critical path.  All 32 lanes must call this.
//
// A strided page (negative reference) is never part of a run: its lane
// fetches it with one strided 16-row box per 64-column chunk.
template <int NCH>
__device__ __forceinline__ void load_page_runs(uint8_t* dst, int chunk_bytes, const TmaPages& maps, int pid, int n,
                                               int bh, uint64_t* bar) {
  const int lane = lane_id();
  const int nxt = __shfl_down_sync(0xffffffffu, pid, 1);
  const int nbh = __shfl_down_sync(0xffffffffu, bh, 1);
  // bit j: page j+1 follows page j (both regular, same batch*head)
  const unsigned cont = __ballot_sync(0xffffffffu, lane + 1 < n && pid >= 0 && nxt == pid + 1 && nbh == bh);
  const bool start = lane < n && (lane == 0 || !((cont >> (lane - 1)) & 1u));
  if (!start) return;
  if (pid < 0) {
    const int base = ~pid;
#pragma unroll
    for (int c = 0; c < NCH; ++c) tma_load_5d(dst + c * chunk_bytes + lane * 2048, &maps.m4s, c * 64, 0, 0, base, bh, bar);
    return;
  }
  int rem = __ffs(~(cont >> lane));  // run length
  int j = lane;
  if (lane == 0 && rem >= 8 && chunk_bytes == 128 * 128) {
    tma_load_4d(dst, &maps.m128w, 0, pid * 16, 0, bh, bar);
    j += 8;
    rem -= 8;
  } else if (NCH > 1 && lane == 0 && rem >= 4 && chunk_bytes == 64 * 128) {
    tma_load_4d(dst, &maps.m64w, 0, pid * 16, 0, bh, bar);
    j += 4;
    rem -= 4;
  }
  auto box = [&](const CUtensorMap* m, int rows) {
#pragma unroll
    for (int c = 0; c < NCH; ++c)
      tma_load_3d(dst + c * chunk_bytes + j * 2048, m, c * 64, (pid + (j - lane)) * 16, bh, bar);
    j += rows / 16;
  };
  while (rem >= 4) {
    box(&maps.m64, 64);
    rem -= 4;
  }
  if (rem >= 2) {
    box(&maps.m32, 32);
    rem -= 2;
  }
  if (rem == 1) box(&maps.m16, 16);
}

__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Store 32 fp32 values (times `mul`) of one row as bf16 to global memory.
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const uint32_t (&r)[32], float mul, bool zero) {
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float a = zero ? 0.f : __uint_as_float(r[2 * i]) * mul;
    const float b = zero ? 0.f : __uint_as_float(r[2 * i + 1]) * mul;
    pk[i] = pack_bf16(a, b);
  }
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) d[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
}

}  // namespace dev
}  // namespace spattn
