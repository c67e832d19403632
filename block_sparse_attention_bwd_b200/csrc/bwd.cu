// Backward kernels: K2 (Delta = rowsum(dO * O)), K3 (dK, dV owned per key
// tile, no atomics) and K4 (dQ owned per query tile, no atomics).
//
// Method (KPage abstract, "KPage: block-sparse attention for partially
// occupied 3D blocks", zhuanzhiai.com, abstract paragraph): the backward pass
// keeps the sparse graph exact by letting the K/V side own its pages.  Here
// the key side packs its valid 16-row pages into 128-row owned tiles exactly
// as the query side does in the forward pass; each key tile walks the query
// pages that reach it (the transposed lists), so dK and dV are accumulated
// in TMEM and written once.  dQ is computed by a second, query-owned pass
// over the forward page lists.  The gradient formulas are the standard ones
// for softmax attention: P = exp(S - LSE), dV = P^T dO, dP = dO V^T,
// dS = P * (dP - Delta), dK = scale dS^T Q, dQ = scale dS K.
//
// Both tile kernels use 12 warps: warps 0 and 11 are TMA producers (one per
// column tensor), warp 1 allocates TMEM and issues the two products of each
// step that read the column tiles, warp 10 issues the accumulating products,
// and warps 2..9 turn each step's scores into P / dS, one tile row per lane,
// two warp groups per step (32 columns each).
#include <algorithm>

#include "kernels.cuh"
#include "tile.cuh"

namespace spattn {
namespace {

using namespace dev;

// ----------------------------------------------------------------------------
// K2: Delta
// ----------------------------------------------------------------------------
template <int D>
__global__ void delta_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ d_o,
                             float* __restrict__ delta, int64_t rows) {
  constexpr int TPR = D / 8;  // threads per row, 8 bf16 (16 B) each
  const int64_t total = rows * TPR;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;  // multiple of 32
  const int lane = threadIdx.x & 31;
  // warp-uniform loop so that the group shuffles below always see full warps
  for (int64_t t0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31); t0 < total; t0 += stride) {
    const int64_t t = t0 + lane;
    const int64_t row = t / TPR;
    const int part = static_cast<int>(t % TPR);
    float acc = 0.f;
    if (t < total) {
      const uint4 a = *reinterpret_cast<const uint4*>(o + row * D + part * 8);
      const uint4 b = *reinterpret_cast<const uint4*>(d_o + row * D + part * 8);
      const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 fa = __bfloat1622float2(pa[i]);
        const float2 fb = __bfloat1622float2(pb[i]);
        acc = fmaf(fa.x, fb.x, acc);
        acc = fmaf(fa.y, fb.y, acc);
      }
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off, TPR);
    if (t < total && part == 0) delta[row] = acc;
  }
}

// ----------------------------------------------------------------------------
// K3: dK, dV (key-owned tiles, query pages as columns, 64 columns per step)
// ----------------------------------------------------------------------------
// TMEM columns: one fp32 staging set (S^T at 0, dP^T at 64), two packed
// bf16 operand sets (P^T at 128 + 64p, dS^T at 160 + 64p), dV at 256, dK at
// 256 + D.  The staging set is free again as soon as the row threads have
// loaded it, so the S^T / dP^T MMAs of step c+1 run while the row threads
// compute step c; the packed set of step c is reused two steps later, after
// the dV / dK MMAs that read it.
//
// Column tiles arrive in stages of one 64-column MMA step (dK / dV) or two
// (dQ, 128 rows, one 32 KB box): a TMA request holds its issuing thread for
// a long time whatever its size, so larger stages keep a producer ahead of the
// tensor core, while more stages give more slack between a stage's release
// and its reuse; dK / dV have room for four 64-row stages per tensor only.
//
// The per-column terms of the backward pass are folded into the two MMAs
// with one extra K = 16 slice each, so the row threads read nothing but
// TMEM: with x = LSE / scale of query column c, split into three bf16 terms
// x = h + m + l (exact to about 2^-27 relative),
//   [K | 1 1 1 0..] . [Q | -h -m -l 0..]^T = S^T - x,  sl2 * (S^T - x) = log2 P^T,
//   [V | 1 1 1 0..] . [dO | -Delta split]^T = dP^T - Delta,
// both accumulated in fp32.  The slices are 16 bf16 wide, in the plain
// (unswizzled) K-major layout: a 128-row block of ones shared by both MMAs,
// and one block per Q / dO stage that the producer writes.
constexpr int kBwdStepPages = 4;                  // 64 columns per MMA step
constexpr int kHalfStage = 64 * 128;              // offset of a two-step stage's second step in a chunk
constexpr int kOnesBytes = 128 * 32;              // 128 rows x 16 bf16, plain layout

// Byte offset of row r (first 8 of its 16 elements) in a plain K-major
// 16-wide block: 8-row core matrices of 256 bytes, the second K half 128 B on.
__device__ __forceinline__ uint32_t aug_row_off(int r) { return static_cast<uint32_t>((r >> 3) * 256 + (r & 7) * 16); }

// First 8 elements of an augmented row: -x as three bf16 terms, then zeros.
__device__ __forceinline__ uint4 aug_row(float x) {
  const float h = __bfloat162float(__float2bfloat16_rn(x));
  const float r1 = x - h;
  const float m = __bfloat162float(__float2bfloat16_rn(r1));
  const float l = r1 - m;
  return make_uint4(pack_bf16(-h, -m), pack_bf16(-l, 0.f), 0u, 0u);
}

template <int D>
struct DkvCfg {
  static constexpr int kNch = D / 64;
  static constexpr int kTile = kNch * kChunkBytes;     // owned 128-row tile
  static constexpr int kStagePages = 4;                  // one step per stage
  static constexpr int kStageChunk = kStagePages * 16 * 128;  // one 64-column chunk of a stage
  static constexpr int kStageTile = kNch * kStageChunk;
  static constexpr int kAugStage = kStagePages * 16 * 32;     // plain-layout slice of a stage
  static constexpr int kQStages = (D == 128) ? 4 : 6;
  static constexpr int kDStages = (D == 128) ? 4 : 6;
  static constexpr int kSmem = 2 * kTile + (kQStages + kDStages) * (kStageTile + kAugStage) + kOnesBytes + 1024 + 512;
};

// 12 warps: 0 and 11 = TMA producers, 1 = TMEM owner and issuer of the MMAs
// that read the step's column tiles into TMEM (S^T/dP^T or S/dP), 2..9 = two
// groups of row threads, 10 = issuer of the accumulating MMAs (dV/dK or dQ).
// Row group g (warps 2+4g .. 5+4g) handles columns 32g .. 32g+31 of every
// 64-column step (warp w reaches TMEM lanes of quarter w%4).  The tensor
// core accepts only a couple of MMAs ahead of the one it runs, so a single
// issuing warp idles it whenever that warp waits; with two issuers one keeps
// it busy while the other waits.
constexpr int kAccWarp = 10;
// Warp 11 is the second producer (dO stages for dK / dV, V stages for dQ;
// warp 0 produces the Q or K stages): a TMA request holds its issuing thread
// for hundreds of cycles, so one producer for both column tensors would set
// the step time.
constexpr int kDkvThreads = 384;
constexpr int kDoWarp = 11;

// Persistent form: one CTA per SM takes work items from a device counter in
// list order (longest first per head), so each SM keeps its rings and TMEM
// across items.  Warp 0 fetches the next item and publishes it in a 4-deep
// queue in shared memory; every other role reads the queue.  Stage, step and
// item counters run across items, so every barrier keeps advancing one phase
// at a time.  At an item boundary the producers load the next item's owned
// K / V (once the last S^T / dP^T products of the previous item have read
// them) and its first stages, and the first S^T / dP^T products of the next
// item run while the row threads finish the previous item and write its dK /
// dV; the accumulating products of the next item wait until those
// accumulators have been read.
constexpr int kItemQueue = 4;
// readers of a queue slot: warps 1, 10, 11 and the 8 row-thread warps
constexpr int kItemReaders = 11;

template <int D>
__global__ void __launch_bounds__(kDkvThreads, 1)
    dkdv_kernel(const __grid_constant__ TmaPages tm_k, const __grid_constant__ TmaPages tm_v,
                const __grid_constant__ TmaPages tm_q, const __grid_constant__ TmaPages tm_do,
                const int32_t* __restrict__ work, int64_t n_work, int* __restrict__ sched,
                const int32_t* __restrict__ col_pages, const uint64_t* __restrict__ col_masks,
                const float* __restrict__ lse, const float* __restrict__ delta, __nv_bfloat16* __restrict__ out_dk,
                __nv_bfloat16* __restrict__ out_dv, int64_t kv_slots, int64_t q_slots, float sl2, float scale,
                int heads, int kv_heads, int kv_group, const uint16_t* __restrict__ col_heads, int* err) {
  using C = DkvCfg<D>;
  constexpr int QS = C::kQStages, DS = C::kDStages, NP = kBwdStepPages, SP = C::kStagePages;
  static_assert(SP == NP, "one MMA step per stage");
  constexpr int NH = SP * 16 / 32;  // stage columns per producer lane
  constexpr int kStageChunk = C::kStageChunk, kAugStage = C::kAugStage;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sK = smem;
  uint8_t* sV = smem + C::kTile;
  uint8_t* sQ = smem + 2 * C::kTile;                 // Q stage s at sQ + s*kStageTile
  uint8_t* sDO = sQ + QS * C::kStageTile;            // dO stage s at sDO + s*kStageTile
  uint8_t* sQa = sDO + DS * C::kStageTile;           // -LSE/scale slice of Q stage s at sQa + s*kAugStage
  uint8_t* sDa = sQa + QS * kAugStage;               // -Delta slice of dO stage s at sDa + s*kAugStage
  uint8_t* sOnes = sDa + DS * kAugStage;             // ones slice of the owned K / V rows
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOnes + kOnesBytes);
  uint64_t* own_full = bars;          // the item's owned K / V rows have landed
  uint64_t* own_free = own_full + 1;  // the item's last S^T / dP^T products have read them
  uint64_t* q_full = own_free + 1;
  uint64_t* q_empty = q_full + QS;
  uint64_t* do_full = q_empty + QS;
  uint64_t* do_empty = do_full + DS;
  uint64_t* st_full = do_empty + DS;  // S^T, dP^T of a step are in the staging set
  uint64_t* st_free = st_full + 1;    // the row threads have loaded the staging set
  uint64_t* pt_full = st_free + 1;    // [2] P^T, dS^T of a step are in packed set p
  uint64_t* acc_done = pt_full + 2;   // the item's dV, dK products have finished
  uint64_t* acc_free = acc_done + 1;  // the row threads have read the item's dV, dK
  uint64_t* acc_b = acc_free + 1;     // [2] dV, dK MMAs of the steps using packed set p finished
  uint64_t* drain = acc_b + 2;        // [2] one per issuing warp
  uint64_t* item_full = drain + 2;    // [kItemQueue]
  uint64_t* item_empty = item_full + kItemQueue;  // [kItemQueue]
  int32_t* items = reinterpret_cast<int32_t*>(item_empty + kItemQueue);  // [kItemQueue]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(items + kItemQueue);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  const Abort ab{abort_flag, err};
  const int warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(own_full, 1);
    mbar_init(own_free, 1);
    mbar_init(&acc_b[0], 1);
    mbar_init(&acc_b[1], 1);
    mbar_init(&drain[1], 1);
    for (int s = 0; s < QS; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    for (int s = 0; s < DS; ++s) {
      mbar_init(&do_full[s], 1);
      mbar_init(&do_empty[s], 1);
    }
    mbar_init(st_full, 1);
    mbar_init(st_free, 256);
    for (int b = 0; b < 2; ++b) mbar_init(&pt_full[b], 256);
    mbar_init(acc_done, 1);
    mbar_init(acc_free, 256);
    mbar_init(drain, 1);
    for (int s = 0; s < kItemQueue; ++s) {
      mbar_init(&item_full[s], 1);
      mbar_init(&item_empty[s], kItemReaders);
    }
    fence_barrier_init();
  }
  {
    // Slices: the ones block holds 1 1 1 0.. in every row; the Q / dO slices
    // start at zero (their second K half is never written again).
    uint4* sl = reinterpret_cast<uint4*>(sQa);
    constexpr int kN16 = ((QS + DS) * kAugStage + kOnesBytes) / 16;
    constexpr int kOnes0 = (QS + DS) * kAugStage / 16;
    for (int i = threadIdx.x; i < kN16; i += kDkvThreads) {
      const bool one = i >= kOnes0 && ((i - kOnes0) & 15) < 8;  // first K half of a ones row
      sl[i] = one ? make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u) : make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }
  if (warp == 1) tmem_alloc(tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t tDV = tmem + 256, tDK = tmem + 256 + D;

  // Item k of this CTA (k = 0, 1, ...): the readers wait for its queue slot,
  // read it and release the slot; -1 ends the loop (also on abort).
  auto read_item = [&](int k) -> int {
    const int s = k % kItemQueue;
    if (!__all_sync(0xffffffffu, mbar_wait(&item_full[s], (k / kItemQueue) & 1, ab))) return -1;
    const int idx = *reinterpret_cast<volatile int32_t*>(&items[s]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&item_empty[s]);
    return idx;
  };

  if (warp == 0 || warp == kDoWarp) {
    // ---------------- producers (whole warps): warp 0 = Q stages, warp 11 = dO stages ----------------
    // Warp 0 also owns the item queue and loads each item's owned K / V rows.
    // Lane j < n owns page j of a stage: it holds the page id (fetched one
    // stage ahead) and issues that page's TMA boxes; every lane also writes
    // the augmented slice rows of two of the stage's 64 query columns.
    const bool is_q = warp == 0;
    const int NS = is_q ? QS : DS;
    uint8_t* stage0 = is_q ? sQ : sDO;
    uint8_t* aug0 = is_q ? sQa : sDa;
    uint64_t* full = is_q ? q_full : do_full;
    uint64_t* empty = is_q ? q_empty : do_empty;
    const TmaPages& tm = is_q ? tm_q : tm_do;
    const float* terms = is_q ? lse : delta;
    const float inv_scale = 1.0f / scale;
    if (lane == 0) {
      tma_prefetch_desc(&tm.m64w);
      tma_prefetch_desc(&tm.m64);
      if (is_q) {
        tma_prefetch_desc(&tm_k.m64);
        tma_prefetch_desc(&tm_v.m64);
      }
    }
    int T = 0;  // stages issued by this warp over all items
    int own_loads = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      int idx;
      if (is_q) {
        const int s = k % kItemQueue;
        if (k >= kItemQueue && !__all_sync(0xffffffffu, mbar_wait(&item_empty[s], ((k / kItemQueue) - 1) & 1, ab)))
          break;
        int v = 0;
        if (lane == 0) {
          v = atomicAdd(sched, 1);
          v = v < n_work ? v : -1;
          items[s] = v;
          mbar_arrive(&item_full[s]);
        }
        idx = __shfl_sync(0xffffffffu, v, 0);
      } else {
        idx = read_item(k);
      }
      if (idx < 0) break;
      const Work wk = load_work(work, idx);
      const int n_cols = wk.e1 - wk.e0;
      if (is_q) {
        // owned K / V rows: their buffers are free once the previous item's
        // last S^T / dP^T products have read them
        if (k >= 1 && !__all_sync(0xffffffffu, mbar_wait(own_free, (k - 1) & 1, ab))) break;
        if (lane == 0) mbar_arrive_expect_tx(own_full, 2 * wk.n_own * C::kNch * 2048);
        __syncwarp();
        const int own_pid = lane < wk.n_own ? wk.own_page(lane) : 0;
        load_page_runs<C::kNch>(sK, kChunkBytes, tm_k, own_pid, wk.n_own, wk.bh, own_full);
        load_page_runs<C::kNch>(sV, kChunkBytes, tm_v, own_pid, wk.n_own, wk.bh, own_full);
        own_loads = k + 1;
      }
      // Lane j holds the page id of column page j of stages t and t+1, and the
      // per-column term (LSE for Q, Delta for dO) of columns lane + 32h of
      // stage t.  Both are fetched one stage ahead, and the fetched values are
      // used only in the next iteration, so their global-load latency overlaps
      // the waits and TMA issue of the current one instead of stalling it.
      const int n_stages = (n_cols + SP - 1) / SP;
      auto page_id = [&](int t) {
        return (t < n_stages && lane < min(SP, n_cols - t * SP)) ? __ldg(col_pages + wk.e0 + t * SP + lane) : 0;
      };
      // Query head of a column page: the item's K/V head owns the query heads
      // q_base .. q_base + kv_group - 1 (grouped-query attention); each entry
      // names its offset.
      const int q_base = (wk.bh / kv_heads) * heads + (wk.bh % kv_heads) * kv_group;
      auto col_bh = [&](int t) {
        return q_base + ((col_heads && t < n_stages && lane < min(SP, n_cols - t * SP))
                             ? static_cast<int>(__ldg(col_heads + wk.e0 + t * SP + lane))
                             : 0);
      };
      // Raw loads only (nothing here reads the loaded registers); a dead
      // column (beyond the stage or the tensor) loads a valid address and is
      // zeroed where the value is used, through its bit in `live`.
      auto fetch_terms = [&](int t, int pg_lane, int bh_lane, float (&x)[NH], uint32_t& live) {
        const int n_t = min(SP, n_cols - t * SP);
        live = 0u;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          const int idx2 = lane + 32 * h;  // column of the stage
          const int pg = __shfl_sync(0xffffffffu, pg_lane, idx2 >> 4);
          const int cb = __shfl_sync(0xffffffffu, bh_lane, idx2 >> 4);
          const int64_t slot = pref_slot(pg, idx2 & 15);
          const bool okc = t < n_stages && (idx2 >> 4) < n_t && slot < q_slots;
          x[h] = __ldg(terms + static_cast<int64_t>(cb) * q_slots + (okc ? slot : 0));
          live |= okc ? (1u << h) : 0u;
        }
      };
      // Augmented row of a column: -LSE / scale for Q (a column that attends
      // nothing, LSE = -inf, is masked everywhere, like a dead one: zeros), or
      // -Delta for dO.
      auto term_row = [&](float t, bool okr) {
        const float x = is_q ? t * inv_scale : t;
        return aug_row(okr && isfinite(x) ? x : 0.f);
      };
      int pid = page_id(0), pid_next = page_id(1);
      int cbh = col_bh(0), cbh_next = col_bh(1);
      float xc[NH];
      uint32_t livec;
      fetch_terms(0, pid, cbh, xc, livec);
      for (int t = 0; t < n_stages; ++t, ++T) {
        const int s = T % NS;
        const int n = min(SP, n_cols - t * SP);
        const int pid_next2 = page_id(t + 2);
        const int cbh_next2 = col_bh(t + 2);
        float xn[NH];
        uint32_t liven;
        fetch_terms(t + 1, pid_next, cbh_next, xn, liven);
        if (T >= NS && !__all_sync(0xffffffffu, mbar_wait(&empty[s], ((T / NS) - 1) & 1, ab))) {
          ok = false;
          break;
        }
#pragma unroll
        for (int h = 0; h < NH; ++h)
          *reinterpret_cast<uint4*>(aug0 + s * kAugStage + aug_row_off(lane + 32 * h)) =
              term_row(xc[h], (livec >> h) & 1u);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_expect_tx(&full[s], n * C::kNch * 2048);
        __syncwarp();
        load_page_runs<C::kNch>(stage0 + s * C::kStageTile, kStageChunk, tm, pid, n, cbh, &full[s]);
        pid = pid_next;
        pid_next = pid_next2;
        cbh = cbh_next;
        cbh_next = cbh_next2;
        livec = liven;
#pragma unroll
        for (int h = 0; h < NH; ++h) xc[h] = xn[h];
      }
    }
    // no copy may still be landing in shared memory when the CTA exits
    if (lane == 0) {
      for (int t = max(0, T - NS); t < T; ++t) mbar_wait_drain(&full[t % NS], (t / NS) & 1);
      if (is_q && own_loads > 0) mbar_wait_drain(own_full, (own_loads - 1) & 1);
    }
  } else if (warp == 1) {
    // ---------------- S^T, dP^T issuer (warp-wide; one elected lane issues) ----------------
    const uint64_t dk0 = sdesc_sw128(smem_u32(sK), 16, 1024);
    const uint64_t dv0 = sdesc_sw128(smem_u32(sV), 16, 1024);
    const uint64_t dqk = sdesc_sw128(smem_u32(sQ), 16, 1024);             // Q stages, K-major
    const uint64_t ddk = sdesc_sw128(smem_u32(sDO), 16, 1024);            // dO stages, K-major
    const uint64_t d_ones = sdesc_plain(smem_u32(sOnes), 128, 256);
    const uint64_t d_qa = sdesc_plain(smem_u32(sQa), 128, 256);
    const uint64_t d_da = sdesc_plain(smem_u32(sDa), 128, 256);
    int G = 0;  // steps over all items
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int idx = read_item(k);
      if (idx < 0) break;
      const Work wk = load_work(work, idx);
      const int n_cols = wk.e1 - wk.e0;
      const int n_steps = (n_cols + NP - 1) / NP;
      ok = __all_sync(0xffffffffu, mbar_wait(own_full, k & 1, ab));
      tc_fence_after();
      for (int st = 0; ok && st < n_steps; ++st, ++G) {
        const int qs = G % QS, ds = G % DS;
        const int n = min(NP, n_cols - st * NP);
        const uint32_t idesc_s = idesc_bf16(128, 16 * n, false, false);
        // the staging set is free once the row threads have loaded step G-1
        bool w = (G < 1 || mbar_wait(st_free, (G - 1) & 1, ab)) && mbar_wait(&q_full[qs], (G / QS) & 1, ab);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        tc_fence_after();
        const uint64_t bq = sdesc_add(dqk, qs * C::kStageTile);
        const uint64_t bd = sdesc_add(ddk, ds * C::kStageTile);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss_w(tmem, sdesc_add(dk0, (kk >> 2) * kChunkBytes + (kk & 3) * 32),
                    sdesc_add(bq, (kk >> 2) * kStageChunk + (kk & 3) * 32), idesc_s, kk > 0);
        umma_ss_w(tmem, d_ones, sdesc_add(d_qa, qs * kAugStage), idesc_s, 1u);
        if (!__all_sync(0xffffffffu, mbar_wait(&do_full[ds], (G / DS) & 1, ab))) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss_w(tmem + 64, sdesc_add(dv0, (kk >> 2) * kChunkBytes + (kk & 3) * 32),
                    sdesc_add(bd, (kk >> 2) * kStageChunk + (kk & 3) * 32), idesc_s, kk > 0);
        umma_ss_w(tmem + 64, d_ones, sdesc_add(d_da, ds * kAugStage), idesc_s, 1u);
        umma_commit_w(st_full);
      }
      // the owned K / V buffers are free once these products have read them
      umma_commit_w(own_free);
    }
    umma_commit_w(&drain[0]);
    mbar_wait_drain(&drain[0], 0);
  } else if (warp == kAccWarp) {
    // ---------------- dV, dK issuer (warp-wide; one elected lane issues) ----------------
    const uint64_t dqm = sdesc_sw128(smem_u32(sQ), kStageChunk, 1024);    // Q stages, MN-major
    const uint64_t ddm = sdesc_sw128(smem_u32(sDO), kStageChunk, 1024);   // dO stages, MN-major
    const uint32_t idesc_acc = idesc_bf16(128, D, false, true);
    int G = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int idx = read_item(k);
      if (idx < 0) break;
      const Work wk = load_work(work, idx);
      const int n_cols = wk.e1 - wk.e0;
      const int n_steps = (n_cols + NP - 1) / NP;
      // the accumulators hold the previous item until its row threads read them
      if (k >= 1 && !__all_sync(0xffffffffu, mbar_wait(acc_free, (k - 1) & 1, ab))) break;
      tc_fence_after();
      for (int st = 0; st < n_steps; ++st, ++G) {
        const int b = G & 1, qs = G % QS, ds = G % DS;
        if (!__all_sync(0xffffffffu, mbar_wait(&pt_full[b], (G >> 1) & 1, ab))) { ok = false; break; }
        tc_fence_after();
        const int n = min(NP, n_cols - st * NP);
        const uint64_t bq = sdesc_add(dqm, qs * C::kStageTile);
        const uint64_t bd = sdesc_add(ddm, ds * C::kStageTile);
#pragma unroll
        for (int j = 0; j < NP; ++j)
          if (j < n) umma_ts_w(tDV, tmem + 128 + 64 * b + 8 * j, sdesc_add(bd, j * 2048), idesc_acc, (st > 0 || j > 0) ? 1u : 0u);
        umma_commit_w(&do_empty[ds]);
#pragma unroll
        for (int j = 0; j < NP; ++j)
          if (j < n)
            umma_ts_w(tDK, tmem + 160 + 64 * b + 8 * j, sdesc_add(bq, j * 2048), idesc_acc, (st > 0 || j > 0) ? 1u : 0u);
        umma_commit_w(&q_empty[qs]);
        umma_commit_w(&acc_b[b]);
      }
      if (ok) umma_commit_w(acc_done);  // every item, with or without steps
    }
    umma_commit_w(&drain[1]);
    mbar_wait_drain(&drain[1], 0);
  } else {
    // ---------------- P^T, dS^T (one key row per thread) + epilogue ----------------
    const int grp = (warp - 2) >> 2;  // column half of each step
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    int G = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int idx = read_item(k);
      if (idx < 0) break;
      const Work wk = load_work(work, idx);
      const int n_cols = wk.e1 - wk.e0;
      const int n_steps = (n_cols + NP - 1) / NP;
      const uint32_t code = wk.row_code(row);
      const int seg = code < 8 ? static_cast<int>(code) : -1;
      StepMasks<NP> raw;
      if (n_steps > 0) raw.fetch(col_masks, wk.e0, min(NP, n_cols), seg);
      for (int st = 0; st < n_steps; ++st, ++G) {
        const int b = G & 1;
        const int N = 16 * min(NP, n_cols - st * NP);
        const bool active = grp * 32 < N;
        uint32_t mw[2];
        raw.bits(mw);
        // mask words of the next step load while this one computes
        if (st + 1 < n_steps) raw.fetch(col_masks, wk.e0 + (st + 1) * NP, min(NP, n_cols - (st + 1) * NP), seg);
        ok = __all_sync(0xffffffffu, mbar_wait(st_full, G & 1, ab));
        if (!ok) break;
        tc_fence_after();
        uint32_t a[32], d[32];
        if (active) {
          tmem_ld32(tmem + lane_off + grp * 32, a);
          tmem_ld32(tmem + 64 + lane_off + grp * 32, d);
          tmem_wait_ld();
        }
        tc_fence_before();
        mbar_arrive(st_free);
        // a = S^T - LSE/scale, d = dP^T - Delta (fp32, from the augmented MMAs)
        uint32_t pp[16], pd[16];
        if (active) {
          const uint32_t m = grp ? mw[1] : mw[0];
          if (m == 0xFFFFFFFFu) {
            // every column allowed: no masking, all values finite
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float x0, x1, s0, s1;
              f2_unpack(f2_mul(f2_pack(__uint_as_float(a[2 * i]), __uint_as_float(a[2 * i + 1])), sl2x2), x0, x1);
              const float p0 = ex2(x0), p1 = ex2(x1);
              f2_unpack(f2_mul(f2_pack(p0, p1), f2_pack(__uint_as_float(d[2 * i]), __uint_as_float(d[2 * i + 1]))), s0,
                        s1);
              pp[i] = pack_bf16(p0, p1);
              pd[i] = pack_bf16(s0, s1);
            }
          } else if (m == 0u) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              pp[i] = 0u;
              pd[i] = 0u;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float x0, x1, s0, s1;
              f2_unpack(f2_mul(f2_pack(__uint_as_float(a[2 * i]), __uint_as_float(a[2 * i + 1])), sl2x2), x0, x1);
              float p0 = ex2(x0), p1 = ex2(x1);
              if (!((m >> (2 * i)) & 1u)) p0 = 0.f;
              if (!((m >> (2 * i + 1)) & 1u)) p1 = 0.f;
              f2_unpack(f2_mul(f2_pack(p0, p1), f2_pack(__uint_as_float(d[2 * i]), __uint_as_float(d[2 * i + 1]))), s0,
                        s1);
              pp[i] = pack_bf16(p0, p1);
              // masked entries: p = 0 exactly, so dS = 0 unless dP - Delta is not finite
              pd[i] = pack_bf16(p0 != 0.f ? s0 : 0.f, p1 != 0.f ? s1 : 0.f);
            }
          }
        }
        // Packed set b still feeds dV(G-2) / dK(G-2).  Every row thread
        // waits, active or not, so that no arrival for step G can land in
        // the pt_full phase of step G-2.
        if (G >= 2 && !__all_sync(0xffffffffu, mbar_wait(&acc_b[b], ((G - 2) >> 1) & 1, ab))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (active) {
          tmem_st16(tmem + 128 + 64 * b + lane_off + grp * 16, pp);
          tmem_st16(tmem + 160 + 64 * b + lane_off + grp * 16, pd);
          tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(&pt_full[b]);
      }
      if (!ok) break;
      // acc_done completes once per item, after the item's last dV / dK products
      ok = __all_sync(0xffffffffu, mbar_wait(acc_done, k & 1, ab));
      if (!ok) break;
      tc_fence_after();
      {
        // group 0 writes dV, group 1 writes scale * dK
        const bool owned = code != 15u && row < 16 * wk.n_own;
        const int64_t slot = owned ? pref_slot(wk.own_page(row >> 4), row & 15) : 0;
        const bool write = owned && slot < kv_slots;
        const int64_t base = (static_cast<int64_t>(wk.bh) * kv_slots + slot) * D;
        const uint32_t tacc = grp == 0 ? tDV : tDK;
        __nv_bfloat16* out = grp == 0 ? out_dv : out_dk;
        const float mul = grp == 0 ? 1.0f : scale;
#pragma unroll
        for (int pc = 0; pc < D / 32; ++pc) {
          uint32_t r[32] = {};
          if (n_steps > 0) {
            tmem_ld32(tacc + lane_off + pc * 32, r);
            tmem_wait_ld();
          }
          if (write) store_row32(out + base + pc * 32, r, mul, n_steps == 0);
        }
      }
      // the next item's dV / dK products may overwrite the accumulators
      tc_fence_before();
      mbar_arrive(acc_free);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ----------------------------------------------------------------------------
// K4: dQ (query-owned tiles, key pages as columns; the forward lists)
// ----------------------------------------------------------------------------
// TMEM columns: the owned Q rows as bf16 pairs at 0 (the A operand of
// S = Q K^T, so that MMA reads only K from shared memory), two fp32 staging
// sets (S at 64 + 64b, dP at 192 + 64b), two packed bf16 dS sets at 320 + 32p,
// dQ at 384.  A staging set is free as soon as the row threads have loaded
// it; a packed set is reused after the dQ MMAs of two steps back.
template <int D>
struct DqCfg {
  static constexpr int kNch = D / 64;
  static constexpr int kTile = kNch * kChunkBytes;        // dO tile (128 rows)
  static constexpr int kStagePages = 8;                   // two steps per stage
  static constexpr int kStageChunk = kStagePages * 16 * 128;
  static constexpr int kStageTile = kNch * kStageChunk;   // 128-row K / V stage
  static constexpr int kKStages = (D == 128) ? 3 : 5;
  static constexpr int kVStages = (D == 128) ? 3 : 5;
  static constexpr int kSmem = kTile + (kKStages + kVStages) * kStageTile + 1024 + 512;
};

template <int D>
__global__ void __launch_bounds__(kDkvThreads, 1)
    dq_kernel(const __nv_bfloat16* __restrict__ q, const __grid_constant__ TmaPages tm_do,
              const __grid_constant__ TmaPages tm_k, const __grid_constant__ TmaPages tm_v,
              const int32_t* __restrict__ work, const int32_t* __restrict__ col_pages,
              const uint64_t* __restrict__ col_masks, const float* __restrict__ lse, const float* __restrict__ delta,
              __nv_bfloat16* __restrict__ out_dq, int64_t q_slots, float sl2, float scale, int heads, int kv_group,
              int* err) {
  using C = DqCfg<D>;
  constexpr int KS = C::kKStages, VS = C::kVStages, NP = kBwdStepPages, SP = C::kStagePages;
  constexpr int SPS = SP / NP;  // steps per stage
  constexpr int kStageChunk = C::kStageChunk;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sDO = smem;
  uint8_t* sK = smem + C::kTile;           // K stage s at sK + s*kStageTile
  uint8_t* sV = sK + KS * C::kStageTile;   // V stage s at sV + s*kStageTile
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + VS * C::kStageTile);
  uint64_t* own_full = bars;
  uint64_t* q_ready = own_full + 1;  // Q rows stored into TMEM by the row threads
  uint64_t* k_full = q_ready + 1;
  uint64_t* k_empty = k_full + KS;
  uint64_t* v_full = k_empty + KS;
  uint64_t* v_empty = v_full + VS;
  uint64_t* sd_full = v_empty + VS;  // [2] S and dP of a step are in staging set b
  uint64_t* s_free = sd_full + 2;    // [2] the row threads have loaded staging set b
  uint64_t* ds_full = s_free + 2;    // [2] dS of a step is in packed set p
  uint64_t* dq_done = ds_full + 2;   // [2] dQ MMAs of the steps using packed set p finished
  uint64_t* acc_done = dq_done + 2;
  uint64_t* drain = acc_done + 1;    // [2] one per issuing warp
  uint32_t* tslot = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  const Abort ab{abort_flag, err};

  const Work wk = load_work(work, blockIdx.x);
  // K/V head of this item's query head (grouped-query attention)
  const int kv_bh = (wk.bh / heads) * (heads / kv_group) + (wk.bh % heads) / kv_group;
  const int n_cols = wk.e1 - wk.e0;
  const int n_steps = (n_cols + NP - 1) / NP;
  const int warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(own_full, 1);
    mbar_init(q_ready, 256);
    for (int s = 0; s < KS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sd_full[b], 1);
      mbar_init(&s_free[b], 256);
      mbar_init(&ds_full[b], 256);
      mbar_init(&dq_done[b], 1);
    }
    mbar_init(acc_done, 1);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t tQ = tmem, tDQ = tmem + 384;
  auto tS = [&](int b) { return tmem + 64 + 64 * b; };
  auto tDP = [&](int b) { return tmem + 192 + 64 * b; };
  auto tPk = [&](int p) { return tmem + 320 + 32 * p; };

  if (warp == 0 || warp == kDoWarp) {
    // ---------------- producers (whole warps): warp 0 = K stages, warp 11 = V stages ----------------
    // Lane j owns page j of a 128-row stage; page ids are fetched one stage
    // ahead.
    const bool is_k = warp == 0;
    const int NS = is_k ? KS : VS;
    uint8_t* stage0 = is_k ? sK : sV;
    uint64_t* full = is_k ? k_full : v_full;
    uint64_t* empty = is_k ? k_empty : v_empty;
    const TmaPages& tm = is_k ? tm_k : tm_v;
    if (is_k) {
      if (lane == 0) {
        tma_prefetch_desc(&tm_do.m64);
        mbar_arrive_expect_tx(own_full, wk.n_own * C::kNch * 2048);
      }
      __syncwarp();
      load_page_runs<C::kNch>(sDO, kChunkBytes, tm_do, lane < wk.n_own ? wk.own_page(lane) : 0, wk.n_own, wk.bh,
                              own_full);
    }
    if (lane == 0) {
      tma_prefetch_desc(&tm.m64w);
      tma_prefetch_desc(&tm.m64);
    }
    __syncwarp();
    const int n_stages = (n_cols + SP - 1) / SP;
    int pid_next = (n_stages > 0 && lane < min(SP, n_cols)) ? __ldg(col_pages + wk.e0 + lane) : 0;
    int issued = 0;
    for (int t = 0; t < n_stages; ++t) {
      const int s = t % NS;
      const int n = min(SP, n_cols - t * SP);
      const int pid = pid_next;
      if (t + 1 < n_stages)
        pid_next = lane < min(SP, n_cols - (t + 1) * SP) ? __ldg(col_pages + wk.e0 + (t + 1) * SP + lane) : 0;
      if (t >= NS && !__all_sync(0xffffffffu, mbar_wait(&empty[s], ((t / NS) - 1) & 1, ab))) break;
      if (lane == 0) mbar_arrive_expect_tx(&full[s], n * C::kNch * 2048);
      __syncwarp();
      load_page_runs<C::kNch>(stage0 + s * C::kStageTile, kStageChunk, tm, pid, n, kv_bh, &full[s]);
      issued = t + 1;
    }
    if (lane == 0) {
      for (int t = max(0, issued - NS); t < issued; ++t) mbar_wait_drain(&full[t % NS], (t / NS) & 1);
      if (is_k) mbar_wait_drain(own_full, 0);
    }
  } else if (warp == 1) {
    // ---------------- S, dP issuer (warp-wide; one elected lane issues) ----------------
    const uint64_t ddo0 = sdesc_sw128(smem_u32(sDO), 16, 1024);
    const uint64_t dkk = sdesc_sw128(smem_u32(sK), 16, 1024);            // K stages, K-major
    const uint64_t dvk = sdesc_sw128(smem_u32(sV), 16, 1024);            // V stages, K-major
    bool ok = __all_sync(0xffffffffu, mbar_wait(own_full, 0, ab) && mbar_wait(q_ready, 0, ab));
    tc_fence_after();
    for (int st = 0; ok && st < n_steps; ++st) {
      const int b = st & 1, t = st / SPS, half = st % SPS, ks = t % KS, vs = t % VS;
      const bool stage_end = half == SPS - 1 || st + 1 == n_steps;
      const int n = min(NP, n_cols - st * NP);
      const uint32_t idesc_s = idesc_bf16(128, 16 * n, false, false);
      // staging set b is free once the row threads have loaded step st-2
      bool w = (st < 2 || mbar_wait(&s_free[b], ((st - 2) >> 1) & 1, ab)) && mbar_wait(&k_full[ks], (t / KS) & 1, ab);
      if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      tc_fence_after();
      const uint64_t bk = sdesc_add(dkk, ks * C::kStageTile + half * kHalfStage);
      const uint64_t bv = sdesc_add(dvk, vs * C::kStageTile + half * kHalfStage);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        umma_ts_w(tS(b), tQ + 8 * kk, sdesc_add(bk, (kk >> 2) * kStageChunk + (kk & 3) * 32), idesc_s, kk > 0);
      if (!__all_sync(0xffffffffu, mbar_wait(&v_full[vs], (t / VS) & 1, ab))) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        umma_ss_w(tDP(b), sdesc_add(ddo0, (kk >> 2) * kChunkBytes + (kk & 3) * 32),
                  sdesc_add(bv, (kk >> 2) * kStageChunk + (kk & 3) * 32), idesc_s, kk > 0);
      if (stage_end) umma_commit_w(&v_empty[vs]);
      umma_commit_w(&sd_full[b]);
    }
    umma_commit_w(&drain[0]);
    mbar_wait_drain(&drain[0], 0);
  } else if (warp == kAccWarp) {
    // ---------------- dQ issuer (warp-wide; one elected lane issues) ----------------
    const uint64_t dkm = sdesc_sw128(smem_u32(sK), kStageChunk, 1024);   // K stages, MN-major
    const uint32_t idesc_acc = idesc_bf16(128, D, false, true);
    bool ok = true;
    for (int st = 0; ok && st < n_steps; ++st) {
      const int p = st & 1, t = st / SPS, half = st % SPS, ks = t % KS;
      const bool stage_end = half == SPS - 1 || st + 1 == n_steps;
      if (!__all_sync(0xffffffffu, mbar_wait(&ds_full[p], (st >> 1) & 1, ab))) { ok = false; break; }
      tc_fence_after();
      const int n = min(NP, n_cols - st * NP);
      const uint64_t bk = sdesc_add(dkm, ks * C::kStageTile + half * kHalfStage);
#pragma unroll
      for (int j = 0; j < NP; ++j)
        if (j < n) umma_ts_w(tDQ, tPk(p) + 8 * j, sdesc_add(bk, j * 2048), idesc_acc, (st > 0 || j > 0) ? 1u : 0u);
      if (stage_end) umma_commit_w(&k_empty[ks]);
      umma_commit_w(&dq_done[p]);
    }
    if (ok && n_steps > 0) umma_commit_w(acc_done);
    umma_commit_w(&drain[1]);
    mbar_wait_drain(&drain[1], 0);
  } else {
    const int grp = (warp - 2) >> 2;  // column half of each step
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t code = wk.row_code(row);
    const int seg = code < 8 ? static_cast<int>(code) : -1;
    const bool owned = code != 15u && row < 16 * wk.n_own;
    const int64_t slot = row < 16 * wk.n_own ? pref_slot(wk.own_page(row >> 4), row & 15) : 0;
    const bool loaded = row < 16 * wk.n_own && slot < q_slots;
    const bool valid_slot = owned && slot < q_slots;
    const int64_t roff = static_cast<int64_t>(wk.bh) * q_slots + slot;
    // Q row into TMEM as bf16 pairs: group g stores pair columns [g*D/4, (g+1)*D/4)
    {
      constexpr int kCols = D / 4;  // 32-bit TMEM columns per group
      uint32_t qr[32] = {};
      if (loaded) {
        const uint4* src = reinterpret_cast<const uint4*>(q + roff * D + grp * (D / 2));
#pragma unroll
        for (int i = 0; i < kCols / 4; ++i) {
          const uint4 v = __ldg(src + i);
          qr[4 * i] = v.x;
          qr[4 * i + 1] = v.y;
          qr[4 * i + 2] = v.z;
          qr[4 * i + 3] = v.w;
        }
      }
      if (kCols == 32) {
        tmem_st32(tQ + lane_off + grp * kCols, qr);
      } else {
        uint32_t h[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) h[i] = qr[i];
        tmem_st16(tQ + lane_off + grp * kCols, h);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(q_ready);
    }
    const float lse2 = (valid_slot && seg >= 0) ? __ldg(lse + roff) * kLog2e : 0.f;
    const float dl = (valid_slot && seg >= 0) ? __ldg(delta + roff) : 0.f;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    const uint64_t nl2 = f2_pack(-lse2, -lse2);
    const uint64_t ndl = f2_pack(-dl, -dl);
    bool ok = true;
    StepMasks<NP> raw;
    if (n_steps > 0) raw.fetch(col_masks, wk.e0, min(NP, n_cols), seg);
    for (int st = 0; st < n_steps; ++st) {
      const int b = st & 1;
      const int N = 16 * min(NP, n_cols - st * NP);
      const bool active = grp * 32 < N;
      uint32_t mw[2];
      raw.bits(mw);
      // mask words of the next step load while this one computes
      if (st + 1 < n_steps) raw.fetch(col_masks, wk.e0 + (st + 1) * NP, min(NP, n_cols - (st + 1) * NP), seg);
      ok = __all_sync(0xffffffffu, mbar_wait(&sd_full[b], (st >> 1) & 1, ab));
      if (!ok) break;
      tc_fence_after();
      uint32_t a[32], d[32];
      if (active) {
        tmem_ld32(tS(b) + lane_off + grp * 32, a);
        tmem_ld32(tDP(b) + lane_off + grp * 32, d);
        tmem_wait_ld();
      }
      tc_fence_before();
      mbar_arrive(&s_free[b]);
      uint32_t pd[16];
      if (active) {
        const uint32_t m = grp ? mw[1] : mw[0];
        if (m == 0xFFFFFFFFu) {
          // every column allowed: no masking, all values finite
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float x0, x1, g0, g1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(a[2 * i]), __uint_as_float(a[2 * i + 1])), sl2x2, nl2), x0, x1);
            f2_unpack(f2_mul(f2_pack(ex2(x0), ex2(x1)),
                             f2_add(f2_pack(__uint_as_float(d[2 * i]), __uint_as_float(d[2 * i + 1])), ndl)),
                      g0, g1);
            pd[i] = pack_bf16(g0, g1);
          }
        } else if (m == 0u) {
#pragma unroll
          for (int i = 0; i < 16; ++i) pd[i] = 0u;
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(a[2 * i]), __uint_as_float(a[2 * i + 1])), sl2x2, nl2), x0, x1);
            float p0 = ex2(x0), p1 = ex2(x1);
            if (!((m >> (2 * i)) & 1u)) p0 = 0.f;
            if (!((m >> (2 * i + 1)) & 1u)) p1 = 0.f;
            float g0, g1;
            f2_unpack(f2_mul(f2_pack(p0, p1), f2_add(f2_pack(__uint_as_float(d[2 * i]), __uint_as_float(d[2 * i + 1])), ndl)),
                      g0, g1);
            pd[i] = pack_bf16(p0 != 0.f ? g0 : 0.f, p1 != 0.f ? g1 : 0.f);
          }
        }
      }
      // Packed set b still feeds dQ(st-2).  Every row thread waits, active or
      // not: dq_done(st-2) implies that ds_full finished the phase of step
      // st-2, so no thread can arrive for step st while that phase is open.
      if (st >= 2 && !__all_sync(0xffffffffu, mbar_wait(&dq_done[b], ((st - 2) >> 1) & 1, ab))) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (active) {
        tmem_st16(tPk(b) + lane_off + grp * 16, pd);
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&ds_full[b]);
    }
    if (ok && n_steps > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(acc_done, 0, ab));
      tc_fence_after();
    }
    if (ok) {
      // group g writes columns [g*D/2, (g+1)*D/2) of dQ
      __nv_bfloat16* dst = out_dq + roff * D;
#pragma unroll
      for (int pc = 0; pc < D / 64; ++pc) {
        const int col = grp * (D / 2) + pc * 32;
        uint32_t r[32] = {};
        if (n_steps > 0) {
          tmem_ld32(tDQ + lane_off + col, r);
          tmem_wait_ld();
        }
        if (valid_slot) store_row32(dst + col, r, scale, n_steps == 0);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_delta(int head_dim, const __nv_bfloat16* o, const __nv_bfloat16* d_o, float* delta, int64_t rows,
                         cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  const int64_t threads = rows * (head_dim / 8);
  const int64_t blocks = std::min<int64_t>((threads + 255) / 256, 148 * 16);
  if (head_dim == 128)
    delta_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, st>>>(o, d_o, delta, rows);
  else
    delta_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, st>>>(o, d_o, delta, rows);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_dkdv_t(const TmaPages& tk, const TmaPages& tv, const TmaPages& tq,
                                 const TmaPages& tdo, const TileArgs& a, const float* lse, const float* delta,
                                 __nv_bfloat16* dk, __nv_bfloat16* dv, cudaStream_t st) {
  using C = DkvCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess || a.n_work == 0) return e;
  // one persistent CTA per SM (at most one item each when there are fewer items)
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess) e = cudaMemsetAsync(a.sched, 0, sizeof(int), st);
  if (e != cudaSuccess) return e;
  const int64_t grid = std::min<int64_t>(a.n_work, std::max(sms, 1));
  dkdv_kernel<D><<<static_cast<unsigned>(grid), kDkvThreads, C::kSmem, st>>>(
      tk, tv, tq, tdo, a.work, a.n_work, a.sched, a.pages, a.masks, lse, delta, dk, dv, a.own_slots, a.col_slots,
      a.scale * kLog2e, a.scale, a.heads, a.kv_heads, a.kv_group, a.col_heads, a.err);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_dq_t(const __nv_bfloat16* q, const TmaPages& tdo, const TmaPages& tk,
                               const TmaPages& tv, const TileArgs& a, const float* lse, const float* delta,
                               __nv_bfloat16* dq, cudaStream_t st) {
  using C = DqCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess || a.n_work == 0) return e;
  dq_kernel<D><<<static_cast<unsigned>(a.n_work), kDkvThreads, C::kSmem, st>>>(
      q, tdo, tk, tv, a.work, a.pages, a.masks, lse, delta, dq, a.own_slots, a.scale * kLog2e, a.scale, a.heads,
      a.kv_group, a.err);
  return cudaGetLastError();
}

cudaError_t launch_dkdv(int head_dim, const TmaPages& tk, const TmaPages& tv, const TmaPages& tq, const TmaPages& tdo,
                        const TileArgs& a, const float* lse, const float* delta, __nv_bfloat16* dk,
                        __nv_bfloat16* dv, cudaStream_t st) {
  return head_dim == 128 ? launch_dkdv_t<128>(tk, tv, tq, tdo, a, lse, delta, dk, dv, st)
                         : launch_dkdv_t<64>(tk, tv, tq, tdo, a, lse, delta, dk, dv, st);
}

cudaError_t launch_dq(int head_dim, const __nv_bfloat16* q, const TmaPages& tdo, const TmaPages& tk,
                      const TmaPages& tv, const TileArgs& a, const float* lse, const float* delta,
                      __nv_bfloat16* dq, cudaStream_t st) {
  return head_dim == 128 ? launch_dq_t<128>(q, tdo, tk, tv, a, lse, delta, dq, st)
                         : launch_dq_t<64>(q, tdo, tk, tv, a, lse, delta, dq, st);
}

}  // namespace spattn
