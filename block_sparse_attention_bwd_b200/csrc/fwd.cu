// K1: forward attention over packed pages, and K5: fill of page-sized holes.
//
// Method (KPage abstract, "KPage: block-sparse attention for partially
// occupied 3D blocks", zhuanzhiai.com, abstract paragraph): valid 16-row K/V
// pages are packed into large tiles while they are loaded, with no compacted
// copy in HBM, and masking stays exact.  The softmax is the online
// (streaming) form used by FlashAttention-style kernels.
//
// One CTA runs one query-owned work item: up to 8 query pages (128 rows,
// TMEM lanes) against its list of key pages, 4 pages (64 columns) per step.
//   warp 0      TMA producer: query pages once, then K and V pages of each
//               step into two-deep rings, one box per run of consecutive
//               pages (or per strided page) and 64-column chunk, gathered
//               straight from [B,H,S,D] memory;
//   warp 1      allocates TMEM and issues tcgen05 MMAs from one thread:
//               S_b = Q K^T into one of two TMEM buffers, then O += P V with
//               P read from TMEM (bf16, written over S_b by the softmax);
//   warps 2..5  one tile row per thread: exact mask from the step's page
//               masks, running max with lazy rescaling, P in bf16 to TMEM,
//               and the epilogue (O / l, LSE in natural log).
// S is double-buffered, so the MMA of step c+1 overlaps the softmax of c.
//
// 64-row route (the kernel form with ROUTE, for work lists that hold routed
// items): rows 0..63 and 64..127 each run over their own two pages of every
// step, as two M = 64 products written to the same 32 columns at TMEM lane
// offsets 0 and 16 (row r of half h at lane 16h + r % 16 + 32 (r / 16)),
// and two M = 64 P.V products that read P from those lanes.
#include "kernels.cuh"
#include "tile.cuh"

namespace spattn {
namespace {

using namespace dev;

// 64 key columns (4 pages) per step; two CTAs share an SM (256 TMEM columns
// and < 113 KB of shared memory each), so the row threads of one CTA compute
// while the tensor core runs the other CTA's MMAs.
constexpr int kFwdStepPages = 4;
constexpr int kFwdStageChunk = 64 * 128;  // one 64-column chunk of a 64-row stage

// F8: Q and K are E4M3 codes (one byte per element, so a 128-byte swizzle
// row holds 128 of them) and S = Q K^T is a kind::f8f6f4 product; V, P and O
// stay bf16.
template <int D, bool F8>
struct FwdCfg {
  static constexpr int kNch = D / 64;                       // 64-column bf16 chunks (V)
  static constexpr int kQKNch = F8 ? D / 128 : D / 64;      // 128-byte chunks of a Q or K row
  static constexpr int kTile = kQKNch * kChunkBytes;        // 128-row query tile
  static constexpr int kKStage = kQKNch * kFwdStageChunk;   // 64-row K stage
  static constexpr int kVStage = kNch * kFwdStageChunk;     // 64-row V stage
  static constexpr int kKStages = (D == 128 && !F8) ? 2 : 4;  // K ring depth
  static constexpr int kVStages = (D == 128) ? 2 : 4;         // V ring depth
  static constexpr int kSmem = kTile + kKStages * kKStage + kVStages * kVStage + 1024 + 512;
  static_assert(!F8 || D == 128, "the E4M3 forward has D = 128 (one 128-byte row per chunk)");
};

// Rescale O only when the running max grows by more than 2^8 (log2 units):
// P stays below 256 and the final O / l is unchanged.
constexpr float kRescaleThreshold = 8.0f;

// 6 warps: 0 = TMA producer, 1 = TMEM owner and MMA issuer, 2..5 = row
// threads (warp w reaches TMEM lanes 32*(w%4) .. 32*(w%4)+31).
constexpr int kFwdThreads = 192;

// ROUTE: the form that reads each item's route flag (the 64-row route of
// Work::halves); without it every item runs as 128 rows over its whole list.
template <int D, bool F8, bool ROUTE>
__global__ void __launch_bounds__(kFwdThreads, 2)
    fwd_kernel(const __grid_constant__ TmaPages tm_q, const __grid_constant__ TmaPages tm_k,
               const __grid_constant__ TmaPages tm_v, const int32_t* __restrict__ work,
               const int32_t* __restrict__ col_pages, const uint64_t* __restrict__ col_masks,
               __nv_bfloat16* __restrict__ out_o, float* __restrict__ out_lse, int64_t q_slots, float sl2,
               int heads, int kv_group, const float* __restrict__ q_descale, const float* __restrict__ k_descale,
               int* err) {
  using C = FwdCfg<D, F8>;
  constexpr int KS = C::kKStages, VS = C::kVStages, NP = kFwdStepPages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sQ = smem;
  uint8_t* sK = smem + C::kTile;          // K stage s at sK + s*kKStage
  uint8_t* sV = sK + KS * C::kKStage;     // V stage s at sV + s*kVStage
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + VS * C::kVStage);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;
  uint64_t* k_empty = k_full + KS;
  uint64_t* v_full = k_empty + KS;
  uint64_t* v_empty = v_full + VS;
  uint64_t* s_full = v_empty + VS;  // [2]
  uint64_t* p_full = s_full + 2;    // [2]
  uint64_t* o_done = p_full + 2;
  uint64_t* drain = o_done + 1;
  uint64_t* o_last = drain + 1;     // the last PV has finished
  uint32_t* tslot = reinterpret_cast<uint32_t*>(o_last + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  const Abort ab{abort_flag, err};

  const Work wk = load_work(work, blockIdx.x);
  // K/V head of this item's query head (grouped-query attention)
  const int kv_bh = (wk.bh / heads) * (heads / kv_group) + (wk.bh % heads) / kv_group;
  const int n_cols = wk.e1 - wk.e0;
  const int n_steps = (n_cols + NP - 1) / NP;
  // 64-row route: every step holds two pages per half (a list of whole steps)
  const bool halves = ROUTE && wk.halves() && (n_cols % NP) == 0;
  const int warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 128);
    }
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    mbar_init(o_last, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tslot, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t tO = tmem + 128;  // S buffers at columns 0 and 64

  if (warp == 0) {
    // ---------------- producer (whole warp): K runs ahead of V ----------------
    // Lane j < n owns page j of a step: it holds the page id (fetched one step
    // ahead) and issues that page's TMA boxes.
    if (lane == 0) {
      tma_prefetch_desc(&tm_q.m64);
      tma_prefetch_desc(&tm_k.m64);
      tma_prefetch_desc(&tm_v.m64);
      tma_prefetch_desc(&tm_k.m16);
      tma_prefetch_desc(&tm_v.m16);
      mbar_arrive_expect_tx(q_full, wk.n_own * C::kQKNch * 2048);
    }
    __syncwarp();
    load_page_runs<C::kQKNch>(sQ, kChunkBytes, tm_q, lane < wk.n_own ? wk.own_page(lane) : 0, wk.n_own, wk.bh,
                              q_full);
    int pid_next = (n_steps > 0 && lane < min(NP, n_cols)) ? __ldg(col_pages + wk.e0 + lane) : 0;
    int k_issued = 0, v_issued = 0;
    for (int st = 0; st < n_steps; ++st) {
      const int n = min(NP, n_cols - st * NP);
      const int pid = pid_next;
      if (st + 1 < n_steps)
        pid_next = lane < min(NP, n_cols - (st + 1) * NP) ? __ldg(col_pages + wk.e0 + (st + 1) * NP + lane) : 0;
      const int ks = st % KS, vs = st % VS;
      if (st >= KS && !__all_sync(0xffffffffu, mbar_wait(&k_empty[ks], ((st / KS) - 1) & 1, ab))) break;
      if (lane == 0) mbar_arrive_expect_tx(&k_full[ks], n * C::kQKNch * 2048);
      __syncwarp();
      load_page_runs<C::kQKNch>(sK + ks * C::kKStage, kFwdStageChunk, tm_k, pid, n, kv_bh, &k_full[ks]);
      k_issued = st + 1;
      if (st >= VS && !__all_sync(0xffffffffu, mbar_wait(&v_empty[vs], ((st / VS) - 1) & 1, ab))) break;
      if (lane == 0) mbar_arrive_expect_tx(&v_full[vs], n * C::kNch * 2048);
      __syncwarp();
      load_page_runs<C::kNch>(sV + vs * C::kVStage, kFwdStageChunk, tm_v, pid, n, kv_bh, &v_full[vs]);
      v_issued = st + 1;
    }
    // no copy may still be landing in shared memory when the CTA exits
    if (lane == 0) {
      for (int st = max(0, k_issued - KS); st < k_issued; ++st) mbar_wait_drain(&k_full[st % KS], (st / KS) & 1);
      for (int st = max(0, v_issued - VS); st < v_issued; ++st) mbar_wait_drain(&v_full[st % VS], (st / VS) & 1);
      mbar_wait_drain(q_full, 0);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (warp-wide; one elected lane issues) ----------------
    const uint64_t dq0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t dk0 = sdesc_sw128(smem_u32(sK), 16, 1024);
    const uint64_t dv0 = sdesc_sw128(smem_u32(sV), kFwdStageChunk, 1024);
    const uint32_t idesc_pv = idesc_bf16(128, D, false, true);
    const uint32_t idesc_pv64 = idesc_bf16(64, D, false, true);
    bool ok = __all_sync(0xffffffffu, mbar_wait(q_full, 0, ab));
    tc_fence_after();
    auto issue_pv = [&](int st) -> bool {
      const int b = st & 1, vs = st % VS;
      const bool w = mbar_wait(&p_full[b], (st >> 1) & 1, ab) && mbar_wait(&v_full[vs], (st / VS) & 1, ab);
      if (!__all_sync(0xffffffffu, w)) return false;
      tc_fence_after();
      const int n = min(NP, n_cols - st * NP);
      const uint64_t dv = sdesc_add(dv0, vs * C::kVStage);
      if (halves) {
        // O_h += P_h V_h: half h's P (lanes from 16h) against the step's pages 2h, 2h+1
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int j = 0; j < 2; ++j)
            umma_ts_w(tO + (static_cast<uint32_t>(16 * h) << 16),
                      tmem + 64 * b + (static_cast<uint32_t>(16 * h) << 16) + 8 * j,
                      sdesc_add(dv, (2 * h + j) * 2048), idesc_pv64, (st > 0 || j > 0) ? 1u : 0u);
      } else {
#pragma unroll
        for (int j = 0; j < NP; ++j)
          if (j < n)
            umma_ts_w(tO, tmem + 64 * b + 8 * j, sdesc_add(dv, j * 2048), idesc_pv, (st > 0 || j > 0) ? 1u : 0u);
      }
      umma_commit_w(&v_empty[vs]);
      umma_commit_w(o_done);
      return true;
    };
    for (int st = 0; ok && st < n_steps; ++st) {
      const int ks = st % KS, b = st & 1;
      // buffer b still holds P(st-2), the TMEM A operand of PV(st-2); let
      // that MMA finish before S(st) overwrites it (waited every step, in
      // order, so the parity is unambiguous)
      const bool w = mbar_wait(&k_full[ks], (st / KS) & 1, ab) && (st < 2 || mbar_wait(o_done, (st - 2) & 1, ab));
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int n = min(NP, n_cols - st * NP);
      const uint64_t dk = sdesc_add(dk0, ks * C::kKStage);
      if (halves) {
        // S_h = Q_h K_h^T (M = 64, N = 32) for h = 0, 1: query rows 64h.. (8 KB
        // into each chunk) against stage rows 32h.. (4 KB), written to the
        // same 32 columns of buffer b at TMEM lanes offset by 16 h, so that
        // row r of half h sits at lane 16 h + r % 16 + 32 (r / 16)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t d = tmem + 64 * b + (static_cast<uint32_t>(16 * h) << 16);
          if constexpr (F8) {
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk)
              umma_ss_e4m3_w(d, sdesc_add(dq0, (kk >> 2) * kChunkBytes + (kk & 3) * 32 + h * 8192),
                             sdesc_add(dk, (kk >> 2) * kFwdStageChunk + (kk & 3) * 32 + h * 4096), idesc_e4m3(64, 32),
                             kk > 0 ? 1u : 0u);
          } else {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              umma_ss_w(d, sdesc_add(dq0, (kk >> 2) * kChunkBytes + (kk & 3) * 32 + h * 8192),
                        sdesc_add(dk, (kk >> 2) * kFwdStageChunk + (kk & 3) * 32 + h * 4096),
                        idesc_bf16(64, 32, false, false), kk > 0 ? 1u : 0u);
          }
        }
      } else if constexpr (F8) {
        // 32 E4M3 elements (32 bytes) of K per MMA
        const uint32_t idesc_s = idesc_e4m3(128, 16 * n);
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)
          umma_ss_e4m3_w(tmem + 64 * b, sdesc_add(dq0, (kk >> 2) * kChunkBytes + (kk & 3) * 32),
                         sdesc_add(dk, (kk >> 2) * kFwdStageChunk + (kk & 3) * 32), idesc_s, kk > 0 ? 1u : 0u);
      } else {
        const uint32_t idesc_s = idesc_bf16(128, 16 * n, false, false);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss_w(tmem + 64 * b, sdesc_add(dq0, (kk >> 2) * kChunkBytes + (kk & 3) * 32),
                    sdesc_add(dk, (kk >> 2) * kFwdStageChunk + (kk & 3) * 32), idesc_s, kk > 0 ? 1u : 0u);
      }
      umma_commit_w(&s_full[b]);
      umma_commit_w(&k_empty[ks]);
      if (st >= 1 && !issue_pv(st - 1)) ok = false;
    }
    if (ok && n_steps > 0 && issue_pv(n_steps - 1)) umma_commit_w(o_last);
    umma_commit_w(drain);
    mbar_wait_drain(drain, 0);
  } else {
    // ---------------- softmax + epilogue (one row per thread) ----------------
    const int q4 = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    // tile row of this thread's TMEM lane 32 q4 + lane: the lane itself, or
    // in the 64-row route row (lane % 16) + 16 q4 of half hh
    const int hh = (lane >> 4) & 1;
    const int row = halves ? 64 * hh + (lane & 15) + 16 * q4 : q4 * 32 + lane;
    const uint32_t code = wk.row_code(row);
    const int seg = code < 8 ? static_cast<int>(code) : -1;
    if constexpr (F8) sl2 *= __ldg(q_descale + wk.bh) * __ldg(k_descale + kv_bh);  // scores of the dequantised Q, K
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    StepMasks<NP> raw;
    if (n_steps > 0) raw.fetch(col_masks, wk.e0, min(NP, n_cols), seg);
    for (int st = 0; st < n_steps; ++st) {
      const int b = st & 1;
      // the 64-row route: 32 columns (this half's two pages) in the low half of S
      const int N = halves ? 32 : 16 * min(NP, n_cols - st * NP);
      uint32_t mw[2];
      raw.bits(mw);
      if (halves && hh) mw[0] = mw[1];
      // mask words of the next step load while this one computes
      if (st + 1 < n_steps) raw.fetch(col_masks, wk.e0 + (st + 1) * NP, min(NP, n_cols - (st + 1) * NP), seg);
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[b], (st >> 1) & 1, ab));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[2][32];
#pragma unroll
      for (int pc = 0; pc < 2; ++pc)
        if (pc * 32 < N) tmem_ld32(tmem + 64 * b + lane_off + pc * 32, sr[pc]);
      tmem_wait_ld();
      // masked row max over four independent chains
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int pc = 0; pc < 2; ++pc) {
        if (pc * 32 < N) {
          if (mw[pc] != 0xFFFFFFFFu) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (!((mw[pc] >> i) & 1u)) sr[pc][i] = 0xFF800000u;  // -inf
          }
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            mx[0] = fmax3(mx[0], __uint_as_float(sr[pc][i]), __uint_as_float(sr[pc][i + 1]));
            mx[1] = fmax3(mx[1], __uint_as_float(sr[pc][i + 2]), __uint_as_float(sr[pc][i + 3]));
            mx[2] = fmax3(mx[2], __uint_as_float(sr[pc][i + 4]), __uint_as_float(sr[pc][i + 5]));
            mx[3] = fmax3(mx[3], __uint_as_float(sr[pc][i + 6]), __uint_as_float(sr[pc][i + 7]));
          }
        }
      }
      const float mx2 = fmax3(mx[0], mx[1], fmaxf(mx[2], mx[3])) * sl2;  // log2 units (scale > 0)
      const bool resc = mx2 > m_used + kRescaleThreshold;
      const float m_new = resc ? mx2 : m_used;
      const float alpha = resc ? ex2(m_used - m_new) : 1.0f;
      l *= alpha;
      m_used = m_new;
      const float neg_mu = (m_used == -INFINITY) ? 0.f : -m_used;
      const uint64_t nmu2 = f2_pack(neg_mu, neg_mu);
      uint64_t ls2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
      for (int pc = 0; pc < 2; ++pc) {
        if (pc * 32 < N) {
          uint32_t pk[16];
          if (mw[pc] == 0u) {
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = 0u;
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float x0, x1;
              f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[pc][2 * i]), __uint_as_float(sr[pc][2 * i + 1])), sl2x2, nmu2),
                        x0, x1);
              const float p0 = ex2(x0), p1 = ex2(x1);
              ls2[i & 1] = f2_add(ls2[i & 1], f2_pack(p0, p1));
              pk[i] = pack_bf16(p0, p1);
            }
          }
          tmem_st16(tmem + 64 * b + lane_off + pc * 16, pk);
        }
      }
      {
        float a0, a1, b0, b1;
        f2_unpack(ls2[0], a0, a1);
        f2_unpack(ls2[1], b0, b1);
        l += (a0 + a1) + (b0 + b1);
      }
      if (st > 0 && __any_sync(0xffffffffu, resc)) {
        // O must hold steps < st before this warp's rows are rescaled, so
        // wait for PV(st-1) here (only here: P(st) needs no wait).  S(st) was
        // issued after PV(st-2) finished and PV(st) waits for this step's
        // arrival, so o_done has completed st-1 or st phases and the parity
        // wait is unambiguous.
        ok = __all_sync(0xffffffffu, mbar_wait(o_done, (st - 1) & 1, ab));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int pc = 0; pc < D / 32; ++pc) {
          uint32_t r[32];
          tmem_ld32(tO + lane_off + pc * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(tO + lane_off + pc * 32, r);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[b]);
    }
    if (ok && n_steps > 0) {
      ok = mbar_wait(o_last, 0, ab);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
    }
    if (ok) {
      const bool owned = code != 15u && row < 16 * wk.n_own;
      const int64_t slot = owned ? pref_slot(wk.own_page(row >> 4), row & 15) : 0;
      const bool write = owned && slot < q_slots;
      const bool empty = !(l > 0.f);
      const float inv = empty ? 0.f : 1.0f / l;
      __nv_bfloat16* dst = out_o + (static_cast<int64_t>(wk.bh) * q_slots + slot) * D;
#pragma unroll
      for (int pc = 0; pc < D / 32; ++pc) {
        uint32_t r[32] = {};
        if (n_steps > 0) {
          tmem_ld32(tO + lane_off + pc * 32, r);
          tmem_wait_ld();
        }
        if (write) store_row32(dst + pc * 32, r, inv, empty || n_steps == 0);
      }
      if (write) out_lse[static_cast<int64_t>(wk.bh) * q_slots + slot] = empty ? -INFINITY : (m_used + lg2(l)) * kLn2;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// Zero the rows that no work item writes: entry e of `fill` is a page and a
// 16-bit row mask; LSE rows (if given) get -inf.
__global__ void fill_kernel(const int32_t* __restrict__ fill, int64_t n_bh, int64_t slots, int head_dim,
                            __nv_bfloat16* __restrict__ t0, __nv_bfloat16* __restrict__ t1, float* __restrict__ lse) {
  const int64_t page = fill[2 * blockIdx.x];
  const uint32_t rows = static_cast<uint32_t>(fill[2 * blockIdx.x + 1]);
  const int vec_per_row = head_dim / 8;  // 16-byte vectors
  for (int64_t bh = blockIdx.y; bh < n_bh; bh += gridDim.y) {
    for (int i = threadIdx.x; i < 16 * vec_per_row; i += blockDim.x) {
      const int r = i / vec_per_row, c = i % vec_per_row;
      const int64_t slot = page * 16 + r;
      if (slot >= slots || !((rows >> r) & 1u)) continue;
      const int64_t off = (bh * slots + slot) * head_dim + c * 8;
      if (t0) *reinterpret_cast<uint4*>(t0 + off) = make_uint4(0, 0, 0, 0);
      if (t1) *reinterpret_cast<uint4*>(t1 + off) = make_uint4(0, 0, 0, 0);
    }
    if (lse && threadIdx.x < 16) {
      const int64_t slot = page * 16 + threadIdx.x;
      if (slot < slots && ((rows >> threadIdx.x) & 1u)) lse[bh * slots + slot] = -INFINITY;
    }
  }
}

template <int D, bool F8, bool ROUTE>
cudaError_t launch_fwd_r(const TmaPages& tq, const TmaPages& tk, const TmaPages& tv, const TileArgs& a,
                         __nv_bfloat16* o, float* lse, const float* q_descale, const float* k_descale,
                         cudaStream_t st) {
  using C = FwdCfg<D, F8>;
  cudaError_t e =
      cudaFuncSetAttribute(fwd_kernel<D, F8, ROUTE>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  if (a.n_work == 0) return cudaSuccess;
  fwd_kernel<D, F8, ROUTE><<<static_cast<unsigned>(a.n_work), kFwdThreads, C::kSmem, st>>>(
      tq, tk, tv, a.work, a.pages, a.masks, o, lse, a.own_slots, a.scale * kLog2e, a.heads, a.kv_group, q_descale,
      k_descale, a.err);
  return cudaGetLastError();
}

template <int D, bool F8>
cudaError_t launch_fwd_t(const TmaPages& tq, const TmaPages& tk, const TmaPages& tv, const TileArgs& a,
                         __nv_bfloat16* o, float* lse, const float* q_descale, const float* k_descale,
                         cudaStream_t st) {
  return a.route64 ? launch_fwd_r<D, F8, true>(tq, tk, tv, a, o, lse, q_descale, k_descale, st)
                   : launch_fwd_r<D, F8, false>(tq, tk, tv, a, o, lse, q_descale, k_descale, st);
}

}  // namespace

cudaError_t launch_fwd(int head_dim, const TmaPages& tq, const TmaPages& tk, const TmaPages& tv, const TileArgs& a,
                       __nv_bfloat16* o, float* lse, cudaStream_t st) {
  return head_dim == 128 ? launch_fwd_t<128, false>(tq, tk, tv, a, o, lse, nullptr, nullptr, st)
                         : launch_fwd_t<64, false>(tq, tk, tv, a, o, lse, nullptr, nullptr, st);
}

cudaError_t launch_fwd_e4m3(const TmaPages& tq8, const TmaPages& tk8, const TmaPages& tv, const TileArgs& a,
                            const float* q_descale, const float* k_descale, __nv_bfloat16* o, float* lse,
                            cudaStream_t st) {
  return launch_fwd_t<128, true>(tq8, tk8, tv, a, o, lse, q_descale, k_descale, st);
}

cudaError_t launch_fill(int head_dim, const int32_t* fill, int64_t n, int64_t bh, int64_t slots,
                        __nv_bfloat16* t0, __nv_bfloat16* t1, float* lse, cudaStream_t st) {
  if (n == 0 || bh == 0) return cudaSuccess;
  dim3 grid(static_cast<unsigned>(n), static_cast<unsigned>(bh < 65535 ? bh : 65535));
  fill_kernel<<<grid, 128, 0, st>>>(fill, bh, slots, head_dim, t0, t1, lse);
  return cudaGetLastError();
}

}  // namespace spattn
