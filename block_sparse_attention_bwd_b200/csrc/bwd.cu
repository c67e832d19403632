// Backward kernels: K2 (Delta = rowsum(dO * O)), K3 (dK, dV owned per key
// tile, no atomics) and K4 (dQ owned per query tile, no atomics).
//
// Method (KPage abstract, "KPage: block-sparse attention for partially
// occupied 3D blocks", zhuanzhiai.com, abstract paragraph): "K/V-owned page
// packing" preserves the sparse graph in the backward pass.  Here the key
// side packs its valid 16-row pages into 128-row owned tiles exactly as the
// query side does in the forward pass; each key tile walks the query pages
// that reach it (the transposed lists), so dK and dV are accumulated in TMEM
// and written once.  dQ is computed by a second, query-owned pass over the
// forward page lists.  The gradient formulas are the standard ones for
// softmax attention: P = exp(S - LSE), dV = P^T dO, dP = dO V^T,
// dS = P * (dP - Delta), dK = scale dS^T Q, dQ = scale dS K.
//
// Both tile kernels use the CTA layout of the forward kernel: warp 0 is the
// TMA producer, warp 1 allocates TMEM and issues tcgen05 MMAs, warps 4..7
// own one tile row each.
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
// TMEM columns: S^T / P^T double buffer at 0 and 64, dP^T / dS^T double
// buffer at 128 and 192, dV at 256, dK at 256 + D.  The MMAs of step c+1
// (S^T, dP^T) run while the row threads turn step c into P^T and dS^T.
constexpr int kBwdStepPages = 4;                  // 64 columns per step
constexpr int kStageChunk = 64 * 128;             // one 64-column chunk of a 64-row stage

template <int D>
struct DkvCfg {
  static constexpr int kNch = D / 64;
  static constexpr int kTile = kNch * kChunkBytes;     // owned 128-row tile
  static constexpr int kStageTile = kNch * kStageChunk;  // 64-row column stage
  static constexpr int kQStages = (D == 128) ? 4 : 6;
  static constexpr int kDStages = (D == 128) ? 4 : 6;
  static constexpr int kLdBytes = 2 * 64 * 4;          // LSE2 and Delta of 64 columns
  static constexpr int kSmem = 2 * kTile + kQStages * kStageTile + kDStages * (kStageTile + kLdBytes) + 1024 + 512;
};

// 10 warps: 0 = TMA producer, 1 = TMEM owner and MMA issuer, 2..9 = two
// groups of row threads; group g (warps 2+4g .. 5+4g) handles columns
// 32g .. 32g+31 of every 64-column step (warp w reaches TMEM lanes of
// quarter w%4).
constexpr int kBwdThreads = 320;

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    dkdv_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                const int32_t* __restrict__ work, const int32_t* __restrict__ col_pages,
                const uint64_t* __restrict__ col_masks, const float* __restrict__ lse,
                const float* __restrict__ delta, __nv_bfloat16* __restrict__ out_dk,
                __nv_bfloat16* __restrict__ out_dv, int64_t kv_slots, int64_t q_slots, float sl2, float scale,
                int* err) {
  using C = DkvCfg<D>;
  constexpr int QS = C::kQStages, DS = C::kDStages, NP = kBwdStepPages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sK = smem;
  uint8_t* sV = smem + C::kTile;
  uint8_t* sQ = smem + 2 * C::kTile;                 // Q stage s at sQ + s*kStageTile
  uint8_t* sDO = sQ + QS * C::kStageTile;            // dO stage s at sDO + s*kStageTile
  float* sLD = reinterpret_cast<float*>(sDO + DS * C::kStageTile);  // stage s: LSE2[64], Delta[64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sLD) + DS * C::kLdBytes);
  uint64_t* own_full = bars;
  uint64_t* q_full = own_full + 1;
  uint64_t* q_empty = q_full + QS;
  uint64_t* do_full = q_empty + QS;
  uint64_t* do_empty = do_full + DS;
  uint64_t* ld_full = do_empty + DS;
  uint64_t* st_full = ld_full + DS;  // [2]
  uint64_t* pt_full = st_full + 2;   // [2]
  uint64_t* acc_done = pt_full + 2;
  uint64_t* acc_step = acc_done + 1;  // completes once per step's dV, dK MMAs
  uint64_t* drain = acc_step + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  const Abort ab{abort_flag, err};

  const Work wk = load_work(work, blockIdx.x);
  const int n_cols = wk.e1 - wk.e0;
  const int n_steps = (n_cols + NP - 1) / NP;
  const int warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(own_full, 1);
    mbar_init(acc_step, 1);
    for (int s = 0; s < QS; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    for (int s = 0; s < DS; ++s) {
      mbar_init(&do_full[s], 1);
      mbar_init(&do_empty[s], 1);
      mbar_init(&ld_full[s], 32);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&st_full[b], 1);
      mbar_init(&pt_full[b], 256);
    }
    mbar_init(acc_done, 1);
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t tDV = tmem + 256, tDK = tmem + 256 + D;

  if (warp == 0) {
    // ---------------- producer (whole warp) ----------------
    // Lane j < n owns page j of a step: it holds the page id (fetched one step
    // ahead) and issues that page's TMA boxes; every lane then fetches LSE2 and
    // Delta for two of the step's 64 query columns.
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(own_full, 2 * wk.n_own * C::kNch * 2048);
    }
    __syncwarp();
    if (lane < wk.n_own)
#pragma unroll
      for (int c = 0; c < C::kNch; ++c) {
        tma_load_3d(sK + c * kChunkBytes + lane * 2048, &tm_k, c * 64, wk.own_page(lane) * 16, wk.bh, own_full);
        tma_load_3d(sV + c * kChunkBytes + lane * 2048, &tm_v, c * 64, wk.own_page(lane) * 16, wk.bh, own_full);
      }
    int pid_next = (n_steps > 0 && lane < min(NP, n_cols)) ? __ldg(col_pages + wk.e0 + lane) : 0;
    int q_issued = 0, d_issued = 0;
    for (int st = 0; st < n_steps; ++st) {
      const int qs = st % QS, ds = st % DS;
      const int n = min(NP, n_cols - st * NP);
      const int pid = pid_next;
      if (st + 1 < n_steps)
        pid_next = lane < min(NP, n_cols - (st + 1) * NP) ? __ldg(col_pages + wk.e0 + (st + 1) * NP + lane) : 0;
      if (st >= QS && !__all_sync(0xffffffffu, mbar_wait(&q_empty[qs], ((st / QS) - 1) & 1, ab))) break;
      if (lane == 0) mbar_arrive_expect_tx(&q_full[qs], n * C::kNch * 2048);
      __syncwarp();
      if (lane < n)
#pragma unroll
        for (int c = 0; c < C::kNch; ++c)
          tma_load_3d(sQ + qs * C::kStageTile + c * kStageChunk + lane * 2048, &tm_q, c * 64, pid * 16, wk.bh, &q_full[qs]);
      q_issued = st + 1;
      if (st >= DS && !__all_sync(0xffffffffu, mbar_wait(&do_empty[ds], ((st / DS) - 1) & 1, ab))) break;
      if (lane == 0) mbar_arrive_expect_tx(&do_full[ds], n * C::kNch * 2048);
      __syncwarp();
      if (lane < n)
#pragma unroll
        for (int c = 0; c < C::kNch; ++c)
          tma_load_3d(sDO + ds * C::kStageTile + c * kStageChunk + lane * 2048, &tm_do, c * 64, pid * 16, wk.bh,
                      &do_full[ds]);
      d_issued = st + 1;
      float* sl = sLD + ds * 128;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int idx = lane + 32 * h;                     // column of the step
        const int pg = __shfl_sync(0xffffffffu, pid, idx >> 4);
        const int64_t slot = static_cast<int64_t>(pg) * 16 + (idx & 15);
        float l2 = 0.f, dl = 0.f;
        if ((idx >> 4) < n && slot < q_slots) {
          const int64_t off = static_cast<int64_t>(wk.bh) * q_slots + slot;
          l2 = __ldg(lse + off) * kLog2e;
          dl = __ldg(delta + off);
        }
        sl[idx] = l2;
        sl[64 + idx] = dl;
      }
      mbar_arrive(&ld_full[ds]);
    }
    if (lane == 0) {
      for (int st = max(0, q_issued - QS); st < q_issued; ++st) mbar_wait_drain(&q_full[st % QS], (st / QS) & 1);
      for (int st = max(0, d_issued - DS); st < d_issued; ++st) mbar_wait_drain(&do_full[st % DS], (st / DS) & 1);
      mbar_wait_drain(own_full, 0);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (warp-wide; one elected lane issues) ----------------
    const uint64_t dk0 = sdesc_sw128(smem_u32(sK), 16, 1024);
    const uint64_t dv0 = sdesc_sw128(smem_u32(sV), 16, 1024);
    const uint64_t dqk = sdesc_sw128(smem_u32(sQ), 16, 1024);             // Q stages, K-major
    const uint64_t ddk = sdesc_sw128(smem_u32(sDO), 16, 1024);            // dO stages, K-major
    const uint64_t dqm = sdesc_sw128(smem_u32(sQ), kStageChunk, 1024);    // Q stages, MN-major
    const uint64_t ddm = sdesc_sw128(smem_u32(sDO), kStageChunk, 1024);   // dO stages, MN-major
    const uint32_t idesc_acc = idesc_bf16(128, D, false, true);
    bool ok = __all_sync(0xffffffffu, mbar_wait(own_full, 0, ab));
    tc_fence_after();
    auto issue_acc = [&](int st) -> bool {
      const int b = st & 1, qs = st % QS, ds = st % DS;
      if (!__all_sync(0xffffffffu, mbar_wait(&pt_full[b], (st >> 1) & 1, ab))) return false;
      tc_fence_after();
      const int n = min(NP, n_cols - st * NP);
      const uint64_t bq = sdesc_add(dqm, qs * C::kStageTile), bd = sdesc_add(ddm, ds * C::kStageTile);
#pragma unroll
      for (int j = 0; j < NP; ++j)
        if (j < n) umma_ts_w(tDV, tmem + 64 * b + 8 * j, sdesc_add(bd, j * 2048), idesc_acc, (st > 0 || j > 0) ? 1u : 0u);
      umma_commit_w(&do_empty[ds]);
#pragma unroll
      for (int j = 0; j < NP; ++j)
        if (j < n)
          umma_ts_w(tDK, tmem + 128 + 64 * b + 8 * j, sdesc_add(bq, j * 2048), idesc_acc, (st > 0 || j > 0) ? 1u : 0u);
      umma_commit_w(&q_empty[qs]);
      umma_commit_w(acc_step);
      return true;
    };
    for (int st = 0; ok && st < n_steps; ++st) {
      const int b = st & 1, qs = st % QS, ds = st % DS;
      const int n = min(NP, n_cols - st * NP);
      const uint32_t idesc_s = idesc_bf16(128, 16 * n, false, false);
      // buffers b still feed dV(st-2) / dK(st-2) as TMEM A operands
      bool w = (st < 2 || mbar_wait(acc_step, (st - 2) & 1, ab)) && mbar_wait(&q_full[qs], (st / QS) & 1, ab);
      if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      tc_fence_after();
      const uint64_t bq = sdesc_add(dqk, qs * C::kStageTile), bd = sdesc_add(ddk, ds * C::kStageTile);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        umma_ss_w(tmem + 64 * b, sdesc_add(dk0, (kk >> 2) * kChunkBytes + (kk & 3) * 32),
                  sdesc_add(bq, (kk >> 2) * kStageChunk + (kk & 3) * 32), idesc_s, kk > 0);
      if (!__all_sync(0xffffffffu, mbar_wait(&do_full[ds], (st / DS) & 1, ab))) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        umma_ss_w(tmem + 128 + 64 * b, sdesc_add(dv0, (kk >> 2) * kChunkBytes + (kk & 3) * 32),
                  sdesc_add(bd, (kk >> 2) * kStageChunk + (kk & 3) * 32), idesc_s, kk > 0);
      umma_commit_w(&st_full[b]);
      if (st >= 1 && !issue_acc(st - 1)) ok = false;
    }
    if (ok && n_steps > 0 && issue_acc(n_steps - 1)) umma_commit_w(acc_done);
    umma_commit_w(drain);
    mbar_wait_drain(drain, 0);
  } else {
    // ---------------- P^T, dS^T (one key row per thread) + epilogue ----------------
    const int grp = (warp - 2) >> 2;  // column half of each step
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t code = wk.row_code(row);
    const int seg = code < 4 ? static_cast<int>(code) : -1;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    bool ok = true;
    uint32_t mw[2];
    if (n_steps > 0) step_masks<NP>(col_masks, wk.e0, min(NP, n_cols), seg, mw);
    for (int st = 0; st < n_steps; ++st) {
      const int b = st & 1, ds = st % DS;
      const int N = 16 * min(NP, n_cols - st * NP);
      const bool active = grp * 32 < N;
      ok = mbar_wait(&st_full[b], (st >> 1) & 1, ab) && mbar_wait(&ld_full[ds], (st / DS) & 1, ab);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t a[32], d[32];
      if (active) {
        tmem_ld32(tmem + 64 * b + lane_off + grp * 32, a);
        tmem_ld32(tmem + 128 + 64 * b + lane_off + grp * 32, d);
      }
      uint32_t mw_next[2] = {0u, 0u};
      if (st + 1 < n_steps) step_masks<NP>(col_masks, wk.e0 + (st + 1) * NP, min(NP, n_cols - (st + 1) * NP), seg, mw_next);
      if (active) {
        tmem_wait_ld();
        const uint32_t m = grp ? mw[1] : mw[0];
        const float4* sl4 = reinterpret_cast<const float4*>(sLD + ds * 128 + grp * 32);
        const float4* sd4 = reinterpret_cast<const float4*>(sLD + ds * 128 + 64 + grp * 32);
        uint32_t pp[16], pd[16];
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const float4 L = sl4[i4];
          const float4 Dl = sd4[i4];
          float x0, x1, x2, x3;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(a[4 * i4]), __uint_as_float(a[4 * i4 + 1])), sl2x2,
                           f2_pack(-L.x, -L.y)), x0, x1);
          f2_unpack(f2_fma(f2_pack(__uint_as_float(a[4 * i4 + 2]), __uint_as_float(a[4 * i4 + 3])), sl2x2,
                           f2_pack(-L.z, -L.w)), x2, x3);
          float p[4] = {ex2(x0), ex2(x1), ex2(x2), ex2(x3)};
#pragma unroll
          for (int h = 0; h < 4; ++h)
            if (!((m >> (4 * i4 + h)) & 1u)) p[h] = 0.f;
          float g0, g1, g2, g3;
          f2_unpack(f2_add(f2_pack(__uint_as_float(d[4 * i4]), __uint_as_float(d[4 * i4 + 1])), f2_pack(-Dl.x, -Dl.y)),
                    g0, g1);
          f2_unpack(f2_add(f2_pack(__uint_as_float(d[4 * i4 + 2]), __uint_as_float(d[4 * i4 + 3])),
                           f2_pack(-Dl.z, -Dl.w)), g2, g3);
          float s0, s1, s2, s3;
          f2_unpack(f2_mul(f2_pack(p[0], p[1]), f2_pack(g0, g1)), s0, s1);
          f2_unpack(f2_mul(f2_pack(p[2], p[3]), f2_pack(g2, g3)), s2, s3);
          pp[2 * i4] = pack_bf16(p[0], p[1]);
          pp[2 * i4 + 1] = pack_bf16(p[2], p[3]);
          // masked entries: p = 0 exactly, so dS = 0 unless dP - Delta is not finite
          pd[2 * i4] = pack_bf16(p[0] != 0.f ? s0 : 0.f, p[1] != 0.f ? s1 : 0.f);
          pd[2 * i4 + 1] = pack_bf16(p[2] != 0.f ? s2 : 0.f, p[3] != 0.f ? s3 : 0.f);
        }
        tmem_st16(tmem + 64 * b + lane_off + grp * 16, pp);
        tmem_st16(tmem + 128 + 64 * b + lane_off + grp * 16, pd);
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&pt_full[b]);
      mw[0] = mw_next[0];
      mw[1] = mw_next[1];
    }
    if (ok && n_steps > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(acc_done, 0, ab));
      tc_fence_after();
    }
    if (ok) {
      // group 0 writes dV, group 1 writes scale * dK
      const bool owned = code != 15u && row < 16 * wk.n_own;
      const int64_t slot = owned ? static_cast<int64_t>(wk.own_page(row >> 4)) * 16 + (row & 15) : 0;
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
// TMEM columns: S / dS double buffer at 0 and 64, dP double buffer at 128
// and 192, dQ at 256.  K stays in its stage until the dQ MMA of its step.
template <int D>
struct DqCfg {
  static constexpr int kNch = D / 64;
  static constexpr int kTile = kNch * kChunkBytes;
  static constexpr int kStageTile = kNch * kStageChunk;
  static constexpr int kKStages = (D == 128) ? 5 : 8;
  static constexpr int kVStages = (D == 128) ? 4 : 8;
  static constexpr int kSmem = 2 * kTile + (kKStages + kVStages) * kStageTile + 1024 + 512;
};

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
              const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
              const int32_t* __restrict__ work, const int32_t* __restrict__ col_pages,
              const uint64_t* __restrict__ col_masks, const float* __restrict__ lse, const float* __restrict__ delta,
              __nv_bfloat16* __restrict__ out_dq, int64_t q_slots, float sl2, float scale, int* err) {
  using C = DqCfg<D>;
  constexpr int KS = C::kKStages, VS = C::kVStages, NP = kBwdStepPages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sQ = smem;
  uint8_t* sDO = smem + C::kTile;
  uint8_t* sK = smem + 2 * C::kTile;       // K stage s at sK + s*kStageTile
  uint8_t* sV = sK + KS * C::kStageTile;   // V stage s at sV + s*kStageTile
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + VS * C::kStageTile);
  uint64_t* own_full = bars;
  uint64_t* k_full = own_full + 1;
  uint64_t* k_empty = k_full + KS;
  uint64_t* v_full = k_empty + KS;
  uint64_t* v_empty = v_full + VS;
  uint64_t* sd_full = v_empty + VS;  // [2]
  uint64_t* ds_full = sd_full + 2;   // [2]
  uint64_t* acc_done = ds_full + 2;
  uint64_t* dq_step = acc_done + 1;  // completes once per step's dQ MMAs
  uint64_t* drain = dq_step + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  const Abort ab{abort_flag, err};

  const Work wk = load_work(work, blockIdx.x);
  const int n_cols = wk.e1 - wk.e0;
  const int n_steps = (n_cols + NP - 1) / NP;
  const int warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(own_full, 1);
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
      mbar_init(&ds_full[b], 256);
    }
    mbar_init(acc_done, 1);
    mbar_init(dq_step, 1);
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t tDQ = tmem + 256;

  if (warp == 0) {
    // ---------------- producer (whole warp; lane j owns page j of a step) ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(own_full, 2 * wk.n_own * C::kNch * 2048);
    }
    __syncwarp();
    if (lane < wk.n_own)
#pragma unroll
      for (int c = 0; c < C::kNch; ++c) {
        tma_load_3d(sQ + c * kChunkBytes + lane * 2048, &tm_q, c * 64, wk.own_page(lane) * 16, wk.bh, own_full);
        tma_load_3d(sDO + c * kChunkBytes + lane * 2048, &tm_do, c * 64, wk.own_page(lane) * 16, wk.bh, own_full);
      }
    int pid_next = (n_steps > 0 && lane < min(NP, n_cols)) ? __ldg(col_pages + wk.e0 + lane) : 0;
    int k_issued = 0, v_issued = 0;
    for (int st = 0; st < n_steps; ++st) {
      const int ks = st % KS, vs = st % VS;
      const int n = min(NP, n_cols - st * NP);
      const int pid = pid_next;
      if (st + 1 < n_steps)
        pid_next = lane < min(NP, n_cols - (st + 1) * NP) ? __ldg(col_pages + wk.e0 + (st + 1) * NP + lane) : 0;
      if (st >= KS && !__all_sync(0xffffffffu, mbar_wait(&k_empty[ks], ((st / KS) - 1) & 1, ab))) break;
      if (lane == 0) mbar_arrive_expect_tx(&k_full[ks], n * C::kNch * 2048);
      __syncwarp();
      if (lane < n)
#pragma unroll
        for (int c = 0; c < C::kNch; ++c)
          tma_load_3d(sK + ks * C::kStageTile + c * kStageChunk + lane * 2048, &tm_k, c * 64, pid * 16, wk.bh, &k_full[ks]);
      k_issued = st + 1;
      if (st >= VS && !__all_sync(0xffffffffu, mbar_wait(&v_empty[vs], ((st / VS) - 1) & 1, ab))) break;
      if (lane == 0) mbar_arrive_expect_tx(&v_full[vs], n * C::kNch * 2048);
      __syncwarp();
      if (lane < n)
#pragma unroll
        for (int c = 0; c < C::kNch; ++c)
          tma_load_3d(sV + vs * C::kStageTile + c * kStageChunk + lane * 2048, &tm_v, c * 64, pid * 16, wk.bh, &v_full[vs]);
      v_issued = st + 1;
    }
    if (lane == 0) {
      for (int st = max(0, k_issued - KS); st < k_issued; ++st) mbar_wait_drain(&k_full[st % KS], (st / KS) & 1);
      for (int st = max(0, v_issued - VS); st < v_issued; ++st) mbar_wait_drain(&v_full[st % VS], (st / VS) & 1);
      mbar_wait_drain(own_full, 0);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (warp-wide; one elected lane issues) ----------------
    const uint64_t dq0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t ddo0 = sdesc_sw128(smem_u32(sDO), 16, 1024);
    const uint64_t dkk = sdesc_sw128(smem_u32(sK), 16, 1024);            // K stages, K-major
    const uint64_t dkm = sdesc_sw128(smem_u32(sK), kStageChunk, 1024);   // K stages, MN-major
    const uint64_t dvk = sdesc_sw128(smem_u32(sV), 16, 1024);            // V stages, K-major
    const uint32_t idesc_acc = idesc_bf16(128, D, false, true);
    bool ok = __all_sync(0xffffffffu, mbar_wait(own_full, 0, ab));
    tc_fence_after();
    auto issue_dq = [&](int st) -> bool {
      const int b = st & 1, ks = st % KS;
      if (!__all_sync(0xffffffffu, mbar_wait(&ds_full[b], (st >> 1) & 1, ab))) return false;
      tc_fence_after();
      const int n = min(NP, n_cols - st * NP);
      const uint64_t bk = sdesc_add(dkm, ks * C::kStageTile);
#pragma unroll
      for (int j = 0; j < NP; ++j)
        if (j < n) umma_ts_w(tDQ, tmem + 64 * b + 8 * j, sdesc_add(bk, j * 2048), idesc_acc, (st > 0 || j > 0) ? 1u : 0u);
      umma_commit_w(&k_empty[ks]);
      umma_commit_w(dq_step);
      return true;
    };
    for (int st = 0; ok && st < n_steps; ++st) {
      const int b = st & 1, ks = st % KS, vs = st % VS;
      const int n = min(NP, n_cols - st * NP);
      const uint32_t idesc_s = idesc_bf16(128, 16 * n, false, false);
      // buffer b still feeds dQ(st-2) as its TMEM A operand
      bool w = (st < 2 || mbar_wait(dq_step, (st - 2) & 1, ab)) && mbar_wait(&k_full[ks], (st / KS) & 1, ab);
      if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      tc_fence_after();
      const uint64_t bk = sdesc_add(dkk, ks * C::kStageTile), bv = sdesc_add(dvk, vs * C::kStageTile);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        umma_ss_w(tmem + 64 * b, sdesc_add(dq0, (kk >> 2) * kChunkBytes + (kk & 3) * 32),
                  sdesc_add(bk, (kk >> 2) * kStageChunk + (kk & 3) * 32), idesc_s, kk > 0);
      if (!__all_sync(0xffffffffu, mbar_wait(&v_full[vs], (st / VS) & 1, ab))) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        umma_ss_w(tmem + 128 + 64 * b, sdesc_add(ddo0, (kk >> 2) * kChunkBytes + (kk & 3) * 32),
                  sdesc_add(bv, (kk >> 2) * kStageChunk + (kk & 3) * 32), idesc_s, kk > 0);
      umma_commit_w(&v_empty[vs]);
      umma_commit_w(&sd_full[b]);
      if (st >= 1 && !issue_dq(st - 1)) ok = false;
    }
    if (ok && n_steps > 0 && issue_dq(n_steps - 1)) umma_commit_w(acc_done);
    umma_commit_w(drain);
    mbar_wait_drain(drain, 0);
  } else {
    const int grp = (warp - 2) >> 2;  // column half of each step
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t code = wk.row_code(row);
    const int seg = code < 4 ? static_cast<int>(code) : -1;
    const bool owned = code != 15u && row < 16 * wk.n_own;
    const int64_t slot = owned ? static_cast<int64_t>(wk.own_page(row >> 4)) * 16 + (row & 15) : 0;
    const bool valid_slot = owned && slot < q_slots;
    const int64_t roff = static_cast<int64_t>(wk.bh) * q_slots + slot;
    const float lse2 = (valid_slot && seg >= 0) ? __ldg(lse + roff) * kLog2e : 0.f;
    const float dl = (valid_slot && seg >= 0) ? __ldg(delta + roff) : 0.f;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    const uint64_t nl2 = f2_pack(-lse2, -lse2);
    const uint64_t ndl = f2_pack(-dl, -dl);
    bool ok = true;
    uint32_t mw[2];
    if (n_steps > 0) step_masks<NP>(col_masks, wk.e0, min(NP, n_cols), seg, mw);
    for (int st = 0; st < n_steps; ++st) {
      const int b = st & 1;
      const int N = 16 * min(NP, n_cols - st * NP);
      const bool active = grp * 32 < N;
      ok = __all_sync(0xffffffffu, mbar_wait(&sd_full[b], (st >> 1) & 1, ab));
      if (!ok) break;
      tc_fence_after();
      uint32_t a[32], d[32];
      if (active) {
        tmem_ld32(tmem + 64 * b + lane_off + grp * 32, a);
        tmem_ld32(tmem + 128 + 64 * b + lane_off + grp * 32, d);
      }
      uint32_t mw_next[2] = {0u, 0u};
      if (st + 1 < n_steps) step_masks<NP>(col_masks, wk.e0 + (st + 1) * NP, min(NP, n_cols - (st + 1) * NP), seg, mw_next);
      if (active) {
        tmem_wait_ld();
        const uint32_t m = grp ? mw[1] : mw[0];
        uint32_t pd[16];
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
        tmem_st16(tmem + 64 * b + lane_off + grp * 16, pd);
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&ds_full[b]);
      mw[0] = mw_next[0];
      mw[1] = mw_next[1];
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
static cudaError_t launch_dkdv_t(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                                 const CUtensorMap& tdo, const TileArgs& a, const float* lse, const float* delta,
                                 __nv_bfloat16* dk, __nv_bfloat16* dv, cudaStream_t st) {
  using C = DkvCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess || a.n_work == 0) return e;
  dkdv_kernel<D><<<static_cast<unsigned>(a.n_work), kBwdThreads, C::kSmem, st>>>(
      tk, tv, tq, tdo, a.work, a.pages, a.masks, lse, delta, dk, dv, a.own_slots, a.col_slots, a.scale * kLog2e,
      a.scale, a.err);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_dq_t(const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                               const CUtensorMap& tv, const TileArgs& a, const float* lse, const float* delta,
                               __nv_bfloat16* dq, cudaStream_t st) {
  using C = DqCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess || a.n_work == 0) return e;
  dq_kernel<D><<<static_cast<unsigned>(a.n_work), kBwdThreads, C::kSmem, st>>>(
      tq, tdo, tk, tv, a.work, a.pages, a.masks, lse, delta, dq, a.own_slots, a.scale * kLog2e, a.scale, a.err);
  return cudaGetLastError();
}

cudaError_t launch_dkdv(int head_dim, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                        const CUtensorMap& tdo, const TileArgs& a, const float* lse, const float* delta,
                        __nv_bfloat16* dk, __nv_bfloat16* dv, cudaStream_t st) {
  return head_dim == 128 ? launch_dkdv_t<128>(tk, tv, tq, tdo, a, lse, delta, dk, dv, st)
                         : launch_dkdv_t<64>(tk, tv, tq, tdo, a, lse, delta, dk, dv, st);
}

cudaError_t launch_dq(int head_dim, const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                      const CUtensorMap& tv, const TileArgs& a, const float* lse, const float* delta,
                      __nv_bfloat16* dq, cudaStream_t st) {
  return head_dim == 128 ? launch_dq_t<128>(tq, tdo, tk, tv, a, lse, delta, dq, st)
                         : launch_dq_t<64>(tq, tdo, tk, tv, a, lse, delta, dq, st);
}

}  // namespace spattn
