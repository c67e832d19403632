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
// K3: dK, dV (key-owned tiles, query pages as columns)
// ----------------------------------------------------------------------------
template <int D>
struct DkvCfg {
  static constexpr int kNch = D / 64;
  static constexpr int kTile = kNch * kChunkBytes;
  static constexpr int kStages = (D == 128) ? 2 : 4;
  static constexpr int kStage = 2 * kTile + 2 * 128 * 4;  // Q, dO tiles + LSE2, Delta of 128 columns
  static constexpr int kSmem = 2 * kTile + kStages * kStage + 1024 + 256;
};

template <int D>
__global__ void __launch_bounds__(256, 1)
    dkdv_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                const int32_t* __restrict__ work, const int32_t* __restrict__ col_pages,
                const uint64_t* __restrict__ col_masks, const float* __restrict__ lse,
                const float* __restrict__ delta, __nv_bfloat16* __restrict__ out_dk,
                __nv_bfloat16* __restrict__ out_dv, int64_t kv_slots, int64_t q_slots, float sl2, float scale,
                int* err) {
  using C = DkvCfg<D>;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sK = smem;
  uint8_t* sV = smem + C::kTile;
  uint8_t* sStage = smem + 2 * C::kTile;  // stage s: Q, dO, LSE2[128], Delta[128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sStage + NS * C::kStage);
  uint64_t* own_full = bars;
  uint64_t* q_full = bars + 1;
  uint64_t* do_full = q_full + NS;
  uint64_t* ld_full = do_full + NS;
  uint64_t* stage_empty = ld_full + NS;
  uint64_t* st_full = stage_empty + NS;
  uint64_t* pt_full = st_full + 1;
  uint64_t* acc_done = pt_full + 1;
  uint64_t* drain = acc_done + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  const Abort ab{abort_flag, err};

  const Work wk = load_work(work, blockIdx.x);
  const int n_cols = wk.e1 - wk.e0;
  const int n_steps = (n_cols + kStepPages - 1) / kStepPages;
  const int warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(own_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&do_full[s], 1);
      mbar_init(&ld_full[s], 32);
      mbar_init(&stage_empty[s], 1);
    }
    mbar_init(st_full, 1);
    mbar_init(pt_full, 128);
    mbar_init(acc_done, 1);
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t tST = tmem, tDPT = tmem + 128, tDV = tmem + 256, tDK = tmem + 256 + D;

  auto stage_q = [&](int s) { return sStage + s * C::kStage; };
  auto stage_do = [&](int s) { return sStage + s * C::kStage + C::kTile; };
  auto stage_l = [&](int s) { return reinterpret_cast<float*>(sStage + s * C::kStage + 2 * C::kTile); };
  auto stage_d = [&](int s) { return reinterpret_cast<float*>(sStage + s * C::kStage + 2 * C::kTile) + 128; };

  if (warp == 0) {
    // ---------------- producer (lane 0: TMA; all lanes: LSE / Delta) ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(own_full, 2 * wk.n_own * C::kNch * 2048);
      for (int p = 0; p < wk.n_own; ++p)
        for (int c = 0; c < C::kNch; ++c) {
          tma_load_3d(sK + c * kChunkBytes + p * 2048, &tm_k, c * 64, wk.own_page(p) * 16, wk.bh, own_full);
          tma_load_3d(sV + c * kChunkBytes + p * 2048, &tm_v, c * 64, wk.own_page(p) * 16, wk.bh, own_full);
        }
    }
    int issued = 0;
    for (int st = 0; st < n_steps; ++st) {
      const int s = st % NS;
      if (st >= NS) {
        bool ok = mbar_wait(&stage_empty[s], ((st / NS) - 1) & 1, ab);
        if (!__all_sync(0xffffffffu, ok)) break;
      }
      const int n = min(kStepPages, n_cols - st * kStepPages);
      const int32_t* pg = col_pages + wk.e0 + st * kStepPages;
      if (lane == 0) {
        mbar_arrive_expect_tx(&q_full[s], n * C::kNch * 2048);
        for (int j = 0; j < n; ++j)
          for (int c = 0; c < C::kNch; ++c)
            tma_load_3d(stage_q(s) + c * kChunkBytes + j * 2048, &tm_q, c * 64, __ldg(pg + j) * 16, wk.bh, &q_full[s]);
        mbar_arrive_expect_tx(&do_full[s], n * C::kNch * 2048);
        for (int j = 0; j < n; ++j)
          for (int c = 0; c < C::kNch; ++c)
            tma_load_3d(stage_do(s) + c * kChunkBytes + j * 2048, &tm_do, c * 64, __ldg(pg + j) * 16, wk.bh,
                        &do_full[s]);
      }
      float* sl = stage_l(s);
      float* sd = stage_d(s);
      for (int idx = lane; idx < 16 * n; idx += 32) {
        const int64_t slot = static_cast<int64_t>(__ldg(pg + (idx >> 4))) * 16 + (idx & 15);
        float l2 = 0.f, dl = 0.f;
        if (slot < q_slots) {
          const int64_t off = static_cast<int64_t>(wk.bh) * q_slots + slot;
          l2 = __ldg(lse + off) * kLog2e;
          dl = __ldg(delta + off);
        }
        sl[idx] = l2;
        sd[idx] = dl;
      }
      mbar_arrive(&ld_full[s]);
      issued = st + 1;
    }
    if (lane == 0) {
      for (int st = max(0, issued - NS); st < issued; ++st) {
        mbar_wait_drain(&q_full[st % NS], (st / NS) & 1);
        mbar_wait_drain(&do_full[st % NS], (st / NS) & 1);
      }
      mbar_wait_drain(own_full, 0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      const uint32_t idesc_acc = idesc_bf16(128, D, false, true);
      bool ok = mbar_wait(own_full, 0, ab);
      tc_fence_after();
      for (int st = 0; ok && st < n_steps; ++st) {
        const int s = st % NS;
        const int n = min(kStepPages, n_cols - st * kStepPages);
        const uint32_t idesc_s = idesc_bf16(128, 16 * n, false, false);
        const uint32_t q_addr = smem_u32(stage_q(s)), do_addr = smem_u32(stage_do(s));
        if (!mbar_wait(&q_full[s], (st / NS) & 1, ab)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
          umma_ss(tST, sdesc_sw128(k_addr + off, 16, 1024), sdesc_sw128(q_addr + off, 16, 1024), idesc_s, kk > 0);
        }
        if (!mbar_wait(&do_full[s], (st / NS) & 1, ab)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
          umma_ss(tDPT, sdesc_sw128(v_addr + off, 16, 1024), sdesc_sw128(do_addr + off, 16, 1024), idesc_s, kk > 0);
        }
        umma_commit(st_full);
        if (!mbar_wait(pt_full, st & 1, ab)) { ok = false; break; }
        tc_fence_after();
        for (int j = 0; j < n; ++j)
          umma_ts(tDV, tST + 8 * j, sdesc_sw128(do_addr + j * 2048, kChunkBytes, 1024), idesc_acc,
                  (st > 0 || j > 0) ? 1u : 0u);
        for (int j = 0; j < n; ++j)
          umma_ts(tDK, tDPT + 8 * j, sdesc_sw128(q_addr + j * 2048, kChunkBytes, 1024), idesc_acc,
                  (st > 0 || j > 0) ? 1u : 0u);
        umma_commit(&stage_empty[s]);
      }
      if (ok && n_steps > 0) umma_commit(acc_done);
      umma_commit(drain);
      mbar_wait_drain(drain, 0);
    }
  } else if (warp >= 4) {
    // ---------------- P^T, dS^T (one key row per thread) + epilogue ----------------
    const int q4 = warp - 4;
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t code = wk.row_code(row);
    const int seg = code < 4 ? static_cast<int>(code) : -1;
    bool ok = true;
    for (int st = 0; st < n_steps; ++st) {
      const int s = st % NS;
      const int n = min(kStepPages, n_cols - st * kStepPages);
      const int N = 16 * n;
      uint32_t mw[4];
      step_masks(col_masks, wk.e0 + st * kStepPages, n, seg, mw);
      ok = mbar_wait(st_full, st & 1, ab) && mbar_wait(&ld_full[s], (st / NS) & 1, ab);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const float* sl = stage_l(s);
      const float* sd = stage_d(s);
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        if (pc * 32 < N) {
          uint32_t a[32], b[32];
          tmem_ld32(tST + lane_off + pc * 32, a);
          tmem_ld32(tDPT + lane_off + pc * 32, b);
          tmem_wait_ld();
          uint32_t pp[16], pd[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float pv[2], dv[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int c = pc * 32 + 2 * i + h;
              const bool on = (mw[pc] >> (2 * i + h)) & 1u;
              const float p = on ? ex2(__uint_as_float(a[2 * i + h]) * sl2 - sl[c]) : 0.f;
              pv[h] = p;
              dv[h] = on ? p * (__uint_as_float(b[2 * i + h]) - sd[c]) : 0.f;
            }
            pp[i] = pack_bf16(pv[0], pv[1]);
            pd[i] = pack_bf16(dv[0], dv[1]);
          }
          tmem_st16(tST + lane_off + pc * 16, pp);
          tmem_st16(tDPT + lane_off + pc * 16, pd);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(pt_full);
    }
    if (ok && n_steps > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(acc_done, 0, ab));
      tc_fence_after();
    }
    if (ok) {
      const bool owned = code != 15u && row < 16 * wk.n_own;
      const int64_t slot = owned ? static_cast<int64_t>(wk.own_page(row >> 4)) * 16 + (row & 15) : 0;
      const bool write = owned && slot < kv_slots;
      const int64_t base = (static_cast<int64_t>(wk.bh) * kv_slots + slot) * D;
#pragma unroll
      for (int pc = 0; pc < D / 32; ++pc) {
        uint32_t r[32] = {};
        if (n_steps > 0) {
          tmem_ld32(tDV + lane_off + pc * 32, r);
          tmem_wait_ld();
        }
        if (write) store_row32(out_dv + base + pc * 32, r, 1.0f, n_steps == 0);
      }
#pragma unroll
      for (int pc = 0; pc < D / 32; ++pc) {
        uint32_t r[32] = {};
        if (n_steps > 0) {
          tmem_ld32(tDK + lane_off + pc * 32, r);
          tmem_wait_ld();
        }
        if (write) store_row32(out_dk + base + pc * 32, r, scale, n_steps == 0);
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
template <int D>
struct DqCfg {
  static constexpr int kNch = D / 64;
  static constexpr int kTile = kNch * kChunkBytes;
  static constexpr int kStages = (D == 128) ? 2 : 4;
  static constexpr int kSmem = 2 * kTile + kStages * 2 * kTile + 1024 + 256;
};

template <int D>
__global__ void __launch_bounds__(256, 1)
    dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
              const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
              const int32_t* __restrict__ work, const int32_t* __restrict__ col_pages,
              const uint64_t* __restrict__ col_masks, const float* __restrict__ lse, const float* __restrict__ delta,
              __nv_bfloat16* __restrict__ out_dq, int64_t q_slots, float sl2, float scale, int* err) {
  using C = DqCfg<D>;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sQ = smem;
  uint8_t* sDO = smem + C::kTile;
  uint8_t* sKV = smem + 2 * C::kTile;  // stage s: K at sKV + 2*s*kTile, V right after
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + NS * 2 * C::kTile);
  uint64_t* own_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + NS;
  uint64_t* kv_empty = v_full + NS;
  uint64_t* sd_full = kv_empty + NS;
  uint64_t* ds_full = sd_full + 1;
  uint64_t* acc_done = ds_full + 1;
  uint64_t* drain = acc_done + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  const Abort ab{abort_flag, err};

  const Work wk = load_work(work, blockIdx.x);
  const int n_cols = wk.e1 - wk.e0;
  const int n_steps = (n_cols + kStepPages - 1) / kStepPages;
  const int warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(own_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(sd_full, 1);
    mbar_init(ds_full, 128);
    mbar_init(acc_done, 1);
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t tS = tmem, tDP = tmem + 128, tDQ = tmem + 256;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(own_full, 2 * wk.n_own * C::kNch * 2048);
      for (int p = 0; p < wk.n_own; ++p)
        for (int c = 0; c < C::kNch; ++c) {
          tma_load_3d(sQ + c * kChunkBytes + p * 2048, &tm_q, c * 64, wk.own_page(p) * 16, wk.bh, own_full);
          tma_load_3d(sDO + c * kChunkBytes + p * 2048, &tm_do, c * 64, wk.own_page(p) * 16, wk.bh, own_full);
        }
      int issued = 0;
      for (int st = 0; st < n_steps; ++st) {
        const int s = st % NS;
        if (st >= NS && !mbar_wait(&kv_empty[s], ((st / NS) - 1) & 1, ab)) break;
        const int n = min(kStepPages, n_cols - st * kStepPages);
        uint8_t* kd = sKV + 2 * s * C::kTile;
        uint8_t* vd = kd + C::kTile;
        const int32_t* pg = col_pages + wk.e0 + st * kStepPages;
        mbar_arrive_expect_tx(&k_full[s], n * C::kNch * 2048);
        for (int j = 0; j < n; ++j)
          for (int c = 0; c < C::kNch; ++c)
            tma_load_3d(kd + c * kChunkBytes + j * 2048, &tm_k, c * 64, __ldg(pg + j) * 16, wk.bh, &k_full[s]);
        mbar_arrive_expect_tx(&v_full[s], n * C::kNch * 2048);
        for (int j = 0; j < n; ++j)
          for (int c = 0; c < C::kNch; ++c)
            tma_load_3d(vd + c * kChunkBytes + j * 2048, &tm_v, c * 64, __ldg(pg + j) * 16, wk.bh, &v_full[s]);
        issued = st + 1;
      }
      for (int st = max(0, issued - NS); st < issued; ++st) {
        mbar_wait_drain(&k_full[st % NS], (st / NS) & 1);
        mbar_wait_drain(&v_full[st % NS], (st / NS) & 1);
      }
      mbar_wait_drain(own_full, 0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(sQ), do_addr = smem_u32(sDO);
      const uint32_t idesc_acc = idesc_bf16(128, D, false, true);
      bool ok = mbar_wait(own_full, 0, ab);
      tc_fence_after();
      for (int st = 0; ok && st < n_steps; ++st) {
        const int s = st % NS;
        const int n = min(kStepPages, n_cols - st * kStepPages);
        const uint32_t idesc_s = idesc_bf16(128, 16 * n, false, false);
        const uint32_t k_addr = smem_u32(sKV + 2 * s * C::kTile);
        const uint32_t v_addr = k_addr + C::kTile;
        if (!mbar_wait(&k_full[s], (st / NS) & 1, ab)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
          umma_ss(tS, sdesc_sw128(q_addr + off, 16, 1024), sdesc_sw128(k_addr + off, 16, 1024), idesc_s, kk > 0);
        }
        if (!mbar_wait(&v_full[s], (st / NS) & 1, ab)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
          umma_ss(tDP, sdesc_sw128(do_addr + off, 16, 1024), sdesc_sw128(v_addr + off, 16, 1024), idesc_s, kk > 0);
        }
        umma_commit(sd_full);
        if (!mbar_wait(ds_full, st & 1, ab)) { ok = false; break; }
        tc_fence_after();
        for (int j = 0; j < n; ++j)
          umma_ts(tDQ, tS + 8 * j, sdesc_sw128(k_addr + j * 2048, kChunkBytes, 1024), idesc_acc,
                  (st > 0 || j > 0) ? 1u : 0u);
        umma_commit(&kv_empty[s]);
      }
      if (ok && n_steps > 0) umma_commit(acc_done);
      umma_commit(drain);
      mbar_wait_drain(drain, 0);
    }
  } else if (warp >= 4) {
    const int q4 = warp - 4;
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
    bool ok = true;
    for (int st = 0; st < n_steps; ++st) {
      const int n = min(kStepPages, n_cols - st * kStepPages);
      const int N = 16 * n;
      uint32_t mw[4];
      step_masks(col_masks, wk.e0 + st * kStepPages, n, seg, mw);
      ok = __all_sync(0xffffffffu, mbar_wait(sd_full, st & 1, ab));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        if (pc * 32 < N) {
          uint32_t a[32], b[32];
          tmem_ld32(tS + lane_off + pc * 32, a);
          tmem_ld32(tDP + lane_off + pc * 32, b);
          tmem_wait_ld();
          uint32_t pd[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float dv[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const bool on = (mw[pc] >> (2 * i + h)) & 1u;
              const float p = on ? ex2(__uint_as_float(a[2 * i + h]) * sl2 - lse2) : 0.f;
              dv[h] = on ? p * (__uint_as_float(b[2 * i + h]) - dl) : 0.f;
            }
            pd[i] = pack_bf16(dv[0], dv[1]);
          }
          tmem_st16(tS + lane_off + pc * 16, pd);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    if (ok && n_steps > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(acc_done, 0, ab));
      tc_fence_after();
    }
    if (ok) {
      __nv_bfloat16* dst = out_dq + roff * D;
#pragma unroll
      for (int pc = 0; pc < D / 32; ++pc) {
        uint32_t r[32] = {};
        if (n_steps > 0) {
          tmem_ld32(tDQ + lane_off + pc * 32, r);
          tmem_wait_ld();
        }
        if (valid_slot) store_row32(dst + pc * 32, r, scale, n_steps == 0);
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
  dkdv_kernel<D><<<static_cast<unsigned>(a.n_work), 256, C::kSmem, st>>>(
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
  dq_kernel<D><<<static_cast<unsigned>(a.n_work), 256, C::kSmem, st>>>(
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
