// Per-slice E4M3 quantisation of Q or K for the FP8 forward.
//
// A [bh, rows, head_dim] bf16 tensor is quantised slice by slice (one slice
// per batch*head): amax = max |x| over the slice, codes = e4m3(x * (448 /
// amax)) rounded to nearest-even and saturated to +-448, descale = amax /
// 448 (1 for an all-zero slice).  Each step is one correctly rounded fp32
// operation, so the codes are fixed by the inputs alone.  The forward then
// scales S = Q8 K8^T by q_descale * k_descale, i.e. it computes attention of
// the dequantised Q and K exactly (up to fp32 accumulation).
#include "kernels.cuh"

namespace spattn {
namespace {

constexpr float kE4m3Max = 448.0f;
constexpr int kQuantThreads = 256;

__device__ __forceinline__ float bf16_abs_max8(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m = fmaxf(m, fabsf(__uint_as_float(w[i] << 16)));
    m = fmaxf(m, fabsf(__uint_as_float(w[i] & 0xFFFF0000u)));
  }
  return m;
}

// amax of slice blockIdx.y into bits[bh] (non-negative floats order like
// their bit patterns, so an integer max is a float max).
__global__ void amax_kernel(const __nv_bfloat16* __restrict__ x, int64_t n_per_bh, unsigned* __restrict__ bits) {
  const int64_t bh = blockIdx.y;
  const uint4* p = reinterpret_cast<const uint4*>(x + bh * n_per_bh);
  const int64_t nv = n_per_bh / 8;
  float m = 0.f;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nv;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    m = fmaxf(m, bf16_abs_max8(__ldg(p + i)));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((threadIdx.x & 31) == 0 && m > 0.f) atomicMax(bits + bh, __float_as_uint(m));
}

// Two fp32 values to two E4M3 codes (lo in the low byte).
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__global__ void quant_kernel(const __nv_bfloat16* __restrict__ x, int64_t n_per_bh, const unsigned* __restrict__ bits,
                             uint8_t* __restrict__ x8) {
  const int64_t bh = blockIdx.y;
  const float amax = __uint_as_float(bits[bh]);
  const float inv = amax > 0.f ? kE4m3Max / amax : 1.0f;
  const uint4* p = reinterpret_cast<const uint4*>(x + bh * n_per_bh);
  uint2* q = reinterpret_cast<uint2*>(x8 + bh * n_per_bh);
  const int64_t nv = n_per_bh / 8;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nv;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 v = __ldg(p + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t c[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      c[j] = e4m3x2(__uint_as_float(w[j] << 16) * inv, __uint_as_float(w[j] & 0xFFFF0000u) * inv);
    q[i] = make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
  }
}

__global__ void descale_kernel(float* __restrict__ d, int64_t bh) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < bh;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float amax = __uint_as_float(reinterpret_cast<const unsigned*>(d)[i]);
    d[i] = amax > 0.f ? amax / kE4m3Max : 1.0f;
  }
}

}  // namespace

cudaError_t launch_quantize_e4m3(const __nv_bfloat16* x, int64_t bh, int64_t elems_per_bh, uint8_t* x8,
                                 float* descale, cudaStream_t st) {
  if (bh == 0) return cudaSuccess;
  cudaError_t e = cudaMemsetAsync(descale, 0, static_cast<size_t>(bh) * sizeof(float), st);
  if (e != cudaSuccess) return e;
  unsigned* bits = reinterpret_cast<unsigned*>(descale);
  if (elems_per_bh > 0) {
    const int64_t nv = elems_per_bh / 8;
    const int64_t per_slice = (nv + kQuantThreads - 1) / kQuantThreads;
    const unsigned gx = static_cast<unsigned>(per_slice < 64 ? per_slice : 64);
    // grid.y covers the slices (at most 65535 per launch)
    for (int64_t b0 = 0; b0 < bh; b0 += 65535) {
      const unsigned gy = static_cast<unsigned>(bh - b0 < 65535 ? bh - b0 : 65535);
      amax_kernel<<<dim3(gx, gy), kQuantThreads, 0, st>>>(x + b0 * elems_per_bh, elems_per_bh, bits + b0);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
      quant_kernel<<<dim3(gx, gy), kQuantThreads, 0, st>>>(x + b0 * elems_per_bh, elems_per_bh, bits + b0,
                                                          x8 + b0 * elems_per_bh);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
  }
  descale_kernel<<<static_cast<unsigned>((bh + 255) / 256 < 1024 ? (bh + 255) / 256 : 1024), 256, 0, st>>>(descale, bh);
  return cudaGetLastError();
}

}  // namespace spattn
