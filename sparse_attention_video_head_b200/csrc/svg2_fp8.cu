// Per-head E4M3 quantisation for the FP8 attention variant (the project's roadmap item "Support FP8
// attention", GitHub README, Open-source Plan).  The pages fix no scaling scheme; this library uses the
// plainest one: one scale per (batch, head) plane of each of Q, K and V.
//
//   amax  = max |x| over the plane (NaN entries do not take part)
//   inv   = fl32(448 / amax), scale = fl32(amax / 448)      (inv = scale = 1 for an all-zero plane)
//   code  = E4M3(fl32(x * inv)), rounded to nearest even and saturated at +-448
//
// 448 is E4M3's largest finite magnitude (OCP 8-bit floating point, E4M3: 4 exponent bits with bias
// 7, 3 mantissa bits, no infinities), so the plane's largest entry maps to +-448.  The value a code
// stands for is E4M3(code) * scale.  Three passes: the maximum (float bits combined with atomicMax,
// which orders non-negative floats like their values, in the caller's scale array), the quantising
// gather (permuted rows, 16 codes per thread), then the maxima turned into scales in place.
#include <cuda_bf16.h>

#include <algorithm>

#include "svg2_device.cuh"
#include "svg2_internal.h"

namespace svg2 {

namespace {

constexpr float kE4m3Max = 448.0f;

__device__ __forceinline__ float abs_max8_bf16(const uint4 v, float m) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) m = fmax3(m, fabsf(bf16lo_to_f32(w[i])), fabsf(bf16hi_to_f32(w[i])));
  return m;
}

// grid (blocks per plane, BH, tensors): blockIdx.z picks X0, X1 or X2; amax is [tensors][BH] float bits.
__global__ void __launch_bounds__(256) amax_kernel(const void* __restrict__ X0, const void* __restrict__ X1,
                                                   const void* __restrict__ X2, bool f32, long long plane,
                                                   int BH, uint32_t* __restrict__ amax) {
  const int bh = blockIdx.y, t = blockIdx.z;
  const void* X = t == 0 ? X0 : (t == 1 ? X1 : X2);
  float m = 0.f;
  const long long step = static_cast<long long>(gridDim.x) * blockDim.x * 8;
  long long i = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
  if (f32) {
    const float* base = static_cast<const float*>(X) + static_cast<size_t>(bh) * plane;
    for (; i < plane; i += step) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(base + i));
      const float4 b = __ldg(reinterpret_cast<const float4*>(base + i) + 1);
      m = fmax3(m, fabsf(a.x), fabsf(a.y));
      m = fmax3(m, fabsf(a.z), fabsf(a.w));
      m = fmax3(m, fabsf(b.x), fabsf(b.y));
      m = fmax3(m, fabsf(b.z), fabsf(b.w));
    }
  } else {
    const __nv_bfloat16* base = static_cast<const __nv_bfloat16*>(X) + static_cast<size_t>(bh) * plane;
    for (; i < plane; i += step) m = abs_max8_bf16(__ldg(reinterpret_cast<const uint4*>(base + i)), m);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax + static_cast<size_t>(t) * BH + bh, __float_as_uint(m));
}

__device__ __forceinline__ float inv_of(uint32_t amax_bits) {
  const float a = __uint_as_float(amax_bits);
  return a > 0.f ? __fdiv_rn(kE4m3Max, a) : 1.f;
}

// 16 source values (bf16 or float32) times inv, as 16 E4M3 codes in one 16-byte word
__device__ __forceinline__ uint4 quant16(const void* src_row, int e, bool f32, float inv) {
  float x[16];
  if (f32) {
    const float4* s = reinterpret_cast<const float4*>(static_cast<const float*>(src_row) + e);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 a = __ldg(s + i);
      x[4 * i] = a.x, x[4 * i + 1] = a.y, x[4 * i + 2] = a.z, x[4 * i + 3] = a.w;
    }
  } else {
    const uint4* s = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(src_row) + e);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint4 a = __ldg(s + i);
      const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) x[8 * i + 2 * j] = bf16lo_to_f32(w[j]), x[8 * i + 2 * j + 1] = bf16hi_to_f32(w[j]);
    }
  }
  uint32_t r[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    r[i] = pack_e4m3x4(__fmul_rn(x[4 * i], inv), __fmul_rn(x[4 * i + 1], inv), __fmul_rn(x[4 * i + 2], inv),
                       __fmul_rn(x[4 * i + 3], inv));
  return make_uint4(r[0], r[1], r[2], r[3]);
}

// Y[r] = E4M3(X[bh, perm[r]] * inv[bh]) row by row (perm == nullptr: the identity); X1/Y1 optional.
__global__ void __launch_bounds__(256) gather_e4m3_kernel(const void* __restrict__ X0, const void* __restrict__ X1,
                                                          bool f32, const int32_t* __restrict__ perm,
                                                          long long rows, int N, int d,
                                                          const uint32_t* __restrict__ amax0,
                                                          const uint32_t* __restrict__ amax1,
                                                          uint8_t* __restrict__ Y0, uint8_t* __restrict__ Y1,
                                                          DeviceStatus* st) {
  const int per_row = d / 16;  // threads per row
  const long long total = rows * per_row;
  const size_t esz = f32 ? 4 : 2;
  for (long long g = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; g < total;
       g += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = g / per_row;
    const int e = static_cast<int>(g - r * per_row) * 16;
    const long long bh = r / N;
    int pr = static_cast<int>(r - bh * N);
    if (perm != nullptr) {
      pr = __ldg(perm + r);
      SVG2_DEBUG_CHECK(pr >= 0 && pr < N, st, kWhereGather, r, pr);
      if (pr < 0 || pr >= N) continue;  // an invalid permutation entry is skipped, never dereferenced
    }
    const long long src = bh * N + pr;
    *reinterpret_cast<uint4*>(Y0 + r * d + e) =
        quant16(static_cast<const char*>(X0) + src * d * esz, e, f32, inv_of(__ldg(amax0 + bh)));
    if (X1 != nullptr)
      *reinterpret_cast<uint4*>(Y1 + r * d + e) =
          quant16(static_cast<const char*>(X1) + src * d * esz, e, f32, inv_of(__ldg(amax1 + bh)));
  }
}

__global__ void amax_to_scale_kernel(uint32_t* __restrict__ v, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float a = __uint_as_float(v[i]);
  v[i] = __float_as_uint(a > 0.f ? __fdiv_rn(a, kE4m3Max) : 1.f);
}

int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

}  // namespace

cudaError_t launch_amax(const void* X0, const void* X1, const void* X2, int tensors, bool f32, int BH, int N, int d,
                        uint32_t* amax, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(amax, 0, static_cast<size_t>(tensors) * BH * sizeof(uint32_t), s);
  if (e != cudaSuccess) return e;
  const long long plane = static_cast<long long>(N) * d;
  const long long want = (plane / 8 + 255) / 256;
  const long long fill = std::max<long long>(1, static_cast<long long>(sm_count()) * 16 / (static_cast<long long>(BH) * tensors));
  const dim3 grid(static_cast<unsigned>(std::max<long long>(1, std::min(want, fill))), BH, tensors);
  amax_kernel<<<grid, 256, 0, s>>>(X0, X1, X2, f32, plane, BH, amax);
  return cudaGetLastError();
}

cudaError_t launch_gather_e4m3(const void* X0, const void* X1, bool f32, const int32_t* perm, int BH, int N, int d,
                               const uint32_t* amax0, const uint32_t* amax1, void* Y0, void* Y1, cudaStream_t s,
                               DeviceStatus* st) {
  const long long rows = static_cast<long long>(BH) * N;
  const long long items = rows * (d / 16);
  const long long cap = static_cast<long long>(sm_count()) * 8;
  const long long want = (items + 255) / 256;
  const int grid = static_cast<int>(std::max<long long>(1, std::min(want, cap)));
  gather_e4m3_kernel<<<grid, 256, 0, s>>>(X0, X1, f32, perm, rows, N, d, amax0, amax1, static_cast<uint8_t*>(Y0),
                                          static_cast<uint8_t*>(Y1), st);
  return cudaGetLastError();
}

cudaError_t launch_amax_to_scale(uint32_t* amax, int n, cudaStream_t s) {
  amax_to_scale_kernel<<<(n + 255) / 256, 256, 0, s>>>(amax, n);
  return cudaGetLastError();
}

}  // namespace svg2
