// Semantic-aware permutation ("Sparse VideoGen2" wiki summary, Method (2); Key claims section 4.1):
// a stable counting sort of cluster labels per (batch, head) and the row gathers / scatters that
// move Q, K, V into cluster-contiguous order and the output back to token order.
//
// Sort: each (b,h) is cut into kSortChunks token chunks.  (1) per-chunk label histograms,
// (2) per label an exclusive scan over labels (offsets) and then over chunks (chunk bases),
// (3) one warp per chunk walks its tokens in order and places them; ranks inside a 32-token
// step come from __match_any_sync, so equal labels keep ascending token order (stable).
// Everything is integer arithmetic, hence bit-exact.  The row moves are HBM-bound copies with
// 16-byte accesses.
#include <cuda_bf16.h>

#include "svg2_device.cuh"
#include "svg2_internal.h"

namespace svg2 {

namespace {

__device__ __forceinline__ int chunk_len(int N) { return (N + kSortChunks - 1) / kSortChunks; }

__global__ void __launch_bounds__(256) sort_hist_kernel(const int32_t* __restrict__ labels, int N, int k,
                                                         int32_t* __restrict__ chunk_hist, DeviceStatus* st) {
  extern __shared__ int32_t hist[];
  const int c = blockIdx.x, bh = blockIdx.y;
  for (int i = threadIdx.x; i < k; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int cl = chunk_len(N);
  const int t0 = c * cl, t1 = min(N, t0 + cl);
  const int32_t* lab = labels + static_cast<size_t>(bh) * N;
  for (int t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
    const int l = lab[t];
    if (l < 0 || l >= k) {
      raise_status(st, kStatusDeviceBounds, kWhereSort, bh, t);
      continue;
    }
    atomicAdd(&hist[l], 1);
  }
  __syncthreads();
  int32_t* out = chunk_hist + (static_cast<size_t>(bh) * kSortChunks + c) * k;
  for (int i = threadIdx.x; i < k; i += blockDim.x) out[i] = hist[i];
}

// One block of 1024 threads per (b,h); k <= 1024 so each thread owns at most one label.
__global__ void __launch_bounds__(1024) sort_scan_kernel(int N, int k, int32_t* __restrict__ chunk_hist,
                                                          int32_t* __restrict__ counts,
                                                          int32_t* __restrict__ offsets) {
  __shared__ int32_t warp_sums[32];
  const int bh = blockIdx.x;
  const int l = threadIdx.x;
  int32_t* ch = chunk_hist + static_cast<size_t>(bh) * kSortChunks * k;
  int total = 0;
  if (l < k) {
    for (int c = 0; c < kSortChunks; ++c) total += ch[c * k + l];
  }
  // block-wide exclusive scan of `total` over l
  const int lane = l & 31, warp = l >> 5;
  int incl = total;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += v;
    }
    warp_sums[lane] = wi - w;
  }
  __syncthreads();
  const int excl = warp_sums[warp] + incl - total;
  if (l < k) {
    if (counts) counts[static_cast<size_t>(bh) * k + l] = total;
    offsets[static_cast<size_t>(bh) * (k + 1) + l] = excl;
    int run = excl;
    for (int c = 0; c < kSortChunks; ++c) {
      const int v = ch[c * k + l];
      ch[c * k + l] = run;
      run += v;
    }
  }
  if (l == k - 1) offsets[static_cast<size_t>(bh) * (k + 1) + k] = excl + total;
}

// One warp per (chunk, b,h): place the chunk's tokens in order.
__global__ void __launch_bounds__(32) sort_scatter_kernel(const int32_t* __restrict__ labels, int N, int k,
                                                           const int32_t* __restrict__ chunk_base,
                                                           int32_t* __restrict__ perm) {
  extern __shared__ int32_t cursor[];
  const int c = blockIdx.x, bh = blockIdx.y;
  const int lane = threadIdx.x;
  const int32_t* base = chunk_base + (static_cast<size_t>(bh) * kSortChunks + c) * k;
  for (int i = lane; i < k; i += 32) cursor[i] = base[i];
  __syncwarp();
  const int cl = chunk_len(N);
  const int t0 = c * cl, t1 = min(N, t0 + cl);
  const int32_t* lab = labels + static_cast<size_t>(bh) * N;
  int32_t* out = perm + static_cast<size_t>(bh) * N;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int tb = t0; tb < t1; tb += 32) {
    const int t = tb + lane;
    int l = -1;
    if (t < t1) {
      l = lab[t];
      if (l < 0 || l >= k) l = -1;
    }
    const uint32_t peers = __match_any_sync(0xffffffffu, l);
    if (l >= 0) {
      const int rank = __popc(peers & lt_mask);
      out[cursor[l] + rank] = t;
    }
    __syncwarp();
    if (l >= 0 && (peers & lt_mask) == 0u) cursor[l] += __popc(peers);
    __syncwarp();
  }
}

// Row copy helpers: one thread moves 8 bf16 values (16 bytes of output).
__device__ __forceinline__ uint4 load8_as_bf16(const void* src_row, int e, bool f32) {
  if (!f32) {
    return __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(src_row) + e));
  }
  const float4* s = reinterpret_cast<const float4*>(static_cast<const float*>(src_row) + e);
  const float4 a = __ldg(s), b = __ldg(s + 1);
  uint4 r;
  r.x = pack_bf16x2(a.x, a.y);
  r.y = pack_bf16x2(a.z, a.w);
  r.z = pack_bf16x2(b.x, b.y);
  r.w = pack_bf16x2(b.z, b.w);
  return r;
}

__global__ void __launch_bounds__(256) gather_rows_kernel(const void* __restrict__ X0, const void* __restrict__ X1,
                                                           bool f32, const int32_t* __restrict__ perm,
                                                           long long rows, int N, int d,
                                                           __nv_bfloat16* __restrict__ Y0,
                                                           __nv_bfloat16* __restrict__ Y1, DeviceStatus* st) {
  const int per_row = d / 8;  // threads per row
  const long long total = rows * per_row;
  const size_t esz = f32 ? 4 : 2;
  for (long long g = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; g < total;
       g += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = g / per_row;
    const int e = static_cast<int>(g - r * per_row) * 8;
    const long long bh = r / N;
    const int pr = __ldg(perm + r);
    SVG2_DEBUG_CHECK(pr >= 0 && pr < N, st, kWhereGather, r, pr);
    if (pr < 0 || pr >= N) continue;  // an invalid permutation entry is skipped, never dereferenced
    const long long src = bh * N + pr;
    const uint4 v0 = load8_as_bf16(static_cast<const char*>(X0) + src * d * esz, e, f32);
    *reinterpret_cast<uint4*>(Y0 + r * d + e) = v0;
    if (X1 != nullptr) {
      const uint4 v1 = load8_as_bf16(static_cast<const char*>(X1) + src * d * esz, e, f32);
      *reinterpret_cast<uint4*>(Y1 + r * d + e) = v1;
    }
  }
}

__global__ void __launch_bounds__(256) scatter_rows_kernel(const __nv_bfloat16* __restrict__ Op,
                                                            const int32_t* __restrict__ perm, long long rows,
                                                            int N, int d, __nv_bfloat16* __restrict__ O,
                                                            DeviceStatus* st) {
  const int per_row = d / 8;
  const long long total = rows * per_row;
  for (long long g = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; g < total;
       g += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = g / per_row;
    const int e = static_cast<int>(g - r * per_row) * 8;
    const long long bh = r / N;
    const int pr = __ldg(perm + r);
    SVG2_DEBUG_CHECK(pr >= 0 && pr < N, st, kWhereGather, r, pr);
    if (pr < 0 || pr >= N) continue;
    const long long dst = bh * N + pr;
    *reinterpret_cast<uint4*>(O + dst * d + e) = __ldg(reinterpret_cast<const uint4*>(Op + r * d + e));
  }
}

int copy_grid(long long work_items) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (work_items + 255) / 256;
  const long long cap = static_cast<long long>(sms) * 8;
  return static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace

cudaError_t launch_sort(const int32_t* labels, int BH, int N, int k, int32_t* perm, int32_t* offsets,
                        int32_t* counts, int32_t* chunk_hist, DeviceStatus* st, cudaStream_t s) {
  const dim3 grid(kSortChunks, BH);
  const size_t smem = static_cast<size_t>(k) * sizeof(int32_t);
  sort_hist_kernel<<<grid, 256, smem, s>>>(labels, N, k, chunk_hist, st);
  sort_scan_kernel<<<BH, 1024, 0, s>>>(N, k, chunk_hist, counts, offsets);
  sort_scatter_kernel<<<grid, 32, smem, s>>>(labels, N, k, chunk_hist, perm);
  return cudaGetLastError();
}

cudaError_t launch_gather(const void* X, bool x_f32, const int32_t* perm, int BH, int N, int d, void* Xp,
                          cudaStream_t s, DeviceStatus* st) {
  const long long rows = static_cast<long long>(BH) * N;
  gather_rows_kernel<<<copy_grid(rows * (d / 8)), 256, 0, s>>>(X, nullptr, x_f32, perm, rows, N, d,
                                                                static_cast<__nv_bfloat16*>(Xp), nullptr, st);
  return cudaGetLastError();
}

cudaError_t launch_gather2(const void* X0, const void* X1, bool x_f32, const int32_t* perm, int BH, int N,
                           int d, void* Xp0, void* Xp1, cudaStream_t s, DeviceStatus* st) {
  const long long rows = static_cast<long long>(BH) * N;
  gather_rows_kernel<<<copy_grid(rows * (d / 8)), 256, 0, s>>>(X0, X1, x_f32, perm, rows, N, d,
                                                                static_cast<__nv_bfloat16*>(Xp0),
                                                                static_cast<__nv_bfloat16*>(Xp1), st);
  return cudaGetLastError();
}

cudaError_t launch_unpermute(const void* Op, const int32_t* perm, int BH, int N, int d, void* O,
                             cudaStream_t s, DeviceStatus* st) {
  const long long rows = static_cast<long long>(BH) * N;
  scatter_rows_kernel<<<copy_grid(rows * (d / 8)), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(Op), perm,
                                                                 rows, N, d, static_cast<__nv_bfloat16*>(O), st);
  return cudaGetLastError();
}

}  // namespace svg2
