// Batched k-means on Q and K per (batch, head) ("Sparse VideoGen2" wiki summary, Method (1);
// Key claims sections 4.1 and 4.3).
//
//  * k-means++ seeding: one CTA per (b,h).  D^2 is kept in float64 and computed exactly as the
//    oracle defines it (sequential, no FMA), so the fixed-point D^2 sampling picks the same seeds.
//    A token is skipped when the triangle inequality proves the new seed cannot be closer
//    (||c_new - c_near||^2 >= 4.0001 D^2), and screened in float32 before the exact recompute.
//  * assignment: tcgen05 GEMM X * C^T on the tensor cores with the centroids split into two bf16
//    terms (hi + lo, residual ~2^-16 |c|), accumulated in TMEM, fused with an argmin epilogue that
//    keeps the best three scores ||c||^2 - 2 x.c per token; when the top scores are closer than the
//    error bound the candidates are re-ranked by exact float32 ||x - c||^2.  A CUDA-core kernel
//    computes exact float32 distances for float32 inputs and d = 64.
//  * update: one warp per cluster sums its members in ascending token order (the stable sort's
//    order) in float64 and divides by the count; an empty cluster keeps its centroid.  It also
//    emits the hi/lo split and ||c||^2 for the next assignment.
#include <cuda.h>
#include <cuda_bf16.h>

#include "svg2_device.cuh"
#include "svg2_internal.h"

namespace svg2 {

namespace {

__device__ __forceinline__ float ld_elem(const void* X, size_t idx, bool f32) {
  if (f32) return __ldg(static_cast<const float*>(X) + idx);
  const unsigned short b = __ldg(static_cast<const unsigned short*>(X) + idx);
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Exact float64 squared distance in the oracle's order: for i ascending, acc = acc + (x_i - c_i)^2.
__device__ __forceinline__ double sqdist_exact(const void* X, size_t row_off, bool f32, const float* c, int d) {
  double acc = 0.0;
  for (int i = 0; i < d; ++i) {
    const double diff = __dsub_rn(static_cast<double>(ld_elem(X, row_off + i, f32)), static_cast<double>(c[i]));
    acc = __dadd_rn(acc, __dmul_rn(diff, diff));
  }
  return acc;
}

__device__ __forceinline__ float sqdist_f32(const void* X, size_t row_off, bool f32, const float* c, int d) {
  float acc = 0.f;
  for (int i = 0; i < d; ++i) {
    const float diff = ld_elem(X, row_off + i, f32) - c[i];
    acc = fmaf(diff, diff, acc);
  }
  return acc;
}

__device__ __forceinline__ unsigned long long fixed_weight(double v, double s) {
  if (!(s > 0.0) || !(v > 0.0)) return 0ull;
  const double r = __ddiv_rn(v, s);
  return static_cast<unsigned long long>(floor(r * 4294967296.0));
}

// Block-wide exclusive scan of a uint64 per thread (blockDim.x == 1024); returns the total.
__device__ unsigned long long block_exscan_u64(unsigned long long v, unsigned long long* excl,
                                               unsigned long long* warp_buf) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  __syncthreads();  // warp_buf reuse across calls
  if (lane == 31) warp_buf[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const unsigned long long w = warp_buf[lane];
    unsigned long long wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    warp_buf[lane] = wi - w;
    if (lane == 31) warp_buf[32] = wi;
  }
  __syncthreads();
  *excl = warp_buf[warp] + incl - v;
  return warp_buf[32];
}

__global__ void __launch_bounds__(1024, 1) kmeanspp_kernel(const void* __restrict__ X, bool f32, int N, int d,
                                                            int k, const double* __restrict__ u,
                                                            float* __restrict__ C, double* __restrict__ Dg,
                                                            int32_t* __restrict__ Ag) {
  __shared__ float cs[128];
  __shared__ float ss[1024];
  __shared__ unsigned long long warp_buf[33];
  __shared__ double red[32];
  __shared__ int pick_sh;
  const int bh = blockIdx.x, tid = threadIdx.x;
  const size_t xbase = static_cast<size_t>(bh) * N * d;
  float* Ch = C + static_cast<size_t>(bh) * k * d;
  double* D = Dg + static_cast<size_t>(bh) * N;
  int32_t* A = Ag + static_cast<size_t>(bh) * N;
  const double* uh = u + static_cast<size_t>(bh) * k;
  const int per = (N + blockDim.x - 1) / blockDim.x;
  const int t0 = min(N, tid * per), t1 = min(N, t0 + per);

  long long pick = static_cast<long long>(floor(uh[0] * static_cast<double>(N)));
  if (pick >= N) pick = N - 1;
  if (pick < 0) pick = 0;
  for (int i = tid; i < d; i += blockDim.x) {
    const float v = ld_elem(X, xbase + static_cast<size_t>(pick) * d + i, f32);
    cs[i] = v;
    Ch[i] = v;
  }
  __syncthreads();
  double lmax = 0.0;
  for (int t = t0; t < t1; ++t) {
    const double v = sqdist_exact(X, xbase + static_cast<size_t>(t) * d, f32, cs, d);
    D[t] = v;
    A[t] = 0;
    lmax = fmax(lmax, v);
  }
  // block max
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lmax = fmax(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
  if ((tid & 31) == 0) red[tid >> 5] = lmax;
  __syncthreads();
  double M0 = 0.0;
  for (int w = 0; w < 32; ++w) M0 = fmax(M0, red[w]);
  unsigned long long qsum = 0ull;
  for (int t = t0; t < t1; ++t) qsum += fixed_weight(D[t], M0);

  for (int s = 1; s < k; ++s) {
    unsigned long long base;
    const unsigned long long U = block_exscan_u64(qsum, &base, warp_buf);
    if (tid == 0) pick_sh = -1;
    __syncthreads();
    if (U == 0ull) {
      if (tid == 0) {
        long long p = static_cast<long long>(floor(uh[s] * static_cast<double>(N)));
        pick_sh = static_cast<int>(p >= N ? N - 1 : p);
      }
    } else {
      unsigned long long target = static_cast<unsigned long long>(floor(uh[s] * static_cast<double>(U)));
      if (target > U - 1ull) target = U - 1ull;
      if (qsum > 0ull && base <= target && target < base + qsum) {
        unsigned long long run = base;
        for (int t = t0; t < t1; ++t) {
          run += fixed_weight(D[t], M0);
          if (run > target) {
            pick_sh = t;
            break;
          }
        }
      }
    }
    __syncthreads();
    const int p = pick_sh < 0 ? N - 1 : pick_sh;
    for (int i = tid; i < d; i += blockDim.x) {
      const float v = ld_elem(X, xbase + static_cast<size_t>(p) * d + i, f32);
      cs[i] = v;
      Ch[static_cast<size_t>(s) * d + i] = v;
    }
    __syncthreads();
    for (int a = tid; a < s; a += blockDim.x) {
      float acc = 0.f;
      const float* ca = Ch + static_cast<size_t>(a) * d;
      for (int i = 0; i < d; ++i) {
        const float diff = cs[i] - ca[i];
        acc = fmaf(diff, diff, acc);
      }
      ss[a] = acc;
    }
    __syncthreads();
    for (int t = t0; t < t1; ++t) {
      const double Dt = D[t];
      if (static_cast<double>(ss[A[t]]) >= 4.0001 * Dt) continue;  // new seed provably farther
      const size_t ro = xbase + static_cast<size_t>(t) * d;
      const float f = sqdist_f32(X, ro, f32, cs, d);
      if (static_cast<double>(f) > Dt * (1.0 + 1e-3)) continue;
      const double nd = sqdist_exact(X, ro, f32, cs, d);
      if (nd < Dt) {
        qsum -= fixed_weight(Dt, M0);
        qsum += fixed_weight(nd, M0);
        D[t] = nd;
        A[t] = s;
      }
    }
  }
}

// Split float32 centroids into bf16 hi + lo parts, zero the padding rows, compute ||c||^2.
__global__ void centroid_prep_kernel(const float* __restrict__ C, int BH, int k, int kpad, int d,
                                     uint16_t* __restrict__ hi, uint16_t* __restrict__ lo,
                                     float* __restrict__ norm) {
  const long long rows = static_cast<long long>(BH) * kpad;
  const int lane = threadIdx.x & 31;
  const long long warp0 = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long r = warp0; r < rows; r += nwarps) {
    const long long bh = r / kpad;
    const int j = static_cast<int>(r - bh * kpad);
    float acc = 0.f;
    for (int i = lane; i < d; i += 32) {
      float c = 0.f;
      if (j < k) c = C[(bh * k + j) * d + i];
      const __nv_bfloat16 h = __float2bfloat16_rn(c);
      const __nv_bfloat16 l = __float2bfloat16_rn(c - __bfloat162float(h));
      hi[r * d + i] = __bfloat16_as_ushort(h);
      lo[r * d + i] = __bfloat16_as_ushort(l);
      acc = fmaf(c, c, acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) norm[r] = acc;
  }
}

// ------------------------------------------------------------------------------------------------
// Exact CUDA-core assignment (float32 inputs, d = 64, or any shape the tensor-core kernel skips)
// ------------------------------------------------------------------------------------------------
constexpr int kExactChunk = 32;

__global__ void __launch_bounds__(128) assign_exact_kernel(const void* __restrict__ X, bool f32, int N, int d,
                                                            int k, const float* __restrict__ C,
                                                            int32_t* __restrict__ labels) {
  __shared__ float cs[kExactChunk * 128];
  const int bh = blockIdx.y;
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  const size_t xo = (static_cast<size_t>(bh) * N + t) * d;
  float best = INFINITY;
  int lab = 0;
  for (int c0 = 0; c0 < k; c0 += kExactChunk) {
    const int nc = min(kExactChunk, k - c0);
    __syncthreads();
    for (int i = threadIdx.x; i < nc * d; i += blockDim.x)
      cs[i] = C[(static_cast<size_t>(bh) * k + c0) * d + i];
    __syncthreads();
    if (t < N) {
      for (int j = 0; j < nc; ++j) {
        const float dist = sqdist_f32(X, xo, f32, cs + j * d, d);
        if (dist < best) {
          best = dist;
          lab = c0 + j;
        }
      }
    }
  }
  if (t < N) labels[static_cast<size_t>(bh) * N + t] = lab;
}

// ------------------------------------------------------------------------------------------------
// Tensor-core assignment (bf16 X, d = 128)
// ------------------------------------------------------------------------------------------------
// Warp roles: 0 = TMA producer, 1 = MMA issuer, 2 = TMEM allocator, 3 = idle, 4..7 = epilogue
// (warp w reads TMEM lanes 32*(w%4) .. +31, i.e. tokens 32*(w-4) .. +31 of the tile).
constexpr int kAsgThreads = 256;
constexpr uint32_t kAsgXStage = 32768;   // 128 tokens x 128 d bf16 (two 16 KB halves)
constexpr uint32_t kAsgCStage = 65536;   // 128 centroids x 128 d x {hi, lo}
constexpr uint32_t kAsgSmem = 2 * kAsgXStage + 2 * kAsgCStage + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t kAsgTmemCols = 512;   // 4 accumulators of 128 columns

struct AsgBars {
  uint64_t x_full[2], x_empty[2], c_full[2], c_empty[2], acc_full[4], acc_empty[4], mma_done;
  uint32_t tmem_base;
};

__device__ __forceinline__ void top3_insert(float s, int j, float& s1, int& i1, float& s2, int& i2, float& s3,
                                            int& i3) {
  if (s < s3) {
    if (s < s2) {
      s3 = s2;
      i3 = i2;
      if (s < s1) {
        s2 = s1;
        i2 = i1;
        s1 = s;
        i1 = j;
      } else {
        s2 = s;
        i2 = j;
      }
    } else {
      s3 = s;
      i3 = j;
    }
  }
}

// Exact float32 distance between the token row held in the swizzled X tile and centroid row c.
__device__ __forceinline__ float tile_row_dist(const uint8_t* xt, int row, const float* __restrict__ c) {
  float acc = 0.f;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      const uint4 v = *reinterpret_cast<const uint4*>(xt + h * 16384 + sw128_offset(row, ch));
      const float4 c0 = __ldg(reinterpret_cast<const float4*>(c + h * 64 + ch * 8));
      const float4 c1 = __ldg(reinterpret_cast<const float4*>(c + h * 64 + ch * 8 + 4));
      float x[8] = {bf16lo_to_f32(v.x), bf16hi_to_f32(v.x), bf16lo_to_f32(v.y), bf16hi_to_f32(v.y),
                    bf16lo_to_f32(v.z), bf16hi_to_f32(v.z), bf16lo_to_f32(v.w), bf16hi_to_f32(v.w)};
      const float cc[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float df = x[e] - cc[e];
        acc = fmaf(df, df, acc);
      }
    }
  }
  return acc;
}

__device__ __forceinline__ float tile_row_norm(const uint8_t* xt, int row) {
  float acc = 0.f;
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      const uint4 v = *reinterpret_cast<const uint4*>(xt + h * 16384 + sw128_offset(row, ch));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = bf16lo_to_f32(w[e]), b = bf16hi_to_f32(w[e]);
        acc = fmaf(a, a, acc);
        acc = fmaf(b, b, acc);
      }
    }
  return acc;
}

__global__ void __launch_bounds__(kAsgThreads, 1)
    assign_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_hi,
                     const __grid_constant__ CUtensorMap tm_lo, int BH, int N, int k, int kpad,
                     const float* __restrict__ C, const float* __restrict__ c_norm, int32_t* __restrict__ labels,
                     DeviceStatus* st) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xs = smem;                       // 2 stages
  uint8_t* cstg = smem + 2 * kAsgXStage;    // 2 stages
  AsgBars* bars = reinterpret_cast<AsgBars*>(cstg + 2 * kAsgCStage);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = (N + kAssignTileM - 1) / kAssignTileM;
  const long long total = static_cast<long long>(BH) * ntiles;
  const int nchunks = kpad / kAssignChunkN;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars->x_full[i]), 1);
      mbar_init(smem_u32(&bars->x_empty[i]), 1 + 4);
      mbar_init(smem_u32(&bars->c_full[i]), 1);
      mbar_init(smem_u32(&bars->c_empty[i]), 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(smem_u32(&bars->acc_full[i]), 1);
      mbar_init(smem_u32(&bars->acc_empty[i]), 4);
    }
    mbar_init(smem_u32(&bars->mma_done), 1);
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(&bars->tmem_base), kAsgTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (elect_one()) {
      prefetch_tensormap(&tm_x);
      prefetch_tensormap(&tm_hi);
      prefetch_tensormap(&tm_lo);
      long long g = 0;  // chunk counter
      int it = 0;
      bool ok = true;
      for (long long w = blockIdx.x; w < total && ok; w += gridDim.x, ++it) {
        const int bh = static_cast<int>(w / ntiles), tile = static_cast<int>(w % ntiles);
        const int xsI = it & 1;
        if (it >= 2) ok = mbar_wait(smem_u32(&bars->x_empty[xsI]), ((it >> 1) - 1) & 1, st, kWhereAssign);
        if (!ok) break;
        const uint32_t xdst = smem_u32(xs + xsI * kAsgXStage);
        mbar_arrive_expect_tx(smem_u32(&bars->x_full[xsI]), kAsgXStage);
        const int y = bh * N + tile * kAssignTileM;
        tma_load_2d(xdst, &tm_x, 0, y, smem_u32(&bars->x_full[xsI]));
        tma_load_2d(xdst + 16384, &tm_x, 64, y, smem_u32(&bars->x_full[xsI]));
        for (int c = 0; c < nchunks; ++c, ++g) {
          const int cs = static_cast<int>(g & 1);
          if (g >= 2) ok = mbar_wait(smem_u32(&bars->c_empty[cs]), ((g >> 1) - 1) & 1, st, kWhereAssign);
          if (!ok) break;
          const uint32_t cdst = smem_u32(cstg + cs * kAsgCStage);
          const uint32_t bar = smem_u32(&bars->c_full[cs]);
          mbar_arrive_expect_tx(bar, kAsgCStage);
          const int yc = bh * kpad + c * kAssignChunkN;
          tma_load_2d(cdst, &tm_hi, 0, yc, bar);
          tma_load_2d(cdst + 16384, &tm_hi, 64, yc, bar);
          tma_load_2d(cdst + 32768, &tm_lo, 0, yc, bar);
          tma_load_2d(cdst + 49152, &tm_lo, 64, yc, bar);
        }
      }
      // Before the CTA may exit, every load it issued must have landed (normally already true).
      const long long drain = kWaitBudgetCycles / 8;
      for (int i = it - 2; i < it; ++i)
        if (i >= 0) mbar_wait(smem_u32(&bars->x_full[i & 1]), (i >> 1) & 1, nullptr, kWhereAssignTail, drain);
      for (long long i = g - 2; i < g; ++i)
        if (i >= 0) mbar_wait(smem_u32(&bars->c_full[i & 1]), (i >> 1) & 1, nullptr, kWhereAssignTail, drain);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (elect_one()) {
      const uint32_t idesc = idesc_bf16_f32(128, kAssignChunkN, 0);
      long long g = 0;
      int it = 0;
      bool ok = true;
      for (long long w = blockIdx.x; w < total && ok; w += gridDim.x, ++it) {
        const int xsI = it & 1;
        ok = mbar_wait(smem_u32(&bars->x_full[xsI]), (it >> 1) & 1, st, kWhereAssign);
        if (!ok) break;
        const uint32_t xa = smem_u32(xs + xsI * kAsgXStage);
        for (int c = 0; c < nchunks; ++c, ++g) {
          const int cs = static_cast<int>(g & 1);
          const int a = static_cast<int>(g & 3);
          ok = mbar_wait(smem_u32(&bars->c_full[cs]), (g >> 1) & 1, st, kWhereAssign);
          if (ok && g >= 4) ok = mbar_wait(smem_u32(&bars->acc_empty[a]), ((g >> 2) - 1) & 1, st, kWhereAssign);
          if (!ok) break;
          tc_fence_after();
          const uint32_t cb = smem_u32(cstg + cs * kAsgCStage);
          const uint32_t d_tmem = tmem + a * kAssignChunkN;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t koff = (ks >> 2) * 16384 + (ks & 3) * 32;
            const uint64_t ad = sdesc_sw128(xa + koff, 16, 1024);
            const uint64_t bh_d = sdesc_sw128(cb + koff, 16, 1024);
            const uint64_t bl_d = sdesc_sw128(cb + 32768 + koff, 16, 1024);
            mma_ss(d_tmem, ad, bh_d, idesc, ks > 0 ? 1u : 0u);
            mma_ss(d_tmem, ad, bl_d, idesc, 1u);
          }
          mma_commit(smem_u32(&bars->acc_full[a]));
          mma_commit(smem_u32(&bars->c_empty[cs]));
        }
        if (ok) mma_commit(smem_u32(&bars->x_empty[xsI]));
      }
      // no MMA may still be writing TMEM when the allocator frees it
      mma_commit(smem_u32(&bars->mma_done));
      mbar_wait(smem_u32(&bars->mma_done), 0, nullptr, kWhereAssignTail, kWaitBudgetCycles / 8);
    }
  } else if (warp >= 4) {
    // ---------------- epilogue: argmin over centroids ----------------
    const int q = warp & 3;
    const int row = q * 32 + lane;
    long long g = 0;
    int it = 0;
    bool ok = true;
    for (long long w = blockIdx.x; w < total && ok; w += gridDim.x, ++it) {
      const int bh = static_cast<int>(w / ntiles), tile = static_cast<int>(w % ntiles);
      const int xsI = it & 1;
      float s1 = INFINITY, s2 = INFINITY, s3 = INFINITY;
      int i1 = 0, i2 = -1, i3 = -1;
      const float* cn = c_norm + static_cast<size_t>(bh) * kpad;
      for (int c = 0; c < nchunks; ++c, ++g) {
        const int a = static_cast<int>(g & 3);
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->acc_full[a]), (g >> 2) & 1, st, kWhereAssign));
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int qq = 0; qq < 4; ++qq) {
          uint32_t v[32];
          tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + a * kAssignChunkN + qq * 32, v);
          tmem_wait_ld();
          const int jb = c * kAssignChunkN + qq * 32;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int j = jb + e;
            if (j < k) {
              const float s = fmaf(-2.f, __uint_as_float(v[e]), __ldg(cn + j));
              top3_insert(s, j, s1, i1, s2, i2, s3, i3);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->acc_empty[a]));
      }
      if (!ok) break;
      // the X tile is still resident (its stage is released only after this epilogue arrives)
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->x_full[xsI]), (it >> 1) & 1, st, kWhereAssignTail));
      if (!ok) break;
      const int n = tile * kAssignTileM + row;
      if (n < N) {
        int best = i1;
        if (i2 >= 0) {
          const uint8_t* xt = xs + xsI * kAsgXStage;
          const float xn = tile_row_norm(xt, row);
          const float tau = ldexpf(xn + fmaxf(__ldg(cn + i1), __ldg(cn + i2)), -10);
          if (s2 - s1 < tau) {
            const float* Cb = C + static_cast<size_t>(bh) * k * 128;
            float bd = tile_row_dist(xt, row, Cb + static_cast<size_t>(i1) * 128);
            const float d2 = tile_row_dist(xt, row, Cb + static_cast<size_t>(i2) * 128);
            if (d2 < bd || (d2 == bd && i2 < best)) {
              bd = d2;
              best = i2;
            }
            if (i3 >= 0 && s3 - s1 < tau) {
              const float d3 = tile_row_dist(xt, row, Cb + static_cast<size_t>(i3) * 128);
              if (d3 < bd || (d3 == bd && i3 < best)) {
                bd = d3;
                best = i3;
              }
            }
          }
        }
        labels[static_cast<size_t>(bh) * N + n] = best;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->x_empty[xsI]));
    }
  }

  __syncwarp();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kAsgTmemCols);
  }
}

// ------------------------------------------------------------------------------------------------
// Update: centroid = mean of members (float64, ascending token order)
// ------------------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) update_kernel(const void* __restrict__ X, bool f32, int BH, int N, int k,
                                                      int kpad, const int32_t* __restrict__ perm,
                                                      const int32_t* __restrict__ offsets,
                                                      float* __restrict__ C, uint16_t* __restrict__ hi,
                                                      uint16_t* __restrict__ lo, float* __restrict__ norm) {
  constexpr int E = D / 32;  // dims per lane
  const int lane = threadIdx.x & 31;
  const long long wid = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5;
  if (wid >= static_cast<long long>(BH) * k) return;
  const int bh = static_cast<int>(wid / k), j = static_cast<int>(wid % k);
  const int o0 = offsets[static_cast<size_t>(bh) * (k + 1) + j];
  const int o1 = offsets[static_cast<size_t>(bh) * (k + 1) + j + 1];
  const int cnt = o1 - o0;
  float* cj = C + (static_cast<size_t>(bh) * k + j) * D;
  float c[E];
  if (cnt > 0) {
    double acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.0;
    const int32_t* pr = perm + static_cast<size_t>(bh) * N;
    const size_t xb = static_cast<size_t>(bh) * N * D + lane * E;
    int r = o0;
    constexpr int U = 8;
    for (; r + U <= o1; r += U) {
      float xv[U][E];
#pragma unroll
      for (int uu = 0; uu < U; ++uu) {
        const size_t ro = xb + static_cast<size_t>(__ldg(pr + r + uu)) * D;
#pragma unroll
        for (int e = 0; e < E; ++e) xv[uu][e] = ld_elem(X, ro + e, f32);
      }
#pragma unroll
      for (int uu = 0; uu < U; ++uu)
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = __dadd_rn(acc[e], static_cast<double>(xv[uu][e]));
    }
    for (; r < o1; ++r) {
      const size_t ro = xb + static_cast<size_t>(__ldg(pr + r)) * D;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = __dadd_rn(acc[e], static_cast<double>(ld_elem(X, ro + e, f32)));
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {
      c[e] = static_cast<float>(__ddiv_rn(acc[e], static_cast<double>(cnt)));
      cj[lane * E + e] = c[e];
    }
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) c[e] = cj[lane * E + e];
  }
  float nrm = 0.f;
  const size_t ro = (static_cast<size_t>(bh) * kpad + j) * D + lane * E;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const __nv_bfloat16 h = __float2bfloat16_rn(c[e]);
    const __nv_bfloat16 l = __float2bfloat16_rn(c[e] - __bfloat162float(h));
    hi[ro + e] = __bfloat16_as_ushort(h);
    lo[ro + e] = __bfloat16_as_ushort(l);
    nrm = fmaf(c[e], c[e], nrm);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) nrm += __shfl_xor_sync(0xffffffffu, nrm, o);
  if (lane == 0) norm[static_cast<size_t>(bh) * kpad + j] = nrm;
}

int num_sms() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

}  // namespace

cudaError_t launch_kmeanspp(const void* X, bool x_f32, int BH, int N, int d, int k, const double* u,
                            float* centroids, double* dist, int32_t* near, cudaStream_t s) {
  kmeanspp_kernel<<<BH, 1024, 0, s>>>(X, x_f32, N, d, k, u, centroids, dist, near);
  return cudaGetLastError();
}

cudaError_t launch_centroid_prep(const float* centroids, int BH, int k, int d, uint16_t* c_hi, uint16_t* c_lo,
                                 float* c_norm, cudaStream_t s) {
  const int kp = kpad_of(k);
  const long long rows = static_cast<long long>(BH) * kp;
  const int blocks = static_cast<int>((rows * 32 + 255) / 256 < 4096 ? (rows * 32 + 255) / 256 : 4096);
  centroid_prep_kernel<<<blocks, 256, 0, s>>>(centroids, BH, k, kp, d, c_hi, c_lo, c_norm);
  return cudaGetLastError();
}

cudaError_t launch_assign(const void* X, bool x_f32, int BH, int N, int d, int k, const float* centroids,
                          const uint16_t* c_hi, const uint16_t* c_lo, const float* c_norm, int32_t* labels,
                          DeviceStatus* st, cudaStream_t s) {
  if (!x_f32 && d == 128) {
    alignas(64) CUtensorMap tx, th, tl;
    const int kp = kpad_of(k);
    cudaError_t e = make_tmap_bf16_rows(&tx, X, static_cast<uint64_t>(BH) * N, 128, kAssignTileM);
    if (e == cudaSuccess) e = make_tmap_bf16_rows(&th, c_hi, static_cast<uint64_t>(BH) * kp, 128, kAssignChunkN);
    if (e == cudaSuccess) e = make_tmap_bf16_rows(&tl, c_lo, static_cast<uint64_t>(BH) * kp, 128, kAssignChunkN);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(assign_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAsgSmem);
    if (e != cudaSuccess) return e;
    const long long tiles = static_cast<long long>(BH) * ((N + kAssignTileM - 1) / kAssignTileM);
    const int grid = static_cast<int>(tiles < num_sms() ? tiles : num_sms());
    assign_tc_kernel<<<grid, kAsgThreads, kAsgSmem, s>>>(tx, th, tl, BH, N, k, kp, centroids, c_norm, labels, st);
    return cudaGetLastError();
  }
  const dim3 grid((N + 127) / 128, BH);
  assign_exact_kernel<<<grid, 128, 0, s>>>(X, x_f32, N, d, k, centroids, labels);
  return cudaGetLastError();
}

cudaError_t launch_update(const void* X, bool x_f32, int BH, int N, int d, int k, const int32_t* perm,
                          const int32_t* offsets, float* centroids, uint16_t* c_hi, uint16_t* c_lo,
                          float* c_norm, cudaStream_t s) {
  const long long warps = static_cast<long long>(BH) * k;
  const int blocks = static_cast<int>((warps * 32 + 255) / 256);
  const int kp = kpad_of(k);
  if (d == 128)
    update_kernel<128><<<blocks, 256, 0, s>>>(X, x_f32, BH, N, k, kp, perm, offsets, centroids, c_hi, c_lo, c_norm);
  else
    update_kernel<64><<<blocks, 256, 0, s>>>(X, x_f32, BH, N, k, kp, perm, offsets, centroids, c_hi, c_lo, c_norm);
  return cudaGetLastError();
}

}  // namespace svg2
