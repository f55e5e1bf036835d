// Batched k-means on Q and K per (batch, head) ("Sparse VideoGen2" wiki summary, Method (1);
// Key claims sections 4.1 and 4.3).
//
//  * k-means++ seeding: one CTA per (b,h).  D^2 is kept in float64 and computed exactly as the
//    oracle defines it (sequential, no FMA), so the fixed-point D^2 sampling picks the same seeds.
//    A token is skipped when the triangle inequality proves the new seed cannot be closer
//    (||c_new - c_near||^2 >= 4.0001 D^2), and screened in float32 before the exact recompute.
//  * assignment: tcgen05 GEMM X * C^T on the tensor cores with the centroids split into two bf16
//    terms (hi + lo, residual ~2^-16 |c|), accumulated in TMEM, fused with an argmin epilogue over
//    the scores ||c||^2 - 2 x.c.  Per token the epilogue keeps the 4 smallest scores that lie
//    within the error tolerance tau of the running minimum; a token left with one candidate is
//    labelled there, a token with several (a near-tie) goes on a list that rerank_kernel decides
//    by exact float32 ||x - c||^2, and a token whose 4-entry list overflowed (a fifth score within
//    tau was dropped) goes on the same list with a flag that makes the re-rank scan all k
//    centroids.  A CUDA-core kernel computes exact float32 distances for float32 inputs and d = 64.
//  * update: one CTA per cluster stages its members' rows (ascending token order, the stable
//    sort's) through shared memory and sums each dimension sequentially in float64, then divides by
//    the count; an empty cluster keeps its centroid.  It also emits the hi/lo split and ||c||^2
//    for the next assignment.
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

// Fallback for candidate sets too large for shared memory: one CTA per (b,h), state in global memory.
__global__ void __launch_bounds__(1024, 1) kmeanspp_kernel(const void* __restrict__ X, bool f32, int Ntok, int stride,
                                                            int d, int k, const double* __restrict__ u,
                                                            float* __restrict__ C, double* __restrict__ Dg,
                                                            int32_t* __restrict__ Ag) {
  const int N = (Ntok + stride - 1) / stride;  // candidates: every stride-th row (the launcher passes 1)
  __shared__ float cs[128];
  __shared__ float ss[1024];
  __shared__ unsigned long long warp_buf[33];
  __shared__ double red[32];
  __shared__ int pick_sh;
  const int bh = blockIdx.x, tid = threadIdx.x;
  const size_t xbase = static_cast<size_t>(bh) * Ntok * d;
  const size_t rstride = static_cast<size_t>(stride) * d;  // elements between candidate rows
  float* Ch = C + static_cast<size_t>(bh) * k * d;
  double* D = Dg + static_cast<size_t>(bh) * Ntok;
  int32_t* A = Ag + static_cast<size_t>(bh) * Ntok;
  const double* uh = u + static_cast<size_t>(bh) * k;
  const int per = (N + blockDim.x - 1) / blockDim.x;
  const int t0 = min(N, tid * per), t1 = min(N, t0 + per);

  long long pick = static_cast<long long>(floor(uh[0] * static_cast<double>(N)));
  if (pick >= N) pick = N - 1;
  if (pick < 0) pick = 0;
  for (int i = tid; i < d; i += blockDim.x) {
    const float v = ld_elem(X, xbase + static_cast<size_t>(pick) * rstride + i, f32);
    cs[i] = v;
    Ch[i] = v;
  }
  __syncthreads();
  double lmax = 0.0;
  for (int t = t0; t < t1; ++t) {
    const double v = sqdist_exact(X, xbase + static_cast<size_t>(t) * rstride, f32, cs, d);
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
      const float v = ld_elem(X, xbase + static_cast<size_t>(p) * rstride + i, f32);
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
      const size_t ro = xbase + static_cast<size_t>(t) * rstride;
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

// ------------------------------------------------------------------------------------------------
// k-means++ seeding kernels with shared-memory state (see kmeanspp_kernel2 below)
// ------------------------------------------------------------------------------------------------
constexpr int kPpThreads = 512;
constexpr int kPpWarps = kPpThreads / 32;
constexpr int kPpMaxPerCta = 15360;   // 10 bytes of state per candidate: 150 KB of shared memory
constexpr int kPpMaxCluster = 16;     // non-portable cluster size limit

__host__ __device__ constexpr size_t pp_smem_bytes(int per_cta) {
  return static_cast<size_t>(per_cta) * 10 + 16;
}

template <int E, bool F32>
__device__ __forceinline__ void pp_load_row(const void* X, size_t row_elem, int lane, float (&v)[E]) {
  if constexpr (F32) {
    const float* p = static_cast<const float*>(X) + row_elem + lane * E;
    if constexpr (E == 4) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(p));
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    } else {
      const float2 a = __ldg(reinterpret_cast<const float2*>(p));
      v[0] = a.x; v[1] = a.y;
    }
  } else {
    const unsigned short* p = static_cast<const unsigned short*>(X) + row_elem + lane * E;
    if constexpr (E == 4) {
      const uint2 a = __ldg(reinterpret_cast<const uint2*>(p));
      v[0] = bf16lo_to_f32(a.x); v[1] = bf16hi_to_f32(a.x); v[2] = bf16lo_to_f32(a.y); v[3] = bf16hi_to_f32(a.y);
    } else {
      const uint32_t a = __ldg(reinterpret_cast<const uint32_t*>(p));
      v[0] = bf16lo_to_f32(a); v[1] = bf16hi_to_f32(a);
    }
  }
}

// Raw row values of lane `lane` (E per lane) as 32-bit words: bf16 pairs, or float32 values.
template <int E, bool F32>
constexpr int pp_words() { return F32 ? E : E / 2; }

template <int E, bool F32>
__device__ __forceinline__ void pp_load_raw(const void* X, size_t row_elem, int lane,
                                            uint32_t (&w)[pp_words<E, F32>()]) {
  if constexpr (F32) {
    static_assert(E == 2, "float32 rows use d = 64 on this path");
    const float2 a = __ldg(reinterpret_cast<const float2*>(static_cast<const float*>(X) + row_elem + lane * E));
    w[0] = __float_as_uint(a.x);
    w[1] = __float_as_uint(a.y);
  } else {
    const unsigned short* p = static_cast<const unsigned short*>(X) + row_elem + lane * E;
    if constexpr (E == 4) {
      const uint2 a = __ldg(reinterpret_cast<const uint2*>(p));
      w[0] = a.x;
      w[1] = a.y;
    } else {
      w[0] = __ldg(reinterpret_cast<const uint32_t*>(p));
    }
  }
}

template <int E, bool F32>
__device__ __forceinline__ void pp_unpack(const uint32_t (&w)[pp_words<E, F32>()], float (&v)[E]) {
  if constexpr (F32) {
#pragma unroll
    for (int i = 0; i < E; ++i) v[i] = __uint_as_float(w[i]);
  } else {
#pragma unroll
    for (int i = 0; i < E / 2; ++i) {
      v[2 * i] = bf16lo_to_f32(w[i]);
      v[2 * i + 1] = bf16hi_to_f32(w[i]);
    }
  }
}

// Exact float64 D^2 of one token row against cs, sequential over i (the oracle's order, no FMA).
template <int D, bool F32>
__device__ __forceinline__ double pp_exact_seq(const void* X, size_t row_elem, const float* cs) {
  double acc = 0.0;
  if constexpr (F32) {
    const float4* r = reinterpret_cast<const float4*>(static_cast<const float*>(X) + row_elem);
#pragma unroll 4
    for (int q = 0; q < D / 4; ++q) {
      const float4 a = __ldg(r + q);
      const float x[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const double df = __dsub_rn(static_cast<double>(x[e]), static_cast<double>(cs[4 * q + e]));
        acc = __dadd_rn(acc, __dmul_rn(df, df));
      }
    }
  } else {
    const uint4* r = reinterpret_cast<const uint4*>(static_cast<const unsigned short*>(X) + row_elem);
#pragma unroll 4
    for (int q = 0; q < D / 8; ++q) {
      const uint4 a = __ldg(r + q);
      const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const double d0 = __dsub_rn(static_cast<double>(bf16lo_to_f32(w[e])), static_cast<double>(cs[8 * q + 2 * e]));
        acc = __dadd_rn(acc, __dmul_rn(d0, d0));
        const double d1 = __dsub_rn(static_cast<double>(bf16hi_to_f32(w[e])), static_cast<double>(cs[8 * q + 2 * e + 1]));
        acc = __dadd_rn(acc, __dmul_rn(d1, d1));
      }
    }
  }
  return acc;
}

template <int E>
__device__ __forceinline__ double pp_exact(const float (&v)[E], const float* cs, int lane) {
  double acc = 0.0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const double df = __dsub_rn(static_cast<double>(v[e]), static_cast<double>(cs[lane * E + e]));
    acc = __dadd_rn(acc, __dmul_rn(df, df));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc = __dadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, o));
  return __shfl_sync(0xffffffffu, acc, 0);  // lane 0's summation order decides
}

__device__ __forceinline__ void pp_sync(int ncl) {
  if (ncl > 1) cluster_sync();
  else __syncthreads();
}

// Store v into `var` of every CTA of the cluster (this CTA's own copy when there is no cluster).
__device__ __forceinline__ void pp_bcast_u64(unsigned long long* var, unsigned long long v, int ncl) {
  if (ncl > 1) {
    for (int r = 0; r < ncl; ++r) st_cluster_u64(var, static_cast<uint32_t>(r), v);
  } else {
    *var = v;
  }
}

// k-means++ seeding over a candidate set: every `stride`-th token (stride 1 = all tokens), S in all.
// One (b,h) runs on the CTAs of one thread-block cluster (1 to kPpMaxCluster of them, chosen at
// launch): each keeps its share of the candidates' state (D^2 in float64 and the nearest seed) in
// shared memory, and the per-seed totals and the pick travel through distributed shared memory.  Lane l of warp w
// owns a contiguous piece of the warp's candidates, so a lane's running fixed-point weight total is
// its piece's total and the sampling search needs no division until the final piece scan.
// Per seed: ||c_new - c_near||^2 >= 4.0001 D^2 proves a candidate cannot get closer; the rest get
// a float32 distance (warp-cooperative, or a transpose-reduce over 32 candidates when many are
// left); those within 1e-3 of their D^2 get the float64 D^2 (per-lane sums over d/32 values, then a
// fixed butterfly across lanes, lane 0's order).  That can differ from a sequential sum in the last
// bit, which moves the fixed-point weight floor(D^2 / M0 * 2^32) only when D^2 / M0 * 2^32 lies
// within ~1e-6 of an integer, and changes a seed only if the sampling target sits exactly on it.
template <int E, bool F32>
__global__ void __launch_bounds__(kPpThreads, 1)
    kmeanspp_kernel2(const void* __restrict__ X, int N, int stride, int S, int k, const double* __restrict__ u,
                     float* __restrict__ C) {
  constexpr int D = E * 32;
  extern __shared__ uint8_t pp_smem[];
  __shared__ float cs[D];
  __shared__ float ss[1024];
  __shared__ unsigned long long wsum[kPpWarps];
  __shared__ unsigned long long cta_tot[kPpMaxCluster];
  __shared__ unsigned long long cta_max[kPpMaxCluster];
  __shared__ unsigned long long pick_bcast;
  __shared__ unsigned long long hit_base;
  __shared__ int hit_warp;
  const int CL = static_cast<int>(cluster_nctas());  // 1 for a launch without clusters
  const uint32_t rank = cluster_rank();
  const int bh = blockIdx.x / CL;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_cta = (S + CL - 1) / CL;
  const int lo = min(S, static_cast<int>(rank) * per_cta), hi = min(S, lo + per_cta);
  const int per_warp = (hi - lo + kPpWarps - 1) / kPpWarps;
  const int wlo = min(hi, lo + warp * per_warp), whi = min(hi, wlo + per_warp);
  const int P = (whi - wlo + 31) / 32;  // candidates per lane piece
  const int plo = min(whi, wlo + lane * P), phi = min(whi, plo + P);
  double* Ds = reinterpret_cast<double*>(pp_smem);
  uint16_t* As = reinterpret_cast<uint16_t*>(pp_smem + static_cast<size_t>(per_cta) * 8);
  const size_t xbase = static_cast<size_t>(bh) * N * D;
  float* Ch = C + static_cast<size_t>(bh) * k * D;
  const double* uh = u + static_cast<size_t>(bh) * k;
  auto row_of = [&](int cand) { return xbase + static_cast<size_t>(cand) * stride * D; };

  auto load_seed = [&](int cand, int s) {
    for (int i = threadIdx.x; i < D; i += blockDim.x) {
      float v;
      if constexpr (F32) v = static_cast<const float*>(X)[row_of(cand) + i];
      else v = bf16lo_to_f32(static_cast<const unsigned short*>(X)[row_of(cand) + i]);
      cs[i] = v;
      if (rank == 0) Ch[static_cast<size_t>(s) * D + i] = v;
    }
  };

  unsigned long long qsum = 0ull;  // fixed-point weight of this lane's piece
  double M0 = 0.0;

  // float64 D^2 of up to 4 candidates at once (warp-cooperative; every lane gets lane 0's sums)
  auto exact4 = [&](const int (&cb)[4], double (&nd)[4]) {
    double acc[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[i] = 0.0;
      if (cb[i] >= 0) {
        float v[E];
        pp_load_row<E, F32>(X, row_of(cb[i]), lane, v);
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const double df = __dsub_rn(static_cast<double>(v[e]), static_cast<double>(cs[lane * E + e]));
          acc[i] = __dadd_rn(acc[i], __dmul_rn(df, df));
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = __dadd_rn(acc[i], __shfl_xor_sync(0xffffffffu, acc[i], o));
#pragma unroll
    for (int i = 0; i < 4; ++i) nd[i] = __shfl_sync(0xffffffffu, acc[i], 0);
  };

  auto update_pass = [&](int s, bool first) {
    for (int i = 0; i < P; ++i) {
      const int c = plo + i;  // this lane's candidate in slice i
      double Dt = INFINITY;
      bool cand = false;
      if (c < phi) {
        if (first) {
          cand = true;
        } else {
          Dt = Ds[c - lo];
          cand = static_cast<double>(ss[As[c - lo]]) < 4.0001 * Dt;  // else provably not closer
        }
      }
      const unsigned m = __ballot_sync(0xffffffffu, cand);
      if (m == 0u) continue;
      bool need = cand;
      if (!first) {
        float f = 0.f;
        if (__popc(m) <= 8) {
          // few candidates: one warp-cooperative float32 distance each, 4 at a time
          unsigned mm = m;
          while (mm) {
            int bl[4];
            float part[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              bl[q] = mm ? __ffs(mm) - 1 : -1;
              if (mm) mm &= mm - 1;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              part[q] = 0.f;
              const int cq = __shfl_sync(0xffffffffu, c, bl[q] < 0 ? 0 : bl[q]);
              if (bl[q] >= 0) {
                float v[E];
                pp_load_row<E, F32>(X, row_of(cq), lane, v);
#pragma unroll
                for (int e = 0; e < E; ++e) {
                  const float df = v[e] - cs[lane * E + e];
                  part[q] = fmaf(df, df, part[q]);
                }
              }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
              for (int q = 0; q < 4; ++q) part[q] += __shfl_xor_sync(0xffffffffu, part[q], o);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float fq = __shfl_sync(0xffffffffu, part[q], 0);
              if (lane == bl[q]) f = fq;
            }
          }
        } else {
          // many candidates: all rows in flight, then a transpose-reduce leaves lane l its own sum
          uint32_t raw[32][pp_words<E, F32>()];
#pragma unroll
          for (int r = 0; r < 32; ++r) {
            const int cr = __shfl_sync(0xffffffffu, c, r);
            if ((m >> r) & 1u) pp_load_raw<E, F32>(X, row_of(cr), lane, raw[r]);
          }
          float pr[32];
#pragma unroll
          for (int r = 0; r < 32; ++r) {
            pr[r] = 0.f;
            if ((m >> r) & 1u) {
              float v[E];
              pp_unpack<E, F32>(raw[r], v);
#pragma unroll
              for (int e = 0; e < E; ++e) {
                const float df = v[e] - cs[lane * E + e];
                pr[r] = fmaf(df, df, pr[r]);
              }
            }
          }
#pragma unroll
          for (int o = 16, n = 16; o > 0; o >>= 1, n >>= 1) {
            const bool upper = (lane & o) != 0;
#pragma unroll
            for (int q = 0; q < n; ++q) {
              const float keep = upper ? pr[q + n] : pr[q];
              const float send = upper ? pr[q] : pr[q + n];
              pr[q] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
          }
          f = pr[0];
        }
        need = cand && static_cast<double>(f) <= Dt * (1.0 + 1e-3);  // float32 error << 1e-3
      }
      unsigned nm = __ballot_sync(0xffffffffu, need);
      while (nm) {
        int bl[4], cb[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          bl[q] = nm ? __ffs(nm) - 1 : -1;
          if (nm) nm &= nm - 1;
          const int cq = __shfl_sync(0xffffffffu, c, bl[q] < 0 ? 0 : bl[q]);
          cb[q] = bl[q] >= 0 ? cq : -1;
        }
        double nd[4];
        exact4(cb, nd);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (lane == bl[q] && nd[q] < Dt) {
            if (!first) {
              qsum -= fixed_weight(Dt, M0);
              qsum += fixed_weight(nd[q], M0);
            }
            Ds[c - lo] = nd[q];
            As[c - lo] = static_cast<uint16_t>(s);
          }
        }
      }
    }
  };

  // ---- seed 0, the initial D^2 and the fixed-point scale M0 (maximum over all candidates)
  long long p0 = static_cast<long long>(floor(uh[0] * static_cast<double>(S)));
  if (p0 >= S) p0 = S - 1;
  if (p0 < 0) p0 = 0;
  load_seed(static_cast<int>(p0), 0);
  __syncthreads();
  update_pass(0, true);
  __syncwarp();
  double lmax = 0.0;
  for (int c = plo; c < phi; ++c) lmax = fmax(lmax, Ds[c - lo]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lmax = fmax(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
  if (lane == 0) wsum[warp] = static_cast<unsigned long long>(__double_as_longlong(lmax));
  __syncthreads();
  if (threadIdx.x == 0) {
    double mx = 0.0;
    for (int w = 0; w < kPpWarps; ++w) mx = fmax(mx, __longlong_as_double(static_cast<long long>(wsum[w])));
    pp_bcast_u64(&cta_max[rank], static_cast<unsigned long long>(__double_as_longlong(mx)), CL);
  }
  pp_sync(CL);
  for (int r = 0; r < CL; ++r) M0 = fmax(M0, __longlong_as_double(static_cast<long long>(cta_max[r])));
  for (int c = plo; c < phi; ++c) qsum += fixed_weight(Ds[c - lo], M0);

  for (int s = 1; s < k; ++s) {
    // ---- totals: lanes -> warps -> CTA -> every CTA of the cluster
    unsigned long long wq = qsum;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wq += __shfl_xor_sync(0xffffffffu, wq, o);
    if (lane == 0) wsum[warp] = wq;
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned long long t = 0;
      for (int w = 0; w < kPpWarps; ++w) t += wsum[w];
      pp_bcast_u64(&cta_tot[rank], t, CL);
    }
    pp_sync(CL);
    unsigned long long U = 0, base = 0;
    for (int r = 0; r < CL; ++r) {
      if (r < static_cast<int>(rank)) base += cta_tot[r];
      U += cta_tot[r];
    }
    if (U == 0ull) {
      if (threadIdx.x == 0 && rank == 0) {
        const long long p = static_cast<long long>(floor(uh[s] * static_cast<double>(S)));
        pp_bcast_u64(&pick_bcast, static_cast<unsigned long long>(p >= S ? S - 1 : p), CL);
      }
    } else {
      unsigned long long target = static_cast<unsigned long long>(floor(uh[s] * static_cast<double>(U)));
      if (target > U - 1ull) target = U - 1ull;
      const unsigned long long mine = cta_tot[rank];
      if (mine > 0ull && base <= target && target < base + mine) {  // block-uniform
        if (threadIdx.x == 0) {
          unsigned long long run = base;
          int w = 0;
          for (; w < kPpWarps - 1; ++w) {
            if (target < run + wsum[w]) break;
            run += wsum[w];
          }
          hit_warp = w;
          hit_base = run;
        }
        __syncthreads();
        if (warp == hit_warp) {
          unsigned long long incl = qsum;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
          }
          unsigned long long run = hit_base + incl - qsum;
          if (qsum > 0ull && run <= target && target < run + qsum) {
            int pk = phi - 1;
            for (int c = plo; c < phi; ++c) {
              run += fixed_weight(Ds[c - lo], M0);
              if (run > target) {
                pk = c;
                break;
              }
            }
            pp_bcast_u64(&pick_bcast, static_cast<unsigned long long>(pk), CL);
          }
        }
      }
    }
    pp_sync(CL);
    const int p = static_cast<int>(pick_bcast);
    load_seed(p, s);
    __syncthreads();
    // ---- squared distances from the new seed to every earlier seed (float32, for pruning): warp w
    // takes seeds w*32 .. w*32+31 of each block of 32*kPpWarps, all 32 rows in flight at once
    for (int a0 = warp * 32; a0 < s; a0 += 32 * kPpWarps) {
      float pr[32];
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        pr[r] = 0.f;
        if (a0 + r < s) {
          const float* ca = Ch + static_cast<size_t>(a0 + r) * D + lane * E;
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const float df = cs[lane * E + e] - ca[e];
            pr[r] = fmaf(df, df, pr[r]);
          }
        }
      }
#pragma unroll
      for (int o = 16, n = 16; o > 0; o >>= 1, n >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int q = 0; q < n; ++q) {
          const float keep = upper ? pr[q + n] : pr[q];
          const float send = upper ? pr[q] : pr[q + n];
          pr[q] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      if (a0 + lane < s) ss[a0 + lane] = pr[0];
    }
    __syncthreads();
    update_pass(s, false);
    __syncthreads();
  }
  if (CL > 1) cluster_sync();  // no CTA leaves while another may still write into its shared memory
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
// Warp roles: 0 = TMA producer, 1 = MMA issuer, 2 = TMEM allocator, 3 = idle, 4..11 = epilogue in
// two warpgroups that split every chunk's 128 columns (warpgroup h takes columns 64h .. 64h+63);
// warp w reads TMEM lanes 32*(w%4) .. +31, i.e. tokens 32*(w%4) .. +31 of the tile.
constexpr int kAsgThreads = 384;
constexpr uint32_t kAsgXStage = 32768;   // 128 tokens x 128 d bf16 (two 16 KB halves)
constexpr uint32_t kAsgCStage = 65536;   // 128 centroids x 128 d x {hi, lo}
constexpr uint32_t kAsgSmem = 2 * kAsgXStage + 2 * kAsgCStage + 1024 /*align*/ + 256 /*barriers*/ +
                               128 * 10 * 4 /*half merge*/;
constexpr uint32_t kAsgTmemCols = 512;   // 4 accumulators of 128 columns
// Flag in the head field of a re-rank entry: the token's candidate list overflowed, so the re-rank
// scans every centroid (heads are below 2^31 because B*H*N is).
constexpr uint32_t kRrFullScan = 0x80000000u;

struct AsgBars {
  uint64_t x_full[2], x_empty[2], c_full[2], c_empty[2], acc_full[4], acc_empty[4], mma_done;
  uint64_t merge_full[4], merge_empty[4];  // per warp quarter: warpgroup 1 -> warpgroup 0 handoff
  uint32_t tmem_base;
};
static_assert(sizeof(AsgBars) <= 256, "barrier block");

__device__ __forceinline__ float tile_row_norm(const uint8_t* xt, int row) {
  float acc[4] = {0.f, 0.f, 0.f, 0.f};  // four chains: the sum is only used for the tolerance
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      const uint4 v = *reinterpret_cast<const uint4*>(xt + h * 16384 + sw128_offset(row, ch));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = bf16lo_to_f32(w[e]), b = bf16hi_to_f32(w[e]);
        acc[e] = fmaf(a, a, acc[e]);
        acc[e] = fmaf(b, b, acc[e]);
      }
    }
  return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// Keep the 4 smallest (score, index) pairs: replace the worst entry if this one is better
// (strictly: among equal scores the one seen first, i.e. the lower index, stays).  `dropped` is the
// smallest score that ever left the list or was refused by it; when it ends up within the final
// tolerance, more than four centroids were candidates and the list alone cannot decide.
__device__ __forceinline__ void cand_insert(float val, int j, float (&cv)[4], int (&ci)[4], float& dropped) {
  int wi = 0;
  float wv = cv[0];
#pragma unroll
  for (int r = 1; r < 4; ++r)
    if (cv[r] > wv) {
      wv = cv[r];
      wi = r;
    }
  if (val < wv) {
    dropped = fminf(dropped, wv);  // an empty slot holds +inf
#pragma unroll
    for (int r = 0; r < 4; ++r)
      if (r == wi) {
        cv[r] = val;
        ci[r] = j;
      }
  } else {
    dropped = fminf(dropped, val);
  }
}

__global__ void __launch_bounds__(kAsgThreads, 1)
    assign_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_hi,
                     const __grid_constant__ CUtensorMap tm_lo, int BH, int N, int k, int kpad,
                     const float* __restrict__ c_norm, int32_t* __restrict__ labels, uint4* __restrict__ rr_list,
                     uint32_t* __restrict__ rr_count, uint32_t rr_cap, DeviceStatus* st,
                     const uint64_t* __restrict__ wait_budget) {
  const long long wb = effective_wait_budget(wait_budget);
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
      mbar_init(smem_u32(&bars->acc_empty[i]), 8);
      mbar_init(smem_u32(&bars->merge_full[i]), 1);
      mbar_init(smem_u32(&bars->merge_empty[i]), 1);
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
        if (it >= 2) ok = mbar_wait(smem_u32(&bars->x_empty[xsI]), ((it >> 1) - 1) & 1, st, kWhereAssign, wb);
        if (!ok) break;
        const uint32_t xdst = smem_u32(xs + xsI * kAsgXStage);
        mbar_arrive_expect_tx(smem_u32(&bars->x_full[xsI]), kAsgXStage);
        const int y = bh * N + tile * kAssignTileM;
        tma_load_2d(xdst, &tm_x, 0, y, smem_u32(&bars->x_full[xsI]));
        tma_load_2d(xdst + 16384, &tm_x, 64, y, smem_u32(&bars->x_full[xsI]));
        for (int c = 0; c < nchunks; ++c, ++g) {
          const int cs = static_cast<int>(g & 1);
          if (g >= 2) ok = mbar_wait(smem_u32(&bars->c_empty[cs]), ((g >> 1) - 1) & 1, st, kWhereAssign, wb);
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
        ok = mbar_wait(smem_u32(&bars->x_full[xsI]), (it >> 1) & 1, st, kWhereAssign, wb);
        if (!ok) break;
        const uint32_t xa = smem_u32(xs + xsI * kAsgXStage);
        for (int c = 0; c < nchunks; ++c, ++g) {
          const int cs = static_cast<int>(g & 1);
          const int a = static_cast<int>(g & 3);
          ok = mbar_wait(smem_u32(&bars->c_full[cs]), (g >> 1) & 1, st, kWhereAssign, wb);
          if (ok && g >= 4) ok = mbar_wait(smem_u32(&bars->acc_empty[a]), ((g >> 2) - 1) & 1, st, kWhereAssign, wb);
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
    // Per 32-column group: scores s = ||c||^2 - 2 x.c (packed pairs), the group minimum
    // (three-input min, four chains), and only if that minimum is within tau of the running
    // minimum, the columns within tau go into a 4-entry candidate list (the minimum itself and
    // near-ties).  tau = 2^-11 (||x||^2 + max(d_min, 0)) is >= 3x the bound on the split-bf16 score
    // error 2^-15 (5 ||x||^2 + 2 d_min), so the true argmin is always among the candidates.  The
    // two warpgroups' lists are merged per token; when more than one candidate survives, the token
    // goes on a list and rerank_kernel, launched next, decides by exact float32 ||x - c||^2 (ties
    // to the lower index), so that the epilogue never waits on centroid rows.
    const int q = warp & 3;
    const int half = (warp - 4) >> 2;
    const int row = q * 32 + lane;
    float* mrg = reinterpret_cast<float*>(bars + 1);  // [128][10]: warpgroup 1's minimum, list, dropped
    long long g = 0;
    int it = 0;
    bool ok = true;
    for (long long w = blockIdx.x; w < total && ok; w += gridDim.x, ++it) {
      const int bh = static_cast<int>(w / ntiles), tile = static_cast<int>(w % ntiles);
      const int xsI = it & 1;
      const float* cn = c_norm + static_cast<size_t>(bh) * kpad;  // 4 KB at most: stays in L1
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->x_full[xsI]), (it >> 1) & 1, st, kWhereAssignTail, wb));
      if (!ok) break;
      const uint8_t* xt = xs + xsI * kAsgXStage;
      const float xn = tile_row_norm(xt, row);
      float gmin = INFINITY;
      float cv[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
      int ci[4] = {-1, -1, -1, -1};
      float dropped = INFINITY;
      for (int c = 0; c < nchunks; ++c, ++g) {
        const int a = static_cast<int>(g & 3);
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->acc_full[a]), (g >> 2) & 1, st, kWhereAssign, wb));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
          const int col0 = half * 64 + qq * 32;
          const int jb = c * kAssignChunkN + col0;
          if (jb >= k) break;  // uniform
          uint32_t v[32];
          tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + a * kAssignChunkN + col0, v);
          tmem_wait_ld();
          float sc[32];
          float4 cn4[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) cn4[e] = __ldg(reinterpret_cast<const float4*>(cn + jb) + e);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float2 r0 = fma2(make_float2(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1])),
                                   make_float2(-2.f, -2.f), make_float2(cn4[e].x, cn4[e].y));
            const float2 r1 = fma2(make_float2(__uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3])),
                                   make_float2(-2.f, -2.f), make_float2(cn4[e].z, cn4[e].w));
            sc[4 * e] = r0.x;
            sc[4 * e + 1] = r0.y;
            sc[4 * e + 2] = r1.x;
            sc[4 * e + 3] = r1.y;
          }
          if (jb + 32 > k) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (jb + e >= k) sc[e] = INFINITY;
          }
          float m4[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
#pragma unroll
          for (int e = 0; e < 32; e += 8)
#pragma unroll
            for (int r = 0; r < 4; ++r) m4[r] = fmin3(m4[r], sc[e + 2 * r], sc[e + 2 * r + 1]);
          const float mloc = fmin3(m4[0], m4[1], fminf(m4[2], m4[3]));
          gmin = fminf(gmin, mloc);
          const float thr = gmin + (xn + fmaxf(gmin + xn, 0.f)) * 0x1p-11f;
          if (mloc <= thr) {  // rare after the first groups: the minimum lies elsewhere
            unsigned hits = 0;
#pragma unroll
            for (int e = 0; e < 32; ++e) hits |= (sc[e] <= thr ? 1u : 0u) << e;
            if (__popc(hits) == 1) {  // the usual case: the group's minimum is its only entry within tau
              cand_insert(mloc, jb + __ffs(hits) - 1, cv, ci, dropped);
              hits = 0u;
            }
            while (hits) {
              const int e = __ffs(hits) - 1;
              hits &= hits - 1;
              float val = sc[0];
#pragma unroll
              for (int r = 1; r < 32; ++r) val = r == e ? sc[r] : val;
              cand_insert(val, jb + e, cv, ci, dropped);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->acc_empty[a]));
      }
      if (!ok) break;
      // merge: warpgroup 1 hands its minimum and list to warpgroup 0 (per token)
      float* mr = mrg + row * 10;
      if (half == 1) {
        if (it > 0)
          ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->merge_empty[q]), (it - 1) & 1, st, kWhereAssign, wb));
        if (!ok) break;
        mr[0] = gmin;
        mr[9] = dropped;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          mr[1 + r] = cv[r];
          mr[5 + r] = __int_as_float(ci[r]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->merge_full[q]));
      } else {
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->merge_full[q]), it & 1, st, kWhereAssign, wb));
        if (!ok) break;
        gmin = fminf(gmin, mr[0]);
        dropped = fminf(dropped, mr[9]);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int j = __float_as_int(mr[5 + r]);
          if (j >= 0) cand_insert(mr[1 + r], j, cv, ci, dropped);  // higher indices than every own entry: ties keep own
        }
        const int n = tile * kAssignTileM + row;
        bool defer = false, full_scan = false;
        uint32_t c01 = 0xffffffffu, c23 = 0xffffffffu;  // the candidates, 16 bits each (0xffff: none)
        if (n < N) {
          const float thr = gmin + (xn + fmaxf(gmin + xn, 0.f)) * 0x1p-11f;
          int best = -1, nc = 0;
          float bv = INFINITY;
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            if (ci[r] >= 0 && cv[r] <= thr) {
              const uint32_t sh = 16u * static_cast<uint32_t>(nc & 1);
              const uint32_t idx = static_cast<uint32_t>(ci[r]) << sh, keep = ~(0xffffu << sh);
              if (nc < 2) c01 = (c01 & keep) | idx;
              else c23 = (c23 & keep) | idx;
              ++nc;
              if (cv[r] < bv || (cv[r] == bv && ci[r] < best)) {
                bv = cv[r];
                best = ci[r];
              }
            }
          }
          // near-tie: the exact distances decide, in rerank_kernel; a list that overflowed (a fifth
          // score within tau was dropped) sends the token to an exact scan over every centroid there
          full_scan = dropped <= thr;
          defer = nc > 1 || full_scan;
          labels[static_cast<size_t>(bh) * N + n] = best < 0 ? 0 : best;
        }
        const unsigned dm = __ballot_sync(0xffffffffu, defer);
        if (dm) {
          uint32_t base = 0;
          if (lane == 0) base = atomicAdd(rr_count, static_cast<uint32_t>(__popc(dm)));
          base = __shfl_sync(0xffffffffu, base, 0);
          const uint32_t slot = base + static_cast<uint32_t>(__popc(dm & ((1u << lane) - 1u)));
          if (defer && slot < rr_cap)
            rr_list[slot] = make_uint4(static_cast<uint32_t>(bh) | (full_scan ? kRrFullScan : 0u),
                                       static_cast<uint32_t>(n), c01, c23);
          else if (defer)  // only past 2^32 - 1 listed tokens in one launch
            raise_status(st, kStatusDeviceBounds, kWhereAssign, slot, static_cast<uint32_t>(n));
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(smem_u32(&bars->merge_empty[q]));  // mr may be overwritten
          mbar_arrive(smem_u32(&bars->x_empty[xsI]));
        }
      }
    }
  }

  __syncwarp();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kAsgTmemCols);
  }
}

// Near-ties of the tensor-core assignment: one warp per listed token computes the exact float32
// ||x - c||^2 of each candidate (lane l holds coordinates 4l .. 4l+3; the partial sums are then
// added across the warp in a fixed butterfly order) and keeps the smallest, ties to the lower index.
// A token whose candidate list overflowed is decided the same way over all k centroids.
constexpr int kRrThreads = 256;

__device__ __forceinline__ float rr_dist(float x0, float x1, float x2, float x3, float4 cv) {
  const float d0 = x0 - cv.x, d1 = x1 - cv.y, d2 = x2 - cv.z, d3 = x3 - cv.w;
  float part = fmaf(d3, d3, fmaf(d2, d2, fmaf(d1, d1, d0 * d0)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  return part;
}

__global__ void __launch_bounds__(kRrThreads) rerank_kernel(const uint16_t* __restrict__ X, int N, int k,
                                                            const float* __restrict__ C,
                                                            const uint4* __restrict__ rr_list,
                                                            const uint32_t* __restrict__ rr_count, uint32_t cap,
                                                            int32_t* __restrict__ labels) {
  const uint32_t total = min(*rr_count, cap);
  const int lane = threadIdx.x & 31;
  const uint32_t warps = gridDim.x * (kRrThreads / 32);
  for (uint32_t i = blockIdx.x * (kRrThreads / 32) + (threadIdx.x >> 5); i < total; i += warps) {
    const uint4 e = rr_list[i];
    const uint32_t hd = e.x & ~kRrFullScan;
    const size_t tok = static_cast<size_t>(hd) * N + e.y;
    const uint2 xr = *reinterpret_cast<const uint2*>(X + tok * 128 + 4 * lane);
    const float x0 = bf16lo_to_f32(xr.x), x1 = bf16hi_to_f32(xr.x), x2 = bf16lo_to_f32(xr.y), x3 = bf16hi_to_f32(xr.y);
    if (e.x & kRrFullScan) {  // uniform across the warp
      const float4* cr = reinterpret_cast<const float4*>(C + static_cast<size_t>(hd) * k * 128) + lane;
      int best = 0;
      float bd = rr_dist(x0, x1, x2, x3, __ldg(cr));
      for (int c = 1; c < k; ++c) {
        const float part = rr_dist(x0, x1, x2, x3, __ldg(cr + static_cast<size_t>(c) * 32));
        if (part < bd) {  // strict: ties keep the lower index
          bd = part;
          best = c;
        }
      }
      if (lane == 0) labels[tok] = best;
      continue;
    }
    int cid[4];
    float4 cv4[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {  // all four rows requested at once (an empty slot reads row 0)
      const uint32_t w = r < 2 ? e.z : e.w;
      const int c = static_cast<int>((w >> (16 * (r & 1))) & 0xffffu);
      cid[r] = c < k ? c : -1;
      cv4[r] = __ldg(reinterpret_cast<const float4*>(C + (static_cast<size_t>(hd) * k + (c < k ? c : 0)) * 128) + lane);
    }
    int best = -1;
    float bd = INFINITY;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int c = cid[r];
      if (c < 0) continue;  // uniform across the warp
      const float part = rr_dist(x0, x1, x2, x3, cv4[r]);
      if (part < bd || (part == bd && c < best)) {
        bd = part;
        best = c;
      }
    }
    if (lane == 0 && best >= 0) labels[tok] = best;
  }
}

// ------------------------------------------------------------------------------------------------
// Update: centroid = mean of members (float64, ascending token order)
// ------------------------------------------------------------------------------------------------
// One CTA per (b,h, cluster).  Member rows (in the stable sort's order) are staged through shared
// memory with cp.async, kUpdRows rows per batch, double-buffered; thread i < d sums dimension i
// over the batch sequentially in float64, which is the oracle's order, so the sums match it bit
// for bit.  Then c = float32(sum / count), the bf16 hi/lo split and ||c||^2.
constexpr int kUpdBufBytes = 16384;  // per buffer: 64 bf16 rows of d = 128
constexpr int kUpdThreads = 256;

template <int D, bool F32>
__global__ void __launch_bounds__(kUpdThreads) update_kernel(const void* __restrict__ X, int BH, int N, int k,
                                                              int kpad, const int32_t* __restrict__ perm,
                                                              const int32_t* __restrict__ offsets,
                                                              float* __restrict__ C, uint16_t* __restrict__ hi,
                                                              uint16_t* __restrict__ lo, float* __restrict__ norm,
                                                              DeviceStatus* st) {
  constexpr int ESZ = F32 ? 4 : 2;
  constexpr int ROWB = D * ESZ;                 // bytes per row
  constexpr int CH = ROWB / 16;                 // 16-byte chunks per row
  constexpr int kUpdRows = kUpdBufBytes / ROWB; // rows per batch
  __shared__ __align__(16) uint8_t buf[2][kUpdBufBytes];
  __shared__ float red[kUpdThreads / 32];
  const int bh = blockIdx.x / k, j = blockIdx.x % k;
  int o0 = offsets[static_cast<size_t>(bh) * (k + 1) + j];
  int o1 = offsets[static_cast<size_t>(bh) * (k + 1) + j + 1];
  SVG2_DEBUG_CHECK(o0 >= 0 && o1 <= N && o0 <= o1, st, kWhereUpdate, o0, o1);
  o0 = o0 < 0 ? 0 : (o0 > N ? N : o0);  // malformed offsets become an empty cluster
  o1 = o1 < o0 ? o0 : (o1 > N ? N : o1);
  const int cnt = o1 - o0;
  const int tid = threadIdx.x;
  float* cj = C + (static_cast<size_t>(bh) * k + j) * D;
  const int32_t* pr = perm + static_cast<size_t>(bh) * N;
  const char* xb = static_cast<const char*>(X) + static_cast<size_t>(bh) * N * ROWB;
  // Each thread copies kPer 16-byte chunks of a batch.  The member indices of a batch are read one
  // batch before its copies are issued, so a copy never waits for its index load.
  constexpr int kPer = kUpdRows * CH / kUpdThreads;
  static_assert(kPer * kUpdThreads == kUpdRows * CH, "chunks per thread");
  auto load_idx = [&](int batch, int (&t)[kPer]) {
    const int r0 = o0 + batch * kUpdRows;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int row = r0 + (tid + i * kUpdThreads) / CH;
      t[i] = row < o1 ? __ldg(pr + row) : 0;
    }
  };
  auto issue = [&](int batch, int b, const int (&t)[kPer]) {
    const int r0 = o0 + batch * kUpdRows;
    const int nr = min(kUpdRows, o1 - r0);
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int q = tid + i * kUpdThreads;
      const int r = q / CH, c = q - r * CH;
      if (r < nr) {
        SVG2_DEBUG_CHECK(t[i] >= 0 && t[i] < N, st, kWhereUpdate, o0 + batch * kUpdRows + r, t[i]);
        const int tk = t[i] < 0 ? 0 : (t[i] >= N ? N - 1 : t[i]);
        cp_async16(smem_u32(&buf[b][r * ROWB + c * 16]), xb + static_cast<size_t>(tk) * ROWB + c * 16);
      }
    }
    cp_async_commit();
  };
  double acc = 0.0;
  const int nb = (cnt + kUpdRows - 1) / kUpdRows;
  int tix[kPer];
  if (nb > 0) {
    load_idx(0, tix);
    issue(0, 0, tix);
  }
  if (nb > 1) load_idx(1, tix);
  for (int b = 0; b < nb; ++b) {
    if (b + 1 < nb) {
      issue(b + 1, (b + 1) & 1, tix);
      if (b + 2 < nb) load_idx(b + 2, tix);  // lands while batch b is summed
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (tid < D) {
      const int nr = min(kUpdRows, cnt - b * kUpdRows);
      const uint8_t* src = buf[b & 1];
      if (nr == kUpdRows) {  // a full batch: every load is issued ahead of the additions
#pragma unroll
        for (int r = 0; r < kUpdRows; ++r) {
          float x;
          if constexpr (F32) x = reinterpret_cast<const float*>(src + r * ROWB)[tid];
          else x = bf16lo_to_f32(reinterpret_cast<const uint16_t*>(src + r * ROWB)[tid]);
          acc = __dadd_rn(acc, static_cast<double>(x));
        }
      } else {
        for (int r = 0; r < nr; ++r) {
          float x;
          if constexpr (F32) x = reinterpret_cast<const float*>(src + r * ROWB)[tid];
          else x = bf16lo_to_f32(reinterpret_cast<const uint16_t*>(src + r * ROWB)[tid]);
          acc = __dadd_rn(acc, static_cast<double>(x));
        }
      }
    }
    __syncthreads();
  }
  float c = 0.f;
  if (tid < D) {
    if (cnt > 0) {
      c = static_cast<float>(__ddiv_rn(acc, static_cast<double>(cnt)));
      cj[tid] = c;
    } else {
      c = cj[tid];
    }
    const size_t ro = (static_cast<size_t>(bh) * kpad + j) * D + tid;
    const __nv_bfloat16 h = __float2bfloat16_rn(c);
    const __nv_bfloat16 l = __float2bfloat16_rn(c - __bfloat162float(h));
    hi[ro] = __bfloat16_as_ushort(h);
    lo[ro] = __bfloat16_as_ushort(l);
  }
  float nrm = c * c;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) nrm += __shfl_xor_sync(0xffffffffu, nrm, o);
  if ((tid & 31) == 0) red[tid >> 5] = nrm;
  __syncthreads();
  if (tid == 0) {
    float t = 0.f;
    for (int w = 0; w < D / 32; ++w) t += red[w];
    norm[static_cast<size_t>(bh) * kpad + j] = t;
  }
}

int num_sms() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

}  // namespace

// Launch configuration of the seeding kernel for `ncl` CTAs per (b,h).
struct PpLaunch {
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  PpLaunch(int BH, int ncl, size_t smem, cudaStream_t s) : cfg{}, attr{} {
    cfg.gridDim = dim3(BH * ncl);
    cfg.blockDim = dim3(kPpThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = ncl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
};

// Cluster size for BH problems of S candidates: the largest size (fewer candidates per CTA, so a
// shorter pass) whose clusters all fit on the GPU at once; past that, more clusters only queue.
template <int E, bool F32>
cudaError_t launch_pp(const void* X, int BH, int N, int stride, int S, int k, const double* u, float* C,
                      cudaStream_t s) {
  auto kern = kmeanspp_kernel2<E, F32>;
  const size_t smem_max = pp_smem_bytes(kPpMaxPerCta);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_max));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  const int cl_min = (S + kPpMaxPerCta - 1) / kPpMaxPerCta;
  if (cl_min > kPpMaxCluster) return cudaErrorInvalidValue;
  int best = cl_min;
  double best_cost = 0.0;
  for (int ncl = cl_min; ncl <= kPpMaxCluster; ++ncl) {
    const int per_cta = (S + ncl - 1) / ncl;
    if (per_cta < 32 * kPpWarps && ncl > cl_min) break;  // fewer than one candidate per lane
    PpLaunch L(BH, ncl, pp_smem_bytes(per_cta), s);
    int active = 0;
    if (cudaOccupancyMaxActiveClusters(&active, kern, &L.cfg) != cudaSuccess || active < 1) {
      cudaGetLastError();  // a size this GPU cannot co-schedule: not a launch error
      continue;
    }
    const int waves = (BH + active - 1) / active;
    // a pass costs about its candidates plus a fixed part (the totals, the pick, the new seed)
    const double cost = waves * (static_cast<double>(per_cta) + (ncl > 1 ? 600.0 : 200.0));
    if (best_cost == 0.0 || cost < best_cost) {
      best_cost = cost;
      best = ncl;
    }
  }
  PpLaunch L(BH, best, pp_smem_bytes((S + best - 1) / best), s);
  return cudaLaunchKernelEx(&L.cfg, kern, X, N, stride, S, k, u, C);
}

int kmeanspp_candidates(int N, int seed_tokens) {
  return (seed_tokens <= 0 || seed_tokens >= N) ? N : seed_tokens;
}

namespace {

// Token of k-means++ candidate j of S < N: one candidate per stratum [floor(j N / S),
// floor((j + 1) N / S)), at offset floor(r w / 2^32) inside it, w the stratum's width and
// r = (j * 2654435769) mod 2^32, a multiplicative hash by the golden ratio.  The offsets vary from
// stratum to stratum, so the candidates do not line up with the video grid's rows and columns.
__device__ __forceinline__ int candidate_token(int j, int N, int S) {
  const unsigned long long lo = static_cast<unsigned long long>(j) * N / S;
  const unsigned long long hi = static_cast<unsigned long long>(j + 1) * N / S;
  const unsigned long long r = static_cast<unsigned int>(static_cast<unsigned int>(j) * 2654435769u);
  return static_cast<int>(lo + ((r * (hi - lo)) >> 32));
}

// Copies the candidate rows of every (b,h) plane into a compact [BH, S, row] buffer, 16 bytes per
// thread and iteration.
__global__ void gather_candidates_kernel(const uint4* __restrict__ X, int N, int S, int vec_per_row,
                                         long long total_vecs, uint4* __restrict__ Xc) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total_vecs;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / vec_per_row;
    const int v = static_cast<int>(i - r * vec_per_row);
    const long long bh = r / S;
    const int j = static_cast<int>(r - bh * S);
    const int n = candidate_token(j, N, S);
    Xc[i] = __ldg(X + (bh * N + n) * vec_per_row + v);
  }
}

}  // namespace

size_t kmeanspp_candidate_bytes(int BH, int N, int d, bool x_f32, int seed_tokens) {
  const int S = kmeanspp_candidates(N, seed_tokens);
  return S < N ? static_cast<size_t>(BH) * S * d * (x_f32 ? 4 : 2) : 0;
}

cudaError_t launch_kmeanspp(const void* X, bool x_f32, int BH, int N, int d, int k, const double* u,
                            float* centroids, double* dist, int32_t* near, uint16_t* seeds_bf16, int seed_tokens,
                            void* cand, size_t cand_bytes, DeviceStatus* st, cudaStream_t s) {
  const int S = kmeanspp_candidates(N, seed_tokens);
  const void* Xs = X;
  int Ns = N;
  if (S < N) {  // seed on the compact copy of the candidate rows
    const size_t need = kmeanspp_candidate_bytes(BH, N, d, x_f32, seed_tokens);
    if (cand == nullptr || cand_bytes < need) return cudaErrorInvalidValue;
    const int vec_per_row = d * (x_f32 ? 4 : 2) / 16;
    const long long total = static_cast<long long>(BH) * S * vec_per_row;
    const long long blocks = (total + 255) / 256;
    gather_candidates_kernel<<<static_cast<unsigned>(blocks < 8192 ? blocks : 8192), 256, 0, s>>>(
        static_cast<const uint4*>(X), N, S, vec_per_row, total, static_cast<uint4*>(cand));
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    Xs = cand;
    Ns = S;
  }
  if (!x_f32 && d == 128) {
    const cudaError_t e = launch_kmeanspp_tc(Xs, BH, Ns, 1, S, k, u, centroids, seeds_bf16, st, s);
    if (e != cudaErrorNotSupported) return e;
  }
  if ((S + kPpMaxCluster - 1) / kPpMaxCluster <= kPpMaxPerCta && !(x_f32 && d == 128)) {
    if (d == 128) return launch_pp<4, false>(Xs, BH, Ns, 1, S, k, u, centroids, s);
    return x_f32 ? launch_pp<2, true>(Xs, BH, Ns, 1, S, k, u, centroids, s)
                 : launch_pp<2, false>(Xs, BH, Ns, 1, S, k, u, centroids, s);
  }
  kmeanspp_kernel<<<BH, 1024, 0, s>>>(Xs, x_f32, Ns, 1, d, k, u, centroids, dist, near);
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
                          uint4* rr_list, uint32_t* rr_count, DeviceStatus* st, const uint64_t* wait_budget,
                          cudaStream_t s) {
  if (!x_f32 && d == 128) {
    alignas(64) CUtensorMap tx, th, tl;
    const int kp = kpad_of(k);
    cudaError_t e = make_tmap_bf16_rows(&tx, X, static_cast<uint64_t>(BH) * N, 128, kAssignTileM);
    if (e == cudaSuccess) e = make_tmap_bf16_rows(&th, c_hi, static_cast<uint64_t>(BH) * kp, 128, kAssignChunkN);
    if (e == cudaSuccess) e = make_tmap_bf16_rows(&tl, c_lo, static_cast<uint64_t>(BH) * kp, 128, kAssignChunkN);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(assign_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAsgSmem);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(rr_count, 0, sizeof(uint32_t), s);
    if (e != cudaSuccess) return e;
    const long long tiles = static_cast<long long>(BH) * ((N + kAssignTileM - 1) / kAssignTileM);
    const int sms = num_sms();
    const int grid = static_cast<int>(tiles < sms ? tiles : sms);
    const size_t bhn = static_cast<size_t>(BH) * N;  // rr_list holds one entry per token
    const uint32_t cap = bhn < 0xffffffffu ? static_cast<uint32_t>(bhn) : 0xffffffffu;
    assign_tc_kernel<<<grid, kAsgThreads, kAsgSmem, s>>>(tx, th, tl, BH, N, k, kp, c_norm, labels, rr_list, rr_count,
                                                          cap, st, wait_budget);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // eight CTAs of 8 warps per SM: each warp waits on its token's rows, so many warps in flight
    rerank_kernel<<<8 * sms, kRrThreads, 0, s>>>(static_cast<const uint16_t*>(X), N, k, centroids, rr_list, rr_count,
                                                 cap, labels);
    return cudaGetLastError();
  }
  const dim3 grid((N + 127) / 128, BH);
  assign_exact_kernel<<<grid, 128, 0, s>>>(X, x_f32, N, d, k, centroids, labels);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------------
// Pruned assignment for the Lloyd iterations after the first (bf16 X, d = 128)
// ------------------------------------------------------------------------------------------------
// The tokens are taken in the previous iteration's label order (its stable sort), 128 per CTA, so a
// tile holds few distinct previous labels a.  For token x of label a, every centroid j with
// ||c_a - c_j|| > 2 ||x - c_a|| is strictly farther from x than c_a (triangle inequality), so it
// cannot be the argmin.  Per tile and label a, R_a = max ||x - c_a|| over the tile's tokens of that
// label; the candidates of the tile are the union over its labels of {j : ||c_a - c_j||^2 <=
// 4 R_a^2 (1 + margin)^2}, the margin covering the float32 rounding of both sides.  Every token then
// takes the exact float32 argmin of ||x - c_j||^2 over the candidates (ascending j, ties to the lower
// index): the label is the one the full search would give, at the cost of a few centroids per tile
// instead of all k.  When the union is large the same loop simply runs over more chunks.
constexpr int kPrThreads = 256;    // two threads per token, 64 coordinates each
constexpr int kPrTile = 128;       // tokens per CTA
constexpr int kPrChunk = 64;       // candidate centroid rows staged in shared memory at a time
constexpr float kPrMargin = 1.001f;

// D2[bh][a][j] = ||c_a - c_j||^2 in float32 (differences, not the expanded form, which would cancel).
// Block = 32 x 32 pairs of one head; 256 threads, each 4 pairs sharing its row a.
__global__ void __launch_bounds__(256) centroid_dist_kernel(const float* __restrict__ C, int k,
                                                           float* __restrict__ D2) {
  __shared__ float ca[32][129];
  __shared__ float cj[32][129];
  const int bh = blockIdx.z, a0 = blockIdx.y * 32, j0 = blockIdx.x * 32;
  const float* Ch = C + static_cast<size_t>(bh) * k * 128;
  for (int i = threadIdx.x; i < 32 * 128; i += 256) {
    const int r = i >> 7, c = i & 127;
    ca[r][c] = a0 + r < k ? Ch[static_cast<size_t>(a0 + r) * 128 + c] : 0.f;
    cj[r][c] = j0 + r < k ? Ch[static_cast<size_t>(j0 + r) * 128 + c] : 0.f;
  }
  __syncthreads();
  const int ai = threadIdx.x >> 3, jb = threadIdx.x & 7;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
  for (int c = 0; c < 128; ++c) {
    const float x = ca[ai][c];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const float df = x - cj[jb + 8 * m][c];
      acc[m] = fmaf(df, df, acc[m]);
    }
  }
  if (a0 + ai < k) {
    float* row = D2 + (static_cast<size_t>(bh) * k + a0 + ai) * k;
#pragma unroll
    for (int m = 0; m < 4; ++m)
      if (j0 + jb + 8 * m < k) row[j0 + jb + 8 * m] = acc[m];
  }
}

__global__ void __launch_bounds__(kPrThreads) pruned_assign_kernel(const uint16_t* __restrict__ X, int N, int k,
                                                                  const float* __restrict__ C,
                                                                  const float* __restrict__ D2,
                                                                  const int32_t* __restrict__ perm,
                                                                  int32_t* __restrict__ labels, DeviceStatus* st) {
  __shared__ __align__(16) float cs[kPrChunk][128];
  __shared__ uint32_t rmax[kMaxClustersAssign];   // R_a^2 (float bits) of the labels in the tile
  __shared__ uint32_t bits[kMaxClustersAssign / 32];
  __shared__ int16_t cand[kMaxClustersAssign];
  __shared__ int16_t tile_labels[kPrTile];
  __shared__ int n_labels, n_cand;
  const int bh = blockIdx.y;
  const int p0 = blockIdx.x * kPrTile;
  const int tok = threadIdx.x >> 1, half = threadIdx.x & 1;
  const int p = p0 + tok;
  const bool valid = p < N;
  const size_t head = static_cast<size_t>(bh) * N;
  const float* Ch = C + static_cast<size_t>(bh) * k * 128;

  for (int i = threadIdx.x; i < (k + 31) / 32; i += kPrThreads) bits[i] = 0u;
  if (threadIdx.x == 0) n_labels = 0;
  int n = 0, a = 0;
  if (valid) {
    n = perm[head + p];
    SVG2_DEBUG_CHECK(n >= 0 && n < N, st, kWherePruned, p, n);
    n = n < 0 ? 0 : (n >= N ? N - 1 : n);
    a = labels[head + n];
    SVG2_DEBUG_CHECK(a >= 0 && a < k, st, kWherePruned, n, a);
    a = a < 0 ? 0 : (a >= k ? k - 1 : a);
  }
  // this thread's 64 coordinates of x
  float x[64];
  {
    const uint4* src = reinterpret_cast<const uint4*>(X + (head + n) * 128 + half * 64);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint4 w = valid ? __ldg(src + q) : make_uint4(0u, 0u, 0u, 0u);
      x[8 * q + 0] = bf16lo_to_f32(w.x); x[8 * q + 1] = bf16hi_to_f32(w.x);
      x[8 * q + 2] = bf16lo_to_f32(w.y); x[8 * q + 3] = bf16hi_to_f32(w.y);
      x[8 * q + 4] = bf16lo_to_f32(w.z); x[8 * q + 5] = bf16hi_to_f32(w.z);
      x[8 * q + 6] = bf16lo_to_f32(w.w); x[8 * q + 7] = bf16hi_to_f32(w.w);
    }
  }
  // r^2 = ||x - c_a||^2 (the two halves summed across the thread pair)
  float r2;
  {
    const float4* ca4 = reinterpret_cast<const float4*>(Ch + static_cast<size_t>(a) * 128 + half * 64);
    float acc = 0.f;
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const float4 c = __ldg(ca4 + q);
      float df = x[4 * q] - c.x;
      acc = fmaf(df, df, acc);
      df = x[4 * q + 1] - c.y;
      acc = fmaf(df, df, acc);
      df = x[4 * q + 2] - c.z;
      acc = fmaf(df, df, acc);
      df = x[4 * q + 3] - c.w;
      acc = fmaf(df, df, acc);
    }
    r2 = acc + __shfl_xor_sync(0xffffffffu, acc, 1);
  }
  __syncthreads();
  // the distinct previous labels of the tile (consecutive runs: the tokens are in label order)
  if (valid && half == 0) {
    int prev = -1;
    if (tok > 0) {
      int np = perm[head + p - 1];
      np = np < 0 ? 0 : (np >= N ? N - 1 : np);
      prev = labels[head + np];
      prev = prev < 0 ? 0 : (prev >= k ? k - 1 : prev);
    }
    if (prev != a) {
      rmax[a] = 0u;
      tile_labels[atomicAdd(&n_labels, 1)] = static_cast<int16_t>(a);
    }
  }
  __syncthreads();
  if (valid && half == 0) atomicMax(&rmax[a], __float_as_uint(r2));  // r2 >= 0: bits order as values
  __syncthreads();
  // union of the labels' candidates
  const int nl = n_labels;
  for (int li = 0; li < nl; ++li) {
    const int al = tile_labels[li];
    const float lim = 4.f * __uint_as_float(rmax[al]) * (kPrMargin * kPrMargin);
    const float* drow = D2 + (static_cast<size_t>(bh) * k + al) * k;
    for (int j = threadIdx.x; j < k; j += kPrThreads)
      if (j == al || __ldg(drow + j) <= lim) atomicOr(&bits[j >> 5], 1u << (j & 31));
  }
  __syncthreads();
  if (threadIdx.x < 32) {  // compact the bit set into an ascending list
    int base = 0;
    for (int w0 = 0; w0 < (k + 31) / 32; w0 += 32) {
      const int w = w0 + threadIdx.x;
      const uint32_t b = w < (k + 31) / 32 ? bits[w] : 0u;
      const int cnt = __popc(b);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (static_cast<int>(threadIdx.x) >= o) incl += v;
      }
      int pos = base + incl - cnt;
      uint32_t bb = b;
      while (bb) {
        const int e = __ffs(bb) - 1;
        bb &= bb - 1;
        cand[pos++] = static_cast<int16_t>(w * 32 + e);
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (threadIdx.x == 0) n_cand = base;
  }
  __syncthreads();
  const int nc = n_cand;
  float best = INFINITY;
  int best_j = 0;
  for (int c0 = 0; c0 < nc; c0 += kPrChunk) {
    const int m = nc - c0 < kPrChunk ? nc - c0 : kPrChunk;
    for (int i = threadIdx.x; i < m * 32; i += kPrThreads) {
      const int r = i >> 5, q = i & 31;
      reinterpret_cast<float4*>(cs[r])[q] =
          __ldg(reinterpret_cast<const float4*>(Ch + static_cast<size_t>(cand[c0 + r]) * 128) + q);
    }
    __syncthreads();
    for (int r = 0; r < m; ++r) {
      const float4* c4 = reinterpret_cast<const float4*>(cs[r] + half * 64);
      float acc = 0.f;
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const float4 c = c4[q];
        float df = x[4 * q] - c.x;
        acc = fmaf(df, df, acc);
        df = x[4 * q + 1] - c.y;
        acc = fmaf(df, df, acc);
        df = x[4 * q + 2] - c.z;
        acc = fmaf(df, df, acc);
        df = x[4 * q + 3] - c.w;
        acc = fmaf(df, df, acc);
      }
      const float d2 = acc + __shfl_xor_sync(0xffffffffu, acc, 1);
      if (d2 < best) {  // ascending candidates: a tie keeps the lower index
        best = d2;
        best_j = cand[c0 + r];
      }
    }
    __syncthreads();
  }
  if (valid && half == 0) labels[head + n] = best_j;
}

cudaError_t launch_assign_pruned(const void* X, int BH, int N, int k, const float* centroids, const int32_t* perm,
                                 float* d2, int32_t* labels, cudaStream_t s, DeviceStatus* st) {
  if (k > kMaxClustersAssign) return cudaErrorInvalidValue;
  const dim3 gd((k + 31) / 32, (k + 31) / 32, BH);
  centroid_dist_kernel<<<gd, 256, 0, s>>>(centroids, k, d2);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const dim3 ga((N + kPrTile - 1) / kPrTile, BH);
  pruned_assign_kernel<<<ga, kPrThreads, 0, s>>>(static_cast<const uint16_t*>(X), N, k, centroids, d2, perm, labels,
                                                  st);
  return cudaGetLastError();
}

cudaError_t launch_update(const void* X, bool x_f32, int BH, int N, int d, int k, const int32_t* perm,
                          const int32_t* offsets, float* centroids, uint16_t* c_hi, uint16_t* c_lo,
                          float* c_norm, cudaStream_t s, DeviceStatus* st) {
  const int blocks = BH * k;
  const int kp = kpad_of(k);
  if (d == 128) {
    if (x_f32)
      update_kernel<128, true><<<blocks, kUpdThreads, 0, s>>>(X, BH, N, k, kp, perm, offsets, centroids, c_hi, c_lo, c_norm, st);
    else
      update_kernel<128, false><<<blocks, kUpdThreads, 0, s>>>(X, BH, N, k, kp, perm, offsets, centroids, c_hi, c_lo, c_norm, st);
  } else {
    if (x_f32)
      update_kernel<64, true><<<blocks, kUpdThreads, 0, s>>>(X, BH, N, k, kp, perm, offsets, centroids, c_hi, c_lo, c_norm, st);
    else
      update_kernel<64, false><<<blocks, kUpdThreads, 0, s>>>(X, BH, N, k, kp, perm, offsets, centroids, c_hi, c_lo, c_norm, st);
  }
  return cudaGetLastError();
}

}  // namespace svg2
