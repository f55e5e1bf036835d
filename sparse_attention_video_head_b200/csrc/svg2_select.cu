// Critical-cluster identification ("Sparse VideoGen2" wiki summary, Key claims section 4.2,
// Eq. 1-2; Method (3)): centroid-based scores weighted by K-cluster size, then top-p selection.
//
// One CTA of 1024 threads per (group of kSelQ Q clusters, b,h); thread j owns K cluster j
// (nK <= 1024) and computes its logits against the whole group, so each K centroid row is read
// once per group (float4 loads streaming through L1) instead of once per Q cluster.
//  * l_ij = (sum_m cq_im * ck_jm) * scale in float64, summed sequentially over m with no FMA
//    (the oracle's order), w_ij = float32(count_j * exp(l_ij - max_j l_ij)) for non-empty j.
//  * top-p in fixed point: u_j = floor(w_j / max w * 2^32) (correctly rounded float64 division),
//    T = ceil(p * sum u); a bitonic sort orders (u desc, j asc), an inclusive integer scan gives
//    the running sums, and a cluster is kept while the sum before it is still below T.  Integer
//    arithmetic after the division, so the mask is bit-exact with the oracle on the same weights.
//  * outputs: uint8 mask, the kept indices ascending (ELL rows), their count and the number of
//    keys they hold (the packed key-stream length used by the attention).
#include "svg2_device.cuh"
#include "svg2_internal.h"

namespace svg2 {

namespace {

constexpr int kSelQ = 8;  // Q clusters per CTA

__device__ double block_max_f64(double v, double* buf) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) buf[threadIdx.x >> 5] = v;
  __syncthreads();
  double r = buf[0];
  for (int w = 1; w < (blockDim.x >> 5); ++w) r = fmax(r, buf[w]);
  return r;
}

// Inclusive scan of uint64 over the block (1024 threads); `buf` holds 33 entries.
__device__ unsigned long long block_inscan_u64(unsigned long long v, unsigned long long* buf,
                                               unsigned long long* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  __syncthreads();
  if (lane == 31) buf[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const unsigned long long w = buf[lane];
    unsigned long long wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    buf[lane] = wi - w;
    if (lane == 31) buf[32] = wi;
  }
  __syncthreads();
  *total = buf[32];
  return buf[warp] + incl;
}

__global__ void __launch_bounds__(1024) select_kernel(const float* __restrict__ cq, const float* __restrict__ ck,
                                                       const float* __restrict__ w_in,
                                                       const int32_t* __restrict__ count_k, int nQ, int nK, int d,
                                                       float top_p, float scale, float* __restrict__ w_out,
                                                       uint8_t* __restrict__ mask, int32_t* __restrict__ sel_count,
                                                       int32_t* __restrict__ sel_idx,
                                                       int32_t* __restrict__ stream_len) {
  __shared__ double cqs[kSelQ][128];
  __shared__ double dbuf[32];
  __shared__ unsigned long long keys[1024];
  __shared__ unsigned long long ubuf[33];
  const int i0 = blockIdx.x * kSelQ, bh = blockIdx.y, j = threadIdx.x;
  const int nq = min(kSelQ, nQ - i0);
  const bool valid = j < nK;
  const int cnt = valid ? count_k[static_cast<size_t>(bh) * nK + j] : 0;

  // logits of K cluster j against every Q cluster of the group: float64, summed over m in order
  // with no FMA (the oracle's order)
  double lg[kSelQ];
#pragma unroll
  for (int qq = 0; qq < kSelQ; ++qq) lg[qq] = -INFINITY;
  if (w_in == nullptr) {
    for (int e = j; e < nq * d; e += blockDim.x)
      cqs[e / d][e % d] = static_cast<double>(cq[(static_cast<size_t>(bh) * nQ + i0) * d + e]);
    __syncthreads();
    if (valid) {
      const float4* ckj = reinterpret_cast<const float4*>(ck + (static_cast<size_t>(bh) * nK + j) * d);
      double acc[kSelQ];
#pragma unroll
      for (int qq = 0; qq < kSelQ; ++qq) acc[qq] = 0.0;
      for (int m4 = 0; m4 < d / 4; ++m4) {
        const float4 c4 = __ldg(ckj + m4);
        const double cv[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
          for (int qq = 0; qq < kSelQ; ++qq) acc[qq] = __dadd_rn(acc[qq], __dmul_rn(cqs[qq][4 * m4 + e], cv[e]));
      }
#pragma unroll
      for (int qq = 0; qq < kSelQ; ++qq) lg[qq] = __dmul_rn(acc[qq], static_cast<double>(scale));
    }
  }

  for (int qq = 0; qq < nq; ++qq) {  // uniform
    const size_t row = static_cast<size_t>(bh) * nQ + i0 + qq;
    double l = -INFINITY;
#pragma unroll
    for (int r = 0; r < kSelQ; ++r)
      if (r == qq) l = lg[r];
    float w = 0.f;
    if (w_in != nullptr) {
      if (valid) w = w_in[row * nK + j];
    } else {
      const double mx = block_max_f64(cnt > 0 ? l : -INFINITY, dbuf);
      if (cnt > 0) w = static_cast<float>(__dmul_rn(static_cast<double>(cnt), exp(__dsub_rn(l, mx))));
      if (w_out != nullptr && valid) w_out[row * nK + j] = w;
    }

    const double wmax = block_max_f64(cnt > 0 ? static_cast<double>(w) : 0.0, dbuf);
    bool keep;
    if (static_cast<double>(top_p) >= 1.0 || !(wmax > 0.0)) {
      keep = cnt > 0;
    } else {
      unsigned long long u = 0ull;
      if (cnt > 0 && w > 0.f) u = static_cast<unsigned long long>(floor(__ddiv_rn(static_cast<double>(w), wmax) * 4294967296.0));
      const unsigned long long kMaxU = (1ull << 33) - 1ull;
      __syncthreads();  // keys[] of the previous Q cluster is no longer read
      keys[j] = valid ? (((kMaxU - u) << 11) | static_cast<unsigned long long>(j)) : ~0ull;
      __syncthreads();
      // bitonic sort, ascending, 1024 keys
      for (int size = 2; size <= 1024; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          const int partner = j ^ stride;
          if (partner > j) {
            const unsigned long long a = keys[j], b = keys[partner];
            const bool up = (j & size) == 0;
            if ((a > b) == up) {
              keys[j] = b;
              keys[partner] = a;
            }
          }
          __syncthreads();
        }
      }
      const unsigned long long kj = keys[j];
      const bool kvalid = kj != ~0ull;
      const unsigned long long uj = kvalid ? (kMaxU - (kj >> 11)) : 0ull;
      unsigned long long U = 0ull;
      const unsigned long long incl = block_inscan_u64(uj, ubuf, &U);
      const unsigned long long T = static_cast<unsigned long long>(ceil(static_cast<double>(top_p) * static_cast<double>(U)));
      const bool keep_sorted = kvalid && (incl - uj) < T;
      __syncthreads();
      // scatter the decision back to cluster order (reuse keys[] as a flag array)
      keys[j] = 0ull;
      __syncthreads();
      if (keep_sorted) keys[static_cast<int>(kj & 2047ull)] = 1ull;
      __syncthreads();
      keep = valid && keys[j] != 0ull;
      if (keep && cnt == 0) keep = false;
    }
    // compaction of kept indices in ascending j, count, and key-stream length
    unsigned long long tot = 0ull;
    const unsigned long long pos = block_inscan_u64(keep ? 1ull : 0ull, ubuf, &tot);
    if (valid) mask[row * nK + j] = keep ? 1 : 0;
    if (keep) sel_idx[row * nK + (pos - 1)] = j;
    unsigned long long len_tot = 0ull;
    block_inscan_u64(keep ? static_cast<unsigned long long>(cnt) : 0ull, ubuf, &len_tot);
    if (j == 0) {
      sel_count[row] = static_cast<int32_t>(tot);
      if (stream_len != nullptr) stream_len[row] = static_cast<int32_t>(len_tot);
    }
  }
}

}  // namespace

cudaError_t launch_select(const float* cq, const float* ck, const float* weights_in, const int32_t* count_k,
                          int BH, int nQ, int nK, int d, float top_p, float scale, float* weights_out,
                          uint8_t* mask, int32_t* sel_count, int32_t* sel_idx, int32_t* stream_len,
                          cudaStream_t s) {
  const dim3 grid((nQ + kSelQ - 1) / kSelQ, BH);
  select_kernel<<<grid, 1024, 0, s>>>(cq, ck, weights_in, count_k, nQ, nK, d, top_p, scale, weights_out, mask,
                                      sel_count, sel_idx, stream_len);
  return cudaGetLastError();
}

}  // namespace svg2
