// k-means++ seeding with the per-seed distance screen on the tensor cores (bf16 tokens, d = 128).
//
// The seeding is the one of "Sparse VideoGen2" (wiki summary, Method (1): k-means++ on the Q and K
// activations of each head), with D^2-proportional sampling made reproducible by fixed-point
// weights floor(D^2 / M0 * 2^32) (M0 = the largest D^2 after the first seed).  Each new seed needs
// one pass over the candidates; that pass is what this kernel does fast:
//
//   * one (b,h) runs on the CTAs of one thread-block cluster, each owning a contiguous range of the
//     candidates, cut into tiles of 128 consecutive candidates;
//   * a tile is fetched by TMA (the candidates are contiguous rows: all tokens, or the compact copy
//     of the candidate rows the launcher makes) and multiplied by the new seed on the tensor core (M = 128 candidates, N = 16 with the seed in
//     column 0, K = 128), giving x . c in TMEM;
//   * the epilogue forms f = ||x||^2 + ||c||^2 - 2 x.c and lists the candidates where f, widened by
//     a rigorous error bound, does not rule out an improvement; after the stream the whole CTA
//     computes their exact float64 D^2 (a sequential sum over the 128 coordinates, the definition's
//     order, one candidate per thread) and the exact value decides;
//   * a tile is skipped without being fetched when no candidate in it can move closer: with a the
//     candidate's nearest seed, ||c_new - c_a||^2 >= 4 D^2 proves ||x - c_new|| >= ||x - c_a||; the
//     table of ||c_new - c_a||^2 is built from the earlier seeds' bf16 rows, which a bulk copy brings
//     into the (then idle) TMA ring while the pick is made;
//   * late in the seeding that test leaves few candidates; when a CTA has at most four rounds of its
//     threads' worth, the pass skips the stream and computes their exact D^2 directly.
//
// Per-tile sums of the fixed-point weights make the sampling search a scan over the tiles, then a
// scan over one tile: the CTA totals meet at a cluster barrier, and the CTA that owns the pick sends
// it to every CTA of the cluster as an 8-byte message on an mbarrier.  The D^2 values, and so the
// seeds, are the same as those of the sequential float64 definition.
#include "svg2_internal.h"
#include "svg2_device.cuh"

namespace svg2 {
namespace {

constexpr int kSdThreads = 320;  // warp 0 TMA, warp 1 MMA + TMEM, warps 2..9 epilogue (2 warpgroups)
constexpr int kSdWarps = kSdThreads / 32;
constexpr int kSdTile = 128;                          // candidates per tile (MMA M)
constexpr int kSdStages = 3;                          // TMA ring depth (a slot frees when its MMA ends)
constexpr int kSdHalf = kSdTile * 128;                // one 64-column half of a tile: 16 KB
constexpr int kSdStageBytes = 2 * kSdHalf;            // 32 KB
constexpr int kSdSeedRows = 16;                       // MMA N: row 0 = the new seed, rows 1..15 zero
constexpr int kSdSeedHalf = kSdSeedRows * 128;        // 2 KB
constexpr int kSdAcc = 8;                             // TMEM accumulators, 16 columns each
constexpr int kSdTmemCols = 128;
constexpr int kSdMaxTiles = 48;
constexpr int kSdMaxPerCta = kSdMaxTiles * kSdTile;   // 6144 candidates per CTA
constexpr int kSdMaxCluster = 16;
constexpr int kSdMaxK = 1024;
// A pass whose pruning test leaves at most this many candidates in a CTA skips the tensor-core
// stream and computes their exact D^2 directly (four rounds of the 320 threads).
constexpr int kSdDirect = 4 * kSdThreads;
constexpr int kSdRingRows = kSdStages * kSdStageBytes / 256;  // bf16 seed rows the ring holds: 384

struct SdBars {
  uint64_t full[kSdStages];
  uint64_t empty[kSdStages];
  uint64_t acc_full[kSdAcc];
  uint64_t acc_empty[kSdAcc];
  uint64_t mma_done;
  uint64_t rows;  // the earlier seeds' bf16 rows copied into the (idle) ring for the pruning table
  uint64_t pick;  // the pass's pick, sent by the CTA that owns it to every CTA of the cluster
  uint32_t tmem_base;
};

// Dynamic shared memory: alignment slack, TMA ring, seed operand, then per candidate D^2 (float64),
// ||x||^2 (float32), the nearest seed (uint16) and a slot of the exact-distance work list (uint16).
__host__ __device__ constexpr size_t sd_smem_bytes(int per_cta) {
  return 1024 + static_cast<size_t>(kSdStages) * kSdStageBytes + 2 * kSdSeedHalf +
         static_cast<size_t>(per_cta) * (8 + 4 + 2 + 2) + 64;
}

__device__ __forceinline__ unsigned long long sd_weight(double v, double m0) {
  if (!(m0 > 0.0) || !(v > 0.0)) return 0ull;
  return static_cast<unsigned long long>(floor(__ddiv_rn(v, m0) * 4294967296.0));
}

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void sd_sync(int ncl) {
  if (ncl > 1) cluster_sync();
  else __syncthreads();
}

__device__ __forceinline__ void sd_bcast(unsigned long long* var, unsigned long long v, int ncl) {
  if (ncl > 1) {
    for (int r = 0; r < ncl; ++r) st_cluster_u64(var, static_cast<uint32_t>(r), v);
  } else {
    *var = v;
  }
}

// The pick goes to every CTA of the cluster with its arrival on their `pick` barrier, so that no
// cluster-wide barrier is needed: each CTA waits for the one message of the pass.
__device__ __forceinline__ void sd_send_pick(unsigned long long* var, uint64_t* bar, unsigned long long v, int ncl) {
  for (int r = 0; r < ncl; ++r) st_async_u64(var, bar, static_cast<uint32_t>(r), v);
}

__global__ void __launch_bounds__(kSdThreads, 1)
    seed_tc_kernel(const __grid_constant__ CUtensorMap tm, const uint16_t* __restrict__ X, int N, int stride, int S,
                   int k, const double* __restrict__ u, float* __restrict__ C, uint16_t* __restrict__ Sb,
                   DeviceStatus* st) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint8_t* seedB = smem + kSdStages * kSdStageBytes;
  __shared__ SdBars bars;
  __shared__ float cs[128];
  __shared__ double csd[128];
  __shared__ float ss[kSdMaxK];
  __shared__ unsigned long long gtot[kSdMaxTiles];
  __shared__ int tflag[kSdMaxTiles];
  __shared__ int tlist[kSdMaxTiles];
  __shared__ int n_active;
  __shared__ int n_exact;
  __shared__ int direct_sh;
  __shared__ unsigned tmask[kSdMaxTiles][4];  // per tile: which candidates pass the pruning test
  __shared__ int toff[kSdMaxTiles];           // their offsets in the direct route's list
  __shared__ int err_sh;
  __shared__ float cc_sh;
  __shared__ unsigned long long cta_tot[2][kSdMaxCluster];  // by pass parity: a CTA may run a pass ahead
  __shared__ unsigned long long cta_max[kSdMaxCluster];
  __shared__ unsigned long long pick_bcast;
  __shared__ unsigned long long wred[kSdWarps];

  const int CL = static_cast<int>(cluster_nctas());
  const uint32_t rank = cluster_rank();
  const int bh = blockIdx.x / CL;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_cta = (S + CL - 1) / CL;
  const int lo = min(S, static_cast<int>(rank) * per_cta), hi = min(S, lo + per_cta);
  const int n = hi - lo;
  const int ntiles = (n + kSdTile - 1) / kSdTile;
  double* Ds = reinterpret_cast<double*>(seedB + 2 * kSdSeedHalf);
  float* xx = reinterpret_cast<float*>(Ds + per_cta);
  uint16_t* As = reinterpret_cast<uint16_t*>(xx + per_cta);
  uint16_t* xlist = As + per_cta;  // candidates whose exact D^2 this pass needs
  const uint16_t* Xh = X + static_cast<size_t>(bh) * N * 128;
  float* Ch = C + static_cast<size_t>(bh) * k * 128;
  uint16_t* Sbh = Sb + static_cast<size_t>(bh) * k * 128;  // the seeds as bf16 rows
  const double* uh = u + static_cast<size_t>(bh) * k;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSdStages; ++i) {
      mbar_init(smem_u32(&bars.full[i]), 1);
      mbar_init(smem_u32(&bars.empty[i]), 1);
    }
    for (int i = 0; i < kSdAcc; ++i) {
      mbar_init(smem_u32(&bars.acc_full[i]), 1);
      mbar_init(smem_u32(&bars.acc_empty[i]), 4);
    }
    mbar_init(smem_u32(&bars.mma_done), 1);
    mbar_init(smem_u32(&bars.rows), 1);
    mbar_init(smem_u32(&bars.pick), 1);
    fence_mbar_init();
    err_sh = 0;
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars.tmem_base), kSdTmemCols);
    tmem_relinquish();
  }
  for (int i = threadIdx.x; i < n; i += kSdThreads) {
    Ds[i] = INFINITY;
    As[i] = 0;
    xx[i] = 0.f;
  }
  for (int i = threadIdx.x; i < 2 * kSdSeedHalf / 16; i += kSdThreads)
    reinterpret_cast<uint4*>(seedB)[i] = make_uint4(0u, 0u, 0u, 0u);
  for (int i = threadIdx.x; i < kSdMaxTiles; i += kSdThreads) gtot[i] = 0ull;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  // The new seed: float32 and float64 copies for the distances, bf16 row 0 of the MMA's B operand
  // (128-byte swizzle, row 0 keeps its chunk order), and, from the first CTA, the output centroid
  // and its bf16 row for the seed-to-seed distances of later passes.
  auto load_seed = [&](int cand, int s) {
    if (threadIdx.x < 64) {
      const int i = 2 * threadIdx.x;
      const uint32_t w = *reinterpret_cast<const uint32_t*>(Xh + static_cast<size_t>(cand) * stride * 128 + i);
      const float a = bf16lo_to_f32(w), b = bf16hi_to_f32(w);
      cs[i] = a;
      cs[i + 1] = b;
      csd[i] = static_cast<double>(a);
      csd[i + 1] = static_cast<double>(b);
      *reinterpret_cast<uint32_t*>(seedB + (i >> 6) * kSdSeedHalf + sw128_offset(0, (i & 63) >> 3) + (i & 7) * 2) = w;
      if (rank == 0) {
        Ch[static_cast<size_t>(s) * 128 + i] = a;
        Ch[static_cast<size_t>(s) * 128 + i + 1] = b;
        *reinterpret_cast<uint32_t*>(Sbh + static_cast<size_t>(s) * 128 + i) = w;
        fence_proxy_async_global();  // every CTA's later bulk copy of the seed rows reads this one
      }
    }
    fence_proxy_async_smem();  // the tensor core reads seedB through the async proxy
  };

  unsigned long long gbase = 0;  // tiles streamed so far (mbarrier phase bookkeeping)
  double M0 = 0.0;
  long long p0 = static_cast<long long>(floor(uh[0] * static_cast<double>(S)));
  if (p0 >= S) p0 = S - 1;
  if (p0 < 0) p0 = 0;
  int pick = static_cast<int>(p0);

  for (int s = 0; s < k; ++s) {
    if (s > 0) {
      // ---- D^2 sampling: CTA total, cluster totals, then the owning CTA scans tiles and one tile
      if (threadIdx.x == 0) mbar_arrive_expect_tx(smem_u32(&bars.pick), 8u);  // this pass's message
      if (warp == 0) {
        unsigned long long t = 0;
        for (int i = lane; i < ntiles; i += 32) t += gtot[i];
        t = warp_sum_u64(t);
        if (lane == 0) sd_bcast(&cta_tot[s & 1][rank], t, CL);
      }
      sd_sync(CL);
      // the seed rows 0 .. s-1 (the last one written in the previous pass, before the barrier) go
      // into the ring now, so that the copy overlaps the pick; the ring is idle until the stream
      if (threadIdx.x == 0 && s < k - 1) {  // (the last seed's pass ends before the table)
        const int nrow = min(s, kSdRingRows);
        const uint32_t bar = smem_u32(&bars.rows);
        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nrow) * 256u);
        for (int r0 = 0; r0 < nrow; r0 += kSdTile)
          bulk_load(smem_u32(ring + r0 * 256), Sbh + static_cast<size_t>(r0) * 128,
                    static_cast<uint32_t>(min(kSdTile, nrow - r0)) * 256u, bar);
      }
      unsigned long long U = 0, base = 0;
      for (int r = 0; r < CL; ++r) {
        if (r < static_cast<int>(rank)) base += cta_tot[s & 1][r];
        U += cta_tot[s & 1][r];
      }
      const unsigned long long mine = cta_tot[s & 1][rank];
      if (U == 0ull) {
        if (threadIdx.x == 0 && rank == 0) {
          const long long p = static_cast<long long>(floor(uh[s] * static_cast<double>(S)));
          sd_send_pick(&pick_bcast, &bars.pick, static_cast<unsigned long long>(p >= S ? S - 1 : p), CL);
        }
      } else if (warp == 0) {
        unsigned long long target = static_cast<unsigned long long>(floor(uh[s] * static_cast<double>(U)));
        if (target > U - 1ull) target = U - 1ull;
        if (mine > 0ull && base <= target && target < base + mine) {
          // the tile: first whose inclusive prefix exceeds the target
          unsigned long long run = base;
          int tsel = -1;
          for (int t0 = 0; t0 < ntiles && tsel < 0; t0 += 32) {
            const unsigned long long g = (t0 + lane < ntiles) ? gtot[t0 + lane] : 0ull;
            unsigned long long incl = g;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const unsigned long long v = __shfl_up_sync(0xffffffffu, incl, o);
              if (lane >= o) incl += v;
            }
            const unsigned hit = __ballot_sync(0xffffffffu, g > 0ull && run + incl > target);
            if (hit) {
              const int l = __ffs(hit) - 1;
              tsel = t0 + l;
              run += __shfl_sync(0xffffffffu, incl - g, l);
            } else {
              run += __shfl_sync(0xffffffffu, incl, 31);
            }
          }
          if (tsel < 0) tsel = ntiles - 1;  // unreachable: the totals say the target lies in this CTA
          // within the tile: lane l holds candidates 4l .. 4l+3 in order
          unsigned long long w4[4], lsum = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int c = tsel * kSdTile + 4 * lane + j;
            w4[j] = c < n ? sd_weight(Ds[c], M0) : 0ull;
            lsum += w4[j];
          }
          unsigned long long incl = lsum;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
          }
          unsigned long long r0 = run + incl - lsum;
          if (lsum > 0ull && r0 <= target && target < r0 + lsum) {
            int pk = tsel * kSdTile + 4 * lane + 3;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              r0 += w4[j];
              if (r0 > target) {
                pk = tsel * kSdTile + 4 * lane + j;
                break;
              }
            }
            sd_send_pick(&pick_bcast, &bars.pick, static_cast<unsigned long long>(lo + pk), CL);
          }
        }
      }
      if (!mbar_wait_cluster(smem_u32(&bars.pick), static_cast<uint32_t>((s - 1) & 1), st, kWhereSeedEpilogue))
        err_sh = 1;
      pick = static_cast<int>(min(pick_bcast, static_cast<unsigned long long>(S - 1)));
    }
    load_seed(pick, s);
    if (s == k - 1) break;  // the last seed's distances are never used
    if (threadIdx.x == 0 && status_set(st)) err_sh = 1;
    __syncthreads();

    // ---- ||c||^2 (warp 0) and squared distances from the new seed to the earlier seeds (pruning)
    if (warp == 0) {
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) a = fmaf(cs[4 * lane + e], cs[4 * lane + e], a);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (lane == 0) cc_sh = a;
    }

    const int nrow = min(s, kSdRingRows);  // rows 0 .. nrow-1 are in the ring
    bool rows_ok = true;
    if (s > 0 && warp * 8 < s)
      rows_ok = mbar_wait(smem_u32(&bars.rows), static_cast<uint32_t>((s - 1) & 1), st, kWhereSeedEpilogue);
    if (s > 0 && rows_ok) {
      // a warp takes 8 seed rows per round: lane (rr, qd) = (lane / 4, lane % 4) sums the quarter
      // qq of the coordinates of row rr, visiting its four 16-byte chunks from a lane-dependent
      // start (rho) so that the ring reads spread over all banks; the new seed's coordinates of
      // that quarter, in the same visiting order, stay in registers
      const int rr = lane >> 2, qd = lane & 3, rho = rr & 3;
      const int qq = (qd + rr) & 3;
      float cq[32];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int ch = (i + rho) & 3;
#pragma unroll
        for (int e = 0; e < 8; ++e) cq[8 * i + e] = cs[32 * qq + 8 * ch + e];
      }
      for (int a0 = warp * 8; a0 < s; a0 += 8 * kSdWarps) {
        const int a = a0 + rr;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (a < s) {
          uint4 v[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int off = qq * 64 + ((i + rho) & 3) * 16;  // bytes within the row
            v[i] = a < nrow ? *reinterpret_cast<const uint4*>(ring + a * 256 + off)
                            : *reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(Sbh) +
                                                              static_cast<size_t>(a) * 256 + off);
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float d0 = bf16lo_to_f32(w[e]) - cq[8 * i + 2 * e];
              const float d1 = bf16hi_to_f32(w[e]) - cq[8 * i + 2 * e + 1];
              acc[e] = fmaf(d0, d0, acc[e]);
              acc[e] = fmaf(d1, d1, acc[e]);
            }
          }
        }
        float t = (acc[0] + acc[1]) + (acc[2] + acc[3]);
        t += __shfl_xor_sync(0xffffffffu, t, 1);
        t += __shfl_xor_sync(0xffffffffu, t, 2);
        if (qd == 0 && a < s) ss[a] = t;
      }
    }
    if (!rows_ok) err_sh = 1;  // (the pruning table is incomplete: the pass streams nothing)
    fence_proxy_async_smem();  // these generic reads of the ring come before the stream's TMA writes
    __syncthreads();

    // ---- tiles that may hold a candidate moving closer (all of them for the first seed)
    if (s == 0) {
      for (int i = threadIdx.x; i < n; i += kSdThreads) xlist[i] = static_cast<uint16_t>(i);
    }
    for (int t0 = warp; t0 < ntiles; t0 += 2 * kSdWarps) {
      // two tiles (t0, t0 + kSdWarps) per round, every load issued before the tests
      bool p[2][4];
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int j = 0; j < 4; ++j) p[h][j] = false;
      if (s > 0) {
        int ai[2][4];
        double dv[2][4];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int c = (t0 + h * kSdWarps) * kSdTile + 32 * j + lane;
            const bool in = t0 + h * kSdWarps < ntiles && c < n;
            ai[h][j] = in ? As[c] : -1;
            dv[h][j] = in ? Ds[c] : 0.0;
          }
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int j = 0; j < 4; ++j)
            p[h][j] = ai[h][j] >= 0 && static_cast<double>(ss[ai[h][j]]) < 4.0001 * dv[h][j];
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int t = t0 + h * kSdWarps;
        unsigned any = 0u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const unsigned m = __ballot_sync(0xffffffffu, p[h][j]);
          if (lane == 0 && t < ntiles) tmask[t][j] = m;
          any |= m;
        }
        if (lane == 0 && t < ntiles) tflag[t] = any ? 1 : 0;
      }
    }
    __syncthreads();
    if (warp == 0) {
      int cnt = 0, tot = 0;  // active tiles; candidates passing the test, with each tile's offset
      for (int t0 = 0; t0 < ntiles; t0 += 32) {
        const int t = t0 + lane;
        const bool f = t < ntiles && tflag[t] != 0;
        const unsigned m = __ballot_sync(0xffffffffu, f);
        if (f) tlist[cnt + __popc(m & ((1u << lane) - 1u))] = t;
        cnt += __popc(m);
        const int c = f ? __popc(tmask[t][0]) + __popc(tmask[t][1]) + __popc(tmask[t][2]) + __popc(tmask[t][3]) : 0;
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        if (t < ntiles) toff[t] = tot + incl - c;
        tot += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) {
        const bool direct = s == 0 || tot <= kSdDirect;  // pass 0: every candidate, listed above
        n_active = (err_sh || direct) ? 0 : cnt;
        n_exact = s == 0 ? n : (direct ? tot : 0);
        direct_sh = s > 0 && direct;
      }
    }
    __syncthreads();
    const int na = n_active;
    if (direct_sh) {  // the direct route: list the candidates that pass the test, in tile order
      for (int t = warp; t < ntiles; t += kSdWarps) {
        if (!tflag[t]) continue;
        int off = toff[t];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const unsigned m = tmask[t][j];
          if ((m >> lane) & 1u) xlist[off + __popc(m & ((1u << lane) - 1u))] = static_cast<uint16_t>(t * kSdTile + 32 * j + lane);
          off += __popc(m);
        }
      }
    }

    // ---- stream the active tiles: TMA -> MMA (x . c) -> screen + exact D^2
    if (warp == 0) {
      if (elect_one()) {
        bool ok = true;
        for (int i = 0; i < na && ok; ++i) {
          const unsigned long long g = gbase + i;
          const int slot = static_cast<int>(g % kSdStages);
          if (g >= kSdStages)
            ok = mbar_wait(smem_u32(&bars.empty[slot]), static_cast<uint32_t>((g / kSdStages - 1) & 1), st,
                           kWhereSeedProducer);
          if (!ok) break;
          const uint32_t dst = smem_u32(ring + slot * kSdStageBytes);
          const uint32_t bar = smem_u32(&bars.full[slot]);
          mbar_arrive_expect_tx(bar, kSdStageBytes);
          const int row = lo + tlist[i] * kSdTile;
          tma_load_3d(dst, &tm, 0, row, bh, bar);
          tma_load_3d(dst + kSdHalf, &tm, 64, row, bh, bar);
        }
      }
    } else if (warp == 1) {
      if (elect_one()) {
        const uint32_t idesc = idesc_bf16_f32(128, kSdSeedRows, 0);
        const uint32_t bsm = smem_u32(seedB);
        bool ok = true;
        for (int i = 0; i < na && ok; ++i) {
          const unsigned long long g = gbase + i;
          const int slot = static_cast<int>(g % kSdStages);
          const int a = static_cast<int>(g % kSdAcc);
          ok = mbar_wait(smem_u32(&bars.full[slot]), static_cast<uint32_t>((g / kSdStages) & 1), st, kWhereSeedMma);
          if (ok && g >= kSdAcc)
            ok = mbar_wait(smem_u32(&bars.acc_empty[a]), static_cast<uint32_t>((g / kSdAcc - 1) & 1), st,
                           kWhereSeedMma);
          if (!ok) break;
          tc_fence_after();
          const uint32_t asm_ = smem_u32(ring + slot * kSdStageBytes);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint64_t ad = sdesc_sw128(asm_ + (ks >> 2) * kSdHalf + (ks & 3) * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(bsm + (ks >> 2) * kSdSeedHalf + (ks & 3) * 32, 16, 1024);
            mma_ss(tmem + a * kSdSeedRows, ad, bd, idesc, ks > 0 ? 1u : 0u);
          }
          mma_commit(smem_u32(&bars.acc_full[a]));
          mma_commit(smem_u32(&bars.empty[slot]));  // the slot is free once these MMAs have read it
        }
      }
    } else {
      const int eg = (warp - 2) >> 2;        // epilogue warpgroup: tiles i with i % 2 == eg
      const int quarter = warp & 3;          // TMEM lanes 32*quarter .. +31
      const int r = 32 * quarter + lane;     // tile row = candidate within the tile
      const float cc = cc_sh;
      bool ok = true;
      for (int i = eg; i < na && ok; i += 2) {
        const unsigned long long g = gbase + i;
        const int a = static_cast<int>(g % kSdAcc);
        const int t = tlist[i];
        ok = mbar_wait(smem_u32(&bars.acc_full[a]), static_cast<uint32_t>((g / kSdAcc) & 1), st, kWhereSeedEpilogue);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const float dot = __uint_as_float(tmem_ld1(tmem + (static_cast<uint32_t>(32 * quarter) << 16) +
                                                   static_cast<uint32_t>(a * kSdSeedRows)));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars.acc_empty[a]));
        const int c = t * kSdTile + r;
        bool need = false;
        if (c < n) {
          // |f - ||x - c||^2| <= 2^-10 (||x||^2 + ||c||^2): float32 norms of 128 terms and a
          // tensor-core dot product of exact bf16 products stay far inside that bound
          const double Dt = Ds[c];
          const float x2 = xx[c];
          const float f = (x2 + cc) - 2.f * dot;
          const float tau = 0.0009765625f * (x2 + cc);
          need = static_cast<double>(ss[As[c]]) < 4.0001 * Dt && static_cast<double>(f) - static_cast<double>(tau) <= Dt;
        }
        const unsigned m = __ballot_sync(0xffffffffu, need);
        if (m) {
          int base = 0;
          if (lane == 0) base = atomicAdd(&n_exact, __popc(m));
          base = __shfl_sync(0xffffffffu, base, 0);
          if (need) xlist[base + __popc(m & ((1u << lane) - 1u))] = static_cast<uint16_t>(c);
        }
      }
    }
    __syncthreads();

    // ---- exact float64 D^2 of the listed candidates, one per thread, rows read from global memory
    const int nx = n_exact;
    for (int j = threadIdx.x; j < nx; j += kSdThreads) {
      const int c = xlist[j];
      const uint4* row = reinterpret_cast<const uint4*>(Xh + static_cast<size_t>(lo + c) * stride * 128);
      uint4 v[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) v[q] = __ldg(row + q);
      double acc = 0.0;
      float x2 = 0.f;  // ||x||^2 for the screen, kept from the first pass
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const uint32_t w[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x0 = bf16lo_to_f32(w[e]), x1 = bf16hi_to_f32(w[e]);
          const double d0 = __dsub_rn(static_cast<double>(x0), csd[8 * q + 2 * e]);
          acc = __dadd_rn(acc, __dmul_rn(d0, d0));
          const double d1 = __dsub_rn(static_cast<double>(x1), csd[8 * q + 2 * e + 1]);
          acc = __dadd_rn(acc, __dmul_rn(d1, d1));
          x2 = fmaf(x0, x0, fmaf(x1, x1, x2));
        }
      }
      if (s == 0) xx[c] = x2;
      const double Dt = Ds[c];
      if (acc < Dt) {
        if (s > 0) atomicAdd(&gtot[c / kSdTile], sd_weight(acc, M0) - sd_weight(Dt, M0));  // modulo 2^64
        Ds[c] = acc;
        As[c] = static_cast<uint16_t>(s);
      }
    }
    __syncthreads();
    gbase += static_cast<unsigned long long>(na);

    if (s == 0) {
      // ---- M0 = the largest D^2 over all candidates, then the per-tile weight sums
      double m = 0.0;
      for (int i = threadIdx.x; i < n; i += kSdThreads) m = fmax(m, Ds[i]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0) wred[warp] = static_cast<unsigned long long>(__double_as_longlong(m));
      __syncthreads();
      if (threadIdx.x == 0) {
        double mx = 0.0;
        for (int w = 0; w < kSdWarps; ++w) mx = fmax(mx, __longlong_as_double(static_cast<long long>(wred[w])));
        sd_bcast(&cta_max[rank], static_cast<unsigned long long>(__double_as_longlong(mx)), CL);
      }
      sd_sync(CL);
      for (int r = 0; r < CL; ++r) M0 = fmax(M0, __longlong_as_double(static_cast<long long>(cta_max[r])));
      for (int t = warp; t < ntiles; t += kSdWarps) {
        unsigned long long q = 0ull;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int c = t * kSdTile + 32 * j + lane;
          if (c < n) q += sd_weight(Ds[c], M0);
        }
        q = warp_sum_u64(q);
        if (lane == 0) gtot[t] = q;
      }
      __syncthreads();
    }
  }

  // ---- teardown: every MMA finished and every TMA load landed before TMEM is freed and the CTA exits
  __syncthreads();
  if (warp == 1 && elect_one()) {
    mma_commit(smem_u32(&bars.mma_done));
    mbar_wait(smem_u32(&bars.mma_done), 0, nullptr, kWhereSeedDrain, kWaitBudgetCycles / 8);
  }
  if (warp == 0 && elect_one()) {
    for (unsigned long long g = gbase >= kSdStages ? gbase - kSdStages : 0ull; g < gbase; ++g)
      mbar_wait(smem_u32(&bars.full[g % kSdStages]), static_cast<uint32_t>((g / kSdStages) & 1), nullptr,
                kWhereSeedDrain, kWaitBudgetCycles / 8);
  }
  if (threadIdx.x == 0 && k > 2)  // the last copy of the seed rows (pass k-2) has landed
    mbar_wait(smem_u32(&bars.rows), static_cast<uint32_t>((k - 3) & 1), nullptr, kWhereSeedDrain,
              kWaitBudgetCycles / 8);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kSdTmemCols);
  if (CL > 1) cluster_sync();  // no CTA leaves while another may still write into its shared memory
}

}  // namespace

cudaError_t launch_kmeanspp_tc(const void* X, int BH, int N, int stride, int S, int k, const double* u,
                               float* centroids, uint16_t* seeds_bf16, DeviceStatus* st, cudaStream_t s) {
  if (k > kSdMaxK || S < 1 || BH < 1) return cudaErrorNotSupported;
  const int cl_min = (S + kSdMaxPerCta - 1) / kSdMaxPerCta;
  if (cl_min > kSdMaxCluster) return cudaErrorNotSupported;
  CUtensorMap tm;
  cudaError_t e = make_tmap_bf16_3d(&tm, X, 128, static_cast<uint64_t>(S), static_cast<uint64_t>(BH),
                                    static_cast<uint64_t>(stride) * 256u, static_cast<uint64_t>(N) * 256u, kSdTile);
  if (e != cudaSuccess) return e;
  auto kern = seed_tc_kernel;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(sd_smem_bytes(kSdMaxPerCta)));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kSdThreads);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // Cluster size: a pass costs about its tiles per CTA plus a fixed part (pick, seed, pruning
  // table); more CTAs per (b,h) only help while every cluster still fits on the GPU at once.
  int best = -1;
  double best_cost = 0.0;
  for (int ncl = cl_min; ncl <= kSdMaxCluster; ++ncl) {
    const int per_cta = (S + ncl - 1) / ncl;
    if (ncl > cl_min && per_cta < kSdTile) break;
    attr[0].val.clusterDim.x = ncl;
    cfg.gridDim = dim3(BH * ncl);
    cfg.dynamicSmemBytes = sd_smem_bytes(per_cta);
    int active = 0;
    if (cudaOccupancyMaxActiveClusters(&active, kern, &cfg) != cudaSuccess || active < 1) {
      cudaGetLastError();
      continue;
    }
    const int waves = (BH + active - 1) / active;
    const double cost = waves * (static_cast<double>((per_cta + kSdTile - 1) / kSdTile) + 3.0);
    if (best < 0 || cost < best_cost) {
      best = ncl;
      best_cost = cost;
    }
  }
  if (best < 0) return cudaErrorNotSupported;
  const int per_cta = (S + best - 1) / best;
  attr[0].val.clusterDim.x = best;
  cfg.gridDim = dim3(BH * best);
  cfg.dynamicSmemBytes = sd_smem_bytes(per_cta);
  return cudaLaunchKernelEx(&cfg, kern, tm, static_cast<const uint16_t*>(X), N, stride, S, k, u, centroids, seeds_bf16,
                            st);
}

}  // namespace svg2
