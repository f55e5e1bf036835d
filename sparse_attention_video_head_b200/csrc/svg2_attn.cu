// Variable-block-size sparse attention ("Sparse VideoGen2" wiki summary, Method (4); Key claims
// section 4.3, Fig. 7(b)) on tcgen05 tensor cores with TMEM accumulators.
//
// Work unit = up to two 128-row Q tiles (A, B) of one Q cluster.  Their keys are the rows of the
// kept K clusters, concatenated into one packed key stream and cut into 128-key tiles, so a
// cluster boundary costs nothing; only the stream's last tile is masked.  The design follows the
// Blackwell execution model rather than the pages' FlashInfer-derived kernel:
//   warps 0-3   softmax + lazy O rescale + epilogue for Q tile A (TMEM lanes = query rows)
//   warps 4-7   the same for Q tile B
//   warps 8, 9, 11  key/value producers (rows 0-47, 48-87, 88-127 of each key tile; warps 8-9 also
//               build the kept clusters' range table): cp.async gathers into the 128-byte-swizzled
//               layout the tensor core reads (two stages).  Three warps on three SMSPs, because each
//               SMSP also runs two softmax warps and the slowest of those sets the pace.
//   warp 10     TMEM allocator (512 columns: S_A, S_B, O_A, O_B), Q tiles by TMA, then the
//               single-thread MMA issuer
// After set-up the softmax warps take 176 registers per thread and the rest 136.  Each Q tile has one
// 128-column S slot: S = Q K^T is one N = 128 product per key tile (full rate; a 64-key product is
// bound by the shared-memory reads of its operands), and P (bf16) overwrites the slot's first 64
// columns as the A operand of the PV product.  MMA order per key tile j: PV_A(j), S_A(j+1),
// PV_B(j), S_B(j+1), so the two tiles' softmaxes run half a period apart and each one's
// exponentials overlap the other's products.  The commit that announces S_x(j+1) also covers
// PV_x(j), so the softmax may rescale O_x in TMEM (only when the row max grows by more than 2^8)
// as soon as it sees S_x(j+1).  Softmax is exact: p = 2^(s*scale*log2e - m), O / l at the end,
// with l summed over the float32 p whose bf16 rounding the PV product uses.
#include <cuda.h>
#include <cuda_bf16.h>

#include <type_traits>

#include "svg2_device.cuh"
#include "svg2_internal.h"

namespace svg2 {

namespace {

// 12 warps in three warpgroups: 8 softmax warps, then 3 key/value producer warps and the MMA issuer.
constexpr int kAttnThreads = 384;
constexpr int kProducerWarp0 = 8, kProducerWarps = 2;  // the warps that build the range table
constexpr int kProducerThreads = 32 * kProducerWarps;
constexpr int kGatherThreads = 96;                      // warps 8, 9 and 11 gather K and V
constexpr int kMmaWarp = 10;
// Register split after set-up (setmaxnreg): 256 x 176 + 128 x 136 = 62464 <= 384 x 168, the launch's
// allocation under __launch_bounds__(384, 1) (ptxas gives 168 registers per thread).
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 176;  // in steps of 8, the split at which neither side spills (168: softmax; 184: the rest)
constexpr int kOtherRegs = 136;
static_assert(256 * kSoftmaxRegs + (kAttnThreads - 256) * kOtherRegs <= kAttnThreads * kLaunchRegs, "register split");
constexpr int kMaxRanges = 1024;
// bytes of one 128-row tile of d values: bf16, or E4M3 codes in the FP8 variant (16 KB column blocks of
// 128-byte swizzled rows)
template <int D, bool F8>
constexpr uint32_t tile_bytes() { return 128u * D * (F8 ? 1u : 2u); }
template <int D, bool F8>
constexpr uint32_t attn_smem() {
  return 6 * tile_bytes<D, F8>() + 1024 /*align*/ + 4096 /*ranges*/ + 4096 + 64 /*cum*/ + 256;
}
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Of every 16 key pairs of a row, this many (the last ones) get 2^x from the cubic on the FMA pipe;
// the rest use the MUFU, whose 16 exponentials per clock per SM would otherwise bound the softmax.
// The FP8 instance's products take half the time, so more of its exponentials go to the FMA pipe.
constexpr int kCubicPairs = 4;
constexpr int kCubicPairsF8 = 4;

struct AttnBars {
  uint64_t q_full, k_full[2], v_full[2], k_empty[2], v_empty[2], o_full, mma_done;
  uint64_t s_full[2], p_full[2][2];  // per Q tile (ring mode: per S slot); P in two 64-key halves
  uint64_t pv_done;                  // ring mode: one phase per PV product
  uint32_t tmem_base;
  int32_t L;
  int32_t nranges;
};

__global__ void plan_count_kernel(const int32_t* __restrict__ q_off, int nQ, int N,
                                  int32_t* __restrict__ head_units, DeviceStatus* st) {
  __shared__ int32_t part[32];
  const int bh = blockIdx.x;
  int acc = 0;
  for (int i = threadIdx.x; i < nQ; i += blockDim.x) {
    const int r0 = q_off[static_cast<size_t>(bh) * (nQ + 1) + i];
    const int n = q_off[static_cast<size_t>(bh) * (nQ + 1) + i + 1] - r0;
    SVG2_DEBUG_CHECK(r0 >= 0 && n >= 0 && r0 + n <= N, st, kWherePlan, i, r0);
    if (r0 < 0 || n <= 0 || r0 + n > N) continue;
    acc += (n + 255) / 256;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += part[w];
    head_units[bh] = t;
  }
}

__global__ void plan_scan_kernel(const int32_t* __restrict__ head_units, int BH, int32_t* __restrict__ head_base) {
  if (threadIdx.x == 0) {
    int run = 0;
    for (int b = 0; b < BH; ++b) {
      head_base[b] = run;
      run += head_units[b];
    }
    head_base[BH] = run;
  }
}

__global__ void plan_write_kernel(const int32_t* __restrict__ q_off, int nQ, int N,
                                  const int32_t* __restrict__ head_base, AttnUnit* __restrict__ units) {
  const int bh = blockIdx.x;
  if (threadIdx.x != 0) return;
  int pos = head_base[bh];
  const int32_t* qo = q_off + static_cast<size_t>(bh) * (nQ + 1);
  for (int i = 0; i < nQ; ++i) {
    const int r0 = qo[i], n = qo[i + 1] - qo[i];
    if (r0 < 0 || n <= 0 || r0 + n > N) continue;  // malformed offsets produce no work
    for (int u = 0; u < n; u += 256) {
      AttnUnit un;
      un.bh = bh;
      un.cluster = i;
      un.row0 = r0 + u;
      un.nrows = min(256, n - u);
      units[pos++] = un;
    }
  }
}

// Element type of the operand planes: bf16, or one-byte E4M3 codes.  The code is wrapped in a struct
// so that the pointers are not of a character type, which may alias anything and then costs the key
// gather's address arithmetic (measured: 8 % on sparse attention).
struct E4m3Code {
  uint8_t bits;
};
template <bool F8>
using AttnElem = std::conditional_t<F8, E4m3Code, __nv_bfloat16>;

// F8: Q, K, V are E4M3 codes with one scale per (b,h) plane each (f8.q, f8.k, f8.v): the scores take
// sq * sk into the softmax scale, the output sv into its normaliser, and P goes to the PV product as
// E4M3.
template <int D, bool F8>
__global__ void __launch_bounds__(kAttnThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const AttnElem<F8>* __restrict__ Kp,
                       const AttnElem<F8>* __restrict__ Vp, const int32_t* __restrict__ k_off,
                       const int32_t* __restrict__ sel_count, const int32_t* __restrict__ sel_idx, int N, int nQ,
                       int nK, float scale, const int32_t* __restrict__ perm_q, __nv_bfloat16* __restrict__ O,
                       const AttnUnit* __restrict__ units, const int32_t* __restrict__ head_base, int BH,
                       const F8Scales f8, DeviceStatus* st, const uint64_t* __restrict__ wait_budget) {
  const int total_units = head_base[BH];
  if (static_cast<int>(blockIdx.x) >= total_units) return;
  if (status_set(st)) return;
  const long long wb = effective_wait_budget(wait_budget);
  const AttnUnit un = units[blockIdx.x];

  constexpr uint32_t kTile = tile_bytes<D, F8>();
  constexpr int kRowBytes = D * (F8 ? 1 : 2);
  constexpr int kHalves = kRowBytes / 128;  // 128-byte swizzle atoms across a row
  constexpr int kKStep = F8 ? 32 : 16;       // contraction elements (32 bytes) per MMA instruction
  constexpr int kSteps = D / kKStep;         // instructions of one S product
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_s = smem;                 // Q_A, Q_B
  uint8_t* k_s = smem + 2 * kTile;     // K stage 0, 1
  uint8_t* v_s = smem + 4 * kTile;     // V stage 0, 1
  int32_t* r_start = reinterpret_cast<int32_t*>(smem + 6 * kTile);
  int32_t* r_cum = r_start + kMaxRanges;  // kMaxRanges + 1 entries
  AttnBars* bars = reinterpret_cast<AttnBars*>(r_cum + kMaxRanges + 16);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = un.bh;
  const bool has_b = un.nrows > 128;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars->k_full[i]), kGatherThreads);
      mbar_init(smem_u32(&bars->v_full[i]), kGatherThreads);
      mbar_init(smem_u32(&bars->k_empty[i]), 1);
      mbar_init(smem_u32(&bars->v_empty[i]), 1);
      mbar_init(smem_u32(&bars->s_full[i]), 1);
      mbar_init(smem_u32(&bars->p_full[i][0]), 4);
      mbar_init(smem_u32(&bars->p_full[i][1]), 4);
    }
    mbar_init(smem_u32(&bars->o_full), 1);
    mbar_init(smem_u32(&bars->mma_done), 1);
    mbar_init(smem_u32(&bars->pv_done), 1);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  if (warp >= kProducerWarp0 && warp < kProducerWarp0 + kProducerWarps) {
    // key-stream range table: start row and stream offset of every kept K cluster
    const int pt = threadIdx.x - 32 * kProducerWarp0;
    const size_t row = static_cast<size_t>(bh) * nQ + un.cluster;
    int cnt = sel_count[row];
    SVG2_DEBUG_CHECK(cnt >= 0 && cnt <= nK, st, kWherePlan, row, cnt);
    cnt = cnt < 0 ? 0 : (cnt > nK ? nK : cnt);
    const int32_t* ko = k_off + static_cast<size_t>(bh) * (nK + 1);
    // each thread handles a contiguous block of entries, then a scan over the block sums
    const int per = (cnt + kProducerThreads - 1) / kProducerThreads;
    const int e0 = min(cnt, pt * per), e1 = min(cnt, e0 + per);
    int local = 0;
    for (int e = e0; e < e1; ++e) {
      int j = sel_idx[row * nK + e];
      SVG2_DEBUG_CHECK(j >= 0 && j < nK, st, kWherePlan, row, j);
      j = j < 0 ? 0 : (j >= nK ? nK - 1 : j);
      const int s0 = ko[j], len = ko[j + 1] - s0;
      SVG2_DEBUG_CHECK(s0 >= 0 && len >= 0 && s0 + len <= N, st, kWherePlan, j, s0);
      r_start[e] = s0;
      r_cum[e] = len;  // temporarily the length
      local += len;
    }
    // scan of `local` across the producer threads via shuffles + shared
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int32_t* wsum = r_cum + kMaxRanges + 1;  // one scratch int per producer warp (inside the 16-int gap)
    if (lane == 31) wsum[warp - kProducerWarp0] = incl;
    asm volatile("bar.sync 1, %0;" ::"n"(kProducerThreads) : "memory");
    int wbase = 0;
    for (int w = 0; w < warp - kProducerWarp0; ++w) wbase += wsum[w];
    int run = wbase + incl - local;
    for (int e = e0; e < e1; ++e) {
      const int len = r_cum[e];
      r_cum[e] = run;
      run += len;
    }
    if (pt == kProducerThreads - 1) {
      bars->L = run;  // the last producer thread holds the last block
      bars->nranges = cnt;
      r_cum[cnt] = run;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int L = bars->L;
  const int nranges = bars->nranges;
  const int T = (L + 127) / 128;  // 128-key tiles of the packed key stream

  // The softmax warpgroups take registers from the producer/MMA warpgroup.
  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kOtherRegs) : "memory");
  }
  if (warp == kMmaWarp) {
    // ---------------- Q by TMA, then MMA issue ----------------
    if (elect_one()) {
      prefetch_tensormap(&tm_q);
      const uint32_t qbar = smem_u32(&bars->q_full);
      const uint32_t qa = smem_u32(q_s), qb = smem_u32(q_s + kTile);
      mbar_arrive_expect_tx(qbar, has_b ? 2 * kTile : kTile);
      const int y = bh * N + un.row0;
#pragma unroll
      for (int hf = 0; hf < kHalves; ++hf) {
        tma_load_2d(qa + hf * 16384, &tm_q, hf * (128 / (kRowBytes / D)), y, qbar);
        if (has_b) tma_load_2d(qb + hf * 16384, &tm_q, hf * (128 / (kRowBytes / D)), y + 128, qbar);
      }
      bool ok = mbar_wait(qbar, 0, st, kWhereAttnMma, wb);
      const uint32_t id_s = F8 ? idesc_e4m3_f32(128, 128, 0) : idesc_bf16_f32(128, 128, 0);
      const uint32_t id_o = F8 ? idesc_e4m3_f32(128, D, 1) : idesc_bf16_f32(128, D, 1);
      const uint32_t kb = smem_u32(k_s), vb = smem_u32(v_s);
      // Descriptors of every operand tile, built once: stepping along K only moves the start
      // address field (bits 0-13, in 16-byte units), which stays far below its 14-bit limit.
      const uint64_t dq0 = sdesc_sw128(qa, 16, 1024), dq1 = sdesc_sw128(qb, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(kb, 16, 1024), dk1 = sdesc_sw128(kb + kTile, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(vb, 16384, 1024), dv1 = sdesc_sw128(vb + kTile, 16384, 1024);
      // S = Q_x K(j)^T over the 128 keys of stage j%2 into the 128 S columns of slot `slot`
      // (slot = x, or in ring mode the slot of tile j); announced on s_full[slot]
      auto issue_s = [&](int x, int stage, int slot) {
        const uint32_t d_tmem = tmem + slot * 128;
        const uint64_t aq = x == 0 ? dq0 : dq1;
        const uint64_t bk = stage == 0 ? dk0 : dk1;
#pragma unroll
        for (int ks = 0; ks < kSteps; ++ks) {
          const uint64_t koff = static_cast<uint64_t>(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
          if constexpr (F8) mma_ss_f8(d_tmem, aq + koff, bk + koff, id_s, ks > 0 ? 1u : 0u);
          else mma_ss(d_tmem, aq + koff, bk + koff, id_s, ks > 0 ? 1u : 0u);
        }
        mma_commit(smem_u32(&bars->s_full[slot]));
      };
      // O_x += P(j) V(j) over keys 64h .. 64h+63: P is packed in the first columns of its S slot,
      // two bf16 or four E4M3 keys per 32-bit column, so each instruction's kKStep keys take 8
      // columns and kKStep 128-byte rows of V
      auto issue_pv = [&](int x, int slot, int stage, int h, bool acc) {
        constexpr int kPvSteps = 64 / kKStep;
        const uint32_t d_tmem = tmem + 256 + x * 128;
        const uint32_t p_tmem = tmem + slot * 128;
        const uint64_t bv = stage == 0 ? dv0 : dv1;
#pragma unroll
        for (int ks = kPvSteps * h; ks < kPvSteps * h + kPvSteps; ++ks) {
          const uint64_t voff = static_cast<uint64_t>((ks * kKStep * 128) >> 4);
          if constexpr (F8) mma_ts_f8(d_tmem, p_tmem + ks * 8, bv + voff, id_o, (acc || ks > 0) ? 1u : 0u);
          else mma_ts(d_tmem, p_tmem + ks * 8, bv + voff, id_o, (acc || ks > 0) ? 1u : 0u);
        }
      };
      if (ok && T > 0) {
        ok = mbar_wait(smem_u32(&bars->k_full[0]), 0, st, kWhereAttnMma, wb);
        if (ok) {
          fence_proxy_async_smem();  // the key rows were written by cp.async (generic proxy)
          tc_fence_after();
          issue_s(0, 0, 0);
          if (has_b) issue_s(1, 0, 1);
          mma_commit(smem_u32(&bars->k_empty[0]));  // K(0) is not read again
        }
      }
      if (!has_b) {
        // Ring mode (one Q tile): S(j) goes to slot j%2, the unused tile's columns serving as the
        // second slot, so S(j+1) is computed while the softmax of j runs.  Order: S(0), S(1), then
        // per tile PV(j) in two halves and S(j+2) into the slot PV(j) has just read.  pv_done marks
        // each PV product (the S commits no longer cover the latest one).
        if (ok && T > 1) {
          ok = mbar_wait(smem_u32(&bars->k_full[1]), 0, st, kWhereAttnMma, wb);
          if (ok) {
            fence_proxy_async_smem();
            tc_fence_after();
            issue_s(0, 1, 1);
            mma_commit(smem_u32(&bars->k_empty[1]));
          }
        }
        // P(j) is announced on the barriers of its slot, phase j/2: while this thread waits for V(j)
        // the softmax may finish P(j+1) too, which on one shared barrier pair would complete two
        // phases before the wait for the second half of P(j) looks, and that wait would never end.
        // P(j+2) needs S(j+2), issued only after both halves of P(j) were taken, so a slot's
        // barriers are never two phases ahead.
        for (int j = 0; j < T && ok; ++j) {
          const int stage = j & 1;
          const uint32_t ppar = (j >> 1) & 1;
          ok = mbar_wait(smem_u32(&bars->p_full[stage][0]), ppar, st, kWhereAttnMma, wb);
          if (ok) ok = mbar_wait(smem_u32(&bars->v_full[stage]), (j >> 1) & 1, st, kWhereAttnMma, wb);
          if (!ok) break;
          fence_proxy_async_smem();
          tc_fence_after();
          issue_pv(0, stage, stage, 0, j > 0);
          ok = mbar_wait(smem_u32(&bars->p_full[stage][1]), ppar, st, kWhereAttnMma, wb);
          if (!ok) break;
          tc_fence_after();
          issue_pv(0, stage, stage, 1, true);
          mma_commit(smem_u32(&bars->pv_done));
          mma_commit(smem_u32(&bars->v_empty[stage]));  // V(j) is not read again
          if (j + 2 < T) {
            ok = mbar_wait(smem_u32(&bars->k_full[stage]), ((j + 2) >> 1) & 1, st, kWhereAttnMma, wb);
            if (!ok) break;
            fence_proxy_async_smem();
            tc_fence_after();
            issue_s(0, stage, stage);
            mma_commit(smem_u32(&bars->k_empty[stage]));  // nor K(j+2)
          }
        }
      }
      // Per tile j: PV_A(j) in two halves as the softmax hands them over, S_A(j+1), then the same
      // for B.  The commit after S_x(j+1) also covers PV_x(j), so when the softmax of x sees
      // S_x(j+1) it may rescale O_x and reuse its S columns.
      for (int j = 0; j < T && ok && has_b; ++j) {
        const int stage = j & 1, nstage = (j + 1) & 1;
        const bool more = j + 1 < T;
        ok = mbar_wait(smem_u32(&bars->p_full[0][0]), j & 1, st, kWhereAttnMma, wb);
        if (ok) ok = mbar_wait(smem_u32(&bars->v_full[stage]), (j >> 1) & 1, st, kWhereAttnMma, wb);
        if (!ok) break;
        fence_proxy_async_smem();
        tc_fence_after();
        issue_pv(0, 0, stage, 0, j > 0);
        ok = mbar_wait(smem_u32(&bars->p_full[0][1]), j & 1, st, kWhereAttnMma, wb);
        if (!ok) break;
        tc_fence_after();
        issue_pv(0, 0, stage, 1, true);
        if (more) {
          ok = mbar_wait(smem_u32(&bars->k_full[nstage]), ((j + 1) >> 1) & 1, st, kWhereAttnMma, wb);
          if (!ok) break;
          fence_proxy_async_smem();
          tc_fence_after();
          issue_s(0, nstage, 0);
        }
        ok = mbar_wait(smem_u32(&bars->p_full[1][0]), j & 1, st, kWhereAttnMma, wb);
        if (!ok) break;
        tc_fence_after();
        issue_pv(1, 1, stage, 0, j > 0);
        ok = mbar_wait(smem_u32(&bars->p_full[1][1]), j & 1, st, kWhereAttnMma, wb);
        if (!ok) break;
        tc_fence_after();
        issue_pv(1, 1, stage, 1, true);
        mma_commit(smem_u32(&bars->v_empty[stage]));  // V(j) is not read again
        if (more) {
          issue_s(1, nstage, 1);
          mma_commit(smem_u32(&bars->k_empty[nstage]));  // nor K(j+1)
        }
      }
      if (ok) mma_commit(smem_u32(&bars->o_full));
      mma_commit(smem_u32(&bars->mma_done));
      mbar_wait(smem_u32(&bars->mma_done), 0, nullptr, kWhereAttnDrain, kWaitBudgetCycles / 8);
      if (!ok) mbar_wait(qbar, 0, nullptr, kWhereAttnDrain, kWaitBudgetCycles / 8);
    }
  } else if (warp == 8 || warp == 9 || warp == 11) {
    // ---------------- key/value gather producer ----------------
    // Warps 8, 9 and 11 fill rows 0-47, 48-87 and 88-127 of each key tile.  Each lane
    // follows the source rows of two stream positions from tile to tile with cursors over the range
    // table (positions only grow, so each cursor crosses every range boundary once, where a search
    // per tile would cost a chain of dependent shared-memory reads); then every cp.async instruction
    // moves whole rows (16 lanes x 16 bytes per row at d = 128), so one instruction touches 2 rows.
    constexpr int CPR = kRowBytes / 16;  // 16-byte chunks per row
    constexpr int RPI = 32 / CPR;        // rows per warp instruction
    constexpr int kIters = 48 / RPI;     // at most this many instructions per tile and operand
    constexpr int kPeriod = 8 / RPI;     // the row's place in its 8-row swizzle group repeats this often
    const int pw = warp == 11 ? 2 : warp - 8;
    const int wr0 = pw == 0 ? 0 : (pw == 1 ? 48 : 88);   // rows 0-47, 48-87, 88-127 (multiples of 8)
    const int nrw = pw == 0 ? 48 : 40;
    const uint32_t kb = smem_u32(k_s), vb = smem_u32(v_s);
    const uint32_t head_row0 = static_cast<uint32_t>(bh) * static_cast<uint32_t>(N);  // B*H*N < 2^31
    const int my_chunk = lane % CPR, my_sub = lane / CPR;
    const int hf = my_chunk >> 3, cc = my_chunk & 7;
    // This thread's byte offset within a tile for instruction it is xo[it % kPeriod] + it * RPI * 128
    // (row rr = it * RPI + my_sub, 128-byte swizzle: chunk cc lands at cc ^ (rr & 7)).
    uint32_t xo[kPeriod];
#pragma unroll
    for (int k = 0; k < kPeriod; ++k)
      xo[k] = hf * 16384 + (wr0 + my_sub) * 128 + ((cc ^ ((k * RPI + my_sub) & 7)) << 4);
    const AttnElem<F8>* kbase = Kp + my_chunk * (16 / sizeof(AttnElem<F8>));
    const AttnElem<F8>* vbase = Vp + my_chunk * (16 / sizeof(AttnElem<F8>));
    int e0c = 0, e1c = 0;  // cursors of this lane's two stream positions: r_cum[e] <= p < r_cum[e + 1]
    auto src_row = [&](int p, int& e) {
      if (p >= L) p = L - 1;
      while (e + 1 < nranges && r_cum[e + 1] <= p) ++e;
      const int r = r_start[e] + (p - r_cum[e]);
      SVG2_DEBUG_CHECK(r >= 0 && r < N, st, kWhereAttnProducer, p, r);
      return r < 0 ? 0 : (r >= N ? N - 1 : r);
    };
    for (int j = 0; j < T; ++j) {
      const int stage = j & 1;
      // global rows of this lane's two stream positions; a K row and its V row share the index
      const uint32_t g0 = head_row0 + static_cast<uint32_t>(src_row(j * 128 + wr0 + lane, e0c));
      const uint32_t g1 = head_row0 + static_cast<uint32_t>(src_row(j * 128 + wr0 + 32 + lane, e1c));
      const uint32_t kdst = kb + stage * kTile, vdst = vb + stage * kTile;
      // K(j) may land as soon as both S products of K(j-2) are done, V(j) once both PV products of
      // V(j-2) are; each lands asynchronously and counts itself on its full barrier
      if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait_sleep(smem_u32(&bars->k_empty[stage]), ((j >> 1) - 1) & 1, st,
                                                             kWhereAttnProducer, 128, wb)))
        break;
#pragma unroll
      for (int it = 0; it < kIters; ++it) {
        if (it * RPI >= nrw) break;
        // row it * RPI + my_sub of the warp's rows: below 32 exactly when it * RPI < 32
        const uint32_t g = __shfl_sync(0xffffffffu, it * RPI < 32 ? g0 : g1, (it * RPI + my_sub) & 31);
        cp_async16(kdst + xo[it % kPeriod] + it * RPI * 128, kbase + static_cast<size_t>(g) * D);
      }
      cp_async_mbar_arrive(smem_u32(&bars->k_full[stage]));
      if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait_sleep(smem_u32(&bars->v_empty[stage]), ((j >> 1) - 1) & 1, st,
                                                             kWhereAttnProducer, 128, wb)))
        break;
#pragma unroll
      for (int it = 0; it < kIters; ++it) {
        if (it * RPI >= nrw) break;
        const uint32_t g = __shfl_sync(0xffffffffu, it * RPI < 32 ? g0 : g1, (it * RPI + my_sub) & 31);
        cp_async16(vdst + xo[it % kPeriod] + it * RPI * 128, vbase + static_cast<size_t>(g) * D);
      }
      cp_async_mbar_arrive(smem_u32(&bars->v_full[stage]));
    }
    cp_async_wait<0>();
  } else if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs) : "memory");
    // ---------------- softmax / correction / epilogue for tile X ----------------
    const int x = warp >> 2;
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int nrows_x = x == 0 ? min(128, un.nrows) : un.nrows - 128;
    if (x == 1 && !has_b) {
      // nothing to do
    } else {
      const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
      const uint32_t t_o = tmem + lane_off + 256 + x * 128;
      const float sl2 = F8 ? scale * kLog2e * f8.q[bh] * f8.k[bh] : scale * kLog2e;
      // Every tcgen05.ld/st below is a warp-collective (.sync.aligned) instruction, so all of it
      // runs under warp-uniform control flow; per-row decisions only select values.
      float m_used = -INFINITY, l = 0.f;
      bool ok = true;
      // ring mode (no tile B): S(j) and P(j) in slot j%2 (parity j/2 of that slot's barriers)
      const bool ring = !has_b;
      for (int j = 0; j < T; ++j) {
        const int slot = ring ? (j & 1) : x;
        const uint32_t par = ring ? ((j >> 1) & 1) : (j & 1);
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->s_full[slot]), par, st, kWhereAttnSoftmax, wb));
        if (!ok) break;
        tc_fence_after();
        const uint32_t t_sj = tmem + lane_off + slot * 128;
        uint32_t sv[128];
        tmem_ld32p(t_sj, sv);
        tmem_ld32p(t_sj + 32, sv + 32);
        tmem_ld32p(t_sj + 64, sv + 64);
        tmem_ld32p(t_sj + 96, sv + 96);
        tmem_wait_ld();
        const int valid = L - j * 128;
        if (valid < 128) {  // the key stream's last tile: columns past its end become -inf (p = 0)
#pragma unroll
          for (int e = 0; e < 128; ++e)
            if (e >= valid) sv[e] = __float_as_uint(-INFINITY);
        }
        // eight independent chains of three-input maxima
        float m8[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) m8[c] = fmaxf(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1]));
#pragma unroll
        for (int e = 16; e < 128; e += 16)
#pragma unroll
          for (int c = 0; c < 8; ++c)
            m8[c] = fmax3(m8[c], __uint_as_float(sv[e + 2 * c]), __uint_as_float(sv[e + 2 * c + 1]));
        const float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
        const float m_new = fmaxf(m_used, mx * sl2);
        const bool grow = m_new > m_used + kRescaleThreshold;
        float f = 1.f;
        if (grow) {
          if (j > 0) f = fast_exp2(m_used - m_new);
          l *= f;
          m_used = m_new;
        }
        if (j > 0 && __any_sync(0xffffffffu, grow)) {
          // O_x must hold every PV product up to j-1, and no MMA writes it until this warpgroup
          // hands over P_x(j).  With two tiles the commit announcing S_x(j) covers PV_x(j-1); in
          // ring mode S(j) was issued before PV(j-1), so that product is awaited on pv_done.
          // Rows that keep their max multiply by 1.
          if (ring) {
            ok = __all_sync(0xffffffffu,
                            mbar_wait(smem_u32(&bars->pv_done), (j - 1) & 1, st, kWhereAttnSoftmax, wb));
            if (!ok) break;
            tc_fence_after();
          }
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(t_o + c * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * f);
            tmem_st32(t_o + c * 32, v);
          }
        }
        // p = 2^(s * scale * log2(e) - m): the argument for two keys at once, the exponentials on
        // the MUFU, the row sum over float32 p (pairs), bf16 pairs written over S as the P operand
        const float2 scl = make_float2(sl2, sl2), negm = make_float2(-m_used, -m_used);
        float2 lsum4[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) lsum4[c] = make_float2(0.f, 0.f);
        // P goes over in two 64-key halves, so that the first half's PV product runs while the
        // second half's exponentials are computed
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          if constexpr (F8) {
            auto p_pair = [&](int e) {  // p of keys 64hh + 2e, 64hh + 2e + 1
              const int col = hh * 64 + 2 * e;
              const float2 t = fma2(make_float2(__uint_as_float(sv[col]), __uint_as_float(sv[col + 1])), scl, negm);
              const float2 pe = ((e & 15) >= 16 - kCubicPairsF8) ? exp2_cubic2(t)
                                                                 : make_float2(fast_exp2(t.x), fast_exp2(t.y));
              lsum4[e & 3] = add2(lsum4[e & 3], pe);
              return pe;
            };
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float2 a = p_pair(2 * e), b = p_pair(2 * e + 1);
              pk[e] = pack_e4m3x4(a.x, a.y, b.x, b.y);
            }
            tmem_st16(t_sj + hh * 16, pk);
          } else {
            uint32_t pk[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int col = hh * 64 + 2 * e;
              const float2 t = fma2(make_float2(__uint_as_float(sv[col]), __uint_as_float(sv[col + 1])), scl, negm);
              float2 pe;
              if ((e & 15) >= 16 - kCubicPairs) pe = exp2_cubic2(t);
              else pe = make_float2(fast_exp2(t.x), fast_exp2(t.y));
              pk[e] = pack_bf16x2(pe.x, pe.y);
              lsum4[e & 3] = add2(lsum4[e & 3], pe);
            }
            tmem_st32(t_sj + hh * 32, pk);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bars->p_full[slot][hh]));
        }
        const float2 ls = add2(add2(lsum4[0], lsum4[1]), add2(lsum4[2], lsum4[3]));
        l += ls.x + ls.y;
      }
      if (ok && T > 0)
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->o_full), 0, st, kWhereAttnSoftmax, wb));
      if (ok) {
        tc_fence_after();
        const int prow = un.row0 + x * 128 + row;
        int tk = -1;
        if (row < nrows_x) {
          tk = perm_q != nullptr ? __ldg(perm_q + static_cast<size_t>(bh) * N + prow) : prow;
          SVG2_DEBUG_CHECK(tk >= 0 && tk < N, st, kWhereAttnSoftmax, prow, tk);
          if (tk < 0 || tk >= N) tk = -1;  // an invalid permutation entry is skipped
        }
        uint4* dst = reinterpret_cast<uint4*>(O + (static_cast<size_t>(bh) * N + (tk < 0 ? 0 : tk)) * D);
        const float inv = (T > 0 && l > 0.f) ? (F8 ? f8.v[bh] : 1.f) / l : 0.f;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          if (T > 0) {
            tmem_ld32(t_o + c * 32, v);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0u;
          }
          if (tk >= 0) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(v[8 * e + 0]) * inv, __uint_as_float(v[8 * e + 1]) * inv);
              w.y = pack_bf16x2(__uint_as_float(v[8 * e + 2]) * inv, __uint_as_float(v[8 * e + 3]) * inv);
              w.z = pack_bf16x2(__uint_as_float(v[8 * e + 4]) * inv, __uint_as_float(v[8 * e + 5]) * inv);
              w.w = pack_bf16x2(__uint_as_float(v[8 * e + 6]) * inv, __uint_as_float(v[8 * e + 7]) * inv);
              dst[c * 4 + e] = w;
            }
          }
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------------------------
// Self-test of the tensor-core path: C = A B^T, then O = bf16(C[:, :128]) V with P from TMEM.
// ------------------------------------------------------------------------------------------------
struct TestBars {
  uint64_t full, mma1, mma2;
  uint32_t tmem_base;
};

__global__ void __launch_bounds__(128, 1)
    selftest_mma_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                        const __grid_constant__ CUtensorMap tm_v, int n, float* __restrict__ C,
                        float* __restrict__ Out, DeviceStatus* st) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_s = smem;                  // 32 KB
  uint8_t* b_s = smem + 32768;          // up to 64 KB (256 rows)
  uint8_t* v_s = smem + 32768 + 65536;  // 32 KB
  TestBars* bars = reinterpret_cast<TestBars*>(v_s + 32768);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->full), 1);
    mbar_init(smem_u32(&bars->mma1), 1);
    mbar_init(smem_u32(&bars->mma2), 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t bhalf = static_cast<uint32_t>(n) * 128u;  // bytes per 64-column half of B
  bool ok = true;
  if (warp == 0 && elect_one()) {
    const uint32_t bar = smem_u32(&bars->full);
    mbar_arrive_expect_tx(bar, 32768 + 2 * bhalf + 32768);
    tma_load_2d(smem_u32(a_s), &tm_a, 0, 0, bar);
    tma_load_2d(smem_u32(a_s) + 16384, &tm_a, 64, 0, bar);
    tma_load_2d(smem_u32(b_s), &tm_b, 0, 0, bar);
    tma_load_2d(smem_u32(b_s) + bhalf, &tm_b, 64, 0, bar);
    tma_load_2d(smem_u32(v_s), &tm_v, 0, 0, bar);
    tma_load_2d(smem_u32(v_s) + 16384, &tm_v, 64, 0, bar);
    ok = mbar_wait(bar, 0, st, kWhereSelftest);
    if (ok) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16_f32(128, static_cast<uint32_t>(n), 0);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t ko = (ks >> 2) * 16384 + (ks & 3) * 32;
        const uint32_t kob = (ks >> 2) * bhalf + (ks & 3) * 32;
        mma_ss(tmem, sdesc_sw128(smem_u32(a_s) + ko, 16, 1024), sdesc_sw128(smem_u32(b_s) + kob, 16, 1024), idesc,
               ks > 0 ? 1u : 0u);
      }
    }
    mma_commit(smem_u32(&bars->mma1));
  }
  __syncwarp();
  ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->mma1), 0, st, kWhereSelftest));
  tc_fence_after();
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const int row = warp * 32 + lane;
  if (ok) {
    for (int c = 0; c < n / 32; ++c) {
      uint32_t v[32];
      tmem_ld32(tmem + lane_off + c * 32, v);
      tmem_wait_ld();
      for (int e = 0; e < 32; ++e) C[static_cast<size_t>(row) * n + c * 32 + e] = __uint_as_float(v[e]);
      if (c < 4) {
        uint32_t pk[16];
        for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
        tmem_st16(tmem + lane_off + 256 + c * 16, pk);
      }
    }
    if (n < 128) {
      uint32_t pk[16];
      for (int e = 0; e < 16; ++e) pk[e] = 0u;
      for (int c = n / 32; c < 4; ++c) tmem_st16(tmem + lane_off + 256 + c * 16, pk);
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0 && elect_one()) {
    if (ok) {
      const uint32_t idesc = idesc_bf16_f32(128, 128, 1);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        mma_ts(tmem + 384, tmem + 256 + ks * 8, sdesc_sw128(smem_u32(v_s) + ks * 2048, 16384, 1024), idesc,
               ks > 0 ? 1u : 0u);
    }
    mma_commit(smem_u32(&bars->mma2));
  }
  __syncwarp();
  ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->mma2), 0, st, kWhereSelftest) && ok);
  tc_fence_after();
  if (ok) {
    for (int c = 0; c < 4; ++c) {
      uint32_t v[32];
      tmem_ld32(tmem + lane_off + 384 + c * 32, v);
      tmem_wait_ld();
      for (int e = 0; e < 32; ++e) Out[static_cast<size_t>(row) * 128 + c * 32 + e] = __uint_as_float(v[e]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Dense attention as the one-cluster case: per (b,h) one Q cluster and one K cluster holding all N
// tokens in their original order, the K cluster selected.
__global__ void dense_plan_kernel(int BH, int N, int32_t* __restrict__ q_off, int32_t* __restrict__ k_off,
                                  int32_t* __restrict__ sel_count, int32_t* __restrict__ sel_idx) {
  const int bh = blockIdx.x * blockDim.x + threadIdx.x;
  if (bh >= BH) return;
  q_off[2 * bh] = 0;
  q_off[2 * bh + 1] = N;
  k_off[2 * bh] = 0;
  k_off[2 * bh + 1] = N;
  sel_count[bh] = 1;
  sel_idx[bh] = 0;
}

}  // namespace

cudaError_t launch_dense_plan(int BH, int N, int32_t* q_off, int32_t* k_off, int32_t* sel_count, int32_t* sel_idx,
                              cudaStream_t s) {
  dense_plan_kernel<<<(BH + 255) / 256, 256, 0, s>>>(BH, N, q_off, k_off, sel_count, sel_idx);
  return cudaGetLastError();
}

namespace {

template <int D, bool F8>
cudaError_t launch_attn_kernel(const CUtensorMap& tq, const void* Kp, const void* Vp, const int32_t* k_off,
                               const int32_t* sel_count, const int32_t* sel_idx, int BH, int N, int nQ, int nK,
                               float scale, const int32_t* perm_q, void* O, const AttnScratch& sc,
                               const F8Scales& f8, DeviceStatus* st, const uint64_t* wait_budget, cudaStream_t s) {
  constexpr uint32_t smem = attn_smem<D, F8>();
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel<D, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long grid = static_cast<long long>(BH) * attn_max_units_per_head(N, nQ);
  sparse_attn_kernel<D, F8><<<static_cast<unsigned>(grid), kAttnThreads, smem, s>>>(
      tq, static_cast<const AttnElem<F8>*>(Kp), static_cast<const AttnElem<F8>*>(Vp), k_off, sel_count, sel_idx, N, nQ, nK,
      scale, perm_q, static_cast<__nv_bfloat16*>(O), sc.units, sc.head_base, BH, f8, st, wait_budget);
  return cudaGetLastError();
}

cudaError_t launch_attn_plan(const int32_t* q_off, int BH, int N, int nQ, const AttnScratch& sc, DeviceStatus* st,
                             cudaStream_t s) {
  plan_count_kernel<<<BH, 256, 0, s>>>(q_off, nQ, N, sc.head_units, st);
  plan_scan_kernel<<<1, 32, 0, s>>>(sc.head_units, BH, sc.head_base);
  plan_write_kernel<<<BH, 32, 0, s>>>(q_off, nQ, N, sc.head_base, sc.units);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sparse_attn(const void* Qp, const void* Kp, const void* Vp, const int32_t* q_off,
                               const int32_t* k_off, const int32_t* sel_count, const int32_t* sel_idx, int BH,
                               int N, int d, int nQ, int nK, float scale, const int32_t* perm_q, void* O,
                               const AttnScratch& sc, DeviceStatus* st, const uint64_t* wait_budget,
                               cudaStream_t s) {
  cudaError_t e = launch_attn_plan(q_off, BH, N, nQ, sc, st, s);
  if (e != cudaSuccess) return e;
  alignas(64) CUtensorMap tq;
  e = make_tmap_bf16_rows(&tq, Qp, static_cast<uint64_t>(BH) * N, static_cast<uint32_t>(d), 128);
  if (e != cudaSuccess) return e;
  if (d == 128)
    return launch_attn_kernel<128, false>(tq, Kp, Vp, k_off, sel_count, sel_idx, BH, N, nQ, nK, scale, perm_q, O, sc,
                                          F8Scales{}, st, wait_budget, s);
  return launch_attn_kernel<64, false>(tq, Kp, Vp, k_off, sel_count, sel_idx, BH, N, nQ, nK, scale, perm_q, O, sc,
                                       F8Scales{}, st, wait_budget, s);
}

cudaError_t launch_sparse_attn_fp8(const void* Qp8, const void* Kp8, const void* Vp8, const F8Scales& f8,
                                   const int32_t* q_off, const int32_t* k_off, const int32_t* sel_count,
                                   const int32_t* sel_idx, int BH, int N, int d, int nQ, int nK, float scale,
                                   const int32_t* perm_q, void* O, const AttnScratch& sc, DeviceStatus* st,
                                   const uint64_t* wait_budget, cudaStream_t s) {
  if (d != 128) return cudaErrorInvalidValue;
  cudaError_t e = launch_attn_plan(q_off, BH, N, nQ, sc, st, s);
  if (e != cudaSuccess) return e;
  alignas(64) CUtensorMap tq;
  e = make_tmap_u8_rows(&tq, Qp8, static_cast<uint64_t>(BH) * N, static_cast<uint32_t>(d), 128);
  if (e != cudaSuccess) return e;
  return launch_attn_kernel<128, true>(tq, Kp8, Vp8, k_off, sel_count, sel_idx, BH, N, nQ, nK, scale, perm_q, O, sc,
                                       f8, st, wait_budget, s);
}

cudaError_t launch_selftest_mma(const void* A, const void* Bm, int n, const void* V, float* C, float* O,
                                DeviceStatus* st, cudaStream_t s) {
  alignas(64) CUtensorMap ta, tb, tv;
  cudaError_t e = make_tmap_bf16_rows(&ta, A, 128, 128, 128);
  if (e == cudaSuccess) e = make_tmap_bf16_rows(&tb, Bm, static_cast<uint64_t>(n), 128, static_cast<uint32_t>(n));
  if (e == cudaSuccess) e = make_tmap_bf16_rows(&tv, V, 128, 128, 128);
  if (e != cudaSuccess) return e;
  const uint32_t smem = 32768 + 65536 + 32768 + 1024 + 256;
  e = cudaFuncSetAttribute(selftest_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  selftest_mma_kernel<<<1, 128, smem, s>>>(ta, tb, tv, n, C, O, st);
  return cudaGetLastError();
}

}  // namespace svg2
