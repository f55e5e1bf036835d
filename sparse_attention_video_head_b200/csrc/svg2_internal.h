// Internal declarations shared by the .cu files of libsvg2 (not part of the public C ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace svg2 {

// Device status word, at offset 0 of every workspace.
struct DeviceStatus {
  uint32_t code;   // svg2_status of the first device error, 0 if none
  uint32_t where;  // kernel tag (kWhere*)
  uint32_t info0;
  uint32_t info1;
};

constexpr uint32_t kStatusDeviceTimeout = 5;  // == SVG2_ERR_DEVICE_TIMEOUT
constexpr uint32_t kStatusDeviceBounds = 6;   // == SVG2_ERR_DEVICE_BOUNDS

// About 0.5 s at the B200's boost clock: far above any legitimate wait inside one tile step.
constexpr long long kWaitBudgetCycles = 1000LL * 1000LL * 1000LL;

// The status area (kStatusBytes at the start of a workspace) holds the DeviceStatus word at offset
// 0 and, at this offset, a uint64 wait budget in clock cycles for the attention and assignment
// kernels' bounded waits: 0 (the value of a zeroed workspace) means kWaitBudgetCycles, and a value
// above kWaitBudgetCycles is clamped to it, so the field can only shorten a wait.
constexpr size_t kWaitBudgetOffset = 16;

// Kernel tags for DeviceStatus::where.
enum : uint32_t {
  kWhereSort = 1,
  kWhereAssign = 2,
  kWhereAttnProducer = 3,
  kWhereAttnMma = 4,
  kWhereAttnSoftmax = 5,
  kWhereSelftest = 6,
  kWhereAssignTail = 7,
  kWhereAttnDrain = 8,
  kWhereSeedProducer = 9,
  kWhereSeedMma = 10,
  kWhereSeedEpilogue = 11,
  kWhereSeedDrain = 12,
  kWhereGather = 13,     // row gathers and the inverse-permutation scatter (debug build)
  kWhereUpdate = 14,     // centroid update (debug build)
  kWherePlan = 15,       // attention work plan and range table (debug build)
  kWherePruned = 16,     // pruned assignment (debug build)
};

constexpr int kStatusBytes = 256;
static_assert(kWaitBudgetOffset >= sizeof(DeviceStatus) && kWaitBudgetOffset + 8 <= kStatusBytes, "status area");

// The wait-budget field of the status area that starts at st (a workspace's first bytes).
inline const uint64_t* wait_budget_of(const DeviceStatus* st) {
  return reinterpret_cast<const uint64_t*>(reinterpret_cast<const char*>(st) + kWaitBudgetOffset);
}
constexpr int kSortChunks = 32;  // token chunks per (b,h) in the stable counting sort
constexpr int kAssignTileM = 128;
constexpr int kAssignChunkN = 128;  // centroids per MMA chunk
constexpr int kMaxClustersAssign = 1024;  // == SVG2_MAX_CLUSTERS
// From this many clusters on, the Lloyd iterations after the first use the pruned assignment
// (centroid-to-centroid distances exclude most clusters per tile of label-ordered tokens).  Its
// exact float32 search beats the tensor-core pass only when that pass is long (large k) and the
// tiles' candidate sets stay small: tokens far from every centroid widen a tile's radius, and on
// the mixture inputs (10 % such tokens) k = 400 ran 3.5 ms slower per iteration on 24 heads while
// k = 500 and k = 1000 ran 0.2-0.3 ms faster.
constexpr int kPrunedMinK = 500;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline int kpad_of(int k) { return (k + kAssignChunkN - 1) / kAssignChunkN * kAssignChunkN; }

// Bump allocator over the caller's workspace; with base == nullptr it only measures.
struct Carve {
  char* base;
  size_t off;
  explicit Carve(void* b) : base(static_cast<char*>(b)), off(0) {}
  template <class T>
  T* take(size_t count) {
    off = align_up(off, 256);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
};

// Scratch of one k-means call (one role).
struct KmeansScratch {
  uint16_t* c_hi;     // [BH, kpad, d] bf16 high part of the centroids
  uint16_t* c_lo;     // [BH, kpad, d] bf16 residual part
  float* c_norm;      // [BH, kpad] squared norms of the centroids
  double* pp_dist;    // [BH, N] k-means++ current D^2
  int32_t* pp_near;   // [BH, N] k-means++ nearest seed
  int32_t* chunk_hist;// [BH, kSortChunks, k]
  int32_t* perm;      // [BH, N] (if the caller passes none)
  int32_t* offsets;   // [BH, k+1]
  uint4* rr_list;     // [BH * N] tokens whose assignment the exact re-rank decides: {bh, n, c0|c1, c2|c3}
  uint32_t* rr_count; // entries in rr_list
  float* d2;          // [BH, k, k] centroid-to-centroid squared distances (k >= kPrunedMinK only)
};

inline void carve_kmeans(Carve& c, int BH, int N, int d, int k, KmeansScratch& s, bool need_perm) {
  const int kp = kpad_of(k);
  s.c_hi = c.take<uint16_t>(static_cast<size_t>(BH) * kp * d);
  s.c_lo = c.take<uint16_t>(static_cast<size_t>(BH) * kp * d);
  s.c_norm = c.take<float>(static_cast<size_t>(BH) * kp);
  s.pp_dist = c.take<double>(static_cast<size_t>(BH) * N);
  s.pp_near = c.take<int32_t>(static_cast<size_t>(BH) * N);
  s.chunk_hist = c.take<int32_t>(static_cast<size_t>(BH) * kSortChunks * k);
  s.perm = need_perm ? c.take<int32_t>(static_cast<size_t>(BH) * N) : nullptr;
  s.offsets = c.take<int32_t>(static_cast<size_t>(BH) * (k + 1));
  s.rr_list = c.take<uint4>(static_cast<size_t>(BH) * N);
  s.rr_count = c.take<uint32_t>(1);
  s.d2 = k >= kPrunedMinK ? c.take<float>(static_cast<size_t>(BH) * k * k) : nullptr;
}

// Attention work plan: one unit = up to two 128-row Q tiles of one Q cluster.
struct AttnUnit {
  int32_t bh;
  int32_t cluster;
  int32_t row0;   // first permuted row of the unit
  int32_t nrows;  // 1..256
};

inline int attn_max_units_per_head(int N, int nQ) { return (N + 255) / 256 + nQ; }

struct AttnScratch {
  AttnUnit* units;     // [BH * max_units_per_head] compacted
  int32_t* head_units; // [BH]
  int32_t* head_base;  // [BH + 1]
};

inline void carve_attn(Carve& c, int BH, int N, int nQ, AttnScratch& s) {
  s.units = c.take<AttnUnit>(static_cast<size_t>(BH) * attn_max_units_per_head(N, nQ));
  s.head_units = c.take<int32_t>(BH);
  s.head_base = c.take<int32_t>(BH + 1);
}

// ---- launchers (host functions defined in the .cu files); all return cudaError_t ----
cudaError_t launch_sort(const int32_t* labels, int BH, int N, int k, int32_t* perm, int32_t* offsets,
                        int32_t* counts, int32_t* chunk_hist, DeviceStatus* st, cudaStream_t s);
// st (may be null) receives the debug build's index reports; the release build never writes it here.
cudaError_t launch_gather(const void* X, bool x_f32, const int32_t* perm, int BH, int N, int d, void* Xp,
                          cudaStream_t s, DeviceStatus* st = nullptr);
cudaError_t launch_gather2(const void* X0, const void* X1, bool x_f32, const int32_t* perm, int BH, int N,
                           int d, void* Xp0, void* Xp1, cudaStream_t s, DeviceStatus* st = nullptr);
cudaError_t launch_unpermute(const void* Op, const int32_t* perm, int BH, int N, int d, void* O,
                             cudaStream_t s, DeviceStatus* st = nullptr);

// k-means++ seeding over the candidates kmeanspp_candidates() counts; when they are fewer than the
// tokens, their rows are first copied into `cand` (at least kmeanspp_candidate_bytes() bytes).
cudaError_t launch_kmeanspp(const void* X, bool x_f32, int BH, int N, int d, int k, const double* u,
                            float* centroids, double* dist, int32_t* near, uint16_t* seeds_bf16, int seed_tokens,
                            void* cand, size_t cand_bytes, DeviceStatus* st, cudaStream_t s);
// k-means++ seeding on the tensor cores (bf16, d = 128); returns cudaErrorNotSupported for shapes
// it does not take, so that the caller can use the CUDA-core kernels.
// seeds_bf16: scratch of BH * k * d bf16 (the seeds' rows, for the seed-to-seed distances).
cudaError_t launch_kmeanspp_tc(const void* X, int BH, int N, int stride, int S, int k, const double* u,
                               float* centroids, uint16_t* seeds_bf16, DeviceStatus* st, cudaStream_t s);
// Number of k-means++ candidates: seed_tokens of the N tokens (one per stratum of the token order),
// or all N when seed_tokens is 0 or at least N.
int kmeanspp_candidates(int N, int seed_tokens);
// Bytes of the compact candidate copy the seeding needs (0 when every token is a candidate).
size_t kmeanspp_candidate_bytes(int BH, int N, int d, bool x_f32, int seed_tokens);
cudaError_t launch_centroid_prep(const float* centroids, int BH, int k, int d, uint16_t* c_hi, uint16_t* c_lo,
                                 float* c_norm, cudaStream_t s);
cudaError_t launch_assign(const void* X, bool x_f32, int BH, int N, int d, int k, const float* centroids,
                          const uint16_t* c_hi, const uint16_t* c_lo, const float* c_norm, int32_t* labels,
                          uint4* rr_list, uint32_t* rr_count, DeviceStatus* st, const uint64_t* wait_budget,
                          cudaStream_t s);
// Lloyd assignment from the previous iteration's stable sort `perm` (bf16 X, d = 128, k <= 1024):
// the centroid-to-centroid table into d2 [BH, k, k], then the pruned exact search per tile.
cudaError_t launch_assign_pruned(const void* X, int BH, int N, int k, const float* centroids, const int32_t* perm,
                                 float* d2, int32_t* labels, cudaStream_t s, DeviceStatus* st = nullptr);
cudaError_t launch_update(const void* X, bool x_f32, int BH, int N, int d, int k, const int32_t* perm,
                          const int32_t* offsets, float* centroids, uint16_t* c_hi, uint16_t* c_lo,
                          float* c_norm, cudaStream_t s, DeviceStatus* st = nullptr);

cudaError_t launch_select(const float* cq, const float* ck, const float* weights_in, const int32_t* count_k,
                          int BH, int nQ, int nK, int d, float top_p, float scale, float* weights_out,
                          uint8_t* mask, int32_t* sel_count, int32_t* sel_idx, int32_t* stream_len,
                          cudaStream_t s);

cudaError_t launch_sparse_attn(const void* Qp, const void* Kp, const void* Vp, const int32_t* q_off,
                               const int32_t* k_off, const int32_t* sel_count, const int32_t* sel_idx, int BH,
                               int N, int d, int nQ, int nK, float scale, const int32_t* perm_q, void* O,
                               const AttnScratch& scratch, DeviceStatus* st, const uint64_t* wait_budget,
                               cudaStream_t s);

// Dequantisation scales of the FP8 attention: one float per (b,h) plane of Q, K and V.
struct F8Scales {
  const float* q = nullptr;
  const float* k = nullptr;
  const float* v = nullptr;
};
// FP8 variant (d = 128): Qp8, Kp8, Vp8 E4M3 codes [BH,N,d], value = E4M3(code) * scale of the plane.
cudaError_t launch_sparse_attn_fp8(const void* Qp8, const void* Kp8, const void* Vp8, const F8Scales& f8,
                                   const int32_t* q_off, const int32_t* k_off, const int32_t* sel_count,
                                   const int32_t* sel_idx, int BH, int N, int d, int nQ, int nK, float scale,
                                   const int32_t* perm_q, void* O, const AttnScratch& sc, DeviceStatus* st,
                                   const uint64_t* wait_budget, cudaStream_t s);
// Per-head E4M3 quantisation (svg2_fp8.cu).  launch_amax zeroes amax [tensors][BH] and writes the
// float bits of max |x| per plane; launch_gather_e4m3 writes Y[r] = E4M3(X[bh, perm[r]] * 448 / amax)
// (perm may be null: the identity; X1/Y1 may be null); launch_amax_to_scale turns each amax into
// the dequantisation scale amax / 448 in place (1 for an all-zero plane).
cudaError_t launch_amax(const void* X0, const void* X1, const void* X2, int tensors, bool f32, int BH, int N, int d,
                        uint32_t* amax, cudaStream_t s);
cudaError_t launch_gather_e4m3(const void* X0, const void* X1, bool f32, const int32_t* perm, int BH, int N, int d,
                               const uint32_t* amax0, const uint32_t* amax1, void* Y0, void* Y1, cudaStream_t s,
                               DeviceStatus* st);
cudaError_t launch_amax_to_scale(uint32_t* amax, int n, cudaStream_t s);
cudaError_t launch_dense_plan(int BH, int N, int32_t* q_off, int32_t* k_off, int32_t* sel_count, int32_t* sel_idx,
                              cudaStream_t s);

cudaError_t launch_selftest_mma(const void* A, const void* Bm, int n, const void* V, float* C, float* O,
                                DeviceStatus* st, cudaStream_t s);

// Tensor map over a [rows, d] bf16 matrix with a box of 64 columns x box_rows rows, 128B swizzle.
// 2D tensor map over rows of d one-byte codes (E4M3), box d x box_rows, 128-byte swizzle (d = 128).
cudaError_t make_tmap_u8_rows(void* map /* CUtensorMap* */, const void* base, uint64_t rows, uint32_t d,
                              uint32_t box_rows);
cudaError_t make_tmap_bf16_rows(void* map /* CUtensorMap* */, const void* base, uint64_t rows, uint32_t d,
                                uint32_t box_rows);

// Tensor map over `planes` matrices of `rows` rows x d bf16 columns with the given pitches in bytes
// (a row pitch above d * 2 selects every n-th row), box of 64 columns x box_rows rows, 128B swizzle.
cudaError_t make_tmap_bf16_3d(void* map /* CUtensorMap* */, const void* base, uint32_t d, uint64_t rows,
                              uint64_t planes, uint64_t row_pitch, uint64_t plane_pitch, uint32_t box_rows);

}  // namespace svg2
