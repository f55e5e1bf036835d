// C-ABI entry points of libsvg2 (declared in include/svg2.h): argument validation, workspace
// carving, tensor-map encoding and the launch sequence of each stage and of the whole layer.
// Host code only; every step of the method runs in the kernels of the other .cu files.
#include <vector>
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>
#include <new>

#include "svg2.h"
#include "svg2_internal.h"

namespace svg2 {

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int to_status(cudaError_t e) { return e == cudaSuccess ? SVG2_OK : SVG2_ERR_CUDA; }

bool valid_dtype(int dt) { return dt == SVG2_BF16 || dt == SVG2_F32; }

// Sizes shared by all stages.
int check_sizes(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1) return SVG2_ERR_INVALID_ARG;
  if (N > SVG2_MAX_TOKENS) return SVG2_ERR_UNSUPPORTED;
  // the (b,h) planes are a grid dimension of their own in several kernels (at most 65535)
  if (static_cast<long long>(B) * H > 65535) return SVG2_ERR_UNSUPPORTED;
  // token rows across all planes are indexed (and addressed by TMA) with 32-bit integers
  if (static_cast<long long>(B) * H * N >= (1LL << 31)) return SVG2_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return SVG2_ERR_UNSUPPORTED;
  return SVG2_OK;
}

int check_k(int k, int N) {
  if (k < 1 || k > N) return SVG2_ERR_INVALID_ARG;
  if (k > SVG2_MAX_CLUSTERS) return SVG2_ERR_UNSUPPORTED;
  return SVG2_OK;
}

int check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (ws == nullptr) return SVG2_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return SVG2_ERR_WORKSPACE;
  if (ws_bytes < need) return SVG2_ERR_WORKSPACE;
  return SVG2_OK;
}

struct LayerCarve {
  DeviceStatus* st;
  KmeansScratch kq, kk;
  int32_t *labels_q, *labels_k, *count_q, *count_k, *perm_q, *perm_k, *q_off, *k_off;
  float* weights;
  uint8_t* mask;
  int32_t *sel_count, *sel_idx, *stream_len;
  void *Qp, *Kp, *Vp, *Op;
  AttnScratch attn;
  uint32_t* f8;  // FP8 attention: per-plane maxima, then scales, of Q [BH], K [BH], V [BH]
};

void carve_layer(Carve& c, int BH, int N, int d, int nQ, int nK, const svg2_layer_outputs* o, LayerCarve& L) {
  L.st = c.take<DeviceStatus>(kStatusBytes / sizeof(DeviceStatus));
  carve_kmeans(c, BH, N, d, nQ, L.kq, false);
  carve_kmeans(c, BH, N, d, nK, L.kk, false);
  auto pick = [&](int32_t* user, size_t n) { return user != nullptr ? user : c.take<int32_t>(n); };
  const size_t BHN = static_cast<size_t>(BH) * N;
  L.labels_q = pick(o ? o->labels_q : nullptr, BHN);
  L.labels_k = pick(o ? o->labels_k : nullptr, BHN);
  L.count_q = pick(o ? o->count_q : nullptr, static_cast<size_t>(BH) * nQ);
  L.count_k = pick(o ? o->count_k : nullptr, static_cast<size_t>(BH) * nK);
  L.perm_q = pick(o ? o->perm_q : nullptr, BHN);
  L.perm_k = pick(o ? o->perm_k : nullptr, BHN);
  L.q_off = pick(o ? o->q_off : nullptr, static_cast<size_t>(BH) * (nQ + 1));
  L.k_off = pick(o ? o->k_off : nullptr, static_cast<size_t>(BH) * (nK + 1));
  L.weights = o ? o->weights : nullptr;  // optional output only
  L.mask = (o && o->mask) ? o->mask : c.take<uint8_t>(static_cast<size_t>(BH) * nQ * nK);
  L.sel_count = pick(o ? o->sel_count : nullptr, static_cast<size_t>(BH) * nQ);
  L.sel_idx = pick(o ? o->sel_idx : nullptr, static_cast<size_t>(BH) * nQ * nK);
  L.stream_len = pick(o ? o->stream_len : nullptr, static_cast<size_t>(BH) * nQ);
  L.Qp = c.take<uint16_t>(BHN * d);
  L.Kp = c.take<uint16_t>(BHN * d);
  L.Vp = c.take<uint16_t>(BHN * d);
  L.Op = c.take<uint16_t>(BHN * d);
  carve_attn(c, BH, N, nQ, L.attn);
  L.f8 = c.take<uint32_t>(3 * static_cast<size_t>(BH));
}

// Bytes from the start of the permuted Q plane to the end of the permuted K plane: both are free
// during the k-means (the gathers fill them afterwards), so the k-means++ candidate rows (at most
// two bytes per element more than one bf16 plane, for float32 inputs) are copied there.
size_t candidate_room(const LayerCarve& L, int BH, int N, int d) {
  return static_cast<size_t>(reinterpret_cast<const char*>(L.Kp) - reinterpret_cast<const char*>(L.Qp)) +
         static_cast<size_t>(BH) * N * d * sizeof(uint16_t);
}

// cand / cand_bytes: room for the compact copy of the k-means++ candidate rows (kmeanspp_candidate_bytes).
cudaError_t run_kmeans(const void* X, bool f32, int BH, int N, int d, int k, int iters, int init, const double* u,
                       int seed_tokens, float* C, int32_t* labels, int32_t* counts, int32_t* perm, int32_t* offsets,
                       const KmeansScratch& s, void* cand, size_t cand_bytes, DeviceStatus* st, cudaStream_t stream) {
  cudaError_t e = cudaSuccess;
  if (init == SVG2_INIT_KMEANSPP)
    e = launch_kmeanspp(X, f32, BH, N, d, k, u, C, s.pp_dist, s.pp_near, s.c_hi, seed_tokens, cand, cand_bytes, st,
                        stream);
  if (e == cudaSuccess) e = launch_centroid_prep(C, BH, k, d, s.c_hi, s.c_lo, s.c_norm, stream);
  for (int it = 0; it < iters && e == cudaSuccess; ++it) {
    // after the first iteration, perm holds the stable sort of the previous labels: the pruned search
    if (it > 0 && s.d2 != nullptr && !f32 && d == 128)
      e = launch_assign_pruned(X, BH, N, k, C, perm, s.d2, labels, stream, st);
    else
      e = launch_assign(X, f32, BH, N, d, k, C, s.c_hi, s.c_lo, s.c_norm, labels, s.rr_list, s.rr_count, st,
                        wait_budget_of(st), stream);
    if (e == cudaSuccess) e = launch_sort(labels, BH, N, k, perm, offsets, counts, s.chunk_hist, st, stream);
    if (e == cudaSuccess)
      e = launch_update(X, f32, BH, N, d, k, perm, offsets, C, s.c_hi, s.c_lo, s.c_norm, stream, st);
  }
  return e;
}

// Stream-ordered store of one 64-bit value into device memory (the status area's wait budget).
__global__ void store_u64_kernel(uint64_t* dst, uint64_t v) { *dst = v; }

cudaError_t launch_store_u64(uint64_t* dst, uint64_t v, cudaStream_t s) {
  store_u64_kernel<<<1, 1, 0, s>>>(dst, v);
  return cudaGetLastError();
}

}  // namespace

cudaError_t make_tmap_bf16_rows(void* map, const void* base, uint64_t rows, uint32_t d, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  if (!aligned(base, 16) || rows == 0 || box_rows == 0 || box_rows > 256) return cudaErrorInvalidValue;
  const cuuint64_t dims[2] = {d, rows};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(static_cast<CUtensorMap*>(map), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
                        dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_u8_rows(void* map, const void* base, uint64_t rows, uint32_t d, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  if (!aligned(base, 16) || rows == 0 || d != 128 || box_rows == 0 || box_rows > 256) return cudaErrorInvalidValue;
  const cuuint64_t dims[2] = {d, rows};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d)};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(static_cast<CUtensorMap*>(map), CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_bf16_3d(void* map, const void* base, uint32_t d, uint64_t rows, uint64_t planes,
                              uint64_t row_pitch, uint64_t plane_pitch, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  if (!aligned(base, 16) || rows == 0 || planes == 0 || box_rows == 0 || box_rows > 256) return cudaErrorInvalidValue;
  if (row_pitch % 16 != 0 || plane_pitch % 16 != 0) return cudaErrorInvalidValue;
  const cuuint64_t dims[3] = {d, rows, planes};
  const cuuint64_t strides[2] = {row_pitch, plane_pitch};
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(static_cast<CUtensorMap*>(map), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
                        dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace svg2

using namespace svg2;

extern "C" {

const char* svg2_status_string(int status) {
  switch (status) {
    case SVG2_OK: return "SVG2_OK";
    case SVG2_ERR_INVALID_ARG: return "SVG2_ERR_INVALID_ARG: invalid argument";
    case SVG2_ERR_UNSUPPORTED: return "SVG2_ERR_UNSUPPORTED: size or type not supported by the library";
    case SVG2_ERR_WORKSPACE: return "SVG2_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case SVG2_ERR_CUDA: return "SVG2_ERR_CUDA: a CUDA call failed";
    case SVG2_ERR_DEVICE_TIMEOUT: return "SVG2_ERR_DEVICE_TIMEOUT: a bounded device wait ran out";
    case SVG2_ERR_DEVICE_BOUNDS: return "SVG2_ERR_DEVICE_BOUNDS: a device index check failed";
    default: return "SVG2: unknown status";
  }
}

int svg2_workspace_size(int B, int H, int N, int d, int nQ, int nK, size_t* bytes) {
  if (bytes == nullptr) return SVG2_ERR_INVALID_ARG;
  int r = check_sizes(B, H, N, d);
  if (r == SVG2_OK) r = check_k(nQ, N);
  if (r == SVG2_OK) r = check_k(nK, N);
  if (r != SVG2_OK) return r;
  Carve c(nullptr);
  LayerCarve L;
  carve_layer(c, B * H, N, d, nQ, nK, nullptr, L);
  *bytes = align_up(c.off, 256);
  return SVG2_OK;
}

int svg2_check_status(void* ws, void* stream, int* device_status, uint32_t* where, uint32_t* info) {
  if (ws == nullptr || device_status == nullptr) return SVG2_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceStatus h{};
  cudaError_t e = cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof(DeviceStatus), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return SVG2_ERR_CUDA;
  *device_status = static_cast<int>(h.code);
  if (where) *where = h.where;
  if (info) {
    info[0] = h.info0;
    info[1] = h.info1;
  }
  return SVG2_OK;
}

int svg2_set_wait_budget(void* ws, uint64_t cycles, void* stream) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return SVG2_ERR_INVALID_ARG;
  const cudaError_t e = launch_store_u64(reinterpret_cast<uint64_t*>(static_cast<char*>(ws) + kWaitBudgetOffset),
                                         cycles, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SVG2_OK : SVG2_ERR_CUDA;
}

int svg2_kmeanspp(const void* X, int dtype, int B, int H, int N, int d, int k, const double* u, int seed_tokens,
                  float* centroids, void* ws, size_t ws_bytes, void* stream) {
  try {
    int r = check_sizes(B, H, N, d);
    if (r == SVG2_OK) r = check_k(k, N);
    if (r != SVG2_OK) return r;
    if (!valid_dtype(dtype) || X == nullptr || u == nullptr || centroids == nullptr || seed_tokens < 0)
      return SVG2_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(centroids, 16)) return SVG2_ERR_INVALID_ARG;
    if (kmeanspp_candidates(N, seed_tokens) < k) return SVG2_ERR_INVALID_ARG;  // fewer candidates than seeds
    const int BH = B * H;
    Carve c(ws);
    DeviceStatus* st = c.take<DeviceStatus>(kStatusBytes / sizeof(DeviceStatus));
    KmeansScratch s;
    carve_kmeans(c, BH, N, d, k, s, false);
    const size_t cand_bytes = kmeanspp_candidate_bytes(BH, N, d, dtype == SVG2_F32, seed_tokens);
    void* cand = c.take<uint8_t>(cand_bytes);
    r = check_ws(ws, ws_bytes, c.off);
    if (r != SVG2_OK) return r;
    return to_status(launch_kmeanspp(X, dtype == SVG2_F32, BH, N, d, k, u, centroids, s.pp_dist, s.pp_near,
                                     s.c_hi, seed_tokens, cand, cand_bytes, st, static_cast<cudaStream_t>(stream)));
  } catch (...) {
    return SVG2_ERR_CUDA;
  }
}

int svg2_kmeans(const void* X, int dtype, int B, int H, int N, int d, int k, int iters, int init, const double* u,
                int seed_tokens, float* centroids, int32_t* labels, int32_t* counts, int32_t* perm, int32_t* offsets, void* ws,
                size_t ws_bytes, void* stream) {
  try {
    int r = check_sizes(B, H, N, d);
    if (r == SVG2_OK) r = check_k(k, N);
    if (r != SVG2_OK) return r;
    if (!valid_dtype(dtype) || iters < 1 || (init != SVG2_INIT_GIVEN && init != SVG2_INIT_KMEANSPP))
      return SVG2_ERR_INVALID_ARG;
    if (X == nullptr || centroids == nullptr || labels == nullptr || counts == nullptr) return SVG2_ERR_INVALID_ARG;
    if (init == SVG2_INIT_KMEANSPP && u == nullptr) return SVG2_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(centroids, 16)) return SVG2_ERR_INVALID_ARG;
    const int BH = B * H;
    Carve c(ws);
    DeviceStatus* st = c.take<DeviceStatus>(kStatusBytes / sizeof(DeviceStatus));
    if (seed_tokens < 0) return SVG2_ERR_INVALID_ARG;
    if (init == SVG2_INIT_KMEANSPP && kmeanspp_candidates(N, seed_tokens) < k)
      return SVG2_ERR_INVALID_ARG;  // fewer candidates than seeds
    KmeansScratch s;
    carve_kmeans(c, BH, N, d, k, s, perm == nullptr);
    const size_t cand_bytes =
        init == SVG2_INIT_KMEANSPP ? kmeanspp_candidate_bytes(BH, N, d, dtype == SVG2_F32, seed_tokens) : 0;
    void* cand = c.take<uint8_t>(cand_bytes);
    r = check_ws(ws, ws_bytes, c.off);
    if (r != SVG2_OK) return r;
    if (perm == nullptr) perm = s.perm;
    if (offsets == nullptr) offsets = s.offsets;
    return to_status(run_kmeans(X, dtype == SVG2_F32, BH, N, d, k, iters, init, u, seed_tokens, centroids, labels, counts, perm,
                                offsets, s, cand, cand_bytes, st, static_cast<cudaStream_t>(stream)));
  } catch (...) {
    return SVG2_ERR_CUDA;
  }
}

static int select_common(const float* cq, const float* ck, const float* w_in, const int32_t* count_k, int B, int H,
                         int nQ, int nK, int d, float top_p, float scale, float* weights, uint8_t* mask,
                         int32_t* sel_count, int32_t* sel_idx, int32_t* stream_len, void* ws, size_t ws_bytes,
                         void* stream) {
  if (B < 1 || H < 1 || nQ < 1 || nK < 1) return SVG2_ERR_INVALID_ARG;
  if (nQ > SVG2_MAX_CLUSTERS || nK > SVG2_MAX_CLUSTERS) return SVG2_ERR_UNSUPPORTED;
  if (w_in == nullptr && d != 64 && d != 128) return SVG2_ERR_UNSUPPORTED;
  if (!(top_p > 0.f) || top_p != top_p) return SVG2_ERR_INVALID_ARG;
  if (count_k == nullptr || mask == nullptr || sel_count == nullptr || sel_idx == nullptr) return SVG2_ERR_INVALID_ARG;
  if (w_in == nullptr && (cq == nullptr || ck == nullptr)) return SVG2_ERR_INVALID_ARG;
  int r = check_ws(ws, ws_bytes, kStatusBytes);
  if (r != SVG2_OK) return r;
  return to_status(launch_select(cq, ck, w_in, count_k, B * H, nQ, nK, d, top_p, scale, weights, mask, sel_count,
                                 sel_idx, stream_len, static_cast<cudaStream_t>(stream)));
}

int svg2_select(const float* cq, const float* ck, const int32_t* count_k, int B, int H, int nQ, int nK, int d,
                float top_p, float scale, float* weights, uint8_t* mask, int32_t* sel_count, int32_t* sel_idx,
                int32_t* stream_len, void* ws, size_t ws_bytes, void* stream) {
  try {
    return select_common(cq, ck, nullptr, count_k, B, H, nQ, nK, d, top_p, scale, weights, mask, sel_count, sel_idx,
                         stream_len, ws, ws_bytes, stream);
  } catch (...) {
    return SVG2_ERR_CUDA;
  }
}

int svg2_select_from_weights(const float* weights, const int32_t* count_k, int B, int H, int nQ, int nK, float top_p,
                             uint8_t* mask, int32_t* sel_count, int32_t* sel_idx, int32_t* stream_len, void* ws,
                             size_t ws_bytes, void* stream) {
  try {
    if (weights == nullptr) return SVG2_ERR_INVALID_ARG;
    return select_common(nullptr, nullptr, weights, count_k, B, H, nQ, nK, 0, top_p, 1.f, nullptr, mask, sel_count,
                         sel_idx, stream_len, ws, ws_bytes, stream);
  } catch (...) {
    return SVG2_ERR_CUDA;
  }
}

int svg2_sort(const int32_t* labels, int B, int H, int N, int k, int32_t* perm, int32_t* offsets, int32_t* counts,
              void* ws, size_t ws_bytes, void* stream) {
  try {
    if (B < 1 || H < 1 || N < 1) return SVG2_ERR_INVALID_ARG;
    if (N > SVG2_MAX_TOKENS) return SVG2_ERR_UNSUPPORTED;
    if (k < 1) return SVG2_ERR_INVALID_ARG;
    if (k > SVG2_MAX_CLUSTERS) return SVG2_ERR_UNSUPPORTED;  // (a sort may have more clusters than tokens)
    int r = SVG2_OK;
    if (labels == nullptr || perm == nullptr || offsets == nullptr) return SVG2_ERR_INVALID_ARG;
    const int BH = B * H;
    Carve c(ws);
    DeviceStatus* st = c.take<DeviceStatus>(kStatusBytes / sizeof(DeviceStatus));
    int32_t* ch = c.take<int32_t>(static_cast<size_t>(BH) * kSortChunks * k);
    r = check_ws(ws, ws_bytes, c.off);
    if (r != SVG2_OK) return r;
    return to_status(launch_sort(labels, BH, N, k, perm, offsets, counts, ch, st, static_cast<cudaStream_t>(stream)));
  } catch (...) {
    return SVG2_ERR_CUDA;
  }
}

int svg2_gather(const void* X, int dtype, const int32_t* perm, int B, int H, int N, int d, void* Xp, void* stream) {
  try {
    const int r = check_sizes(B, H, N, d);
    if (r != SVG2_OK) return r;
    if (!valid_dtype(dtype) || X == nullptr || perm == nullptr || Xp == nullptr) return SVG2_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(Xp, 16)) return SVG2_ERR_INVALID_ARG;
    return to_status(launch_gather(X, dtype == SVG2_F32, perm, B * H, N, d, Xp, static_cast<cudaStream_t>(stream)));
  } catch (...) {
    return SVG2_ERR_CUDA;
  }
}

int svg2_permute(const void* X, int dtype, const int32_t* labels, int B, int H, int N, int d, int k, void* Xp,
                 int32_t* perm, int32_t* offsets, int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
  try {
    int r = svg2_sort(labels, B, H, N, k, perm, offsets, counts, ws, ws_bytes, stream);
    if (r != SVG2_OK) return r;
    return svg2_gather(X, dtype, perm, B, H, N, d, Xp, stream);
  } catch (...) {
    return SVG2_ERR_CUDA;
  }
}

int svg2_sparse_attn(const void* Qp, const void* Kp, const void* Vp, const int32_t* q_off, const int32_t* k_off,
                     const int32_t* sel_count, const int32_t* sel_idx, int B, int H, int N, int d, int nQ, int nK,
                     float scale, const int32_t* perm_q, void* O, void* ws, size_t ws_bytes, void* stream) {
  try {
    int r = check_sizes(B, H, N, d);
    if (r == SVG2_OK) r = check_k(nQ, N);
    if (r == SVG2_OK) r = check_k(nK, N);
    if (r != SVG2_OK) return r;
    if (Qp == nullptr || Kp == nullptr || Vp == nullptr || q_off == nullptr || k_off == nullptr ||
        sel_count == nullptr || sel_idx == nullptr || O == nullptr)
      return SVG2_ERR_INVALID_ARG;
    if (!aligned(Qp, 16) || !aligned(Kp, 16) || !aligned(Vp, 16) || !aligned(O, 16)) return SVG2_ERR_INVALID_ARG;
    if (scale != scale) return SVG2_ERR_INVALID_ARG;
    const int BH = B * H;
    Carve c(ws);
    DeviceStatus* st = c.take<DeviceStatus>(kStatusBytes / sizeof(DeviceStatus));
    AttnScratch a;
    carve_attn(c, BH, N, nQ, a);
    r = check_ws(ws, ws_bytes, c.off);
    if (r != SVG2_OK) return r;
    return to_status(launch_sparse_attn(Qp, Kp, Vp, q_off, k_off, sel_count, sel_idx, BH, N, d, nQ, nK, scale, perm_q,
                                        O, a, st, wait_budget_of(st), static_cast<cudaStream_t>(stream)));
  } catch (...) {
    return SVG2_ERR_CUDA;
  }
}

int svg2_quantize_e4m3(const void* X, int dtype, const int32_t* perm, int B, int H, int N, int d, void* X8,
                       float* scale, void* stream) {
  try {
    const int r = check_sizes(B, H, N, d);
    if (r != SVG2_OK) return r;
    if (!valid_dtype(dtype) || X == nullptr || X8 == nullptr || scale == nullptr) return SVG2_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(X8, 16) || !aligned(scale, 4)) return SVG2_ERR_INVALID_ARG;
    const int BH = B * H;
    const bool f32 = dtype == SVG2_F32;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t* amax = reinterpret_cast<uint32_t*>(scale);  // the maxima live in `scale` until the last pass
    cudaError_t e = launch_amax(X, nullptr, nullptr, 1, f32, BH, N, d, amax, s);
    if (e == cudaSuccess) e = launch_gather_e4m3(X, nullptr, f32, perm, BH, N, d, amax, nullptr, X8, nullptr, s, nullptr);
    if (e == cudaSuccess) e = launch_amax_to_scale(amax, BH, s);
    return to_status(e);
  } catch (...) {
    return SVG2_ERR_CUDA;
  }
}

int svg2_sparse_attn_fp8(const void* Qp8, const void* Kp8, const void* Vp8, const float* scale_q, const float* scale_k,
                         const float* scale_v, const int32_t* q_off, const int32_t* k_off, const int32_t* sel_count,
                         const int32_t* sel_idx, int B, int H, int N, int d, int nQ, int nK, float scale,
                         const int32_t* perm_q, void* O, void* ws, size_t ws_bytes, void* stream) {
  try {
    int r = check_sizes(B, H, N, d);
    if (r == SVG2_OK) r = check_k(nQ, N);
    if (r == SVG2_OK) r = check_k(nK, N);
    if (r != SVG2_OK) return r;
    if (d != 128) return SVG2_ERR_UNSUPPORTED;
    if (Qp8 == nullptr || Kp8 == nullptr || Vp8 == nullptr || scale_q == nullptr || scale_k == nullptr ||
        scale_v == nullptr || q_off == nullptr || k_off == nullptr || sel_count == nullptr || sel_idx == nullptr ||
        O == nullptr)
      return SVG2_ERR_INVALID_ARG;
    if (!aligned(Qp8, 16) || !aligned(Kp8, 16) || !aligned(Vp8, 16) || !aligned(O, 16) || !aligned(scale_q, 4) ||
        !aligned(scale_k, 4) || !aligned(scale_v, 4))
      return SVG2_ERR_INVALID_ARG;
    if (scale != scale) return SVG2_ERR_INVALID_ARG;
    const int BH = B * H;
    Carve c(ws);
    DeviceStatus* st = c.take<DeviceStatus>(kStatusBytes / sizeof(DeviceStatus));
    AttnScratch a;
    carve_attn(c, BH, N, nQ, a);
    r = check_ws(ws, ws_bytes, c.off);
    if (r != SVG2_OK) return r;
    return to_status(launch_sparse_attn_fp8(Qp8, Kp8, Vp8, F8Scales{scale_q, scale_k, scale_v}, q_off, k_off,
                                            sel_count, sel_idx, BH, N, d, nQ, nK, scale, perm_q, O, a, st,
                                            wait_budget_of(st), static_cast<cudaStream_t>(stream)));
  } catch (...) {
    return SVG2_ERR_CUDA;
  }
}

namespace {
struct DenseCarve {
  DeviceStatus* st;
  int32_t *q_off, *k_off, *sel_count, *sel_idx;
  AttnScratch attn;
};
void carve_dense(Carve& c, int BH, int N, DenseCarve& D) {
  D.st = c.take<DeviceStatus>(kStatusBytes / sizeof(DeviceStatus));
  D.q_off = c.take<int32_t>(static_cast<size_t>(BH) * 2);
  D.k_off = c.take<int32_t>(static_cast<size_t>(BH) * 2);
  D.sel_count = c.take<int32_t>(BH);
  D.sel_idx = c.take<int32_t>(BH);
  carve_attn(c, BH, N, 1, D.attn);
}
}  // namespace

int svg2_dense_attn_workspace_size(int B, int H, int N, int d, size_t* bytes) {
  if (bytes == nullptr) return SVG2_ERR_INVALID_ARG;
  const int r = check_sizes(B, H, N, d);
  if (r != SVG2_OK) return r;
  Carve c(nullptr);
  DenseCarve D;
  carve_dense(c, B * H, N, D);
  *bytes = align_up(c.off, 256);
  return SVG2_OK;
}

int svg2_dense_attn(const void* Q, const void* K, const void* V, int B, int H, int N, int d, float scale, void* O,
                    void* ws, size_t ws_bytes, void* stream) {
  try {
    int r = check_sizes(B, H, N, d);
    if (r != SVG2_OK) return r;
    if (Q == nullptr || K == nullptr || V == nullptr || O == nullptr) return SVG2_ERR_INVALID_ARG;
    if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16)) return SVG2_ERR_INVALID_ARG;
    if (!(scale == scale) || scale == INFINITY || scale == -INFINITY) return SVG2_ERR_INVALID_ARG;
    const int BH = B * H;
    Carve c(ws);
    DenseCarve D;
    carve_dense(c, BH, N, D);
    r = check_ws(ws, ws_bytes, c.off);
    if (r != SVG2_OK) return r;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_dense_plan(BH, N, D.q_off, D.k_off, D.sel_count, D.sel_idx, s);
    if (e == cudaSuccess)
      e = launch_sparse_attn(Q, K, V, D.q_off, D.k_off, D.sel_count, D.sel_idx, BH, N, d, 1, 1, scale, nullptr, O,
                             D.attn, D.st, wait_budget_of(D.st), s);
    return to_status(e);
  } catch (...) {
    return SVG2_ERR_CUDA;
  }
}

int svg2_unpermute(const void* Op, const int32_t* perm, int B, int H, int N, int d, void* O, void* stream) {
  try {
    const int r = check_sizes(B, H, N, d);
    if (r != SVG2_OK) return r;
    if (Op == nullptr || perm == nullptr || O == nullptr) return SVG2_ERR_INVALID_ARG;
    if (!aligned(Op, 16) || !aligned(O, 16)) return SVG2_ERR_INVALID_ARG;
    return to_status(launch_unpermute(Op, perm, B * H, N, d, O, static_cast<cudaStream_t>(stream)));
  } catch (...) {
    return SVG2_ERR_CUDA;
  }
}

// Checks shared by svg2_layer and svg2_layer_host (everything but the tensor pointers).
static int check_layer_params(const svg2_params* p, int dtype, int B, int H, int N, int d, const double* uq,
                              const double* uk, const float* cq, const float* ck) {
  if (p == nullptr) return SVG2_ERR_INVALID_ARG;
  int r = check_sizes(B, H, N, d);
  if (r == SVG2_OK) r = check_k(p->nQ, N);
  if (r == SVG2_OK) r = check_k(p->nK, N);
  if (r != SVG2_OK) return r;
  if (!valid_dtype(dtype) || p->iters < 1 || (p->init != SVG2_INIT_GIVEN && p->init != SVG2_INIT_KMEANSPP))
    return SVG2_ERR_INVALID_ARG;
  if (p->seed_tokens < 0) return SVG2_ERR_INVALID_ARG;
  if (p->init == SVG2_INIT_KMEANSPP && kmeanspp_candidates(N, p->seed_tokens) < (p->nQ > p->nK ? p->nQ : p->nK))
    return SVG2_ERR_INVALID_ARG;  // fewer candidates than seeds
  if (!(p->top_p > 0.f) || p->scale != p->scale) return SVG2_ERR_INVALID_ARG;
  if (cq == nullptr || ck == nullptr) return SVG2_ERR_INVALID_ARG;
  if (p->init == SVG2_INIT_KMEANSPP && (uq == nullptr || uk == nullptr)) return SVG2_ERR_INVALID_ARG;
  if (p->attn_fp8 != 0 && p->attn_fp8 != 1) return SVG2_ERR_INVALID_ARG;
  if (p->attn_fp8 && d != 128) return SVG2_ERR_UNSUPPORTED;
  return SVG2_OK;
}

int svg2_layer(const void* Q, const void* K, const void* V, int dtype, int B, int H, int N, int d,
               const svg2_params* p, const double* uq, const double* uk, float* cq, float* ck, void* O,
               const svg2_layer_outputs* outs, void* ws, size_t ws_bytes, void* stream) {
  try {
    int r = check_layer_params(p, dtype, B, H, N, d, uq, uk, cq, ck);
    if (r != SVG2_OK) return r;
    if (Q == nullptr || K == nullptr || V == nullptr || O == nullptr) return SVG2_ERR_INVALID_ARG;
    if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16) || !aligned(cq, 16) ||
        !aligned(ck, 16))
      return SVG2_ERR_INVALID_ARG;
    const int BH = B * H;
    Carve c(ws);
    LayerCarve L;
    carve_layer(c, BH, N, d, p->nQ, p->nK, outs, L);
    r = check_ws(ws, ws_bytes, c.off);
    if (r != SVG2_OK) return r;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool f32 = dtype == SVG2_F32;
    // the permuted planes are free until the gathers: the k-means++ candidates are copied there
    void* cand = L.Qp;
    const size_t cand_bytes = candidate_room(L, BH, N, d);
    cudaError_t e = run_kmeans(Q, f32, BH, N, d, p->nQ, p->iters, p->init, uq, p->seed_tokens, cq, L.labels_q, L.count_q, L.perm_q,
                               L.q_off, L.kq, cand, cand_bytes, L.st, s);
    if (e == cudaSuccess)
      e = run_kmeans(K, f32, BH, N, d, p->nK, p->iters, p->init, uk, p->seed_tokens, ck, L.labels_k, L.count_k, L.perm_k, L.k_off,
                     L.kk, cand, cand_bytes, L.st, s);
    if (e == cudaSuccess)
      e = launch_select(cq, ck, nullptr, L.count_k, BH, p->nQ, p->nK, d, p->top_p, p->scale, L.weights, L.mask,
                        L.sel_count, L.sel_idx, L.stream_len, s);
    const F8Scales f8{reinterpret_cast<const float*>(L.f8), reinterpret_cast<const float*>(L.f8 + BH),
                      reinterpret_cast<const float*>(L.f8 + 2 * BH)};
    if (p->attn_fp8) {
      // E4M3 rows go to the first half of each permuted bf16 plane's room
      if (e == cudaSuccess) e = launch_amax(Q, K, V, 3, f32, BH, N, d, L.f8, s);
      if (e == cudaSuccess) e = launch_gather_e4m3(Q, nullptr, f32, L.perm_q, BH, N, d, L.f8, nullptr, L.Qp, nullptr, s, L.st);
      if (e == cudaSuccess)
        e = launch_gather_e4m3(K, V, f32, L.perm_k, BH, N, d, L.f8 + BH, L.f8 + 2 * BH, L.Kp, L.Vp, s, L.st);
      if (e == cudaSuccess) e = launch_amax_to_scale(L.f8, 3 * BH, s);
    } else {
      if (e == cudaSuccess) e = launch_gather(Q, f32, L.perm_q, BH, N, d, L.Qp, s, L.st);
      if (e == cudaSuccess) e = launch_gather2(K, V, f32, L.perm_k, BH, N, d, L.Kp, L.Vp, s, L.st);
    }
    if (e == cudaSuccess && p->attn_fp8) {
      e = launch_sparse_attn_fp8(L.Qp, L.Kp, L.Vp, f8, L.q_off, L.k_off, L.sel_count, L.sel_idx, BH, N, d, p->nQ,
                                 p->nK, p->scale, p->fuse_unpermute ? L.perm_q : nullptr, p->fuse_unpermute ? O : L.Op,
                                 L.attn, L.st, wait_budget_of(L.st), s);
      if (e == cudaSuccess && !p->fuse_unpermute) e = launch_unpermute(L.Op, L.perm_q, BH, N, d, O, s, L.st);
    } else if (e == cudaSuccess) {
      if (p->fuse_unpermute) {
        e = launch_sparse_attn(L.Qp, L.Kp, L.Vp, L.q_off, L.k_off, L.sel_count, L.sel_idx, BH, N, d, p->nQ, p->nK,
                               p->scale, L.perm_q, O, L.attn, L.st, wait_budget_of(L.st), s);
      } else {
        e = launch_sparse_attn(L.Qp, L.Kp, L.Vp, L.q_off, L.k_off, L.sel_count, L.sel_idx, BH, N, d, p->nQ, p->nK,
                               p->scale, nullptr, L.Op, L.attn, L.st, wait_budget_of(L.st), s);
        if (e == cudaSuccess) e = launch_unpermute(L.Op, L.perm_q, BH, N, d, O, s, L.st);
      }
    }
    return to_status(e);
  } catch (...) {
    return SVG2_ERR_CUDA;
  }
}

int svg2_layer_host(const void* Qh, const void* Kh, const void* Vh, void* Oh, void* Qd, void* Kd, void* Vd, void* Od,
                    int dtype, int B, int H, int N, int d, const svg2_params* p, const double* uq, const double* uk,
                    float* cq, float* ck, int heads_per_group, void* ws, size_t ws_bytes, void* stream,
                    void* copy_stream) {
  try {
    int r = check_layer_params(p, dtype, B, H, N, d, uq, uk, cq, ck);
    if (r != SVG2_OK) return r;
    if (Qh == nullptr || Kh == nullptr || Vh == nullptr || Oh == nullptr) return SVG2_ERR_INVALID_ARG;
    if (Qd == nullptr || Kd == nullptr || Vd == nullptr || Od == nullptr || heads_per_group < 0)
      return SVG2_ERR_INVALID_ARG;
    if (!aligned(Qd, 16) || !aligned(Kd, 16) || !aligned(Vd, 16) || !aligned(Od, 16) || !aligned(cq, 16) ||
        !aligned(ck, 16))
      return SVG2_ERR_INVALID_ARG;
    const int BH = B * H;
    Carve c(ws);
    LayerCarve L;
    carve_layer(c, BH, N, d, p->nQ, p->nK, nullptr, L);
    r = check_ws(ws, ws_bytes, c.off);
    if (r != SVG2_OK) return r;
    const int G = heads_per_group == 0 ? BH : (heads_per_group < BH ? heads_per_group : BH);
    // groups of G planes, except that the last G are split into halves, quarters, ... down to one
    // plane, so that the copy back that nothing overlaps (the last group's) is small
    std::vector<int> gsize;
    if (heads_per_group == 0) {
      gsize.push_back(BH);
    } else {
      int left = BH;
      while (left > G) {
        gsize.push_back(G);
        left -= G;
      }
      while (left > 1) {
        const int h = (left + 1) / 2;
        gsize.push_back(h);
        left -= h;
      }
      if (left == 1) gsize.push_back(1);
    }
    const int ngroups = static_cast<int>(gsize.size());
    const bool f32 = dtype == SVG2_F32;
    const size_t esz = f32 ? 4 : 2;
    const size_t bytes_in = static_cast<size_t>(BH) * N * d * esz;
    const size_t plane_out = static_cast<size_t>(N) * d * 2;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaStream_t cs = copy_stream != nullptr ? static_cast<cudaStream_t>(copy_stream) : s;

    // K is uploaded, and clustered, in two halves of the planes, so that the first half's k-means
    // starts while the second half is still in flight; V goes up per attention group, so that a
    // group's gathers and attention need only its own planes.
    const int nkc = BH >= 2 ? 2 : 1;
    const int kc_split = (BH + 1) / 2;
    // events: entry (copies wait for prior work on `stream`), Q landed, all copies done, each K
    // half landed, each group's V landed, each group's output ready
    std::vector<cudaEvent_t> ev(3 + nkc + 2 * ngroups, nullptr);
    cudaError_t e = cudaSuccess;
    for (auto& x : ev)
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming);
    auto release = [&]() {
      for (auto x : ev)
        if (x) cudaEventDestroy(x);  // deferred by the runtime until the recorded work completes
    };
    if (e != cudaSuccess) {
      release();
      return SVG2_ERR_CUDA;
    }
    cudaEvent_t entry = ev[0], q_in = ev[1], all_out = ev[2];
    cudaEvent_t* k_in = ev.data() + 3;
    cudaEvent_t* v_in = k_in + nkc;
    cudaEvent_t* o_out = v_in + ngroups;
    auto ok = [&](cudaError_t x) {
      if (e == cudaSuccess) e = x;
      return e == cudaSuccess;
    };
    const size_t plane_in = static_cast<size_t>(N) * d * esz;  // bytes of one input plane
    auto kc_range = [&](int c, int& h0c, int& hnc) {
      h0c = c == 0 ? 0 : kc_split;
      hnc = nkc == 1 ? BH : (c == 0 ? kc_split : BH - kc_split);
    };
    ok(cudaEventRecord(entry, s));
    ok(cudaStreamWaitEvent(cs, entry, 0));
    // inputs in the order the computation needs them: K first (its k-means, with more clusters than
    // Q's, is the longer of the two and hides the upload of Q), then Q, then V
    for (int c = 0; c < nkc; ++c) {
      int h0c, hnc;
      kc_range(c, h0c, hnc);
      ok(cudaMemcpyAsync(static_cast<char*>(Kd) + h0c * plane_in, static_cast<const char*>(Kh) + h0c * plane_in,
                         hnc * plane_in, cudaMemcpyHostToDevice, cs));
      ok(cudaEventRecord(k_in[c], cs));
    }
    ok(cudaMemcpyAsync(Qd, Qh, bytes_in, cudaMemcpyHostToDevice, cs));
    ok(cudaEventRecord(q_in, cs));
    {
      size_t h0 = 0;
      for (int g = 0; g < ngroups; h0 += static_cast<size_t>(gsize[g]), ++g) {
        ok(cudaMemcpyAsync(static_cast<char*>(Vd) + h0 * plane_in, static_cast<const char*>(Vh) + h0 * plane_in,
                           gsize[g] * plane_in, cudaMemcpyHostToDevice, cs));
        ok(cudaEventRecord(v_in[g], cs));
      }
    }
    // k-means of K, half by half (the planes are independent problems; the scratch serves the
    // halves in turn on the one stream)
    for (int c = 0; c < nkc && e == cudaSuccess; ++c) {
      int h0c, hnc;
      kc_range(c, h0c, hnc);
      ok(cudaStreamWaitEvent(s, k_in[c], 0));
      const size_t hb = static_cast<size_t>(h0c);
      if (e == cudaSuccess)
        e = run_kmeans(static_cast<const char*>(Kd) + hb * plane_in, f32, hnc, N, d, p->nK, p->iters, p->init,
                       uk != nullptr ? uk + hb * p->nK : nullptr, p->seed_tokens, ck + hb * p->nK * d,
                       L.labels_k + hb * N, L.count_k + hb * p->nK, L.perm_k + hb * N, L.k_off + hb * (p->nK + 1),
                       L.kk, L.Qp, candidate_room(L, BH, N, d), L.st, s);
    }
    ok(cudaStreamWaitEvent(s, q_in, 0));
    if (e == cudaSuccess)
      e = run_kmeans(Qd, f32, BH, N, d, p->nQ, p->iters, p->init, uq, p->seed_tokens, cq, L.labels_q, L.count_q,
                     L.perm_q, L.q_off, L.kq, L.Qp, candidate_room(L, BH, N, d), L.st, s);
    if (e == cudaSuccess)
      e = launch_select(cq, ck, nullptr, L.count_k, BH, p->nQ, p->nK, d, p->top_p, p->scale, nullptr, L.mask,
                        L.sel_count, L.sel_idx, L.stream_len, s);
    // FP8 attention: L.f8 holds Q's scales [BH], then per group its K scales and V scales [hn each]
    if (p->attn_fp8) {
      if (e == cudaSuccess) e = launch_amax(Qd, nullptr, nullptr, 1, f32, BH, N, d, L.f8, s);
      if (e == cudaSuccess) e = launch_gather_e4m3(Qd, nullptr, f32, L.perm_q, BH, N, d, L.f8, nullptr, L.Qp, nullptr, s, L.st);
      if (e == cudaSuccess) e = launch_amax_to_scale(L.f8, BH, s);
    } else if (e == cudaSuccess) {
      e = launch_gather(Qd, f32, L.perm_q, BH, N, d, L.Qp, s, L.st);
    }
    // per head group: gather its K and V planes once its V has landed, attend, and copy the output
    // back while the next group runs
    const size_t plane_p = static_cast<size_t>(N) * d;  // elements of one permuted plane
    size_t h0 = 0;
    for (int g = 0; g < ngroups && e == cudaSuccess; h0 += static_cast<size_t>(gsize[g]), ++g) {
      const int hn = gsize[g];
      ok(cudaStreamWaitEvent(s, v_in[g], 0));
      if (p->attn_fp8) {
        const char* kg = static_cast<const char*>(Kd) + h0 * plane_in;
        const char* vg = static_cast<const char*>(Vd) + h0 * plane_in;
        uint32_t* fk = L.f8 + BH + 2 * h0;  // this group's K scales, then its V scales
        if (e == cudaSuccess) e = launch_amax(kg, vg, nullptr, 2, f32, hn, N, d, fk, s);
        if (e == cudaSuccess)
          e = launch_gather_e4m3(kg, vg, f32, L.perm_k + h0 * N, hn, N, d, fk, fk + hn,
                                 static_cast<uint8_t*>(L.Kp) + h0 * plane_p, static_cast<uint8_t*>(L.Vp) + h0 * plane_p,
                                 s, L.st);
        if (e == cudaSuccess) e = launch_amax_to_scale(fk, 2 * hn, s);
        if (e != cudaSuccess) break;
        const F8Scales f8{reinterpret_cast<const float*>(L.f8) + h0, reinterpret_cast<const float*>(fk),
                          reinterpret_cast<const float*>(fk + hn)};
        e = launch_sparse_attn_fp8(static_cast<const uint8_t*>(L.Qp) + h0 * plane_p,
                                   static_cast<const uint8_t*>(L.Kp) + h0 * plane_p,
                                   static_cast<const uint8_t*>(L.Vp) + h0 * plane_p, f8, L.q_off + h0 * (p->nQ + 1),
                                   L.k_off + h0 * (p->nK + 1), L.sel_count + h0 * p->nQ,
                                   L.sel_idx + h0 * static_cast<size_t>(p->nQ) * p->nK, hn, N, d, p->nQ, p->nK,
                                   p->scale, L.perm_q + h0 * N, static_cast<char*>(Od) + h0 * plane_out, L.attn, L.st,
                                   wait_budget_of(L.st), s);
      } else {
        if (e == cudaSuccess)
          e = launch_gather2(static_cast<const char*>(Kd) + h0 * plane_in, static_cast<const char*>(Vd) + h0 * plane_in,
                             f32, L.perm_k + h0 * N, hn, N, d, static_cast<uint16_t*>(L.Kp) + h0 * plane_p,
                             static_cast<uint16_t*>(L.Vp) + h0 * plane_p, s, L.st);
        if (e != cudaSuccess) break;
        e = launch_sparse_attn(static_cast<const uint16_t*>(L.Qp) + h0 * plane_p,
                               static_cast<const uint16_t*>(L.Kp) + h0 * plane_p,
                               static_cast<const uint16_t*>(L.Vp) + h0 * plane_p, L.q_off + h0 * (p->nQ + 1),
                               L.k_off + h0 * (p->nK + 1), L.sel_count + h0 * p->nQ,
                               L.sel_idx + h0 * static_cast<size_t>(p->nQ) * p->nK, hn, N, d, p->nQ, p->nK, p->scale,
                               L.perm_q + h0 * N, static_cast<char*>(Od) + h0 * plane_out, L.attn, L.st,
                               wait_budget_of(L.st), s);
      }
      ok(cudaEventRecord(o_out[g], s));
      ok(cudaStreamWaitEvent(cs, o_out[g], 0));
      ok(cudaMemcpyAsync(static_cast<char*>(Oh) + h0 * plane_out, static_cast<const char*>(Od) + h0 * plane_out,
                         hn * plane_out, cudaMemcpyDeviceToHost, cs));
    }
    ok(cudaEventRecord(all_out, cs));
    ok(cudaStreamWaitEvent(s, all_out, 0));
    release();
    return to_status(e);
  } catch (...) {
    return SVG2_ERR_CUDA;
  }
}

int svg2_selftest_mma(const void* A, const void* Bm, int n, const void* V, float* C, float* O, void* ws,
                      size_t ws_bytes, void* stream) {
  try {
    if (A == nullptr || Bm == nullptr || V == nullptr || C == nullptr || O == nullptr) return SVG2_ERR_INVALID_ARG;
    if (n != 64 && n != 128 && n != 256) return SVG2_ERR_UNSUPPORTED;
    if (!aligned(A, 16) || !aligned(Bm, 16) || !aligned(V, 16)) return SVG2_ERR_INVALID_ARG;
    const int r = check_ws(ws, ws_bytes, kStatusBytes);
    if (r != SVG2_OK) return r;
    return to_status(launch_selftest_mma(A, Bm, n, V, C, O, static_cast<DeviceStatus*>(ws),
                                         static_cast<cudaStream_t>(stream)));
  } catch (...) {
    return SVG2_ERR_CUDA;
  }
}

}  // extern "C"
