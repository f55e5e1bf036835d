// svg2_sparse_attn_noalloc: the sparse-attention entry point for callers that cannot allocate
// device memory (no cudaMalloc, no caching allocator), for example code that runs where a
// workspace cannot be obtained at call time.  Its scratch — the status word and the attention
// work plan — lives in one file-scope __device__ array of fixed size instead of a caller
// workspace.  The caller still passes every input and output buffer.
#include <cuda_runtime.h>

#include <atomic>

#include "svg2.h"
#include "svg2_internal.h"

namespace svg2 {
namespace {

// Held by every GPU that loads this library, until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];

// Device address of the array for the current device (host code only sees a stand-in for the
// symbol, so the address is looked up with cudaGetSymbolAddress once per device).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SVG2_ERR_CUDA;
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return SVG2_ERR_CUDA;
    g_scratch_addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return SVG2_OK;
}

}  // namespace
}  // namespace svg2

using namespace svg2;

extern "C" SVG2_API int svg2_sparse_attn_noalloc(const void* Qp, const void* Kp, const void* Vp, const int32_t* q_off,
                                                 const int32_t* k_off, const int32_t* sel_count,
                                                 const int32_t* sel_idx, int B, int H, int N, int d, int nQ,
                                                 int nK, float scale, const int32_t* perm_q, void* O,
                                                 uint32_t* device_status, void* stream) {
  try {
    if (B < 1 || H < 1 || N < 1 || nQ < 1 || nK < 1 || nQ > N || nK > N) return SVG2_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SVG2_ERR_UNSUPPORTED;
    if (nQ > SVG2_MAX_CLUSTERS || nK > SVG2_MAX_CLUSTERS || N > SVG2_MAX_TOKENS) return SVG2_ERR_UNSUPPORTED;
    if (Qp == nullptr || Kp == nullptr || Vp == nullptr || q_off == nullptr || k_off == nullptr ||
        sel_count == nullptr || sel_idx == nullptr || O == nullptr)
      return SVG2_ERR_INVALID_ARG;
    const uintptr_t mis = reinterpret_cast<uintptr_t>(Qp) | reinterpret_cast<uintptr_t>(Kp) |
                          reinterpret_cast<uintptr_t>(Vp) | reinterpret_cast<uintptr_t>(O);
    if ((mis & 15u) != 0 || scale != scale) return SVG2_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(device_status) & 15u) != 0) return SVG2_ERR_INVALID_ARG;
    const long long BH = static_cast<long long>(B) * H;
    if (BH > 65535 || BH * N >= (1LL << 31)) return SVG2_ERR_UNSUPPORTED;
    // the same layout the workspace path uses: status word, then the work plan
    Carve measure(nullptr);
    measure.take<DeviceStatus>(kStatusBytes / sizeof(DeviceStatus));
    AttnScratch unused;
    carve_attn(measure, static_cast<int>(BH), N, nQ, unused);
    if (measure.off > kNoAllocScratchBytes) return SVG2_ERR_UNSUPPORTED;  // sizes beyond the fixed array
    void* base = nullptr;
    int r = scratch_address(&base);
    if (r != SVG2_OK) return r;
    Carve c(base);
    DeviceStatus* st = c.take<DeviceStatus>(kStatusBytes / sizeof(DeviceStatus));
    AttnScratch a;
    carve_attn(c, static_cast<int>(BH), N, nQ, a);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (device_status != nullptr) {
      st = reinterpret_cast<DeviceStatus*>(device_status);  // the caller's word (starts at zero)
    } else if (cudaMemsetAsync(st, 0, sizeof(DeviceStatus), s) != cudaSuccess) {
      return SVG2_ERR_CUDA;  // the library's own word is cleared so an old error cannot stop this call
    }
    const cudaError_t e = launch_sparse_attn(Qp, Kp, Vp, q_off, k_off, sel_count, sel_idx, static_cast<int>(BH), N,
                                             d, nQ, nK, scale, perm_q, O, a, st, nullptr, s);
    return e == cudaSuccess ? SVG2_OK : SVG2_ERR_CUDA;
  } catch (...) {
    return SVG2_ERR_CUDA;
  }
}
