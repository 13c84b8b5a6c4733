// hkv_select_pages_noalloc: page-level retrieval for callers that cannot allocate
// device memory.
//
// Some callers may not call cudaMalloc (or any allocator) at all: a host framework
// that owns every byte of device memory and hands plugins only the tensors of the
// call, a runtime whose memory plan is fixed before it starts serving, or a latency-
// critical loop where an allocation could stall the device.  They cannot supply the
// workspace hkv_select_pages needs for its column-sum partials.  This variant keeps
// that scratch in a file-scope device array instead, sized once when the library
// is loaded (every GPU that loads the library holds it until the process exits).
//
// The array is shared by every call on a device and keeps the previous call's
// contents.  What must start at zero (the status word) is cleared on the stream at
// the start of each call; the partial sums are fully overwritten.  Calls whose
// kernels overlap on the GPU (different streams without ordering) race on the
// array and must not be issued.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

// 256-byte status header + column-sum partials (kColMaxSplits x H x d floats).
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB: H * d <= 7084
static __device__ __align__(256) unsigned char g_select_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_select_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// cudaGetSymbolAddress once per device (with that device current) and cached.
hsa_status_t scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return hsa::api_fail(HSA_ERR_CUDA, "hkv_select_pages_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return hsa::api_fail(HSA_ERR_UNSUPPORTED, "hkv_select_pages_noalloc: device %d beyond %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_select_scratch);
    if (e != cudaSuccess || p == nullptr)
      return hsa::api_fail(HSA_ERR_CUDA, "hkv_select_pages_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return HSA_OK;
}

}  // namespace

extern "C" hsa_status_t hkv_select_pages_noalloc(const float* kbar_pages, int NP, const int32_t* cand_range,
                                                 const hsa_bf16* Q, int Lq, int H, int d, int Kp, int32_t* sel_out,
                                                 float* scores_out, int32_t* status_out, hsa_stream_t stream) {
  const char* fn = "hkv_select_pages_noalloc";
  if (H < 1 || d <= 0) return hsa::api_fail(HSA_ERR_INVALID_ARG, "%s: H = %d, d = %d must be >= 1", fn, H, d);
  if (d != 64 && d != 128) return hsa::api_fail(HSA_ERR_UNSUPPORTED, "%s: d = %d (supported: 64, 128)", fn, d);
  if (NP < 1 || Lq < 1) return hsa::api_fail(HSA_ERR_INVALID_ARG, "%s: NP = %d, Lq = %d must be >= 1", fn, NP, Lq);
  if (Kp < 1 || Kp > NP || Kp > 64)
    return hsa::api_fail(HSA_ERR_INVALID_ARG, "%s: Kp = %d must be in [1, min(NP, 64)]", fn, Kp);
  if ((size_t)H * d * 8 + (size_t)NP * 8 > 200 * 1024)
    return hsa::api_fail(HSA_ERR_UNSUPPORTED, "%s: H*d*8 + NP*8 bytes exceed the shared-memory budget", fn);
  if (NP > H * d) return hsa::api_fail(HSA_ERR_UNSUPPORTED, "%s: NP = %d pages exceed H*d = %d", fn, NP, H * d);
  const size_t need = 256 + (size_t)hsa::kColMaxSplits * H * d * sizeof(float);
  if (need > kNoAllocScratchBytes)
    return hsa::api_fail(HSA_ERR_UNSUPPORTED, "%s: H*d = %d needs %zu scratch bytes, the static maximum is %zu", fn,
                         H * d, need, kNoAllocScratchBytes);
  const void* ptrs[] = {kbar_pages, Q};
  for (const void* p : ptrs)
    if (!p || (reinterpret_cast<uintptr_t>(p) & 15u))
      return hsa::api_fail(HSA_ERR_INVALID_ARG, "%s: kbar_pages and Q must be non-NULL and 16-byte aligned", fn);
  if (!sel_out) return hsa::api_fail(HSA_ERR_INVALID_ARG, "%s: sel_out is NULL", fn);

  void* base = nullptr;
  hsa_status_t st = scratch_address(&base);
  if (st != HSA_OK) return st;
  int* status = status_out ? reinterpret_cast<int*>(status_out) : static_cast<int*>(base);
  float* part = reinterpret_cast<float*>(static_cast<char*>(base) + 256);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), stream);
  if (e == cudaSuccess) e = hsa::launch_page_scores_partial(Q, Lq, H * d, kbar_pages, NP, cand_range, part, stream);
  if (e == cudaSuccess)
    e = hsa::launch_select_pages_final(part, Lq, NP, cand_range, Kp, sel_out, scores_out, status, stream);
  if (e != cudaSuccess) return hsa::api_fail(HSA_ERR_CUDA, "%s: %s", fn, cudaGetErrorString(e));
  return HSA_OK;
}
