// hkv_select_pages_noalloc: page-level retrieval for callers that cannot allocate
// device memory.
//
// Some callers may not call cudaMalloc (or any allocator) at all: a host framework
// that owns every byte of device memory and hands plugins only the tensors of the
// call, a runtime whose memory plan is fixed before it starts serving, or a latency-
// critical loop where an allocation could stall the device.  They cannot supply the
// workspace hkv_select_pages needs for its partial page scores.  This variant keeps
// that scratch in a file-scope device array instead (2.3 MiB, enough for 2048
// pages), which every GPU that loads the library holds until the process exits.
//
// The array is shared by every call on a device and keeps the previous call's
// contents.  What must start at zero (the status word) is cleared on the stream at
// the start of each call; the partial sums are fully overwritten.  Calls whose
// kernels overlap on the GPU (different streams without ordering) race on the
// array and must not be issued.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

// Largest page count the static scratch serves.  Pass 1 of the page scoring writes
// one partial score per page for each of its row splits (at most kColMaxSplits).
constexpr int kNoAllocMaxPages = 2048;
// 256-byte status header + the partial scores: 256 + 296 * 2048 * 4 bytes (2.3 MiB).
constexpr size_t kNoAllocScratchBytes = 256 + size_t(hsa::kColMaxSplits) * kNoAllocMaxPages * sizeof(float);
static __device__ __align__(256) unsigned char g_select_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
struct ScratchAddr {
  CUcontext ctx = nullptr;  // context the address was looked up in
  void* ptr = nullptr;
};
ScratchAddr g_scratch[kMaxDevices];

PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
std::once_flag g_ctx_once;

// Device address of g_select_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// cudaGetSymbolAddress (with that device current) and cached together with the
// context it belongs to; a new primary context (after cudaDeviceReset, say) loads
// the array at another address, and the lookup is then made again.
hsa_status_t scratch_address(void** out) {
  const char* fn = "hkv_select_pages_noalloc";
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return hsa::api_fail(HSA_ERR_CUDA, "%s: cudaGetDevice: %s", fn, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return hsa::api_fail(HSA_ERR_UNSUPPORTED, "%s: device %d beyond %d", fn, dev, kMaxDevices);
  std::call_once(g_ctx_once, [] {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
  });
  if (!g_ctx_current) return hsa::api_fail(HSA_ERR_CUDA, "%s: cuCtxGetCurrent is unavailable", fn);
  CUcontext ctx = nullptr;  // NULL until the runtime has set up this device's context
  if (g_ctx_current(&ctx) != CUDA_SUCCESS) return hsa::api_fail(HSA_ERR_CUDA, "%s: cuCtxGetCurrent failed", fn);
  std::lock_guard<std::mutex> lock(g_mu);
  ScratchAddr& sa = g_scratch[dev];
  if (sa.ptr == nullptr || ctx == nullptr || sa.ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_select_scratch);  // sets up the context if needed
    if (e != cudaSuccess || p == nullptr)
      return hsa::api_fail(HSA_ERR_CUDA, "%s: cudaGetSymbolAddress: %s", fn, cudaGetErrorString(e));
    if (g_ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr)
      return hsa::api_fail(HSA_ERR_CUDA, "%s: no current CUDA context", fn);
    sa.ptr = p;
    sa.ctx = ctx;
  }
  *out = sa.ptr;
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
  // pass 1 writes page_score_splits(Lq) partial scores per page
  const size_t need = 256 + (size_t)hsa::page_score_splits(Lq) * NP * sizeof(float);
  if (NP > kNoAllocMaxPages || need > kNoAllocScratchBytes)
    return hsa::api_fail(HSA_ERR_UNSUPPORTED,
                         "%s: NP = %d pages need %zu scratch bytes; the static maximum is %d pages (%zu bytes)", fn,
                         NP, need, kNoAllocMaxPages, kNoAllocScratchBytes);
  if (NP > H * d) return hsa::api_fail(HSA_ERR_UNSUPPORTED, "%s: NP = %d pages exceed H*d = %d", fn, NP, H * d);
  const void* ptrs[] = {kbar_pages, Q};
  for (const void* p : ptrs)
    if (!p || (reinterpret_cast<uintptr_t>(p) & 15u))
      return hsa::api_fail(HSA_ERR_INVALID_ARG, "%s: kbar_pages and Q must be non-NULL and 16-byte aligned", fn);
  if (!sel_out) return hsa::api_fail(HSA_ERR_INVALID_ARG, "%s: sel_out is NULL", fn);

  if (hsa::injected_fault() == HSA_FAULT_LAUNCH) return hsa::api_fail(HSA_ERR_CUDA, "%s: injected launch failure", fn);
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
