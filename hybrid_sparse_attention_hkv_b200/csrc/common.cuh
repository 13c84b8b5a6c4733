// Device helpers shared by the HKV / HSA kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/hsa.h"

namespace hsa {

constexpr int kBlockInter = 128;
constexpr int kBlockIntra = 64;

// ------------------------------------------------------------------ status word
// The first 256 bytes of every workspace are its header:
//   int32 [0]  device status (an hsa_status_t); kernels record only the first failure
//   int32 [1]  nonzero once a bounded wait has run out: every other wait of the same
//              workspace then gives up at its next poll instead of running out on its
//              own, so a protocol that stalls ends in one wait limit, not one per wait
//   uint32[2]  kWaitTag when word 3 holds a limit set by hsa_set_wait_limit
//   uint32[3]  limit of every bounded device wait, in microseconds
//   int32 [4]  site of the first wait that ran out (0: none, or a wait without a site)
//   int32 [5]  CTA index of that wait
constexpr uint32_t kWaitTag = 0x54494157u;  // "WAIT"
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;

__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Wait limit of a kernel whose `status` points at a workspace header: the host-set
// limit when the tag is present, else 2 s.
__device__ __forceinline__ uint64_t wait_limit_ns(const int* status) {
  if (status != nullptr) {
    const uint32_t* w = reinterpret_cast<const uint32_t*>(status);
    if (w[2] == kWaitTag && w[3] != 0u) return (uint64_t)w[3] * 1000ull;
  }
  return kDefaultWaitLimitNs;
}

// ------------------------------------------------------------------ bf16
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Round x to bf16 (hi) and the remainder x - hi to bf16 (lo): x ~= hi + lo with
// about 16 significant bits.
__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

__device__ __forceinline__ void add8(float* acc, uint4 v) {
  acc[0] += bf16_lo(v.x); acc[1] += bf16_hi(v.x);
  acc[2] += bf16_lo(v.y); acc[3] += bf16_hi(v.y);
  acc[4] += bf16_lo(v.z); acc[5] += bf16_hi(v.z);
  acc[6] += bf16_lo(v.w); acc[7] += bf16_hi(v.w);
}

// ------------------------------------------------------------------ memory
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace hsa
