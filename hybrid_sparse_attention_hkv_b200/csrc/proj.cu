// Linformer-style projection of the HSA linear branch ("WorldAttention pairs
// hierarchical KV caching with hybrid sparse attention..." news summary, HSA
// paragraph: low-rank projection, O(L r) cost):
//     EK_h = E_h [Kc; Kq]_h,   FV_h = F_h [Vc; Vq]_h,   E_h, F_h in R^{r x L}.
// The tensor-core pass (proj_tc.cu) splits the long reduction dimension L across
// CTAs; this file adds the split partial sums in a fixed order and stores them as
// bf16 hi/lo pairs for the split-precision attention that follows.
#include "common.cuh"
#include "kernels.h"

namespace hsa {

// Sum the split partials (fixed order), add `add` when given, and store either the
// fp32 sums (sum_out) or hi = bf16(v), lo = bf16(v - hi).
__global__ void proj_reduce_kernel(const float* __restrict__ part, int splits, long long per_which,
                                   const float* __restrict__ add, float* __restrict__ sum_out,
                                   uint16_t* __restrict__ EKhi, uint16_t* __restrict__ EKlo,
                                   uint16_t* __restrict__ FVhi, uint16_t* __restrict__ FVlo) {
  const long long i4 = (long long)blockIdx.x * blockDim.x + threadIdx.x;  // float4 index over 2 * per_which
  if (i4 * 4 >= 2 * per_which) return;
  const long long e = i4 * 4;
  const int which = e >= per_which;
  const long long off = e - which * per_which;
  float4 acc = make_float4(0, 0, 0, 0);
  for (int s = 0; s < splits; ++s) {
    const float4 v = *reinterpret_cast<const float4*>(part + ((long long)s * 2 + which) * per_which + off);
    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
  }
  if (add) {
    const float4 v = *reinterpret_cast<const float4*>(add + e);
    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
  }
  if (sum_out) {
    *reinterpret_cast<float4*>(sum_out + e) = acc;
    return;
  }
  __nv_bfloat16 h[4], l[4];
  split_bf16(acc.x, h[0], l[0]);
  split_bf16(acc.y, h[1], l[1]);
  split_bf16(acc.z, h[2], l[2]);
  split_bf16(acc.w, h[3], l[3]);
  uint16_t* hi = which ? FVhi : EKhi;
  uint16_t* lo = which ? FVlo : EKlo;
  uint2 hv, lv;
  hv.x = (uint32_t)__bfloat16_as_ushort(h[0]) | ((uint32_t)__bfloat16_as_ushort(h[1]) << 16);
  hv.y = (uint32_t)__bfloat16_as_ushort(h[2]) | ((uint32_t)__bfloat16_as_ushort(h[3]) << 16);
  lv.x = (uint32_t)__bfloat16_as_ushort(l[0]) | ((uint32_t)__bfloat16_as_ushort(l[1]) << 16);
  lv.y = (uint32_t)__bfloat16_as_ushort(l[2]) | ((uint32_t)__bfloat16_as_ushort(l[3]) << 16);
  *reinterpret_cast<uint2*>(hi + off) = hv;
  *reinterpret_cast<uint2*>(lo + off) = lv;
}

cudaError_t launch_proj_reduce(const float* part, int splits, int H, int d, int r, const float* add,
                               float* sum_out, uint16_t* EKhi, uint16_t* EKlo, uint16_t* FVhi, uint16_t* FVlo,
                               cudaStream_t s) {
  const long long per_which = (long long)H * r * d;
  const long long n4 = 2 * per_which / 4;
  proj_reduce_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, s>>>(part, splits, per_which, add, sum_out, EKhi, EKlo,
                                                                  FVhi, FVlo);
  return cudaGetLastError();
}

}  // namespace hsa
