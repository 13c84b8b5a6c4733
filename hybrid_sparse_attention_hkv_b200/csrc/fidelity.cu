// Fidelity of the two HSA branches against dense attention ("WorldAttention pairs
// hierarchical KV caching with hybrid sparse attention..." news summary, HSA
// paragraph and Figure 6: how much of full attention's global mass and output the
// linear branch keeps), as a diagnostic on any inputs:
//   cos_x   = <o_x, o_ref> / (|o_x| |o_ref|)           per head, over rows and columns
//   rel_x   = |o_x - o_ref| / |o_ref|
//   mass_sp = mean over rows of exp(lse_sp - lse_ref)  the dense softmax mass of the
//             keys the sparse branch kept (lse: ln sum_k exp(q.k scale) over the
//             keys a branch attends to)
// Pass 1: per (head, row split) fp64 partial sums; pass 2: per head, the splits in
// order.  Deterministic.
#include "common.cuh"
#include "kernels.h"

namespace hsa {
namespace {

constexpr int kFidThreads = 256;
constexpr int kParts = 8;  // dot_l, |l|^2, |ref|^2, dot_s, |s|^2, mass, |l-ref|^2, |s-ref|^2

__device__ double block_sum(double v, double* red) {
  v = warp_sum(v);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x == 0)
    for (int w = 0; w < kFidThreads / 32; ++w) t += red[w];
  return t;  // valid in thread 0
}

__global__ void __launch_bounds__(kFidThreads) fidelity_partial_kernel(const float* __restrict__ o_ref,
                                                                       const float* __restrict__ lse_ref,
                                                                       const float* __restrict__ o_sp,
                                                                       const float* __restrict__ lse_sp,
                                                                       const float* __restrict__ o_lin, int Lq, int H,
                                                                       int d, double* __restrict__ part) {
  __shared__ double red[kFidThreads / 32];
  const int h = blockIdx.x, split = blockIdx.y;
  const int rows_per = (Lq + kFidelitySplits - 1) / kFidelitySplits;
  const int r0 = split * rows_per, r1 = min(Lq, r0 + rows_per);
  double acc[kParts] = {0, 0, 0, 0, 0, 0, 0, 0};
  const long long n = (long long)max(0, r1 - r0) * d;
  for (long long i = threadIdx.x; i < n; i += kFidThreads) {
    const long long t = r0 + i / d, c = i % d;
    const long long idx = (t * H + h) * d + c;
    const double r = o_ref[idx], s = o_sp[idx], l = o_lin[idx];
    acc[0] += l * r;
    acc[1] += l * l;
    acc[2] += r * r;
    acc[3] += s * r;
    acc[4] += s * s;
    acc[6] += (l - r) * (l - r);
    acc[7] += (s - r) * (s - r);
  }
  for (int t = r0 + threadIdx.x; t < r1; t += kFidThreads) acc[5] += exp((double)lse_sp[(long long)t * H + h] -
                                                                        (double)lse_ref[(long long)t * H + h]);
  for (int k = 0; k < kParts; ++k) {
    const double v = block_sum(acc[k], red);
    if (threadIdx.x == 0) part[((long long)h * kFidelitySplits + split) * kParts + k] = v;
  }
}

__global__ void fidelity_final_kernel(const double* __restrict__ part, int Lq, int H, double* __restrict__ report) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= H) return;
  double s[kParts] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int q = 0; q < kFidelitySplits; ++q)
    for (int k = 0; k < kParts; ++k) s[k] += part[((long long)h * kFidelitySplits + q) * kParts + k];
  double* out = report + (long long)h * 5;
  out[0] = s[0] / sqrt(s[1] * s[2]);
  out[1] = s[3] / sqrt(s[4] * s[2]);
  out[2] = s[5] / Lq;
  out[3] = sqrt(s[6] / s[2]);
  out[4] = sqrt(s[7] / s[2]);
}

}  // namespace

cudaError_t launch_fidelity(const float* o_ref, const float* lse_ref, const float* o_sp, const float* lse_sp,
                            const float* o_lin, int Lq, int H, int d, double* part, double* report, cudaStream_t s) {
  fidelity_partial_kernel<<<dim3(H, kFidelitySplits), kFidThreads, 0, s>>>(o_ref, lse_ref, o_sp, lse_sp, o_lin, Lq,
                                                                           H, d, part);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  fidelity_final_kernel<<<(H + 127) / 128, 128, 0, s>>>(part, Lq, H, report);
  return cudaGetLastError();
}

}  // namespace hsa
