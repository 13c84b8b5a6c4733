// Linformer-style projection of the HSA linear branch ("WorldAttention pairs
// hierarchical KV caching with hybrid sparse attention..." news summary, HSA
// paragraph: low-rank projection, O(L r) cost):
//     EK_h = E_h [Kc; Kq]_h,   FV_h = F_h [Vc; Vq]_h,   E_h, F_h in R^{r x L}.
// A GEMM with a long reduction dimension (L) and a small output (r x d per head),
// so the reduction is split across CTAs; partial sums are reduced in a fixed order
// and stored as bf16 hi/lo pairs for the split-precision attention that follows.
#include "common.cuh"
#include "kernels.h"

namespace hsa {

constexpr int kPM = 128;  // rows of E per CTA
constexpr int kPK = 64;   // reduction chunk
constexpr int kPStages = 3;
constexpr int kPThreads = 256;

struct ProjArgs {
  const uint16_t* E;
  const uint16_t* F;
  long long ef_stride;
  const uint16_t* Kc;
  const uint16_t* Kq;
  const uint16_t* Vc;
  const uint16_t* Vq;
  int H, r, Lq;
  long long Lc, L;
  long long k_per_split;
  int splits;
  float* part;  // [splits][2][H][r][D]
};

// grid: x = 128-row tile of r, y = head, z = split * 2 + which (0: E.K, 1: F.V)
template <int D>
__global__ void __launch_bounds__(kPThreads) proj_kernel(const ProjArgs a) {
  constexpr int WARPS_M = 2, WARPS_N = 4;
  constexpr int WM = kPM / WARPS_M;  // 64
  constexpr int WN = D / WARPS_N;    // 32 (D=128) or 16 (D=64)
  constexpr int MT = WM / 16;        // m16 tiles per warp
  constexpr int NT = WN / 8;         // n8 tiles per warp
  extern __shared__ __align__(128) unsigned char smem[];
  uint16_t* sA = reinterpret_cast<uint16_t*>(smem);      // [stages][128][64]
  uint16_t* sB = sA + kPStages * kPM * kPK;              // [stages][64][D]

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int wm = warp % WARPS_M, wn = warp / WARPS_M;
  const int m0 = blockIdx.x * kPM, h = blockIdx.y;
  const int which = blockIdx.z & 1, split = blockIdx.z >> 1;
  const uint16_t* A = (which ? a.F : a.E) + (long long)h * a.ef_stride;
  const uint16_t* Bc = which ? a.Vc : a.Kc;
  const uint16_t* Bq = which ? a.Vq : a.Kq;
  const long long k_begin = (long long)split * a.k_per_split;
  const long long k_end = min(a.L, k_begin + a.k_per_split);
  const int nchunks = k_begin < k_end ? (int)((k_end - k_begin + kPK - 1) / kPK) : 0;

  auto issue = [&](int ch, int st) {
    const long long k0 = k_begin + (long long)ch * kPK;
    uint16_t* dA = sA + st * kPM * kPK;
    uint16_t* dB = sB + st * kPK * D;
    // A: 128 rows x 8 chunks
    for (int x = tid; x < kPM * (kPK / 8); x += kPThreads) {
      const int rr = x / (kPK / 8), c = x % (kPK / 8);
      const long long k = k0 + c * 8;
      const bool ok = (m0 + rr) < a.r && k < k_end;
      const uint16_t* g = A + (ok ? ((long long)(m0 + rr) * a.L + k) : 0);
      cp_async16(smem_u32(dA + rr * kPK + swz(rr, c) * 8), g, ok ? 16 : 0);
    }
    // B: 64 rows (reduction index) x D/8 chunks; row k is Kc[k] (k < Lc) or Kq[k - Lc]
    for (int x = tid; x < kPK * (D / 8); x += kPThreads) {
      const int rr = x / (D / 8), c = x % (D / 8);
      const long long k = k0 + rr;
      const bool ok = k < k_end;
      const uint16_t* g = Bq;  // any valid address when zero-filling (Bc is NULL without history)
      if (ok) g = k < a.Lc ? Bc + ((k * a.H + h) * D + c * 8) : Bq + (((k - a.Lc) * a.H + h) * D + c * 8);
      cp_async16(smem_u32(dB + rr * D + swz(rr, c) * 8), g, ok ? 16 : 0);
    }
  };

  float acc[MT][NT][4];
#pragma unroll
  for (int i = 0; i < MT; ++i)
#pragma unroll
    for (int j = 0; j < NT; ++j) acc[i][j][0] = acc[i][j][1] = acc[i][j][2] = acc[i][j][3] = 0.f;

#pragma unroll
  for (int st = 0; st < kPStages - 1; ++st) {
    if (st < nchunks) issue(st, st);
    cp_async_commit();
  }
  for (int ch = 0; ch < nchunks; ++ch) {
    cp_async_wait<kPStages - 2>();
    __syncthreads();
    const int nxt = ch + kPStages - 1;
    if (nxt < nchunks) issue(nxt, nxt % kPStages);
    cp_async_commit();
    const uint16_t* tA = sA + (ch % kPStages) * kPM * kPK;
    const uint16_t* tB = sB + (ch % kPStages) * kPK * D;
#pragma unroll
    for (int kk = 0; kk < kPK / 16; ++kk) {
      uint32_t af[MT][4];
#pragma unroll
      for (int i = 0; i < MT; ++i) {
        const int row = wm * WM + i * 16 + (lane % 16);
        const int chunk = 2 * kk + lane / 16;
        ldsm_x4(smem_u32(tA + row * kPK + swz(row, chunk) * 8), af[i][0], af[i][1], af[i][2], af[i][3]);
      }
#pragma unroll
      for (int jp = 0; jp < NT / 2; ++jp) {
        const int mi = lane / 8;
        const int krow = kk * 16 + (lane % 8) + 8 * (mi % 2);
        const int chunk = (wn * WN) / 8 + 2 * jp + (mi / 2);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_u32(tB + krow * D + swz(krow, chunk) * 8), b0, b1, b2, b3);
#pragma unroll
        for (int i = 0; i < MT; ++i) {
          mma_bf16(acc[i][2 * jp], af[i], b0, b1);
          mma_bf16(acc[i][2 * jp + 1], af[i], b2, b3);
        }
      }
    }
  }
  cp_async_wait<0>();

  float* out = a.part + ((((long long)split * 2 + which) * a.H + h) * a.r) * D;
#pragma unroll
  for (int i = 0; i < MT; ++i) {
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int row = m0 + wm * WM + i * 16 + lane / 4;
      const int col = wn * WN + j * 8 + 2 * (lane % 4);
      if (row < a.r) *reinterpret_cast<float2*>(out + (long long)row * D + col) = make_float2(acc[i][j][0], acc[i][j][1]);
      if (row + 8 < a.r)
        *reinterpret_cast<float2*>(out + (long long)(row + 8) * D + col) = make_float2(acc[i][j][2], acc[i][j][3]);
    }
  }
}

int proj_splits(int H, int r, long long L) {
  const int base = ((r + kPM - 1) / kPM) * H * 2;
  long long want = (4LL * 148 + base - 1) / base;        // about four CTAs per SM
  long long maxs = (L + 4 * kPK - 1) / (4 * kPK);         // at least 4 chunks per split
  if (want > maxs) want = maxs;
  if (want < 1) want = 1;
  return (int)want;
}

cudaError_t launch_proj(const uint16_t* E, const uint16_t* F, long long ef_head_stride, const uint16_t* Kc,
                        const uint16_t* Kq, const uint16_t* Vc, const uint16_t* Vq, int H, int d, int r,
                        long long Lc, int Lq, int splits, float* part, cudaStream_t s) {
  ProjArgs a;
  a.E = E; a.F = F; a.ef_stride = ef_head_stride;
  a.Kc = Kc; a.Kq = Kq; a.Vc = Vc; a.Vq = Vq;
  a.H = H; a.r = r; a.Lq = Lq; a.Lc = Lc; a.L = Lc + Lq;
  const long long chunks = (a.L + kPK - 1) / kPK;
  a.k_per_split = ((chunks + splits - 1) / splits) * kPK;
  a.splits = splits;
  a.part = part;
  dim3 grid((r + kPM - 1) / kPM, H, splits * 2);
  const size_t smem = (size_t)kPStages * (kPM * kPK + kPK * d) * 2;
  cudaError_t e;
  if (d == 128) {
    e = cudaFuncSetAttribute(proj_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    proj_kernel<128><<<grid, kPThreads, smem, s>>>(a);
  } else {
    e = cudaFuncSetAttribute(proj_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    proj_kernel<64><<<grid, kPThreads, smem, s>>>(a);
  }
  return cudaGetLastError();
}

// Sum the split partials (fixed order) and store hi = bf16(v), lo = bf16(v - hi).
__global__ void proj_reduce_kernel(const float* __restrict__ part, int splits, long long per_which,
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

cudaError_t launch_proj_reduce(const float* part, int splits, int H, int d, int r, uint16_t* EKhi,
                               uint16_t* EKlo, uint16_t* FVhi, uint16_t* FVlo, cudaStream_t s) {
  const long long per_which = (long long)H * r * d;
  const long long n4 = 2 * per_which / 4;
  proj_reduce_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, s>>>(part, splits, per_which, EKhi, EKlo, FVhi, FVlo);
  return cudaGetLastError();
}

}  // namespace hsa
