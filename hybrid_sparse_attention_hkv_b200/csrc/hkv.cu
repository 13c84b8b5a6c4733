// HKV kernels: page summaries, prompt-level and page-level retrieval, and the
// active-cache gather ("WorldAttention pairs hierarchical KV caching with hybrid
// sparse attention..." news summary, HKV and kernel paragraphs).
//
// All of these are HBM (or host-link) bound: they stream bf16 rows once with
// 16-byte vector loads, one thread per 16-byte column chunk, and reduce in fp32
// in a fixed order (deterministic results).
#include <float.h>

#include "common.cuh"
#include "kernels.h"

namespace hsa {

// ------------------------------------------------------------------ column sums
// part[s][c] = sum over the rows of split s of X[row][c]; X: [n, C] bf16, C % 8 == 0.
// A CTA owns a contiguous row range; thread t reads 16-byte column vector (t % CV)
// of rows r0 + (t / CV), r0 + (t / CV) + RP, ...  (RP = 256 / CV row phases).
__global__ void __launch_bounds__(256) colsum_partial_kernel(const uint16_t* __restrict__ X, long long n, int C,
                                                             long long rows_per_split, float* __restrict__ part) {
  __shared__ float red[2048];
  const int CV = C / 8;
  const long long r0 = (long long)blockIdx.x * rows_per_split;
  const long long r1 = min(n, r0 + rows_per_split);
  float* out = part + (long long)blockIdx.x * C;
  if (CV <= 256) {
    const int RP = 256 / CV;
    const int v = threadIdx.x % CV, rp = threadIdx.x / CV;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (rp < RP) {
#pragma unroll 4
      for (long long r = r0 + rp; r < r1; r += RP) add8(acc, ld_nc_v4(X + r * C + v * 8));
#pragma unroll
      for (int k = 0; k < 8; ++k) red[rp * C + v * 8 + k] = acc[k];
    }
    __syncthreads();
    for (int c = threadIdx.x; c < C; c += 256) {
      float s = 0.f;
      for (int q = 0; q < RP; ++q) s += red[q * C + c];
      out[c] = s;
    }
  } else {
    for (int v = threadIdx.x; v < CV; v += 256) {
      float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll 4
      for (long long r = r0; r < r1; ++r) add8(acc, ld_nc_v4(X + r * C + v * 8));
#pragma unroll
      for (int k = 0; k < 8; ++k) out[v * 8 + k] = acc[k];
    }
  }
}

int colsum_splits(long long n) {
  long long s = (n + 15) / 16;
  return (int)(s < 1 ? 1 : (s > kColMaxSplits ? kColMaxSplits : s));
}

cudaError_t launch_colsum_partial(const uint16_t* X, long long n, int C, float* part, cudaStream_t s) {
  int splits = colsum_splits(n);
  long long rps = (n + splits - 1) / splits;
  colsum_partial_kernel<<<splits, 256, 0, s>>>(X, n, C, rps, part);
  return cudaGetLastError();
}

// kbar[c] = (sum_s part[s][c]) / n
__global__ void page_summary_final_kernel(const float* __restrict__ part, int splits, long long n, int C,
                                          float* __restrict__ kbar) {
  int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= C) return;
  float s = 0.f;
  for (int q = 0; q < splits; ++q) s += part[(long long)q * C + c];
  kbar[c] = s / (float)n;
}

cudaError_t launch_page_summary_final(const float* part, long long n, int C, float* kbar, cudaStream_t s) {
  page_summary_final_kernel<<<(C + 255) / 256, 256, 0, s>>>(part, colsum_splits(n), n, C, kbar);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ page-level retrieval
// One CTA: qbar = column means of Q, s_p = qbar . kbar_p for candidates, top-Kp
// (ties -> lower page id), written ascending.
__global__ void __launch_bounds__(1024) select_pages_final_kernel(
    const float* __restrict__ part, int splits, long long Lq, int C, const float* __restrict__ kbar, int NP,
    const int32_t* __restrict__ cand_range, int Kp, int32_t* __restrict__ sel_out, float* __restrict__ scores_out,
    int* status) {
  extern __shared__ float sm[];
  float* qbar = sm;           // [C]
  float* score = sm + C;      // [NP]
  int* taken = reinterpret_cast<int*>(score + NP);  // [NP]
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32, nwarps = blockDim.x / 32;
  for (int c = tid; c < C; c += blockDim.x) {
    float s = 0.f;
    for (int q = 0; q < splits; ++q) s += part[(long long)q * C + c];
    qbar[c] = s / (float)Lq;
  }
  int first = 0, end = NP;
  if (cand_range) {
    first = cand_range[0];
    end = cand_range[1];
  }
  const bool bad = first < 0 || end > NP || end - first < Kp;
  for (int p = tid; p < NP; p += blockDim.x) {
    score[p] = -INFINITY;
    taken[p] = 0;
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) set_status(status, HSA_ERR_DEVICE);
    for (int k = tid; k < Kp; k += blockDim.x) sel_out[k] = -1;
    if (scores_out)
      for (int p = tid; p < NP; p += blockDim.x) scores_out[p] = -INFINITY;
    return;
  }
  for (int p = first + warp; p < end; p += nwarps) {
    const float* kb = kbar + (long long)p * C;
    float s = 0.f;
    for (int c = lane; c < C; c += 32) s = fmaf(qbar[c], kb[c], s);
    s = warp_sum(s);
    if (lane == 0) score[p] = s;
  }
  __syncthreads();
  if (scores_out)
    for (int p = tid; p < NP; p += blockDim.x) scores_out[p] = score[p];
  if (tid == 0) {
    int chosen[64];
    int nchosen = 0;
    for (int k = 0; k < Kp; ++k) {
      int best = -1;
      float bv = -INFINITY;
      for (int p = first; p < end; ++p) {
        if (taken[p]) continue;
        if (best < 0 || score[p] > bv) {  // strict: a tie keeps the lower page id
          best = p;
          bv = score[p];
        }
      }
      taken[best] = 1;
      if (nchosen < 64) chosen[nchosen++] = best;
    }
    // ascending page order (insertion sort, Kp <= 64)
    for (int a = 1; a < nchosen; ++a) {
      int v = chosen[a], b = a - 1;
      while (b >= 0 && chosen[b] > v) {
        chosen[b + 1] = chosen[b];
        --b;
      }
      chosen[b + 1] = v;
    }
    for (int k = 0; k < nchosen; ++k) sel_out[k] = chosen[k];
  }
}

cudaError_t launch_select_pages_final(const float* part, long long Lq, int C, const float* kbar_pages, int NP,
                                      const int32_t* cand_range, int Kp, int32_t* sel_out, float* scores_out,
                                      int* status, cudaStream_t s) {
  size_t smem = (size_t)C * 4 + (size_t)NP * 8;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(select_pages_final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  select_pages_final_kernel<<<1, 1024, smem, s>>>(part, colsum_splits(Lq), Lq, C, kbar_pages, NP, cand_range, Kp,
                                                  sel_out, scores_out, status);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ prompt-level retrieval
__device__ double block_sum_d(double v, double* red) {
  v = warp_sum(v);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x < 32) {
    t = threadIdx.x < blockDim.x / 32 ? red[threadIdx.x] : 0.0;
    t = warp_sum(t);
    if (threadIdx.x == 0) red[32] = t;
  }
  __syncthreads();
  return red[32];
}

__global__ void __launch_bounds__(256) select_prompt_kernel(const float* __restrict__ e_cur,
                                                            const float* __restrict__ e_seg, int n_seg, int dim,
                                                            const int32_t* __restrict__ seg_begin,
                                                            int32_t* seg_out, int32_t* cand_range_out) {
  __shared__ double red[33];
  double nc = 0.0;
  for (int i = threadIdx.x; i < dim; i += blockDim.x) nc += (double)e_cur[i] * e_cur[i];
  nc = block_sum_d(nc, red);
  int best = 0;
  double bestc = -2.0;
  for (int s = 0; s < n_seg; ++s) {
    const float* e = e_seg + (long long)s * dim;
    double dt = 0.0, ns = 0.0;
    for (int i = threadIdx.x; i < dim; i += blockDim.x) {
      dt += (double)e_cur[i] * e[i];
      ns += (double)e[i] * e[i];
    }
    dt = block_sum_d(dt, red);
    ns = block_sum_d(ns, red);
    double c = dt / sqrt(nc * ns);
    if (s == 0 || c > bestc) {  // strict: ties keep the lowest segment
      bestc = c;
      best = s;
    }
  }
  if (threadIdx.x == 0) {
    *seg_out = best;
    cand_range_out[0] = seg_begin[best];
    cand_range_out[1] = seg_begin[best + 1];
  }
}

cudaError_t launch_select_prompt(const float* e_cur, const float* e_seg, int n_seg, int dim,
                                 const int32_t* seg_begin, int32_t* seg_out, int32_t* cand_range_out,
                                 cudaStream_t s) {
  select_prompt_kernel<<<1, 256, 0, s>>>(e_cur, e_seg, n_seg, dim, seg_begin, seg_out, cand_range_out);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ gather
// Unit = (K or V, 128-row block j of the output, head h): 128 rows x d columns.
// Row R of the output comes from page sel[R / P_tok], row R % P_tok.  Each thread
// moves one 16-byte chunk of NIT rows (all loads issued before the stores).  For
// K units the 128-row block mean per head is accumulated on the way (fp32,
// fixed order) and written to kbar128[j, h, :].
template <int D>
__global__ void __launch_bounds__(256) gather_kernel(const uint16_t* const* __restrict__ page_k,
                                                     const uint16_t* const* __restrict__ page_v, int NP,
                                                     const int32_t* __restrict__ sel, long long P_tok, int H,
                                                     long long Lc, uint16_t* __restrict__ Kc,
                                                     uint16_t* __restrict__ Vc, float* __restrict__ kbar128,
                                                     int* status) {
  constexpr int TPR = D / 8;
  constexpr int RPI = 256 / TPR;
  constexpr int NIT = 128 / RPI;
  __shared__ float red[RPI][D];
  const long long nblk = (Lc + 127) / 128;
  long long unit = blockIdx.x;
  const int h = (int)(unit % H);
  unit /= H;
  const long long j = unit % nblk;
  const int kv = (int)(unit / nblk);
  const int c = threadIdx.x % TPR, rp = threadIdx.x / TPR;
  const uint16_t* const* pages = kv ? page_v : page_k;
  uint16_t* dst = kv ? Vc : Kc;

  uint4 v[NIT];
  bool ok[NIT];
#pragma unroll
  for (int it = 0; it < NIT; ++it) {
    const long long R = j * 128 + rp + it * RPI;
    ok[it] = false;
    if (R < Lc) {
      const int slot = (int)(R / P_tok);
      const long long t = R - (long long)slot * P_tok;
      const int p = sel[slot];
      const uint16_t* base = (p >= 0 && p < NP) ? pages[p] : nullptr;
      // page pointers come from a device table: check range and 16-byte alignment here
      if (base != nullptr && (reinterpret_cast<uintptr_t>(base) & 15u) == 0) {
        v[it] = ld_nc_v4(base + (t * H + h) * D + c * 8);
        ok[it] = true;
      } else {
        set_status(status, HSA_ERR_DEVICE);
      }
    }
  }
#pragma unroll
  for (int it = 0; it < NIT; ++it) {
    const long long R = j * 128 + rp + it * RPI;
    if (ok[it]) *reinterpret_cast<uint4*>(dst + (R * H + h) * D + c * 8) = v[it];
  }
  if (kv == 0 && kbar128 != nullptr) {
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int it = 0; it < NIT; ++it)
      if (ok[it]) add8(acc, v[it]);
#pragma unroll
    for (int k = 0; k < 8; ++k) red[rp][c * 8 + k] = acc[k];
    __syncthreads();
    const long long rows = min((long long)128, Lc - j * 128);
    for (int col = threadIdx.x; col < D; col += 256) {
      float s = 0.f;
#pragma unroll
      for (int q = 0; q < RPI; ++q) s += red[q][col];
      kbar128[(j * H + h) * D + col] = s / (float)rows;
    }
  }
}

cudaError_t launch_gather(const uint16_t* const* page_k, const uint16_t* const* page_v, int NP,
                          const int32_t* sel, int Kp, long long P_tok, int H, int d, uint16_t* Kc,
                          uint16_t* Vc, float* kbar128, int* status, cudaStream_t s) {
  const long long Lc = (long long)Kp * P_tok;
  const long long nblk = (Lc + 127) / 128;
  const long long grid = 2 * nblk * H;
  if (d == 128)
    gather_kernel<128><<<(unsigned)grid, 256, 0, s>>>(page_k, page_v, NP, sel, P_tok, H, Lc, Kc, Vc, kbar128, status);
  else
    gather_kernel<64><<<(unsigned)grid, 256, 0, s>>>(page_k, page_v, NP, sel, P_tok, H, Lc, Kc, Vc, kbar128, status);
  return cudaGetLastError();
}

}  // namespace hsa
