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
// copy_dst (optional): every row read is also written there (page seal: the copy
// into the store and the summary in one pass).
__global__ void __launch_bounds__(256) colsum_partial_kernel(const uint16_t* __restrict__ X, long long n, int C,
                                                             long long rows_per_split, float* __restrict__ part,
                                                             uint16_t* __restrict__ copy_dst) {
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
      for (long long r = r0 + rp; r < r1; r += RP) {
        const uint4 w = ld_nc_v4(X + r * C + v * 8);
        if (copy_dst) *reinterpret_cast<uint4*>(copy_dst + r * C + v * 8) = w;
        add8(acc, w);
      }
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
      for (long long r = r0; r < r1; ++r) {
        const uint4 w = ld_nc_v4(X + r * C + v * 8);
        if (copy_dst) *reinterpret_cast<uint4*>(copy_dst + r * C + v * 8) = w;
        add8(acc, w);
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) out[v * 8 + k] = acc[k];
    }
  }
}

int colsum_splits(long long n) {
  long long s = (n + 15) / 16;  // 16 rows per split
  return (int)(s < 1 ? 1 : (s > kColMaxSplits ? kColMaxSplits : s));
}

// Sum of part[q][c] over the splits, with four independent accumulators so that
// the loads of consecutive splits overlap.
__device__ __forceinline__ float sum_splits(const float* __restrict__ part, int splits, int C, int c) {
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  int q = 0;
  for (; q + 4 <= splits; q += 4) {
    a0 += part[(long long)q * C + c];
    a1 += part[(long long)(q + 1) * C + c];
    a2 += part[(long long)(q + 2) * C + c];
    a3 += part[(long long)(q + 3) * C + c];
  }
  for (; q < splits; ++q) a0 += part[(long long)q * C + c];
  return (a0 + a1) + (a2 + a3);
}

cudaError_t launch_colsum_partial(const uint16_t* X, long long n, int C, float* part, uint16_t* copy_dst,
                                  cudaStream_t s) {
  int splits = colsum_splits(n);
  long long rps = (n + splits - 1) / splits;
  colsum_partial_kernel<<<splits, 256, 0, s>>>(X, n, C, rps, part, copy_dst);
  return cudaGetLastError();
}

// kbar[c] = (sum_s part[s][c]) / n
__global__ void page_summary_final_kernel(const float* __restrict__ part, int splits, long long n, int C,
                                          float* __restrict__ kbar) {
  int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= C) return;
  kbar[c] = sum_splits(part, splits, C, c) / (float)n;
}

cudaError_t launch_page_summary_final(const float* part, long long n, int C, float* kbar, cudaStream_t s) {
  page_summary_final_kernel<<<(C + 255) / 256, 256, 0, s>>>(part, colsum_splits(n), n, C, kbar);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ page-level retrieval
// s_p = qbar . kbar_p with qbar the column mean of Q.  Pass 1 splits Q's rows over
// many CTAs; each CTA sums its rows' columns in shared memory and dots that sum
// with every candidate page's kbar, writing one partial score per page.  Pass 2
// (one CTA) adds the partials in split order, divides by Lq, ranks the candidates
// (ties -> lower page id) and writes the top Kp ascending.  Both passes reduce in
// a fixed order (deterministic).
constexpr int kScoreThreads = 256;

int page_score_splits(long long Lq) {
  long long s = (Lq + 15) / 16;  // at least 16 rows per split
  return (int)(s < 1 ? 1 : (s > kColMaxSplits ? kColMaxSplits : s));
}

__global__ void __launch_bounds__(kScoreThreads) page_scores_partial_kernel(
    const uint16_t* __restrict__ Q, long long Lq, int C, long long rows_per_split, const float* __restrict__ kbar,
    int NP, const int32_t* __restrict__ cand_range, float* __restrict__ part) {
  extern __shared__ float colsum[];  // [C]
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const long long r0 = (long long)blockIdx.x * rows_per_split;
  const long long r1 = min(Lq, r0 + rows_per_split);
  for (int v = tid; v < C / 8; v += kScoreThreads) {
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    long long r = r0;
    for (; r + 16 <= r1; r += 16) {  // 16 loads in flight
      uint4 w[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) w[k] = ld_nc_v4(Q + (r + k) * C + v * 8);
      asm volatile("" ::: "memory");  // keep the batch of loads ahead of their uses
#pragma unroll
      for (int k = 0; k < 16; ++k) add8(acc, w[k]);
    }
    for (; r < r1; ++r) add8(acc, ld_nc_v4(Q + r * C + v * 8));
#pragma unroll
    for (int k = 0; k < 8; ++k) colsum[v * 8 + k] = acc[k];
  }
  __syncthreads();
  int first = 0, end = NP;
  if (cand_range) {
    first = max(cand_range[0], 0);
    end = min(cand_range[1], NP);
  }
  float* out = part + (long long)blockIdx.x * NP;
  for (int p = first + warp; p < end; p += kScoreThreads / 32) {
    const float* kb = kbar + (long long)p * C;
    float sacc = 0.f;
    constexpr int kBatch = 8;  // float4 loads in flight per lane
    for (int c0 = lane * 4; c0 < C; c0 += 128 * kBatch) {
      float4 k4[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int c = c0 + u * 128;
        k4[u] = c < C ? __ldg(reinterpret_cast<const float4*>(kb + c)) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      asm volatile("" ::: "memory");  // keep the batch of loads ahead of their uses
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int c = c0 + u * 128;
        if (c < C) {
          sacc = fmaf(colsum[c], k4[u].x, sacc);
          sacc = fmaf(colsum[c + 1], k4[u].y, sacc);
          sacc = fmaf(colsum[c + 2], k4[u].z, sacc);
          sacc = fmaf(colsum[c + 3], k4[u].w, sacc);
        }
      }
    }
    sacc = warp_sum(sacc);
    if (lane == 0) out[p] = sacc;
  }
}

constexpr int kFinalThreads = 1024;

__global__ void __launch_bounds__(kFinalThreads) select_pages_final_kernel(
    const float* __restrict__ part, int splits, long long Lq, int NP, const int32_t* __restrict__ cand_range,
    int Kp, int32_t* __restrict__ sel_out, float* __restrict__ scores_out, int* status) {
  extern __shared__ float score[];  // [NP]
  __shared__ int warp_cnt[kFinalThreads / 32];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  int first = 0, end = NP;
  if (cand_range) {
    first = cand_range[0];
    end = cand_range[1];
  }
  if (first < 0 || end > NP || end - first < Kp) {
    if (tid == 0) set_status(status, HSA_ERR_DEVICE);
    for (int k = tid; k < Kp; k += kFinalThreads) sel_out[k] = -1;
    if (scores_out)
      for (int p = tid; p < NP; p += kFinalThreads) scores_out[p] = -INFINITY;
    return;
  }
  for (int p = warp; p < NP; p += kFinalThreads / 32) {
    float sacc = 0.f;
    if (p >= first && p < end)
      for (int q = lane; q < splits; q += 32) sacc += part[(long long)q * NP + p];
    sacc = warp_sum(sacc);
    if (lane == 0) score[p] = (p >= first && p < end) ? sacc / (float)Lq : -INFINITY;
  }
  __syncthreads();
  if (scores_out)
    for (int p = tid; p < NP; p += kFinalThreads) scores_out[p] = score[p];
  // a candidate is kept when fewer than Kp candidates rank before it
  int base = 0;
  for (int p0 = 0; p0 < NP; p0 += kFinalThreads) {
    const int p = p0 + tid;
    bool keep = false;
    if (p >= first && p < end) {
      const float sp = score[p];
      int rank = 0;
      for (int q = first; q < end && rank < Kp; ++q) {
        const float sq = score[q];
        rank += (sq > sp) || (sq == sp && q < p);
      }
      keep = rank < Kp;
    }
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) warp_cnt[warp] = __popc(bal);
    __syncthreads();
    int before = base;
    for (int w = 0; w < warp; ++w) before += warp_cnt[w];
    if (keep) {
      const int pos = before + __popc(bal & ((1u << lane) - 1u));
      if (pos < Kp) sel_out[pos] = p;
    }
    __syncthreads();
    for (int w = 0; w < kFinalThreads / 32; ++w) base += warp_cnt[w];
    __syncthreads();
  }
}

// s_p = (sum over the splits of part[q][p]) / Lq for the candidates, -inf elsewhere
// (the page scores of this call's heads, before any ranking).
__global__ void page_scores_sum_kernel(const float* __restrict__ part, int splits, long long Lq, int NP,
                                       const int32_t* __restrict__ cand_range, float* __restrict__ scores) {
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= NP) return;
  int first = 0, end = NP;
  if (cand_range) {
    first = cand_range[0];
    end = cand_range[1];
  }
  float s = 0.f;
  for (int q = 0; q < splits; ++q) s += part[(long long)q * NP + p];
  scores[p] = (p >= first && p < end) ? s / (float)Lq : -INFINITY;
}

cudaError_t launch_page_scores_sum(const float* part, long long Lq, int NP, const int32_t* cand_range, float* scores,
                                   cudaStream_t s) {
  page_scores_sum_kernel<<<(NP + 255) / 256, 256, 0, s>>>(part, page_score_splits(Lq), Lq, NP, cand_range, scores);
  return cudaGetLastError();
}

cudaError_t launch_page_scores_partial(const uint16_t* Q, long long Lq, int C, const float* kbar_pages, int NP,
                                       const int32_t* cand_range, float* part, cudaStream_t s) {
  const int splits = page_score_splits(Lq);
  const long long rps = (Lq + splits - 1) / splits;
  const size_t smem = (size_t)C * 4;
  if (smem > kDefaultSmemOptIn) {
    cudaError_t e = cudaFuncSetAttribute(page_scores_partial_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  page_scores_partial_kernel<<<splits, kScoreThreads, smem, s>>>(Q, Lq, C, rps, kbar_pages, NP, cand_range, part);
  return cudaGetLastError();
}

cudaError_t launch_select_pages_final(const float* part, long long Lq, int NP, const int32_t* cand_range, int Kp,
                                      int32_t* sel_out, float* scores_out, int* status, cudaStream_t s) {
  const size_t smem = (size_t)NP * 4;
  if (smem > kDefaultSmemOptIn) {
    cudaError_t e = cudaFuncSetAttribute(select_pages_final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  select_pages_final_kernel<<<1, kFinalThreads, smem, s>>>(part, page_score_splits(Lq), Lq, NP, cand_range, Kp,
                                                           sel_out, scores_out, status);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ retrieval policies
// The retrieval ablations of the method's evaluation rank the candidate pages by
// something other than the mean-key score: by recency (the page id: the most recent
// pages) or by caller-drawn random keys (a uniform random subset).  One split of
// "partial scores" holds those keys; select_pages_final then ranks them exactly as
// it ranks page scores (ties -> lower page id) and writes the top Kp ascending.
__global__ void policy_keys_kernel(int policy, const float* __restrict__ rand_keys, int NP, float* __restrict__ part) {
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= NP) return;
  part[p] = policy == kPolicyRecent ? (float)p : rand_keys[p];
}

cudaError_t launch_policy_keys(int policy, const float* rand_keys, int NP, float* part, cudaStream_t s) {
  policy_keys_kernel<<<(NP + 255) / 256, 256, 0, s>>>(policy, rand_keys, NP, part);
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

// ------------------------------------------------------------------ 64-row key sums of a page
// sums[b][c] = sum over the rows [64 b, min(64 b + 64, n)) of X[row][c], fp32 in row
// order (a page's keys, once when it is sealed).  Thread = 16-byte column chunk.
constexpr int kSumThreads = 128;

__global__ void __launch_bounds__(kSumThreads) block_sums64_kernel(const uint16_t* __restrict__ X, long long n, int C,
                                                                  float* __restrict__ sums) {
  const long long b = blockIdx.x;
  const int cc = blockIdx.y * kSumThreads + threadIdx.x;
  if (cc * 8 >= C) return;
  const long long r0 = b * 64, r1 = min(n, r0 + 64);
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  long long r = r0;
  for (; r + 8 <= r1; r += 8) {
    uint4 w[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) w[u] = ld_nc_v4(X + (r + u) * C + cc * 8);
#pragma unroll
    for (int u = 0; u < 8; ++u) add8(acc, w[u]);
  }
  for (; r < r1; ++r) add8(acc, ld_nc_v4(X + r * C + cc * 8));
  float4* out = reinterpret_cast<float4*>(sums + b * C + cc * 8);
  out[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  out[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

cudaError_t launch_block_sums64(const uint16_t* X, long long n, int C, float* sums, cudaStream_t s) {
  const long long nb = (n + 63) / 64;
  const int cols = (C / 8 + kSumThreads - 1) / kSumThreads;
  block_sums64_kernel<<<dim3((unsigned)nb, cols), kSumThreads, 0, s>>>(X, n, C, sums);
  return cudaGetLastError();
}

// kbar128[j] of the active cache gathered from pages sel[0..Kp) (P_tok a multiple of
// 64, so each 64-row half of a 128-row block lies in one page): the two halves'
// stored sums, added in order, over the block's rows.  Needs only the selection,
// not the gathered copy.
__global__ void __launch_bounds__(kSumThreads) kc128_from_pages_kernel(const float* __restrict__ sums, int NP,
                                                                      long long nb64_page,
                                                                      const int32_t* __restrict__ sel, long long Lc,
                                                                      int C, float* __restrict__ kbar128,
                                                                      int* status) {
  const long long j = blockIdx.x;
  const int cc = blockIdx.y * kSumThreads + threadIdx.x;
  if (cc * 8 >= C) return;
  const long long P_tok = nb64_page * 64;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int u = 0; u < 2; ++u) {
    const long long r = j * 128 + u * 64;  // first gathered row of this half
    if (r >= Lc) break;
    const int p = sel[r / P_tok];
    if (p < 0 || p >= NP) {
      set_status(status, HSA_ERR_DEVICE);
      continue;
    }
    const float4* src = reinterpret_cast<const float4*>(sums + ((long long)p * nb64_page + (r % P_tok) / 64) * C + cc * 8);
    const float4 a = src[0], b = src[1];
    acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
    acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
  }
  const float inv = 1.f / (float)min(128LL, Lc - j * 128);
  float4* out = reinterpret_cast<float4*>(kbar128 + j * C + cc * 8);
  out[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
  out[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
}

cudaError_t launch_kc128_from_pages(const float* sums, int NP, long long P_tok, const int32_t* sel, int Kp, int C,
                                    float* kbar128, int* status, cudaStream_t s) {
  const long long Lc = (long long)Kp * P_tok;
  const long long nKc = (Lc + 127) / 128;
  const int cols = (C / 8 + kSumThreads - 1) / kSumThreads;
  kc128_from_pages_kernel<<<dim3((unsigned)nKc, cols), kSumThreads, 0, s>>>(sums, NP, P_tok / 64, sel, Lc, C,
                                                                           kbar128, status);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ gather
// Unit = (K or V, 128-row block j of the output): 128 full rows (all heads).
// Row R of the output comes from page sel[R / P_tok], row R % P_tok; a row is
// H*d contiguous bf16 in both the page and the output.  Thread t owns the 16-byte
// column chunk t of every row of the block and keeps 8 rows in flight; for K units
// it also accumulates the 128-row block mean of its 8 columns (fp32, fixed order)
// and writes kbar128[j, :, :] directly.  Page ids and page pointers come from
// device memory and are checked here (range, 16-byte alignment).
constexpr int kGatherUnroll = 8;

constexpr int kGatherMaxThreads = 640;  // one thread per 16-byte column up to H*d = 5120

__global__ void __launch_bounds__(kGatherMaxThreads) gather_kernel(
    const uint16_t* const* __restrict__ page_k, const uint16_t* const* __restrict__ page_v, int NP,
    const int32_t* __restrict__ sel, long long P_tok, int C, long long Lc, uint16_t* __restrict__ Kc,
    uint16_t* __restrict__ Vc, float* __restrict__ kbar128, int* status) {
  const long long nblk = (Lc + 127) / 128;
  const long long j = blockIdx.x % nblk;
  const int kv = (int)(blockIdx.x / nblk);
  const int CV = C / 8;
  const uint16_t* const* pages = kv ? page_v : page_k;
  uint16_t* dst = kv ? Vc : Kc;
  const long long r0 = j * 128;
  const int rows = (int)min((long long)128, Lc - r0);
  const bool pool = kv == 0 && kbar128 != nullptr;
  const int slot0 = (int)(r0 / P_tok);
  const long long t0 = r0 - (long long)slot0 * P_tok;
  for (int cc = threadIdx.x; cc < CV; cc += blockDim.x) {
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    // current page of this block's rows (rows are consecutive: advance slot by slot)
    int slot = -1;
    const uint16_t* base = nullptr;
    long long t = t0;
    int cur = slot0;
    for (int i0 = 0; i0 < rows; i0 += kGatherUnroll) {
      uint4 v[kGatherUnroll];
      bool ok[kGatherUnroll];
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u) {
        ok[u] = false;
        if (i0 + u < rows) {
          while (t >= P_tok) {
            t -= P_tok;
            ++cur;
          }
          if (cur != slot) {
            slot = cur;
            const int p = sel[slot];
            base = (p >= 0 && p < NP) ? pages[p] : nullptr;
            if (base == nullptr || (reinterpret_cast<uintptr_t>(base) & 15u) != 0) {
              base = nullptr;
              set_status(status, HSA_ERR_DEVICE);
            }
          }
          if (base != nullptr) {
            v[u] = ld_nc_v4(base + t * C + cc * 8);
            ok[u] = true;
          }
          ++t;
        }
      }
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u) {
        if (ok[u]) {
          *reinterpret_cast<uint4*>(dst + (r0 + i0 + u) * C + cc * 8) = v[u];
          if (pool) add8(acc, v[u]);
        }
      }
    }
    if (pool) {
      float* out = kbar128 + j * C + cc * 8;
      const float inv = 1.f / (float)rows;
#pragma unroll
      for (int k = 0; k < 8; ++k) out[k] = acc[k] * inv;
    }
  }
}

cudaError_t launch_gather(const uint16_t* const* page_k, const uint16_t* const* page_v, int NP,
                          const int32_t* sel, int Kp, long long P_tok, int H, int d, uint16_t* Kc,
                          uint16_t* Vc, float* kbar128, int* status, cudaStream_t s) {
  const long long Lc = (long long)Kp * P_tok;
  const long long nblk = (Lc + 127) / 128;
  const int CV = H * d / 8;
  const int threads = CV >= kGatherMaxThreads ? kGatherMaxThreads : ((CV + 31) / 32) * 32;
  gather_kernel<<<(unsigned)(2 * nblk), threads, 0, s>>>(page_k, page_v, NP, sel, P_tok, H * d, Lc, Kc, Vc,
                                                         kbar128, status);
  return cudaGetLastError();
}

}  // namespace hsa
