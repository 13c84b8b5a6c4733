// HSA block pooling and head-adaptive block selection ("WorldAttention pairs
// hierarchical KV caching with hybrid sparse attention..." news summary, HSA
// paragraph: per head, the minimal block set whose cumulative attention mass
// reaches tau_h; Binter = 128 against the cached KV, Bintra = 64 in the chunk).
#include <float.h>
#include <limits.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace hsa {

// ------------------------------------------------------------------ pooling
// Unit = (source, 128-row block i, head h).  Sources: 0 = Q (writes the two 64-row
// means and the 128-row mean), 1 = Kq (two 64-row means), 2 = Kc (128-row mean).
// A partial block is the mean of its real rows.  fp32 sums in a fixed order.
template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const uint16_t* __restrict__ Q, const uint16_t* __restrict__ Kq,
                                                   const uint16_t* __restrict__ Kc, int H, int Lq, long long Lc,
                                                   int nQ128, float* __restrict__ q128, float* __restrict__ q64,
                                                   float* __restrict__ kq64, float* __restrict__ kc128) {
  constexpr int TPR = D / 8;
  constexpr int RPI = 256 / TPR;
  constexpr int NIT = 128 / RPI;
  __shared__ float red[2][RPI][D];
  long long unit = blockIdx.x;
  const int h = (int)(unit % H);
  unit /= H;
  int src;
  long long i;
  if (unit < nQ128) {
    src = 0;
    i = unit;
  } else if (unit < 2 * nQ128) {
    src = 1;
    i = unit - nQ128;
  } else {
    src = 2;
    i = unit - 2 * nQ128;
  }
  const uint16_t* X = src == 0 ? Q : (src == 1 ? Kq : Kc);
  const long long n = src == 2 ? Lc : (long long)Lq;
  const int c = threadIdx.x % TPR, rp = threadIdx.x / TPR;
  float a0[8] = {0, 0, 0, 0, 0, 0, 0, 0}, a1[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  uint4 v[NIT];
#pragma unroll
  for (int it = 0; it < NIT; ++it) {
    const long long R = i * 128 + rp + it * RPI;
    v[it] = R < n ? ld_nc_v4(X + (R * H + h) * D + c * 8) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int it = 0; it < NIT; ++it) {
    if (it * RPI < 64) add8(a0, v[it]);  // rows rp + it*RPI < 64 exactly when it*RPI < 64
    else add8(a1, v[it]);
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    red[0][rp][c * 8 + k] = a0[k];
    red[1][rp][c * 8 + k] = a1[k];
  }
  __syncthreads();
  const long long base = i * 128;
  const int n0 = (int)max(0LL, min(64LL, n - base));
  const int n1 = (int)max(0LL, min(64LL, n - base - 64));
  for (int col = threadIdx.x; col < D; col += 256) {
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int q = 0; q < RPI; ++q) {
      s0 += red[0][q][col];
      s1 += red[1][q][col];
    }
    if (src == 0) {
      q64[((2 * i) * H + h) * D + col] = s0 / (float)n0;
      if (n1 > 0) q64[((2 * i + 1) * H + h) * D + col] = s1 / (float)n1;
      q128[(i * H + h) * D + col] = (s0 + s1) / (float)(n0 + n1);
    } else if (src == 1) {
      kq64[((2 * i) * H + h) * D + col] = s0 / (float)n0;
      if (n1 > 0) kq64[((2 * i + 1) * H + h) * D + col] = s1 / (float)n1;
    } else {
      kc128[(i * H + h) * D + col] = (s0 + s1) / (float)(n0 + n1);
    }
  }
}

cudaError_t launch_pool(const uint16_t* Q, const uint16_t* Kq, const uint16_t* Kc, int H, int d, int Lq,
                        long long Lc, float* q128, float* q64, float* kq64, float* kc128, cudaStream_t s) {
  const int nQ128 = (Lq + 127) / 128;
  const long long nKc = kc128 ? (Lc + 127) / 128 : 0;  // Kc pooled here only when asked
  const long long grid = (2LL * nQ128 + nKc) * H;
  if (grid == 0) return cudaSuccess;
  if (d == 128)
    pool_kernel<128><<<(unsigned)grid, 256, 0, s>>>(Q, Kq, Kc, H, Lq, Lc, nQ128, q128, q64, kq64, kc128);
  else
    pool_kernel<64><<<(unsigned)grid, 256, 0, s>>>(Q, Kq, Kc, H, Lq, Lc, nQ128, q128, q64, kq64, kc128);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ block scores
// s[h][i][j] = scale * qbar_i . kbar_j for every selection row i of one map and every
// key block j (j < nA from kA, the rest from kB), fp32, summed over d in order.  One
// CTA per (64 key blocks, 32 rows, head): both tiles are loaded whole into shared
// memory (16-byte loads, all in flight at once), so a key block's mean is read once
// per 32 rows rather than once per row, in one memory round trip.
constexpr int kScoreRows = 32, kScoreKeys = 64;

template <int D>
__global__ void __launch_bounds__(256) block_scores_kernel(const float* __restrict__ q, int R,
                                                           const float* __restrict__ kA, int nA,
                                                           const float* __restrict__ kB, int K, int H, float scale,
                                                           float* __restrict__ out) {
  extern __shared__ __align__(16) float sm_scores[];
  constexpr int P = D + 4;  // row pitch (floats): 16-byte rows, rows 4 banks apart
  float* sq = sm_scores;                   // [kScoreRows][P]
  float* sk = sm_scores + kScoreRows * P;  // [kScoreKeys][P]
  const int h = blockIdx.z;
  const int i0 = blockIdx.y * kScoreRows, j0 = blockIdx.x * kScoreKeys;
  constexpr int V = D / 4;  // float4 per row
  for (int t = threadIdx.x; t < kScoreRows * V; t += 256) {
    const int r = t / V, c = t % V, i = i0 + r;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i < R) v = __ldg(reinterpret_cast<const float4*>(q + ((long long)i * H + h) * D) + c);
    *reinterpret_cast<float4*>(sq + r * P + 4 * c) = v;
  }
  for (int t = threadIdx.x; t < kScoreKeys * V; t += 256) {
    const int r = t / V, c = t % V, j = j0 + r;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (j < nA) v = __ldg(reinterpret_cast<const float4*>(kA + ((long long)j * H + h) * D) + c);
    else if (j < K) v = __ldg(reinterpret_cast<const float4*>(kB + ((long long)(j - nA) * H + h) * D) + c);
    *reinterpret_cast<float4*>(sk + r * P + 4 * c) = v;
  }
  __syncthreads();
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;  // rows 2 ty, 2 ty + 1; keys tx + 16 u
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 8
  for (int c = 0; c < D; ++c) {
    const float a0 = sq[(2 * ty) * P + c], a1 = sq[(2 * ty + 1) * P + c];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float b = sk[(tx + 16 * u) * P + c];
      acc[0][u] = fmaf(a0, b, acc[0][u]);
      acc[1][u] = fmaf(a1, b, acc[1][u]);
    }
  }
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int i = i0 + 2 * ty + rr;
    if (i >= R) continue;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = j0 + tx + 16 * u;
      if (j < K) out[((long long)h * R + i) * K + j] = acc[rr][u] * scale;
    }
  }
}

template <int D>
cudaError_t launch_scores(const float* q, int R, const float* kA, int nA, const float* kB, int K, int H, float scale,
                          float* out, cudaStream_t s) {
  if (R == 0 || K == 0) return cudaSuccess;
  const size_t smem = (size_t)(kScoreRows + kScoreKeys) * (D + 4) * sizeof(float);
  if (smem > 48 * 1024) {
    const cudaError_t e =
        cudaFuncSetAttribute(block_scores_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const dim3 grid((unsigned)((K + kScoreKeys - 1) / kScoreKeys), (unsigned)((R + kScoreRows - 1) / kScoreRows),
                  (unsigned)H);
  block_scores_kernel<D><<<grid, 256, smem, s>>>(q, R, kA, nA, kB, K, H, scale, out);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ block selection
// One CTA per selection row (head h, query block i, map inter|intra; in joint mode
// one row per (head, 64-row query block) over the Kc blocks followed by the Kq
// blocks, whose kept ids are split into the row's inter and intra lists):
//   s_j = qbar_i . kbar_j * scale                 (fp32, one warp per block)
//   e_j = exp(s_j - max_j s_j);  total = sum_j e_j (fp64)
//   rank by e descending (ties -> lower j)        (bitonic sort in shared memory)
//   k* = first k with sum_{m<k} e_(m) >= tau * total   (fp64 prefix sums)
//   emit the k* kept ids ascending                (flag + ordered compaction)
// tau >= 1 keeps every block.
constexpr int kSelThreads = 256;

__device__ __forceinline__ bool ranks_before(float ea, int ia, float eb, int ib) {
  return ea > eb || (ea == eb && ia < ib);
}

// Exclusive prefix sum of one value per thread over the block; `total` receives the
// block's sum in every thread.  warp_tot: shared, kSelThreads / 32 + 1 entries.
template <typename T>
__device__ T block_excl_scan(T v, T* warp_tot, T& total) {
  constexpr int kWarps = kSelThreads / 32;
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  T x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    T y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    T w = lane < kWarps ? warp_tot[lane] : T(0);
    T wx = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      T y = __shfl_up_sync(0xffffffffu, wx, o);
      if (lane >= o) wx += y;
    }
    if (lane < kWarps) warp_tot[lane] = wx - w;  // exclusive warp offsets
    if (lane == kWarps - 1) warp_tot[kWarps] = wx;
  }
  __syncthreads();
  T r = warp_tot[warp] + x - v;
  total = warp_tot[kWarps];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kSelThreads) block_select_kernel(
    const float* __restrict__ scores, const float* __restrict__ tau, int H, int nQ128, int nKc, int nQ64, int nKq,
    bool joint, int32_t* __restrict__ inter_idx, int32_t* __restrict__ inter_cnt, int32_t* __restrict__ intra_idx,
    int32_t* __restrict__ intra_cnt) {
  extern __shared__ __align__(16) unsigned char smraw[];
  __shared__ double dred[40];
  __shared__ int ired[40];
  __shared__ float fred[40];
  __shared__ int s_kstar;

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  int row = blockIdx.x;
  // the row's keys: nK scores (block_scores_kernel); kept ids < nA go to idx_out /
  // cnt_out, the others (minus nA) to idx_out2 / cnt_out2
  int h, i, nK, nA;
  const float* srow;
  int32_t* idx_out;
  int32_t* cnt_out;
  int32_t* idx_out2 = nullptr;
  int32_t* cnt_out2 = nullptr;
  if (joint) {
    h = row / nQ64;
    i = row % nQ64;
    nA = nKc;
    nK = nKc + nKq;
    srow = scores + ((long long)h * nQ64 + i) * nK;
    idx_out = inter_idx + ((long long)h * nQ64 + i) * nKc;
    cnt_out = inter_cnt + (long long)h * nQ64 + i;
    idx_out2 = intra_idx + ((long long)h * nQ64 + i) * nKq;
    cnt_out2 = intra_cnt + (long long)h * nQ64 + i;
  } else if (row < H * nQ128) {
    h = row / nQ128;
    i = row % nQ128;
    nK = nA = nKc;
    srow = scores + ((long long)h * nQ128 + i) * nKc;
    idx_out = inter_idx + ((long long)h * nQ128 + i) * nKc;
    cnt_out = inter_cnt + (long long)h * nQ128 + i;
  } else {
    row -= H * nQ128;
    h = row / nQ64;
    i = row % nQ64;
    nK = nA = nKq;
    srow = scores + (long long)H * nQ128 * nKc + ((long long)h * nQ64 + i) * nKq;
    idx_out = intra_idx + ((long long)h * nQ64 + i) * nKq;
    cnt_out = intra_cnt + (long long)h * nQ64 + i;
  }
  if (nK == 0) {
    if (tid == 0) {
      *cnt_out = 0;
      if (cnt_out2) *cnt_out2 = 0;
    }
    return;
  }
  const float t = tau[h];
  if (t >= 1.0f) {
    for (int j = tid; j < nK; j += kSelThreads) {
      if (j < nA) idx_out[j] = j;
      else idx_out2[j - nA] = j - nA;
    }
    if (tid == 0) {
      *cnt_out = nA;
      if (cnt_out2) *cnt_out2 = nK - nA;
    }
    return;
  }
  int NB2 = 1;
  while (NB2 < nK) NB2 <<= 1;
  float* e = reinterpret_cast<float*>(smraw);   // [NB2]
  int* id = reinterpret_cast<int*>(e + NB2);    // [NB2]
  int* flag = id + NB2;                          // [NB2]

  for (int j = tid; j < nK; j += kSelThreads) e[j] = srow[j];
  __syncthreads();
  // row max
  float m = -INFINITY;
  for (int j = tid; j < nK; j += kSelThreads) m = fmaxf(m, e[j]);
  m = warp_max(m);
  if (lane == 0) fred[warp] = m;
  __syncthreads();
  if (tid == 0) {
    float mm = fred[0];
    for (int w = 1; w < kSelThreads / 32; ++w) mm = fmaxf(mm, fred[w]);
    fred[32] = mm;
  }
  __syncthreads();
  m = fred[32];
  for (int j = tid; j < NB2; j += kSelThreads) {
    if (j < nK) {
      e[j] = expf(e[j] - m);
      id[j] = j;
    } else {
      e[j] = -1.0f;  // sentinel ranks last
      id[j] = INT_MAX;
    }
    flag[j] = 0;
  }
  __syncthreads();
  // total mass in fp64 (fixed order: strided per thread, then a tree)
  double tot = 0.0;
  for (int j = tid; j < nK; j += kSelThreads) tot += (double)e[j];
  tot = warp_sum(tot);
  if (lane == 0) dred[warp] = tot;
  __syncthreads();
  if (tid == 0) {
    double s = 0.0;
    for (int w = 0; w < kSelThreads / 32; ++w) s += dred[w];
    dred[32] = s;
  }
  __syncthreads();
  tot = dred[32];
  // bitonic sort into rank order
  for (int k = 2; k <= NB2; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int x = tid; x < NB2; x += kSelThreads) {
        const int y = x ^ jj;
        if (y > x) {
          const bool first_half = (x & k) == 0;
          const bool xb = ranks_before(e[x], id[x], e[y], id[y]);
          if (first_half != xb) {
            float te = e[x]; e[x] = e[y]; e[y] = te;
            int ti = id[x]; id[x] = id[y]; id[y] = ti;
          }
        }
      }
      __syncthreads();
    }
  }
  // prefix sums over the ranked masses: each thread owns a contiguous chunk
  const int CH = (nK + kSelThreads - 1) / kSelThreads;
  const int b0 = tid * CH, b1 = min(nK, b0 + CH);
  double local = 0.0;
  for (int x = b0; x < b1; ++x) local += (double)e[x];
  double tot_scan;
  const double before = block_excl_scan<double>(local, dred, tot_scan);
  if (tid == 0) s_kstar = nK;
  __syncthreads();
  const double thr = (double)t * tot;
  double cum = before;
  for (int x = b0; x < b1; ++x) {
    cum += (double)e[x];
    if (cum >= thr) {
      atomicMin(&s_kstar, x + 1);
      break;
    }
  }
  __syncthreads();
  const int kstar = s_kstar;
  for (int x = tid; x < kstar; x += kSelThreads) flag[id[x]] = 1;
  __syncthreads();
  // ordered compaction of the kept ids (ids >= nA into the second list, minus nA)
  int cnt = 0, cnt2 = 0;
  for (int x = b0; x < b1; ++x) {
    if (x < nA) cnt += flag[x];
    else cnt2 += flag[x];
  }
  int total_kept, total_kept2;
  int pos = block_excl_scan<int>(cnt, ired, total_kept);
  int pos2 = block_excl_scan<int>(cnt2, ired, total_kept2);
  for (int x = b0; x < b1; ++x) {
    if (!flag[x]) continue;
    if (x < nA) idx_out[pos++] = x;
    else idx_out2[pos2++] = x - nA;
  }
  if (tid == 0) {
    *cnt_out = total_kept;
    if (cnt_out2) *cnt_out2 = total_kept2;
  }
}

size_t block_scores_floats(int H, int Lq, long long Lc) {
  const long long nQ128 = (Lq + 127) / 128, nQ64 = (Lq + 63) / 64, nKc = (Lc + 127) / 128;
  const long long separate = nQ128 * nKc + nQ64 * nQ64, joint = nQ64 * (nKc + nQ64);
  return (size_t)H * (size_t)(separate > joint ? separate : joint);
}

cudaError_t launch_block_select(const float* q128, const float* kc128, const float* q64, const float* kq64,
                                const float* tau, int H, int d, int Lq, long long Lc, float scale, bool joint,
                                float* scores, int32_t* inter_idx, int32_t* inter_cnt, int32_t* intra_idx,
                                int32_t* intra_cnt, cudaStream_t s) {
  const int nQ128 = (Lq + 127) / 128, nQ64 = (Lq + 63) / 64;
  const int nKc = (int)((Lc + 127) / 128), nKq = nQ64;
  // the scores of every row: [H][nQ64][nKc + nKq] (joint), or [H][nQ128][nKc] followed
  // by [H][nQ64][nKq] (separate)
  auto scores_of = [&](auto tag) -> cudaError_t {
    constexpr int D = decltype(tag)::value;
    if (joint) return launch_scores<D>(q64, nQ64, kc128, nKc, kq64, nKc + nKq, H, scale, scores, s);
    const cudaError_t e = launch_scores<D>(q128, nQ128, kc128, nKc, kc128, nKc, H, scale, scores, s);
    if (e != cudaSuccess) return e;
    return launch_scores<D>(q64, nQ64, kq64, nKq, kq64, nKq, H, scale, scores + (long long)H * nQ128 * nKc, s);
  };
  cudaError_t e = d == 128 ? scores_of(std::integral_constant<int, 128>()) : scores_of(std::integral_constant<int, 64>());
  if (e != cudaSuccess) return e;
  int nmax = joint ? nKc + nKq : (nKc > nKq ? nKc : nKq), NB2 = 1;
  while (NB2 < nmax) NB2 <<= 1;
  const size_t smem = (size_t)NB2 * 12;
  const int grid = joint ? H * nQ64 : H * (nQ128 + nQ64);
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(block_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  block_select_kernel<<<grid, kSelThreads, smem, s>>>(scores, tau, H, nQ128, nKc, nQ64, nKq, joint, inter_idx,
                                                      inter_cnt, intra_idx, intra_cnt);
  return cudaGetLastError();
}

}  // namespace hsa
