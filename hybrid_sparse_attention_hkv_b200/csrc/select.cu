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
  if (smem > kDefaultSmemOptIn) {
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
//   s_j = qbar_i . kbar_j * scale                 (fp32, block_scores_kernel)
//   e_j = exp(s_j - max_j s_j);  total = sum_j e_j (fp64)
//   rank by e descending (ties -> lower j)        (bitonic sort, rank_masses)
//   k* = first k with sum_{m<k} e_(m) >= tau * total   (fp64 prefix sums)
//   emit the k* kept ids ascending                (flag + ordered compaction)
// tau >= 1 keeps every block.
constexpr int kSelThreads = 256;
constexpr int kMaxSortKeys = 16 * kSelThreads;  // longest row ranked in registers; longer rows sort block-wide


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

// Rank a row's masses: e[0..nK) (>= 0) and their ids, into e / id in rank order
// (masses descending, equal masses the lower id first), N = E x 256 >= nK a power of
// two.  Keys mass bits << 32 | ~id order exactly so (the bits of non-negative floats
// order as their values; padding keys are 0 and rank last).  Bitonic sort with each
// thread holding E consecutive keys in registers: steps between a thread's own keys
// swap registers, steps within a warp exchange by shuffles, and only the steps of
// stride >= 32 E go through shared memory (`keys`, [N], over e and id): six
// synchronised passes for any N, against log2(N) (log2(N) + 1) / 2 for a block-wide
// network.
template <int E>
__device__ void rank_masses(float* e, int* id, int nK, unsigned long long* keys) {
  constexpr int N = E * kSelThreads;
  const int tid = threadIdx.x;
  unsigned long long v[E];
#pragma unroll
  for (int r = 0; r < E; ++r) {
    const int x = tid * E + r;
    v[r] = x < nK ? ((unsigned long long)__float_as_uint(e[x]) << 32) | (unsigned)(0xFFFFFFFFu - (unsigned)x) : 0ull;
  }
  __syncthreads();  // e is read before any pass writes the keys over it
  auto cas = [](unsigned long long a, unsigned long long b, bool keep_max) -> unsigned long long {
    return keep_max ? (a > b ? a : b) : (a < b ? a : b);
  };
  // both loops unrolled: every register index below is a compile-time constant
  constexpr int LOG2N = E == 1 ? 8 : E == 2 ? 9 : E == 4 ? 10 : E == 8 ? 11 : 12;
  static_assert((1 << LOG2N) == N, "N = E x 256, a power of two");
#pragma unroll
  for (int ks = 1; ks <= LOG2N; ++ks) {
    const int k = 1 << ks;
#pragma unroll
    for (int js = ks - 1; js >= 0; --js) {
      const int j = 1 << js;
      if (j < E) {  // partner in this thread's registers
#pragma unroll
        for (int r = 0; r < E; ++r) {
          if ((r & j) == 0) {
            const int x = tid * E + r;
            const bool desc = (x & k) == 0;  // this block of k ends descending
            const unsigned long long a = v[r], b = v[r + j];
            v[r] = cas(a, b, desc);
            v[r + j] = cas(a, b, !desc);
          }
        }
      } else if (j < 32 * E) {  // partner in this warp: lane ^ (j / E)
        const int m = j / E;
#pragma unroll
        for (int r = 0; r < E; ++r) {
          const int x = tid * E + r;
          const unsigned olo = __shfl_xor_sync(0xffffffffu, (unsigned)v[r], m);
          const unsigned ohi = __shfl_xor_sync(0xffffffffu, (unsigned)(v[r] >> 32), m);
          const unsigned long long o = ((unsigned long long)ohi << 32) | olo;
          v[r] = cas(v[r], o, ((x & k) == 0) == ((x & j) == 0));  // the lower of the pair keeps the max in a descending block
        }
      } else {  // partner in another warp: through shared memory
#pragma unroll
        for (int r = 0; r < E; ++r) keys[tid * E + r] = v[r];
        __syncthreads();
#pragma unroll
        for (int r = 0; r < E; ++r) {
          const int x = tid * E + r;
          v[r] = cas(v[r], keys[x ^ j], ((x & k) == 0) == ((x & j) == 0));
        }
        __syncthreads();
      }
    }
  }
#pragma unroll
  for (int r = 0; r < E; ++r) {
    const int x = tid * E + r;
    e[x] = __uint_as_float((unsigned)(v[r] >> 32));
    id[x] = (int)(0xFFFFFFFFu - (unsigned)v[r]);
  }
  __syncthreads();
}

template <int EMAX>  // the largest E = N / 256 of the launch's rows
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
  int NB2 = kSelThreads;  // sort size: a power of two >= nK, at least one key a thread
  while (NB2 < nK) NB2 <<= 1;
  float* e = reinterpret_cast<float*>(smraw);   // [NB2] masses (rank order after the sort)
  int* id = reinterpret_cast<int*>(e + NB2);    // [NB2] block ids (rank order after the sort)
  int* flag = id + NB2;                          // [NB2]
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(smraw);  // [NB2], over e and id

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
    if (j < nK) e[j] = expf(e[j] - m);
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
  // NB2 <= EMAX x 256 (the launch's largest row); only the sizes up to it are built,
  // so that a launch of short rows keeps few registers a thread.  Rows longer than the
  // register network takes (kMaxSortKeys) rank with block-wide passes in shared memory.
  const int E = NB2 / kSelThreads;
  if (NB2 > kMaxSortKeys) {
    for (int j = tid; j < NB2; j += kSelThreads) {
      id[j] = j < nK ? j : INT_MAX;
      if (j >= nK) e[j] = -1.0f;  // padding ranks last
    }
    __syncthreads();
    for (int k = 2; k <= NB2; k <<= 1) {
      for (int jj = k >> 1; jj > 0; jj >>= 1) {
        for (int x = tid; x < NB2; x += kSelThreads) {
          const int y = x ^ jj;
          if (y > x) {
            const bool before = e[x] > e[y] || (e[x] == e[y] && id[x] < id[y]);
            if (((x & k) == 0) != before) {
              const float te = e[x]; e[x] = e[y]; e[y] = te;
              const int ti = id[x]; id[x] = id[y]; id[y] = ti;
            }
          }
        }
        __syncthreads();
      }
    }
  } else if (E == 1) rank_masses<1>(e, id, nK, keys);
  else if constexpr (EMAX >= 2) {
    if (E == 2) rank_masses<2>(e, id, nK, keys);
    else if constexpr (EMAX >= 4) {
      if (E == 4) rank_masses<4>(e, id, nK, keys);
      else if constexpr (EMAX >= 8) {
        if (E == 8) rank_masses<8>(e, id, nK, keys);
        else if constexpr (EMAX >= 16) rank_masses<16>(e, id, nK, keys);
      }
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
  int nmax = joint ? nKc + nKq : (nKc > nKq ? nKc : nKq), NB2 = kSelThreads;
  while (NB2 < nmax) NB2 <<= 1;
  const size_t smem = (size_t)NB2 * 12;
  const int grid = joint ? H * nQ64 : H * (nQ128 + nQ64);
  auto go = [&](auto kernel) -> cudaError_t {
    if (smem > kDefaultSmemOptIn) {
      const cudaError_t r = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (r != cudaSuccess) return r;
    }
    kernel<<<grid, kSelThreads, smem, s>>>(scores, tau, H, nQ128, nKc, nQ64, nKq, joint, inter_idx, inter_cnt,
                                           intra_idx, intra_cnt);
    return cudaGetLastError();
  };
  switch (NB2 / kSelThreads) {
    case 1: return go(block_select_kernel<1>);
    case 2: return go(block_select_kernel<2>);
    case 4: return go(block_select_kernel<4>);
    case 8: return go(block_select_kernel<8>);
    default: return go(block_select_kernel<16>);
  }
}

}  // namespace hsa
