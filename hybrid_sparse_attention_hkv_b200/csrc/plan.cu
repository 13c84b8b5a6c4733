// Work plan of the attention kernel (one CTA).
//
// The cost of a (head, 128-query tile) is its kept cached blocks plus half its
// kept chunk blocks (64 rows each; the sum of its two halves' counts, an upper
// bound on their union).  A list whose cost exceeds a segment length S -- the
// step's cost per SM divided by kPlanUnitsPerSM -- is cut into ceil(cost / S)
// segments; the kernel cuts its actual tile list at the same fractions of its
// cost.  Units are ordered head by head, the costliest head first, and within a
// head by query tile: the CTAs running at one time then share a few heads' K/V in
// L2, and the hardware's in-order CTA dispatch starts the long heads first.  The
// order of units does not change any result: each unit writes its own output rows
// or its own partial slot, and the slots of a list are merged in segment order.
#include "common.cuh"
#include "kernels.h"

namespace hsa {
namespace {

constexpr int kPlanThreads = 1024;
constexpr int kPlanMaxHeads = 512;
constexpr size_t kPlanMaxSmem = 160 * 1024;  // three ints per (head, query tile)

// Block-wide exclusive scan of one int per thread (kPlanThreads threads).
__device__ int block_exclusive_scan(int v, int* s_warp, int& total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) s_warp[w] = incl;
  __syncthreads();
  if (w == 0) {
    int x = s_warp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += t;
    }
    s_warp[lane] = x;  // inclusive prefix of warp totals
  }
  __syncthreads();
  const int before = (w > 0 ? s_warp[w - 1] : 0) + incl - v;
  total = s_warp[kPlanThreads / 32 - 1];
  __syncthreads();
  return before;
}

// Cost of (head, query tile) i in 128-row tile units (x2, to count chunk tiles exactly).
__device__ __forceinline__ int cost2(const AttnArgs& a, int i, int nQ128, int nQ64, int nKc, int nKq) {
  const int h = i / nQ128, qb = i % nQ128;
  int ni = 0;
  if (a.joint) {  // inter lists per 64-query half: their sum bounds the union
    for (int half = 0; half < 2; ++half) {
      const int i64 = 2 * qb + half;
      if (i64 < nQ64) ni += min(max(a.inter_cnt[(long long)h * nQ64 + i64], 0), nKc);
    }
    ni = min(ni, nKc);
  } else {
    ni = min(max(a.inter_cnt[i], 0), nKc);
  }
  int nc = 0;
  for (int half = 0; half < 2; ++half) {
    const int i64 = 2 * qb + half;
    if (i64 < nQ64) nc += min(max(a.intra_cnt[(long long)h * nQ64 + i64], 0), nKq);
  }
  return 2 * ni + nc;
}

__global__ void __launch_bounds__(kPlanThreads) attn_plan_kernel(const AttnArgs a, int nQ128, int nQ64, int nKc,
                                                                 int nKq) {
  __shared__ int head_units[kPlanMaxHeads], head_rank[kPlanMaxHeads], head_order[kPlanMaxHeads],
      head_start[kPlanMaxHeads];
  __shared__ unsigned long long head_cost[kPlanMaxHeads];
  extern __shared__ int list_scratch[];  // [3][HQ]
  int* list_slot = list_scratch;
  int* list_pre = list_scratch + a.H * nQ128;
  int* list_cost = list_scratch + 2 * a.H * nQ128;
  __shared__ int s_warp[32];
  __shared__ long long s_sum[32];
  __shared__ int s_seg, s_units, s_slots;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int HQ = a.H * nQ128;
  // 1. total cost -> segment length S (in cost2 units)
  long long t = 0;
  for (int i = tid; i < HQ; i += kPlanThreads) {
    const int c2 = cost2(a, i, nQ128, nQ64, nKc, nKq);
    list_cost[i] = c2;
    t += c2;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  if (lane == 0) s_sum[w] = t;
  __syncthreads();
  if (tid == 0) {
    long long tot = 0;
    for (int k = 0; k < kPlanThreads / 32; ++k) tot += s_sum[k];
    const long long per_sm = (tot + kPlanSMs - 1) / kPlanSMs;
    s_seg = (int)max(2LL * kPlanMinSegment, (per_sm + kPlanUnitsPerSM - 1) / kPlanUnitsPerSM);
    s_units = 0;
    s_slots = 0;
  }
  __syncthreads();
  const int S = s_seg;
  // 2. segments per list; per-head unit counts and costs; exclusive prefix P(i) of
  //    unit counts over lists (kept for the head starts); first slots of split lists
  for (int i = tid; i < a.H; i += kPlanThreads) {
    head_units[i] = 0;
    head_cost[i] = 0;
  }
  __syncthreads();
  for (int c = 0; c < HQ; c += kPlanThreads) {
    const int i = c + tid;
    const int c2 = i < HQ ? list_cost[i] : 0;
    const int nseg = i < HQ ? max(1, (c2 + S - 1) / S) : 0;
    int stot, utot;
    const int slot = block_exclusive_scan(nseg > 1 ? nseg : 0, s_warp, stot) + s_slots;
    const int upre = block_exclusive_scan(nseg, s_warp, utot) + s_units;
    if (i < HQ) {
      const int h = i / nQ128;
      a.tile_done[i] = 0;
      list_slot[i] = nseg > 1 ? slot : -1;  // scratch: first slot, then unit prefix below
      list_pre[i] = upre;
      atomicAdd(&head_units[h], nseg);
      atomicAdd(&head_cost[h], (unsigned long long)c2);
    }
    __syncthreads();
    if (tid == 0) {
      s_slots += stot;
      s_units += utot;
    }
    __syncthreads();
  }
  if (s_units > a.max_units || s_slots > a.max_slots) {
    if (tid == 0) {
      set_status(a.status, HSA_ERR_DEVICE);
      *a.n_units = 0;
    }
    return;
  }
  // 3. head order: costliest first (ties: lower head); head_start = units before it
  for (int h = tid; h < a.H; h += kPlanThreads) {
    int rank = 0;
    for (int o = 0; o < a.H; ++o)
      rank += head_cost[o] > head_cost[h] || (head_cost[o] == head_cost[h] && o < h);
    head_rank[h] = rank;
  }
  __syncthreads();
  if (tid == 0) {
    for (int h = 0; h < a.H; ++h) head_order[head_rank[h]] = h;
    int run = 0;
    for (int k = 0; k < a.H; ++k) {
      head_start[head_order[k]] = run;
      run += head_units[head_order[k]];
    }
  }
  __syncthreads();
  // 4. place the units
  for (int i = tid; i < HQ; i += kPlanThreads) {
    const int h = i / nQ128;
    const int nseg = max(1, (list_cost[i] + S - 1) / S);
    const int pos = head_start[h] + list_pre[i] - list_pre[h * nQ128];
    for (int k = 0; k < nseg; ++k) a.units[pos + k] = make_int4(i, k, nseg, list_slot[i]);
  }
  if (tid == 0) *a.n_units = s_units;
}

}  // namespace

cudaError_t launch_attn_plan(const AttnArgs& a, cudaStream_t s) {
  const int nQ128 = (a.Lq + 127) / 128, nQ64 = (a.Lq + 63) / 64;
  const int nKc = (int)((a.Lc + 127) / 128), nKq = nQ64;
  if (a.H > kPlanMaxHeads) return cudaErrorInvalidConfiguration;
  const size_t smem = (size_t)3 * a.H * nQ128 * sizeof(int);
  if (smem > kPlanMaxSmem) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(attn_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  attn_plan_kernel<<<1, kPlanThreads, smem, s>>>(a, nQ128, nQ64, nKc, nKq);
  return cudaGetLastError();
}

}  // namespace hsa
