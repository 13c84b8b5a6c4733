// HSA attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA): the
// block-sparse branch, the Linformer branch and their gated merge in one kernel
// ("WorldAttention pairs hierarchical KV caching with hybrid sparse attention..."
// news summary, HSA paragraph: exact attention over each head's kept blocks, a
// low-rank linear global branch, learned gates merging the two).
//
// One CTA per work unit (plan.cu): a segment of the key-tile list of one (head,
// 128-query tile).  The list, in order:
//   linear tiles  64 rows of EK / FV (split bf16 hi + lo), r / 64 of them, in
//                 segment 0 only;
//   cached tiles  one 128-row tile per kept inter block of the cached KV (with the
//                 joint block selection, the union of the two 64-query halves'
//                 inter lists, each tile tagged with the halves that keep it);
//   chunk tiles   the union of the two 64-query halves' kept 64-row intra blocks,
//                 each tagged with the halves that use it; blocks with the same tag
//                 are paired into 128-row tiles (two 64-row boxes in one slot), so
//                 that a chunk block costs half a tile's fixed pipeline latency.
// A segment takes the sparse tiles whose cumulative cost (2 per 128-row tile, 1 per
// lone 64-row chunk tile) falls in its share of the list's cost.  A unit covering its whole
// list writes the output; a segment of a split list writes its unnormalised O_s
// with its running (max, sum) to a partial slot (segment 0 adds the weighted
// linear branch), and the CTA that finishes the list's last segment merges the
// slots in segment order.
// 7 warps:
//   warp 0      TMA producer of the Q tile (once) and of each key tile's K part
//               (K, or EK_hi + EK_lo) into a 3-slot ring of 128-byte-swizzled
//               buffers (a slot frees when its S MMA ends);
//   warp 6      TMA producer of the V parts (V, or FV_hi + FV_lo) into a 2-slot
//               ring (a slot frees when its P.V MMA ends);
//   warp 1      MMA issuer (one elected lane): S_j = Q K_j^T (+ Q EK_lo^T) into one of two
//               TMEM S buffers, then O += P_j V_j with P_j read from TMEM (written
//               over S_j; for linear tiles P_hi FV_hi + P_lo FV_hi + P_hi FV_lo
//               into a second accumulator O_l);
//   warps 2-5   softmax, one TMEM lane (= query row) per thread, one running
//               max / sum per branch: exp2, row sums, P as packed bf16 back into
//               TMEM; the running max is raised (and that O rescaled in TMEM) only
//               when it grows by more than 2^8; finally o_s = O_s / l_s,
//               o_l = O_l / l_l, out = g o_s + (1 - g) o_l, stored.
// The tensor core computes S_{j+1} while the softmax warps work on S_j.
// Every wait is bounded (HSA_ERR_TIMEOUT in the workspace status on expiry) and names
// its site (kind << 24 | warp << 16 | tile), recorded for the first wait of the
// workspace that runs out.  The softmax warps' per-tile waits are per-lane (a
// warp-wide vote after each of them cost 7% of the kernel's time); the producers, the
// MMA warp, which issues with elect.sync, and the waits before the first and after the
// last tile, where the warps go on to warp-collective TMEM access and teardown, take
// the warp's common answer.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace hsa {
using namespace sm100;

namespace {

constexpr int kTcThreads = 224;  // 7 warps
constexpr int kKStages = 3;      // K ring: a slot frees as soon as its S MMA completes
constexpr int kVStages = 2;      // V ring: a slot frees when its P.V MMA completes
constexpr int kRegionBytes = 128 * 128;  // one [128 rows x 64 bf16] swizzled region
// wait sites (header word 4 of the first wait that runs out: kind << 24 | warp << 16 | tile)
constexpr int kSiteKEmpty = 1, kSiteVEmpty = 2, kSiteQ = 3, kSiteKFull = 4, kSitePFull = 6, kSiteVFull = 7,
              kSiteSFull = 8, kSiteODone = 13;
__device__ __forceinline__ int wait_site(int kind, int warp, int j) { return (kind << 24) | (warp << 16) | (j & 0xFFFF); }

struct TcMaps {
  CUtensorMap q, kc, vc, kq, vq, ekhi, eklo, fvhi, fvlo;
};

// Key-tile code: (first row << 4) | (type << 2) | half-mask; a pair of chunk blocks
// ja < jb (64-row block ids < 8192): (ja << 17) | (jb << 4) | (type << 2) | half-mask.
constexpr int kTileCached = 0;  // 128 rows of Kc / Vc
constexpr int kTileChunk = 1;   // 64 rows of Kq / Vq
constexpr int kTileLinear = 2;  // 64 rows of EK / FV (hi + lo)
constexpr int kTilePair = 3;    // two 64-row blocks of Kq / Vq used by the same query halves

template <int D>
struct TcLayout {
  static constexpr int kQBytes = (D / 64) * kRegionBytes;
  static constexpr int kKVBytes = (D / 64) * kRegionBytes;  // one 128-row K or V tile
  static constexpr int kBytes = kQBytes + (kKStages + kVStages) * kKVBytes;
};

__device__ __forceinline__ int tc_tile_code(long long start, int type, int mask) {
  return (int)(start << 4) | (type << 2) | mask;
}
__device__ __forceinline__ int tile_type(int code) { return (code >> 2) & 3; }
__device__ __forceinline__ int tile_start(int code) { return code >> 4; }
__device__ __forceinline__ int tile_rows(int code) {
  const int t = tile_type(code);
  return (t == kTileCached || t == kTilePair) ? 128 : 64;
}
__device__ __forceinline__ int pair_code(int ja, int jb, int mask) {
  return (ja << 17) | (jb << 4) | (kTilePair << 2) | mask;
}
__device__ __forceinline__ int pair_first(int code) { return code >> 17; }
__device__ __forceinline__ int pair_second(int code) { return (code >> 4) & 0x1FFF; }

// 16 output values of row `grow`, head h, columns [16c, 16c + 16), fp32 or bf16.
__device__ __forceinline__ void store_out16(const AttnArgs& a, int grow, int h, int D, int c, const float (&v)[16]) {
  const long long idx = ((long long)grow * a.H + h) * D + c * 16;
  if (a.out_bf16) {
    uint4 w0, w1;
    w0.x = pack_bf16x2(v[0], v[1]); w0.y = pack_bf16x2(v[2], v[3]);
    w0.z = pack_bf16x2(v[4], v[5]); w0.w = pack_bf16x2(v[6], v[7]);
    w1.x = pack_bf16x2(v[8], v[9]); w1.y = pack_bf16x2(v[10], v[11]);
    w1.z = pack_bf16x2(v[12], v[13]); w1.w = pack_bf16x2(v[14], v[15]);
    *reinterpret_cast<uint4*>(a.out_bf16 + idx) = w0;
    *reinterpret_cast<uint4*>(a.out_bf16 + idx + 8) = w1;
  } else {
#pragma unroll
    for (int k = 0; k < 16; k += 4)
      *reinterpret_cast<float4*>(a.out_f32 + idx + k) = make_float4(v[k], v[k + 1], v[k + 2], v[k + 3]);
  }
}

// ------------------------------------------------------------------ kernel
// Online-softmax step of one query row over one key tile of ROWS columns held in
// sr[] (raw scores): update the running max m (raised only when it grows by more
// than 2^8, returning the factor alpha for O), write P = 2^(s*sl2 - m) as packed
// bf16 pairs over the first ROWS/2 columns of the S buffer, and fold the row sum
// into l.  MASKED: only the first `valid` keys exist.
__device__ __forceinline__ float fmax3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
template <int ROWS, bool MASKED>
__device__ __forceinline__ void softmax_tile(const uint32_t (&sr)[128], int valid, float sl2, float& m, float& l,
                                             float& alpha, bool& rescale, uint32_t tS) {
  float pm[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) pm[q] = -INFINITY;
  if (MASKED) {
#pragma unroll
    for (int k = 0; k < ROWS; ++k)
      if (k < valid) pm[k & 7] = fmaxf(pm[k & 7], __uint_as_float(sr[k]));
  } else {
#pragma unroll
    for (int k = 0; k < ROWS; k += 2) pm[(k >> 1) & 7] = fmax3f(pm[(k >> 1) & 7], __uint_as_float(sr[k]), __uint_as_float(sr[k + 1]));
  }
  const float mx = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])), fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
  const float mn = mx * sl2;
  if (mn > m + 8.f) {
    if (m != -INFINITY) {
      alpha = ex2_approx(m - mn);
      rescale = true;
    }
    m = mn;
  }
  const float2 a2 = make_float2(sl2, sl2), b2 = make_float2(-m, -m);
  float2 acc[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < ROWS / 32; ++c) {
    uint32_t pk[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int i = c * 32 + 2 * k;
      const float2 t = __ffma2_rn(make_float2(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])), a2, b2);
      // every exp2 on the SFU: the softmax is bound by its latency, not by the SFU's
      // throughput, so moving some to a polynomial on the FMA pipe (measured: a quarter,
      // an eighth) lengthens it
      float p0 = ex2_approx(t.x), p1 = ex2_approx(t.y);
      if (MASKED) {
        if (i >= valid) p0 = 0.f;
        if (i + 1 >= valid) p1 = 0.f;
      }
      acc[k & 3] = __fadd2_rn(acc[k & 3], make_float2(p0, p1));
      pk[k] = pack_bf16x2(p0, p1);
    }
    tmem_st16(tS + c * 16, pk);  // P (bf16 pairs) over the first half of S
  }
  const float2 s01 = __fadd2_rn(acc[0], acc[1]), s23 = __fadd2_rn(acc[2], acc[3]);
  const float2 st = __fadd2_rn(s01, s23);
  l = l * alpha + (st.x + st.y);
}

// Linear-branch variant over 64 projected rows (no masking): P is written as two
// bf16 parts, hi = bf16(p) over columns [0, 32) and lo = bf16(p - hi) over
// [32, 64) of the S buffer, so that P.FV keeps about 16 significant bits.
__device__ __forceinline__ void softmax_tile_split(const uint32_t (&sr)[64], float sl2, float& m, float& l,
                                                   float& alpha, bool& rescale, uint32_t tS) {
  float pm[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) pm[q] = -INFINITY;
#pragma unroll
  for (int k = 0; k < 64; ++k) pm[k & 7] = fmaxf(pm[k & 7], __uint_as_float(sr[k]));
  const float mx = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])), fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
  const float mn = mx * sl2;
  if (mn > m + 8.f) {
    if (m != -INFINITY) {
      alpha = ex2_approx(m - mn);
      rescale = true;
    }
    m = mn;
  }
  const float2 a2 = make_float2(sl2, sl2), b2 = make_float2(-m, -m);
  float2 acc[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    uint32_t hi[16], lo[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int i = c * 32 + 2 * k;
      const float2 t = __ffma2_rn(make_float2(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])), a2, b2);
      const float p0 = ex2_approx(t.x), p1 = ex2_approx(t.y);
      acc[k & 3] = __fadd2_rn(acc[k & 3], make_float2(p0, p1));
      __nv_bfloat16 h0, l0, h1, l1;
      split_bf16(p0, h0, l0);
      split_bf16(p1, h1, l1);
      hi[k] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
      lo[k] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
    }
    tmem_st16(tS + c * 16, hi);
    tmem_st16(tS + 32 + c * 16, lo);
  }
  const float2 s01 = __fadd2_rn(acc[0], acc[1]), s23 = __fadd2_rn(acc[2], acc[3]);
  const float2 st = __fadd2_rn(s01, s23);
  l = l * alpha + (st.x + st.y);
}

// MMA issue by the whole MMA warp (one elected lane issues), every loop unrolled at
// compile time: the descriptors of one tile are its base descriptor plus constant
// address offsets (in 16-byte units, the descriptor's low field), so consecutive
// MMAs issue back to back.
// S (+)= Q K^T over D / 16 steps of 16; K tile of ROWS rows (K-major, 128-byte swizzle).
template <int D, int ROWS>
__device__ __forceinline__ void issue_qk(uint32_t tS, uint64_t qd, uint64_t kd, bool accumulate_first) {
  constexpr uint32_t idesc = idesc_bf16(128, ROWS, false, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t qo = (uint64_t)(((kk / 4) * kRegionBytes + (kk % 4) * 32) >> 4);
    const uint64_t ko = (uint64_t)(((kk / 4) * (ROWS * 128) + (kk % 4) * 32) >> 4);
    mma_ss_elect(tS, qd + qo, kd + ko, idesc, (accumulate_first || kk > 0) ? 1u : 0u);
  }
}
// O (+)= P V over ROWS / 16 steps; P from TMEM, V tile of ROWS rows (MN-major).
template <int D, int ROWS>
__device__ __forceinline__ void issue_pv(uint32_t tO, uint32_t tP, uint64_t vd, bool accumulate_first) {
  constexpr uint32_t idesc = idesc_bf16(128, D, false, true);
#pragma unroll
  for (int kk = 0; kk < ROWS / 16; ++kk)
    mma_ts_elect(tO, tP + kk * 8, vd + (uint64_t)((kk * 2048) >> 4), idesc, (accumulate_first || kk > 0) ? 1u : 0u);
}

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
    sparse_attn_tc_kernel(const __grid_constant__ TcMaps maps, const AttnArgs a, int nQ128, int nKc, int nQ64,
                          int nKq) {
  using Lay = TcLayout<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = smem;
  unsigned char* sK = smem + Lay::kQBytes;                    // [kKStages] K tiles
  unsigned char* sV = sK + kKStages * Lay::kKVBytes;          // [kVStages] V tiles
  int* tiles = reinterpret_cast<int*>(smem + Lay::kBytes);  // [r/64 + nKc + nKq]
  int* flags = tiles + (a.EKhi ? a.r / 64 : 0) + nKc + nKq; // [nKq]
  int* scratch = flags + nKq;                                 // [nKq]
  int* flagc = scratch + nKq;                                 // [nKc] (joint selection)
  __shared__ __align__(8) uint64_t bar_q, bar_k_full[kKStages], bar_k_empty[kKStages], bar_v_full[kVStages],
      bar_v_empty[kVStages], bar_s_full[2], bar_p_full[2], bar_o_done, bar_final;
  __shared__ uint32_t s_tmem;
  __shared__ int s_ntiles, s_n2, s_ninter;

  __shared__ int s_last;

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  int* status = a.status;
  const uint64_t wlim = wait_limit_ns(status);
  const int HQ = a.H * nQ128;
  const bool planned = a.units != nullptr;
  // both loads in flight together (units[] holds the grid's max_units entries)
  const int4 unit = planned ? a.units[blockIdx.x] : make_int4((int)blockIdx.x, 0, 1, -1);
  const int n_units = planned ? *a.n_units : HQ;
  if ((int)blockIdx.x >= n_units) return;  // spare CTA of the upper-bound grid
  const int tq = unit.x, seg = unit.y, nseg = unit.z, slot0 = unit.w;
  if (tq < 0 || tq >= HQ || nseg < 1 || seg < 0 || seg >= nseg ||
      (nseg > 1 && (slot0 < 0 || slot0 + nseg > a.max_slots))) {
    if (tid == 0) set_status(status, HSA_ERR_DEVICE);
    return;
  }
  const int qb = tq % nQ128, h = tq / nQ128;
  const int q0 = qb * 128;

  if (warp == 0) {
    tmem_alloc(&s_tmem, 512);
    tmem_relinquish();
  }
  if (tid == 32) {
    mbar_init(&bar_q, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&bar_k_full[s], 1);
      mbar_init(&bar_k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&bar_v_full[s], 1);
      mbar_init(&bar_v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar_s_full[b], 1);
      mbar_init(&bar_p_full[b], 128);
    }
    mbar_init(&bar_o_done, 1);
    mbar_init(&bar_final, 1);
    fence_barrier_init();
  }

  // ---- key-tile list (linear tiles, cached tiles, chunk tiles).  Selection counts
  // and ids come from caller buffers: counts are clamped, out-of-range ids skipped.
  const bool any_lin = a.EKhi != nullptr;
  const bool do_lin = any_lin && seg == 0;  // the linear tiles belong to segment 0
  const bool do_sparse = a.inter_cnt != nullptr;
  const int n_lin = do_lin ? a.r / 64 : 0;
  const int n_inter0 = (do_sparse && !a.joint) ? min(max(a.inter_cnt[(long long)h * nQ128 + qb], 0), nKc) : 0;
  for (int t = tid; t < n_lin; t += kTcThreads) tiles[t] = tc_tile_code((long long)t * 64, kTileLinear, 3);
  if (do_sparse) {
    const int32_t* ilist = a.inter_idx + ((long long)h * nQ128 + qb) * nKc;
    for (int m = tid; m < n_inter0; m += kTcThreads) {
      const long long j = ilist[m];
      const bool ok = j >= 0 && j < nKc;
      if (!ok) set_status(status, HSA_ERR_DEVICE);
      tiles[n_lin + m] = ok ? tc_tile_code(j * 128, kTileCached, 3) : tc_tile_code(0, kTileCached, 0);
    }
    for (int j = tid; j < nKq; j += kTcThreads) flags[j] = 0;
    if (a.joint)
      for (int j = tid; j < nKc; j += kTcThreads) flagc[j] = 0;
  }
  __syncthreads();
  if (do_sparse && a.joint) {  // the two 64-query halves' inter lists
    for (int half = 0; half < 2; ++half) {
      const int i64 = 2 * qb + half;
      if (i64 < nQ64) {
        const int cnt = min(max(a.inter_cnt[(long long)h * nQ64 + i64], 0), nKc);
        const int32_t* lst = a.inter_idx + ((long long)h * nQ64 + i64) * nKc;
        for (int m = tid; m < cnt; m += kTcThreads) {
          const int j = lst[m];
          if (j >= 0 && j < nKc) atomicOr(&flagc[j], 1 << half);
          else set_status(status, HSA_ERR_DEVICE);
        }
      }
    }
  }
  if (do_sparse) {
    for (int half = 0; half < 2; ++half) {
      const int i64 = 2 * qb + half;
      if (i64 < nQ64) {
        const int cnt = min(max(a.intra_cnt[(long long)h * nQ64 + i64], 0), nKq);
        const int32_t* lst = a.intra_idx + ((long long)h * nQ64 + i64) * nKq;
        for (int m = tid; m < cnt; m += kTcThreads) {
          const int j = lst[m];
          if (j >= 0 && j < nKq) atomicOr(&flags[j], 1 << half);
          else set_status(status, HSA_ERR_DEVICE);
        }
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    int n_inter = n_inter0;
    if (do_sparse && a.joint) {  // cached blocks kept by either half, ascending, tagged
      n_inter = 0;
      for (int b = 0; b < nKc; b += 32) {
        const int j = b + lane;
        const int f = j < nKc ? flagc[j] : 0;
        const unsigned bal = __ballot_sync(0xffffffffu, f != 0);
        if (f) tiles[n_lin + n_inter + __popc(bal & ((1u << lane) - 1u))] = tc_tile_code((long long)j * 128, kTileCached, f);
        n_inter += __popc(bal);
      }
    }
    // chunk blocks by tag (both halves, half 0 only, half 1 only), ascending within a
    // tag, paired; a tag's odd block out stays a 64-row tile at the end of the list.
    // The partial last block (the largest id) is always the second of its pair.
    int base = n_lin + n_inter;
    int single[3] = {-1, -1, -1};
    if (do_sparse) {
      for (int c = 0; c < 3; ++c) {
        const int tag = c == 0 ? 3 : c;
        int cnt = 0;
        for (int b = 0; b < nKq; b += 32) {
          const int j = b + lane;
          const bool in = j < nKq && flags[j] == tag;
          const unsigned bal = __ballot_sync(0xffffffffu, in);
          if (in) scratch[cnt + __popc(bal & ((1u << lane) - 1u))] = j;
          cnt += __popc(bal);
        }
        __syncwarp();
        for (int k = lane; k < cnt / 2; k += 32) tiles[base + k] = pair_code(scratch[2 * k], scratch[2 * k + 1], tag);
        base += cnt / 2;
        if (cnt & 1) single[c] = scratch[cnt - 1];
        __syncwarp();
      }
    }
    const int n2 = base - n_lin;  // 128-row sparse tiles: cached + pairs
    for (int c = 0; c < 3; ++c) {
      if (single[c] >= 0) {
        if (lane == 0) tiles[base] = tc_tile_code((long long)single[c] * 64, kTileChunk, c == 0 ? 3 : c);
        ++base;
      }
    }
    if (lane == 0) {
      s_ntiles = base;
      s_n2 = n2;
      s_ninter = n_inter;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // this segment's share of the sparse tiles, by cost (a 128-row tile costs 2, a lone
  // 64-row chunk tile 1; the 128-row tiles come first)
  const int n2 = s_n2;
  const int n_inter = s_ninter;
  const int n1 = s_ntiles - n_lin - n2;
  const long long cost = 2LL * n2 + n1;
  auto cut = [&](long long x) -> int {  // sparse tiles whose cumulative cost before them is < x
    return x <= 2LL * n2 ? (int)((x + 1) / 2) : n2 + (int)(x - 2LL * n2);
  };
  const int t0 = cut(cost * seg / nseg), t1 = cut(cost * (seg + 1) / nseg);
  const int T = n_lin + (t1 - t0);
  // tile j of this unit: the linear tiles, then sparse tiles t0 .. t1 - 1
  auto tile_at = [&](int j) -> int { return j < n_lin ? tiles[j] : tiles[j + t0]; };
  if (T == 0 && nseg == 1 && tid == 0) set_status(status, HSA_ERR_DEVICE);  // no key tile: empty selection
  const uint32_t tmem = s_tmem;
  const uint32_t tOs = tmem + 256, tOl = tmem + 256 + D;
  constexpr int kHalfSlot = (D / 64) * 64 * 128;  // 64 rows x D bf16: hi part / lo part of a slot

  if (warp == 0) {
    // ------------------------------------------------------------ Q + K producer
    if (lane == 0) {
      prefetch_tensormap(&maps.q);
      mbar_arrive_expect_tx(&bar_q, Lay::kQBytes);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) tma_load_2d(sQ + c * kRegionBytes, &maps.q, &bar_q, h * D + c * 64, q0);
    }
    for (int j = 0; j < T; ++j) {
      const int s = j % kKStages;
      if (!mbar_wait_warp(&bar_k_empty[s], ((j / kKStages) & 1) ^ 1, status, wlim, wait_site(kSiteKEmpty, warp, j)))
        break;
      if (lane == 0) {
        const int code = tile_at(j);
        const int type = tile_type(code);
        const int rows = tile_rows(code);
        unsigned char* dK = sK + s * Lay::kKVBytes;
        mbar_arrive_expect_tx(&bar_k_full[s], type == kTileLinear ? 2 * kHalfSlot : (D / 64) * rows * 128);
        if (type == kTileLinear) {
          const int y = h * a.r + tile_start(code);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            tma_load_2d(dK + c * 64 * 128, &maps.ekhi, &bar_k_full[s], c * 64, y);
            tma_load_2d(dK + kHalfSlot + c * 64 * 128, &maps.eklo, &bar_k_full[s], c * 64, y);
          }
        } else if (type == kTilePair) {  // rows 0-63 and 64-127 of the slot from two blocks
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            tma_load_2d(dK + c * 128 * 128, &maps.kq, &bar_k_full[s], h * D + c * 64, pair_first(code) * 64);
            tma_load_2d(dK + c * 128 * 128 + 64 * 128, &maps.kq, &bar_k_full[s], h * D + c * 64,
                        pair_second(code) * 64);
          }
        } else {
          const CUtensorMap* mk = type == kTileChunk ? &maps.kq : &maps.kc;
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_2d(dK + c * rows * 128, mk, &bar_k_full[s], h * D + c * 64, tile_start(code));
        }
      }
      __syncwarp();
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ V producer
    for (int j = 0; j < T; ++j) {
      const int s = j % kVStages;
      if (!mbar_wait_warp(&bar_v_empty[s], ((j / kVStages) & 1) ^ 1, status, wlim, wait_site(kSiteVEmpty, warp, j)))
        break;
      if (lane == 0) {
        const int code = tile_at(j);
        const int type = tile_type(code);
        const int rows = tile_rows(code);
        unsigned char* dV = sV + s * Lay::kKVBytes;
        mbar_arrive_expect_tx(&bar_v_full[s], type == kTileLinear ? 2 * kHalfSlot : (D / 64) * rows * 128);
        if (type == kTileLinear) {
          const int y = h * a.r + tile_start(code);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            tma_load_2d(dV + c * 64 * 128, &maps.fvhi, &bar_v_full[s], c * 64, y);
            tma_load_2d(dV + kHalfSlot + c * 64 * 128, &maps.fvlo, &bar_v_full[s], c * 64, y);
          }
        } else if (type == kTilePair) {
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            tma_load_2d(dV + c * 128 * 128, &maps.vq, &bar_v_full[s], h * D + c * 64, pair_first(code) * 64);
            tma_load_2d(dV + c * 128 * 128 + 64 * 128, &maps.vq, &bar_v_full[s], h * D + c * 64,
                        pair_second(code) * 64);
          }
        } else {
          const CUtensorMap* mv = type == kTileChunk ? &maps.vq : &maps.vc;
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_2d(dV + c * rows * 128, mv, &bar_v_full[s], h * D + c * 64, tile_start(code));
        }
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    bool ok = mbar_wait_warp(&bar_q, 0, status, wlim, wait_site(kSiteQ, warp, 0));
    tc_fence_after();
    const uint64_t qd = sdesc_sw128(smem_u32(sQ), 16, 1024);
    // The warp stays converged: waits take the warp's common answer, tile codes and
    // descriptors are warp-uniform, one elected lane issues each MMA and commit.
    // K and V arrive by TMA on their mbarriers, which orders them for the tensor
    // core; only P, written to TMEM by the softmax warps, needs the tcgen05 fence.
    auto issue_s = [&](int j) -> bool {
      const int s = j % kKStages;
      if (!mbar_wait_warp(&bar_k_full[s], (j / kKStages) & 1, status, wlim, wait_site(kSiteKFull, warp, j))) return false;
      const int code = tile_at(j);
      const uint64_t kd = sdesc_sw128(smem_u32(sK + s * Lay::kKVBytes), 16, 1024);
      const uint32_t tS = tmem + (j & 1) * 128;
      if (tile_type(code) == kTileLinear) {  // EK_hi then EK_lo, 64 rows each
        issue_qk<D, 64>(tS, qd, kd, false);
        issue_qk<D, 64>(tS, qd, kd + (uint64_t)(kHalfSlot >> 4), true);
      } else if (tile_rows(code) == 128) {
        issue_qk<D, 128>(tS, qd, kd, false);
      } else {
        issue_qk<D, 64>(tS, qd, kd, false);
      }
      mma_commit_elect(&bar_k_empty[s]);
      mma_commit_elect(&bar_s_full[j & 1]);
      return true;
    };
    if (ok && T > 0) ok = issue_s(0);
    for (int j = 0; ok && j < T; ++j) {
      if (j + 1 < T && !issue_s(j + 1)) break;
      if (!mbar_wait_warp(&bar_p_full[j & 1], (j >> 1) & 1, status, wlim, wait_site(kSitePFull, warp, j))) break;
      const int sv = j % kVStages;
      if (!mbar_wait_warp(&bar_v_full[sv], (j / kVStages) & 1, status, wlim, wait_site(kSiteVFull, warp, j))) break;
      tc_fence_after();
      const int code = tile_at(j);
      const uint32_t v_base = smem_u32(sV + sv * Lay::kKVBytes);
      const uint32_t tP = tmem + (j & 1) * 128;
      if (tile_type(code) == kTileLinear) {
        // O_l += P_hi FV_hi + P_lo FV_hi + P_hi FV_lo; first linear tile initialises O_l
        const uint64_t vhi = sdesc_sw128(v_base, 64 * 128, 1024);
        const uint64_t vlo = sdesc_sw128(v_base + kHalfSlot, 64 * 128, 1024);
        issue_pv<D, 64>(tOl, tP, vhi, j > 0);
        issue_pv<D, 64>(tOl, tP + 32, vhi, true);
        issue_pv<D, 64>(tOl, tP, vlo, true);
      } else if (tile_rows(code) == 128) {  // the first sparse tile initialises O_s
        issue_pv<D, 128>(tOs, tP, sdesc_sw128(v_base, 128 * 128, 1024), j > n_lin);
      } else {
        issue_pv<D, 64>(tOs, tP, sdesc_sw128(v_base, 64 * 128, 1024), j > n_lin);
      }
      mma_commit_elect(&bar_v_empty[sv]);
      mma_commit_elect(&bar_o_done);
      // one-shot: completes once every MMA of the unit has completed
      if (j == T - 1) mma_commit_elect(&bar_final);
    }
  } else if (warp >= 2 && warp <= 5) {
    // ------------------------------------------------------------ softmax + epilogue
    const int wq = warp & 3;
    const int row = 32 * wq + lane;
    const int half_bit = wq < 2 ? 1 : 2;  // warp-uniform: rows 0..63 are half 0
    const uint32_t loff = (uint32_t)(32 * wq) << 16;
    const float sl2 = a.scale * 1.4426950408889634f;
    float ms = -INFINITY, ls = 0.f;  // sparse branch running max / sum
    float ml = -INFINITY, ll = 0.f;  // linear branch running max / sum
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const int b = j & 1;
      if (!mbar_wait(&bar_s_full[b], (j >> 1) & 1, status, wlim, wait_site(kSiteSFull, warp, j))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int code = tile_at(j);
      const int type = tile_type(code);
      const int rows = tile_rows(code);
      const long long nrows = (type == kTileChunk || type == kTilePair) ? (long long)a.Lq : a.Lc;
      const int valid = type == kTileLinear ? 64
                        : type == kTilePair ? 64 + (int)min(64LL, nrows - 64LL * pair_second(code))
                                            : (int)min((long long)rows, nrows - tile_start(code));
      const bool used = (code & half_bit) != 0;
      const uint32_t tS = tmem + b * 128 + loff;
      float alpha = 1.f;
      bool rescale = false;
      if (type == kTileLinear) {  // tile-uniform
        uint32_t h64[64];
        tmem_ld64_sync(tS, h64);
        softmax_tile_split(h64, sl2, ml, ll, alpha, rescale, tS);
      } else if (used) {  // warp-uniform (a warp's 32 rows lie in one 64-row half)
        uint32_t sr[128];
        if (rows == 128) {
          tmem_ld128_sync(tS, sr);
          if (valid == 128) softmax_tile<128, false>(sr, valid, sl2, ms, ls, alpha, rescale, tS);
          else softmax_tile<128, true>(sr, valid, sl2, ms, ls, alpha, rescale, tS);
        } else {
          uint32_t h64[64];
          tmem_ld64_sync(tS, h64);
#pragma unroll
          for (int k = 0; k < 64; ++k) sr[k] = h64[k];
          if (valid == 64) softmax_tile<64, false>(sr, valid, sl2, ms, ls, alpha, rescale, tS);
          else softmax_tile<64, true>(sr, valid, sl2, ms, ls, alpha, rescale, tS);
        }
      } else {
        uint32_t zero[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) zero[k] = 0u;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (c * 32 < rows) tmem_st16(tS + c * 16, zero);
      }
      tmem_st_wait();
      if (__any_sync(0xffffffffu, rescale)) {
        // O holds the P.V products of tiles 0..j-1 once the last of them has completed
        // (P.V of tile j cannot have started: it waits for this P).  Without a rescale
        // nothing here touches O, and the wait is skipped.
        if (j > 0 && !mbar_wait(&bar_o_done, (j - 1) & 1, status, wlim, wait_site(kSiteODone, warp, j))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tO = type == kTileLinear ? tOl : tOs;
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          uint32_t r[16];
          tmem_ld16_sync(tO + loff + c * 16, r);
#pragma unroll
          for (int k = 0; k < 16; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * alpha);
          tmem_st16(tO + loff + c * 16, r);
        }
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(&bar_p_full[b]);
    }
    // Wait for every P.V product of the unit on the one-shot barrier the MMA warp
    // commits after its last P.V (phase 0, so the parity names it unambiguously; the
    // per-tile barrier can be up to two phases ahead or behind here).  The wait polls
    // (bounded): the softmax warps have no other work left, and sleeping waits here
    // cost 1 % of the kernel's time.
    auto wait_poll = [&](uint64_t* bar, uint32_t par) -> bool {
      bool r = false;
      for (uint32_t i = 0; i < kSpinLimit && !r; ++i) r = mbar_try_wait(bar, par);
      if (!r) set_status(status, HSA_ERR_TIMEOUT);
      return __all_sync(0xffffffffu, r);
    };
    if (ok && (T == 0 || wait_poll(&bar_final, 0))) {
      tc_fence_after();
      const int grow = q0 + row;
      const bool valid_row = grow < a.Lq;
      // out = g o_s + (1 - g) o_l with g = sigmoid(gate logit) when both branches run
      const float g = (do_sparse && any_lin && a.gate_logit) ? 1.f / (1.f + expf(-a.gate_logit[h])) : 1.f;
      const float wl = do_lin ? (do_sparse ? 1.f - g : 1.f) / ll : 0.f;
      if (nseg == 1) {
        if (do_sparse && valid_row && !(ls > 0.f)) set_status(status, HSA_ERR_DEVICE);
        const float ws = (do_sparse && ls > 0.f) ? g / ls : 0.f;
        if (do_sparse && valid_row && a.lse_out)  // ln sum_k exp(q.k * scale) = (m + log2 l) ln 2
          a.lse_out[(long long)grow * a.H + h] = ls > 0.f ? (ms + log2f(ls)) * 0.6931471805599453f : -INFINITY;
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          uint32_t rs[16], rl[16];
          if (do_sparse) tmem_ld16_sync(tOs + loff + c * 16, rs);
          if (do_lin) tmem_ld16_sync(tOl + loff + c * 16, rl);
          if (valid_row) {
            float v[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const float vs = do_sparse ? __uint_as_float(rs[k]) * ws : 0.f;
              const float vl = do_lin ? __uint_as_float(rl[k]) * wl : 0.f;
              v[k] = vs + vl;
            }
            store_out16(a, grow, h, D, c, v);
          }
        }
      } else {
        // one segment of a split list: unnormalised O_s and (max, sum); segment 0
        // also leaves the weighted linear branch at the list's first slot
        const int slot = slot0 + seg;
        float* po = a.part_o + ((long long)slot * 128 + row) * D;
        float* pl = a.part_lin + ((long long)slot0 * 128 + row) * D;
        const bool had_sparse = T > n_lin;
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          uint32_t rs[16], rl[16];
          if (had_sparse) tmem_ld16_sync(tOs + loff + c * 16, rs);
          if (do_lin) tmem_ld16_sync(tOl + loff + c * 16, rl);
          if (valid_row) {
#pragma unroll
            for (int k = 0; k < 16; k += 4) {
              *reinterpret_cast<float4*>(po + c * 16 + k) =
                  had_sparse ? make_float4(__uint_as_float(rs[k]), __uint_as_float(rs[k + 1]),
                                           __uint_as_float(rs[k + 2]), __uint_as_float(rs[k + 3]))
                             : make_float4(0.f, 0.f, 0.f, 0.f);
              if (do_lin)
                *reinterpret_cast<float4*>(pl + c * 16 + k) =
                    make_float4(__uint_as_float(rl[k]) * wl, __uint_as_float(rl[k + 1]) * wl,
                                __uint_as_float(rl[k + 2]) * wl, __uint_as_float(rl[k + 3]) * wl);
            }
          }
        }
        if (valid_row) a.part_ml[(long long)slot * 128 + row] = make_float2(had_sparse && ls > 0.f ? ms : -INFINITY, ls);
        __threadfence();
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (nseg > 1) {
    // the CTA that finishes a split list's last segment merges its segments, in
    // segment order (which CTA that is does not change the result)
    if (tid == 0) s_last = atomicAdd(&a.tile_done[tq], 1) == nseg - 1;
    __syncthreads();
    if (s_last && warp >= 2 && warp <= 5) {
      __threadfence();
      const int row = 32 * (warp & 3) + lane, grow = q0 + row;
      if (grow < a.Lq) {
        float M = -INFINITY;
        for (int k = 0; k < nseg; ++k) M = fmaxf(M, __ldcg(&a.part_ml[(long long)(slot0 + k) * 128 + row]).x);
        float L = 0.f;
        for (int k = 0; k < nseg; ++k) {
          const float2 m_l = __ldcg(&a.part_ml[(long long)(slot0 + k) * 128 + row]);
          if (m_l.x != -INFINITY) L += m_l.y * exp2f(m_l.x - M);
        }
        if (!(L > 0.f)) set_status(status, HSA_ERR_DEVICE);
        if (a.lse_out) a.lse_out[(long long)grow * a.H + h] = L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
        const float g = (any_lin && a.gate_logit) ? 1.f / (1.f + expf(-a.gate_logit[h])) : 1.f;
        const float ws = L > 0.f ? g / L : 0.f;
        const float* pl = a.part_lin + ((long long)slot0 * 128 + row) * D;
#pragma unroll 1
        for (int c = 0; c < D / 16; ++c) {
          float v[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) v[k] = 0.f;
          for (int sg = 0; sg < nseg; ++sg) {
            const float m_s = __ldcg(&a.part_ml[(long long)(slot0 + sg) * 128 + row]).x;
            if (m_s == -INFINITY) continue;  // no tile of this segment reaches the row
            const float w = exp2f(m_s - M);
            const float* po = a.part_o + ((long long)(slot0 + sg) * 128 + row) * D + c * 16;
#pragma unroll
            for (int k = 0; k < 16; k += 4) {
              const float4 o4 = __ldcg(reinterpret_cast<const float4*>(po + k));
              v[k] += o4.x * w; v[k + 1] += o4.y * w; v[k + 2] += o4.z * w; v[k + 3] += o4.w * w;
            }
          }
#pragma unroll
          for (int k = 0; k < 16; ++k) v[k] *= ws;
          if (any_lin) {
#pragma unroll
            for (int k = 0; k < 16; k += 4) {
              const float4 l4 = __ldcg(reinterpret_cast<const float4*>(pl + c * 16 + k));
              v[k] += l4.x; v[k + 1] += l4.y; v[k + 2] += l4.z; v[k + 3] += l4.w;
            }
          }
          store_out16(a, grow, h, D, c, v);
        }
      }
    }
  }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

cudaError_t get_encoder() {
  std::call_once(g_encode_once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode ? cudaSuccess : cudaErrorNotSupported;
}

// [rows, cols] bf16 row-major, boxes of 64 columns x box_rows rows, 128-byte swizzle.
cudaError_t make_map(CUtensorMap* m, const void* base, long long rows, long long cols, int box_rows) {
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int D>
cudaError_t launch_tc(const AttnArgs& a, cudaStream_t s) {
  const int nQ128 = (a.Lq + 127) / 128, nQ64 = (a.Lq + 63) / 64;
  const int nKc = (int)((a.Lc + 127) / 128), nKq = nQ64;
  cudaError_t e = get_encoder();
  if (e != cudaSuccess) return e;
  TcMaps maps;
  const long long HD = (long long)a.H * D;
  if ((e = make_map(&maps.q, a.Q, a.Lq, HD, 128)) != cudaSuccess) return e;
  if ((e = make_map(&maps.kq, a.Kq, a.Lq, HD, 64)) != cudaSuccess) return e;
  if ((e = make_map(&maps.vq, a.Vq, a.Lq, HD, 64)) != cudaSuccess) return e;
  // maps a launch never reads point at the chunk tensors
  const bool hist = a.Lc > 0 && a.Kc != nullptr;
  if ((e = make_map(&maps.kc, hist ? a.Kc : a.Kq, hist ? a.Lc : a.Lq, HD, 128)) != cudaSuccess) return e;
  if ((e = make_map(&maps.vc, hist ? a.Vc : a.Vq, hist ? a.Lc : a.Lq, HD, 128)) != cudaSuccess) return e;
  const bool lin = a.EKhi != nullptr;
  const long long pr = (long long)a.H * a.r;
  if ((e = make_map(&maps.ekhi, lin ? a.EKhi : a.Kq, lin ? pr : a.Lq, lin ? D : HD, 64)) != cudaSuccess) return e;
  if ((e = make_map(&maps.eklo, lin ? a.EKlo : a.Kq, lin ? pr : a.Lq, lin ? D : HD, 64)) != cudaSuccess) return e;
  if ((e = make_map(&maps.fvhi, lin ? a.FVhi : a.Vq, lin ? pr : a.Lq, lin ? D : HD, 64)) != cudaSuccess) return e;
  if ((e = make_map(&maps.fvlo, lin ? a.FVlo : a.Vq, lin ? pr : a.Lq, lin ? D : HD, 64)) != cudaSuccess) return e;
  const int n_lin = lin ? a.r / 64 : 0;
  const size_t smem = 1024 + TcLayout<D>::kBytes + (size_t)(n_lin + 2 * nKc + 3 * nKq) * 4;
  if (smem > 232448) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(sparse_attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = a.units ? a.max_units : a.H * nQ128;
  sparse_attn_tc_kernel<D><<<grid, kTcThreads, smem, s>>>(maps, a, nQ128, nKc, nQ64, nKq);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t s) {
  return a.d == 128 ? launch_tc<128>(a, s) : launch_tc<64>(a, s);
}

}  // namespace hsa
