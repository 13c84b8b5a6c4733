// Linformer projection of the HSA linear branch on the 5th-generation tensor cores
// ("WorldAttention pairs hierarchical KV caching with hybrid sparse attention..."
// news summary, HSA paragraph: low-rank projection, O(L r)):
//     EK_h = E_h [Kc; Kq]_h,   FV_h = F_h [Vc; Vq]_h,   E_h, F_h in R^{r x L}.
//
// One CTA per (group of 128-row tiles of r, HP heads, split of L, E.K or F.V); with
// one E shared by all heads, HP = 2 adjacent heads share every E tile (one MMA of
// N = 2 d covers both), which halves the E traffic:
//   warp 0      TMA producer: per 64-row chunk of L, the E (or F) tiles [128 x 64]
//               of every r tile and the K (or V) chunk [64 x HP d] of the heads, into a
//               ring of 128-byte-swizzled stages; chunks of the cached KV and of the
//               chunk KV are separate (E's column offset Lc for the latter), so no
//               chunk straddles the two tensors;
//   warp 1      MMA issuer: acc_t += E_t chunk (K-major) x K chunk (MN-major), the
//               accumulators of all r tiles resident in TMEM for the whole split;
//   warps 2-5   epilogue: TMEM -> fp32 partial sums in global memory, reduced over
//               the splits in a fixed order by proj_reduce_kernel (proj.cu).
// Every wait is bounded (HSA_ERR_TIMEOUT in the workspace status on expiry).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace hsa {
using namespace sm100;

namespace {

constexpr int kPjThreads = 192;
constexpr int kChunk = 64;  // rows of L per pipeline stage

struct PjMaps {
  CUtensorMap e, f, kc, vc, kq, vq;
};

struct PjArgs {
  int H, r, Lq;
  long long Lc;
  int per_head;      // E/F maps hold H stacked [r, L] matrices
  int n_chunks_c;    // ceil(Lc / 64)
  int n_chunks;      // n_chunks_c + ceil(Lq / 64)
  int chunk_lo, chunk_hi;  // chunks [chunk_lo, chunk_hi) of [0, n_chunks) make up this launch
  int chunks_per_split;
  float* part;       // [splits][2][H][r][D]
  int* status;
};

template <int NB, int MT>  // NB = HP x d accumulator columns per r tile
struct PjLayout {
  static constexpr int kEBytes = 128 * kChunk * 2;       // one [128 x 64] tile: 16 KB
  static constexpr int kBBytes = kChunk * NB * 2;        // [64 x NB]
  static constexpr int kStageBytes = MT * kEBytes + kBBytes;
  static constexpr int kStages = (200 * 1024) / kStageBytes > 6 ? 6 : (200 * 1024) / kStageBytes;
  static constexpr int kBytes = kStages * kStageBytes;
  static constexpr int kTmemCols = MT * NB <= 32 ? 32 : (MT * NB <= 64 ? 64 : (MT * NB <= 128 ? 128 : (MT * NB <= 256 ? 256 : 512)));
  static_assert(MT * NB <= 512, "accumulators exceed TMEM");
};

// ------------------------------------------------------------------ kernel
template <int D, int MT, int HP>
__global__ void __launch_bounds__(kPjThreads, 1) proj_tc_kernel(const __grid_constant__ PjMaps maps, const PjArgs a) {
  constexpr int NB = HP * D;
  using Lay = PjLayout<NB, MT>;
  constexpr int NS = Lay::kStages;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bar_full[NS], bar_empty[NS], bar_acc;
  __shared__ uint32_t s_tmem;

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const uint64_t wlim = wait_limit_ns(a.status);
  const int rg = blockIdx.x, h0 = blockIdx.y * HP;  // first head of this CTA
  const int which = blockIdx.z & 1, split = blockIdx.z >> 1;
  const int c_begin = a.chunk_lo + split * a.chunks_per_split;
  const int c_end = min(a.chunk_hi, c_begin + a.chunks_per_split);
  const int nc = max(0, c_end - c_begin);
  const CUtensorMap* mE = which ? &maps.f : &maps.e;
  const CUtensorMap* mBc = which ? &maps.vc : &maps.kc;
  const CUtensorMap* mBq = which ? &maps.vq : &maps.kq;
  const int erow0 = (a.per_head ? h0 * a.r : 0) + rg * MT * 128;  // per-head E only with HP = 1

  if (warp == 0) {
    tmem_alloc(&s_tmem, Lay::kTmemCols);
    tmem_relinquish();
  }
  if (tid == 32) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar_full[s], 1);
      mbar_init(&bar_empty[s], 1);
    }
    mbar_init(&bar_acc, 1);
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tacc = s_tmem;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(mE);
      prefetch_tensormap(mBc);
      prefetch_tensormap(mBq);
    }
    for (int i = 0; i < nc; ++i) {
      const int s = i % NS;
      if (!mbar_wait(&bar_empty[s], ((i / NS) & 1) ^ 1, a.status, wlim)) break;
      if (lane == 0) {
        const int c = c_begin + i;
        const bool cached = c < a.n_chunks_c;
        const int brow = cached ? c * kChunk : (c - a.n_chunks_c) * kChunk;
        const int ecol = cached ? c * kChunk : (int)a.Lc + (c - a.n_chunks_c) * kChunk;
        unsigned char* st = smem + s * Lay::kStageBytes;
        mbar_arrive_expect_tx(&bar_full[s], Lay::kStageBytes);
#pragma unroll
        for (int t = 0; t < MT; ++t) tma_load_2d(st + t * Lay::kEBytes, mE, &bar_full[s], ecol, erow0 + t * 128);
#pragma unroll
        for (int c2 = 0; c2 < NB / 64; ++c2)
          tma_load_2d(st + MT * Lay::kEBytes + c2 * (kChunk * 128), cached ? mBc : mBq, &bar_full[s],
                      h0 * D + c2 * 64, brow);
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    const uint32_t idesc = idesc_bf16(128, NB, false, true);
    bool ok = true;
    for (int i = 0; i < nc; ++i) {
      const int s = i % NS;
      if (!mbar_wait(&bar_full[s], (i / NS) & 1, a.status, wlim)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t st = smem_u32(smem + s * Lay::kStageBytes);
        const uint32_t b_base = st + MT * Lay::kEBytes;
#pragma unroll
        for (int t = 0; t < MT; ++t) {
#pragma unroll
          for (int kk = 0; kk < kChunk / 16; ++kk) {
            const uint64_t ad = sdesc_sw128(st + t * Lay::kEBytes + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(b_base + kk * 2048, kChunk * 128, 1024);
            mma_ss(tacc + t * NB, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit(&bar_empty[s]);
      }
      __syncwarp();
    }
    if (lane == 0 && ok && nc > 0) mma_commit(&bar_acc);
    __syncwarp();
  } else {
    const int wq = warp & 3;
    const int row = 32 * wq + lane;
    const uint32_t loff = (uint32_t)(32 * wq) << 16;
    const bool have = nc > 0 && mbar_wait_warp(&bar_acc, 0, a.status, wlim);
    if (nc == 0 || have) {
      tc_fence_after();
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        const int m = (rg * MT + t) * 128 + row;
#pragma unroll
        for (int c = 0; c < NB / 16; ++c) {
          // columns [hh d, hh d + d) of the accumulator belong to head h0 + hh
          float* out = a.part + ((((long long)split * 2 + which) * a.H + h0 + (c * 16) / D) * a.r) * D;
          uint32_t v[16];
          if (nc > 0) {
            tmem_ld16_sync(tacc + loff + t * NB + c * 16, v);
          } else {
#pragma unroll
            for (int k = 0; k < 16; ++k) v[k] = 0u;
          }
          if (m < a.r) {
            float4* dst = reinterpret_cast<float4*>(out + (long long)m * D + (c * 16) % D);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              dst[k] = make_float4(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]),
                                   __uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3]));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tacc, Lay::kTmemCols);
  }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 g_enc = nullptr;
std::once_flag g_enc_once;

cudaError_t encoder() {
  std::call_once(g_enc_once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_enc ? cudaSuccess : cudaErrorNotSupported;
}

cudaError_t map2d(CUtensorMap* m, const void* base, long long rows, long long cols, int box_rows) {
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int D, int MT, int HP>
cudaError_t launch_mt(const PjMaps& maps, const PjArgs& a, int groups, int splits, cudaStream_t s) {
  using Lay = PjLayout<HP * D, MT>;
  const size_t smem = 1024 + Lay::kBytes;
  cudaError_t e =
      cudaFuncSetAttribute(proj_tc_kernel<D, MT, HP>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  proj_tc_kernel<D, MT, HP><<<dim3(groups, a.H / HP, 2 * splits), kPjThreads, smem, s>>>(maps, a);
  return cudaGetLastError();
}

// Heads per CTA: 2 when one E serves every head and H is even, else 1.
int proj_heads_per_cta(int H, bool per_head) { return (!per_head && H % 2 == 0) ? 2 : 1; }
// r tiles per CTA: at most 4, and at most 512 TMEM columns of accumulators.
int proj_tiles_per_cta(int r, int d, int hp) {
  const int tiles = (r + 127) / 128;
  const int cap = 512 / (hp * d) < 4 ? 512 / (hp * d) : 4;
  return tiles < cap ? tiles : cap;
}

}  // namespace

// Splits of the chunk range of a launch (`part` selects all chunks, the cached KV's
// or the current chunk's), chosen for the shared-E launch (the workspace is sized
// with the largest); a per-head-E launch uses the same count with twice the CTAs.
static long long part_chunks(long long Lc, int Lq, int part) {
  const long long cc = (Lc + kChunk - 1) / kChunk, cq = (Lq + kChunk - 1) / kChunk;
  return part == kProjCached ? cc : (part == kProjChunk ? cq : cc + cq);
}

int proj_tc_splits(int H, int d, int r, long long Lc, int Lq, int part) {
  const long long chunks = part_chunks(Lc, Lq, part);
  const int hp = proj_heads_per_cta(H, false);
  const int mt = proj_tiles_per_cta(r, d, hp);
  const int groups = ((r + 127) / 128 + mt - 1) / mt;
  const long long base = (long long)groups * (H / hp) * 2;
  int best = 1;
  double best_eff = 0.0;
  for (int s = 1; s <= 16 && s <= chunks; ++s) {
    const long long units = base * s;
    const long long waves = (units + 147) / 148;
    const double eff = (double)units / (double)(waves * 148);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = s;
    }
  }
  return best;
}

cudaError_t launch_proj_tc(const uint16_t* E, const uint16_t* F, long long ef_head_stride, const uint16_t* Kc,
                           const uint16_t* Kq, const uint16_t* Vc, const uint16_t* Vq, int H, int d, int r,
                           long long Lc, int Lq, int which_part, int splits, float* part, int* status,
                           cudaStream_t s) {
  cudaError_t e = encoder();
  if (e != cudaSuccess) return e;
  const long long L = Lc + Lq;
  const long long HD = (long long)H * d;
  PjMaps maps;
  const long long erows = ef_head_stride ? (long long)H * r : r;
  if ((e = map2d(&maps.e, E, erows, L, 128)) != cudaSuccess) return e;
  if ((e = map2d(&maps.f, F, erows, L, 128)) != cudaSuccess) return e;
  if ((e = map2d(&maps.kq, Kq, Lq, HD, kChunk)) != cudaSuccess) return e;
  if ((e = map2d(&maps.vq, Vq, Lq, HD, kChunk)) != cudaSuccess) return e;
  if ((e = map2d(&maps.kc, Lc > 0 ? Kc : Kq, Lc > 0 ? Lc : Lq, HD, kChunk)) != cudaSuccess) return e;
  if ((e = map2d(&maps.vc, Lc > 0 ? Vc : Vq, Lc > 0 ? Lc : Lq, HD, kChunk)) != cudaSuccess) return e;
  PjArgs a;
  a.H = H; a.r = r; a.Lq = Lq; a.Lc = Lc;
  a.per_head = ef_head_stride != 0;
  a.n_chunks_c = (int)((Lc + kChunk - 1) / kChunk);
  a.n_chunks = a.n_chunks_c + (Lq + kChunk - 1) / kChunk;
  a.chunk_lo = which_part == kProjChunk ? a.n_chunks_c : 0;
  a.chunk_hi = which_part == kProjCached ? a.n_chunks_c : a.n_chunks;
  a.chunks_per_split = (a.chunk_hi - a.chunk_lo + splits - 1) / splits;
  a.part = part;
  a.status = status;
  const int hp = proj_heads_per_cta(H, a.per_head != 0);
  const int mt = proj_tiles_per_cta(r, d, hp);
  const int groups = ((r + 127) / 128 + mt - 1) / mt;
  if (d == 128) {
    if (hp == 2) {
      switch (mt) {
        case 1: return launch_mt<128, 1, 2>(maps, a, groups, splits, s);
        default: return launch_mt<128, 2, 2>(maps, a, groups, splits, s);
      }
    }
    switch (mt) {
      case 1: return launch_mt<128, 1, 1>(maps, a, groups, splits, s);
      case 2: return launch_mt<128, 2, 1>(maps, a, groups, splits, s);
      case 3: return launch_mt<128, 3, 1>(maps, a, groups, splits, s);
      default: return launch_mt<128, 4, 1>(maps, a, groups, splits, s);
    }
  }
  if (hp == 2) {
    switch (mt) {
      case 1: return launch_mt<64, 1, 2>(maps, a, groups, splits, s);
      case 2: return launch_mt<64, 2, 2>(maps, a, groups, splits, s);
      case 3: return launch_mt<64, 3, 2>(maps, a, groups, splits, s);
      default: return launch_mt<64, 4, 2>(maps, a, groups, splits, s);
    }
  }
  switch (mt) {
    case 1: return launch_mt<64, 1, 1>(maps, a, groups, splits, s);
    case 2: return launch_mt<64, 2, 1>(maps, a, groups, splits, s);
    case 3: return launch_mt<64, 3, 1>(maps, a, groups, splits, s);
    default: return launch_mt<64, 4, 1>(maps, a, groups, splits, s);
  }
}

}  // namespace hsa
