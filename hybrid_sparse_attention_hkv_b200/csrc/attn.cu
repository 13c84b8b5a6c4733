// HSA attention kernels ("WorldAttention pairs hierarchical KV caching with hybrid
// sparse attention..." news summary, HSA paragraph).
//
//  * sparse branch: exact online-softmax attention of a 128-query tile of one head
//    over the key tiles its block selection keeps (inter: 128-key blocks of the
//    cached KV, shared by the whole tile; intra: 64-key blocks of the chunk, kept
//    per 64-query half), with the per-head gated merge fused into the epilogue;
//  * linear branch: softmax(Q EK^T * scale) FV over the r projected rows, with
//    EK and FV held as split bf16 pairs (hi + lo) so that the products keep
//    about 16 significant bits.
//
// Warp-level bf16 tensor-core MMA (m16n8k16), 8 warps x 16 query rows, key tiles
// of 64 rows double-buffered in shared memory by cp.async.
#include <float.h>

#include "common.cuh"
#include "kernels.h"

namespace hsa {

constexpr int kBM = 128;  // query rows per CTA
constexpr int kBN = 64;   // keys per tile
constexpr int kThreads = 256;

// Tile code: (first key row << 3) | (source << 2) | half-mask.
// source 0 = cached KV (Kc/Vc), 1 = chunk KV (Kq/Vq); mask bit 0 = rows 0..63 of the
// query tile use it, bit 1 = rows 64..127 use it.
__device__ __forceinline__ int tile_code(long long start, int src, int mask) {
  return (int)(start << 3) | (src << 2) | mask;
}

template <int D>
__device__ __forceinline__ void load_rows(uint16_t* sdst, const uint16_t* base, long long start, long long nrows,
                                          int H, int h, int tid) {
  constexpr int CPR = D / 8;  // 16-byte chunks per row
#pragma unroll
  for (int x = tid; x < kBN * CPR; x += kThreads) {
    const int r = x / CPR, c = x % CPR;
    const long long R = start + r;
    const bool ok = R < nrows;
    const uint16_t* g = base + ((ok ? R : 0) * H + h) * D + c * 8;
    cp_async16(smem_u32(sdst + r * D + swz(r, c) * 8), g, ok ? 16 : 0);
  }
}

// S(16 x 64) = Q(16 x D) K^T for one warp: qf = Q fragments, sK = 64 x D tile.
template <int D>
__device__ __forceinline__ void qk_tile(float (&s)[8][4], const uint32_t (&qf)[D / 16][4], const uint16_t* sK,
                                        int lane) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      const int mi = lane / 8;
      const int key = np * 16 + (lane % 8) + 8 * (mi / 2);
      const int chunk = 2 * kk + (mi % 2);
      uint32_t b0, b1, b2, b3;
      ldsm_x4(smem_u32(sK + key * D + swz(key, chunk) * 8), b0, b1, b2, b3);
      mma_bf16(s[2 * np], qf[kk], b0, b1);
      mma_bf16(s[2 * np + 1], qf[kk], b2, b3);
    }
  }
}

// O(16 x D) += P(16 x 64) V(64 x D): pf = P as A fragments (4 k-steps of 16 keys).
template <int D>
__device__ __forceinline__ void pv_tile(float (&o)[D / 8][4], const uint32_t (&pf)[4][4], const uint16_t* sV,
                                        int lane) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
    for (int nd = 0; nd < D / 16; ++nd) {
      const int mi = lane / 8;
      const int key = kk * 16 + (lane % 8) + 8 * (mi % 2);
      const int chunk = 2 * nd + (mi / 2);
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(smem_u32(sV + key * D + swz(key, chunk) * 8), b0, b1, b2, b3);
      mma_bf16(o[2 * nd], pf[kk], b0, b1);
      mma_bf16(o[2 * nd + 1], pf[kk], b2, b3);
    }
  }
}

// Online-softmax update for one 64-key tile.  s holds raw scores (masked = -inf);
// rows g (c0, c1) and g + 8 (c2, c3).  Returns P (exp2 of scaled scores) in s.
template <int D>
__device__ __forceinline__ void softmax_update(float (&s)[8][4], float (&o)[D / 8][4], float& m0, float& m1,
                                               float& l0, float& l1, float sl2) {
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    mx0 = fmaxf(mx0, fmaxf(s[j][0], s[j][1]));
    mx1 = fmaxf(mx1, fmaxf(s[j][2], s[j][3]));
  }
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
  const float mn0 = fmaxf(m0, mx0 * sl2), mn1 = fmaxf(m1, mx1 * sl2);
  const float a0 = exp2f(m0 - mn0), a1 = exp2f(m1 - mn1);
  m0 = mn0;
  m1 = mn1;
  float r0 = 0.f, r1 = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    s[j][0] = exp2f(fmaf(s[j][0], sl2, -mn0));
    s[j][1] = exp2f(fmaf(s[j][1], sl2, -mn0));
    s[j][2] = exp2f(fmaf(s[j][2], sl2, -mn1));
    s[j][3] = exp2f(fmaf(s[j][3], sl2, -mn1));
    r0 += s[j][0] + s[j][1];
    r1 += s[j][2] + s[j][3];
  }
  l0 = l0 * a0 + r0;
  l1 = l1 * a1 + r1;
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    o[n][0] *= a0;
    o[n][1] *= a0;
    o[n][2] *= a1;
    o[n][3] *= a1;
  }
}

template <int D>
__device__ __forceinline__ void load_q(uint16_t* sQ, const uint16_t* Q, int q0, int Lq, int H, int h, int tid) {
  constexpr int CPR = D / 8;
  for (int x = tid; x < kBM * CPR; x += kThreads) {
    const int r = x / CPR, c = x % CPR;
    const int R = q0 + r;
    const bool ok = R < Lq;
    const uint16_t* g = Q + ((long long)(ok ? R : 0) * H + h) * D + c * 8;
    cp_async16(smem_u32(sQ + r * D + swz(r, c) * 8), g, ok ? 16 : 0);
  }
}

template <int D>
__device__ __forceinline__ void q_frags(uint32_t (&qf)[D / 16][4], const uint16_t* sQ, int warp, int lane) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const int row = warp * 16 + (lane % 16);
    const int chunk = 2 * kk + lane / 16;
    ldsm_x4(smem_u32(sQ + row * D + swz(row, chunk) * 8), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
  }
}

// Normalise and store the 16 x D warp tile; optional gated merge with o_lin.
template <int D>
__device__ __forceinline__ void store_out(const AttnArgs& a, float (&o)[D / 8][4], float l0, float l1, int q0,
                                          int h, int warp, int lane, bool merge, float g) {
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float inv0 = 1.f / l0, inv1 = 1.f / l1;
  const float gm = 1.f - g;
  const int row0 = q0 + warp * 16 + lane / 4, row1 = row0 + 8;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int row = half ? row1 : row0;
    if (row >= a.Lq) continue;
    const float inv = half ? inv1 : inv0;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      const int col = n * 8 + 2 * (lane % 4);
      const long long idx = ((long long)row * a.H + h) * D + col;
      float v0 = o[n][2 * half] * inv, v1 = o[n][2 * half + 1] * inv;
      if (merge) {
        const float2 ol = *reinterpret_cast<const float2*>(a.o_lin + idx);
        v0 = g * v0 + gm * ol.x;
        v1 = g * v1 + gm * ol.y;
      }
      if (a.out_bf16)
        *reinterpret_cast<uint32_t*>(a.out_bf16 + idx) = pack_bf16x2(v0, v1);
      else
        *reinterpret_cast<float2*>(a.out_f32 + idx) = make_float2(v0, v1);
    }
  }
}

// ------------------------------------------------------------------ sparse branch
template <int D>
__global__ void __launch_bounds__(kThreads, 1) sparse_attn_kernel(const AttnArgs a, int nQ128, int nKc, int nQ64,
                                                                  int nKq) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint16_t* sQ = reinterpret_cast<uint16_t*>(smem);
  uint16_t* sK = sQ + kBM * D;        // [2][64][D]
  uint16_t* sV = sK + 2 * kBN * D;    // [2][64][D]
  int* tiles = reinterpret_cast<int*>(sV + 2 * kBN * D);  // [2*nKc + nKq]
  int* flags = tiles + 2 * nKc + nKq;                      // [nKq]
  __shared__ int s_ntiles;

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int qb = blockIdx.x % nQ128, h = blockIdx.x / nQ128;
  const int q0 = qb * kBM;

  load_q<D>(sQ, a.Q, q0, a.Lq, a.H, h, tid);
  cp_async_commit();

  // tile list: two 64-key tiles per selected inter block, then the union of the two
  // 64-query halves' intra blocks in ascending order, tagged with who uses them.
  // Counts and ids come from the caller's selection buffers: clamp the counts and
  // skip ids outside [0, nK) (recorded as HSA_ERR_DEVICE) so shared memory and the
  // key loads stay in bounds whatever the buffers hold.
  const int n_inter = min(max(a.inter_cnt[(long long)h * nQ128 + qb], 0), nKc);
  const int32_t* ilist = a.inter_idx + ((long long)h * nQ128 + qb) * nKc;
  for (int m = tid; m < n_inter; m += kThreads) {
    const long long j = ilist[m];
    const bool ok = j >= 0 && j < nKc;
    if (!ok) set_status(a.status, HSA_ERR_DEVICE);
    tiles[2 * m] = ok ? tile_code(j * 128, 0, 3) : 0;
    tiles[2 * m + 1] = ok ? tile_code(j * 128 + 64, 0, (j * 128 + 64 < a.Lc) ? 3 : 0) : 0;
  }
  for (int j = tid; j < nKq; j += kThreads) flags[j] = 0;
  __syncthreads();
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int i64 = 2 * qb + half;
    if (i64 < nQ64) {
      const int cnt = min(max(a.intra_cnt[(long long)h * nQ64 + i64], 0), nKq);
      const int32_t* lst = a.intra_idx + ((long long)h * nQ64 + i64) * nKq;
      for (int m = tid; m < cnt; m += kThreads) {
        const int j = lst[m];
        if (j >= 0 && j < nKq) atomicOr(&flags[j], 1 << half);
        else set_status(a.status, HSA_ERR_DEVICE);
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    int base = 2 * n_inter;
    for (int b = 0; b < nKq; b += 32) {
      const int j = b + lane;
      const int f = j < nKq ? flags[j] : 0;
      const unsigned bal = __ballot_sync(0xffffffffu, f != 0);
      if (f) tiles[base + __popc(bal & ((1u << lane) - 1u))] = tile_code((long long)j * 64, 1, f);
      base += __popc(bal);
    }
    if (lane == 0) s_ntiles = base;
  }
  __syncthreads();
  const int T = s_ntiles;
  const int my_bit = warp < 4 ? 1 : 2;

  auto issue = [&](int t, int st) {
    const int code = tiles[t];
    const long long start = (long long)(code >> 3);
    const int src = (code >> 2) & 1;
    const long long nrows = src ? (long long)a.Lq : a.Lc;
    load_rows<D>(sK + st * kBN * D, src ? a.Kq : a.Kc, start, nrows, a.H, h, tid);
    load_rows<D>(sV + st * kBN * D, src ? a.Vq : a.Vc, start, nrows, a.H, h, tid);
  };
  if (T > 0) issue(0, 0);
  cp_async_commit();
  cp_async_wait<1>();
  __syncthreads();
  uint32_t qf[D / 16][4];
  q_frags<D>(qf, sQ, warp, lane);

  float o[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const float sl2 = a.scale * 1.4426950408889634f;

  for (int t = 0; t < T; ++t) {
    if (t + 1 < T) issue(t + 1, (t + 1) & 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const int code = tiles[t];
    if (code & my_bit) {
      const int st = t & 1;
      float s[8][4];
#pragma unroll
      for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
      qk_tile<D>(s, qf, sK + st * kBN * D, lane);
      const long long start = (long long)(code >> 3);
      const long long nrows = ((code >> 2) & 1) ? (long long)a.Lq : a.Lc;
      const long long valid = nrows - start;
      if (valid < kBN) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int key = j * 8 + 2 * (lane % 4);
          if (key >= valid) s[j][0] = s[j][2] = -INFINITY;
          if (key + 1 >= valid) s[j][1] = s[j][3] = -INFINITY;
        }
      }
      softmax_update<D>(s, o, m0, m1, l0, l1, sl2);
      uint32_t pf[4][4];
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        pf[kk][0] = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
        pf[kk][1] = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
        pf[kk][2] = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        pf[kk][3] = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
      }
      pv_tile<D>(o, pf, sV + st * kBN * D, lane);
    }
    __syncthreads();
  }

  const bool merge = a.gate_logit != nullptr;
  float g = 1.f;
  if (merge) g = 1.f / (1.f + expf(-a.gate_logit[h]));
  store_out<D>(a, o, l0, l1, q0, h, warp, lane, merge, g);
}

// ------------------------------------------------------------------ linear branch
template <int D>
__device__ __forceinline__ void load_proj_rows(uint16_t* sdst, const uint16_t* base, int row0, int tid) {
  constexpr int CPR = D / 8;
#pragma unroll
  for (int x = tid; x < kBN * CPR; x += kThreads) {
    const int r = x / CPR, c = x % CPR;
    cp_async16(smem_u32(sdst + r * D + swz(r, c) * 8), base + (long long)(row0 + r) * D + c * 8, 16);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) linear_attn_kernel(const AttnArgs a, int nQ128) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint16_t* sQ = reinterpret_cast<uint16_t*>(smem);
  uint16_t* sT = sQ + kBM * D;  // [2 stages][4: EKhi, EKlo, FVhi, FVlo][64][D]
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int qb = blockIdx.x % nQ128, h = blockIdx.x / nQ128;
  const int q0 = qb * kBM;
  const long long hoff = (long long)h * a.r * D;
  const int T = a.r / kBN;

  load_q<D>(sQ, a.Q, q0, a.Lq, a.H, h, tid);
  cp_async_commit();
  auto issue = [&](int t, int st) {
    uint16_t* dst = sT + st * 4 * kBN * D;
    load_proj_rows<D>(dst + 0 * kBN * D, a.EKhi + hoff, t * kBN, tid);
    load_proj_rows<D>(dst + 1 * kBN * D, a.EKlo + hoff, t * kBN, tid);
    load_proj_rows<D>(dst + 2 * kBN * D, a.FVhi + hoff, t * kBN, tid);
    load_proj_rows<D>(dst + 3 * kBN * D, a.FVlo + hoff, t * kBN, tid);
  };
  issue(0, 0);
  cp_async_commit();
  cp_async_wait<1>();
  __syncthreads();
  uint32_t qf[D / 16][4];
  q_frags<D>(qf, sQ, warp, lane);

  float o[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const float sl2 = a.scale * 1.4426950408889634f;

  for (int t = 0; t < T; ++t) {
    if (t + 1 < T) issue(t + 1, (t + 1) & 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint16_t* st = sT + (t & 1) * 4 * kBN * D;
    float s[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
    qk_tile<D>(s, qf, st + 0 * kBN * D, lane);  // Q EK_hi^T
    qk_tile<D>(s, qf, st + 1 * kBN * D, lane);  // + Q EK_lo^T
    softmax_update<D>(s, o, m0, m1, l0, l1, sl2);
    uint32_t ph[4][4], pl[4][4];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int j = 2 * kk + (q >> 1);
        const int e = (q & 1) * 2;
        __nv_bfloat16 h0, l0b, h1, l1b;
        split_bf16(s[j][e], h0, l0b);
        split_bf16(s[j][e + 1], h1, l1b);
        ph[kk][q] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
        pl[kk][q] = (uint32_t)__bfloat16_as_ushort(l0b) | ((uint32_t)__bfloat16_as_ushort(l1b) << 16);
      }
    }
    pv_tile<D>(o, ph, st + 2 * kBN * D, lane);  // P_hi FV_hi
    pv_tile<D>(o, pl, st + 2 * kBN * D, lane);  // + P_lo FV_hi
    pv_tile<D>(o, ph, st + 3 * kBN * D, lane);  // + P_hi FV_lo
    __syncthreads();
  }
  store_out<D>(a, o, l0, l1, q0, h, warp, lane, false, 1.f);
}

// ------------------------------------------------------------------ launchers
cudaError_t launch_sparse_attn(const AttnArgs& a, cudaStream_t s) {
  const int nQ128 = (a.Lq + 127) / 128, nQ64 = (a.Lq + 63) / 64;
  const int nKc = (int)((a.Lc + 127) / 128), nKq = nQ64;
  const size_t smem = (size_t)(kBM + 4 * kBN) * a.d * 2 + (size_t)(2 * nKc + 2 * nKq) * 4;
  const int grid = a.H * nQ128;
  cudaError_t e;
  if (a.d == 128) {
    e = cudaFuncSetAttribute(sparse_attn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    sparse_attn_kernel<128><<<grid, kThreads, smem, s>>>(a, nQ128, nKc, nQ64, nKq);
  } else {
    e = cudaFuncSetAttribute(sparse_attn_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    sparse_attn_kernel<64><<<grid, kThreads, smem, s>>>(a, nQ128, nKc, nQ64, nKq);
  }
  return cudaGetLastError();
}

cudaError_t launch_linear_attn(const AttnArgs& a, cudaStream_t s) {
  const int nQ128 = (a.Lq + 127) / 128;
  const size_t smem = (size_t)(kBM + 8 * kBN) * a.d * 2;
  const int grid = a.H * nQ128;
  cudaError_t e;
  if (a.d == 128) {
    e = cudaFuncSetAttribute(linear_attn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    linear_attn_kernel<128><<<grid, kThreads, smem, s>>>(a, nQ128);
  } else {
    e = cudaFuncSetAttribute(linear_attn_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    linear_attn_kernel<64><<<grid, kThreads, smem, s>>>(a, nQ128);
  }
  return cudaGetLastError();
}

}  // namespace hsa
