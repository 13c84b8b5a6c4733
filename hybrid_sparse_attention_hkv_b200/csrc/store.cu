// Tiered page store of the hierarchical KV cache ("WorldAttention pairs
// hierarchical KV caching with hybrid sparse attention..." news summary, HKV
// paragraph: KV pages live in a hierarchy of memories ranked by cost, unselected
// pages are demoted to cheaper memory so that GPU occupancy stays bounded; project
// page, Method figure "three-tier hierarchical KV cache").
//
// Two tiers here: every sealed page lives in page-locked host memory mapped into the
// device address space (the authoritative copy, pages are immutable once sealed),
// and up to S pages also live in an HBM slot pool.  A device page table holds, per
// page, the address the gather reads: its slot when resident, else its host copy.
// Residency is decided on the device, from the device-side page selection, so a step
// never waits for the host:
//   fetch     for the selected pages: a resident page is touched; a missing one takes
//             the lowest free slot, else the least recently used slot whose page is
//             not selected (ties -> lower slot), whose page is demoted (its table
//             entry points back at its host copy); the page is then copied host ->
//             slot over the host link and its table entry points at the slot.
//   prefetch  the m best-scoring pages outside a protected set (the current
//             selection), in score order (ties -> lower page), are made resident the
//             same way, without evicting a protected page; meant for a side stream
//             while the chunk's denoising steps run, so that the next chunk's fetch
//             finds its pages in HBM.
// Every decision is made by one thread in a fixed order (deterministic); the copies
// are then spread over many CTAs.
//
// State buffer layout (bytes; every part 256-byte aligned):
//   [0, 256)         int32 tick, n_copy
//   table_k          uint64 [NP]  page addresses read by the gather (K)
//   table_v          uint64 [NP]  (V)
//   slot_of_page     int32 [NP]   -1 = not resident
//   page_of_slot     int32 [S]    -1 = free
//   stamp            int32 [S]    tick of the last use
//   copy_list        int2  [S]    (page, slot) pairs to copy after a fetch / prefetch
#include "common.cuh"
#include "kernels.h"

namespace hsa {
namespace {

inline size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

struct StoreLayout {
  size_t table_k, table_v, slot_of_page, page_of_slot, stamp, copy_list, total;
};

StoreLayout store_layout(int NP, int S) {
  StoreLayout L;
  size_t off = 256;
  L.table_k = off; off += al256((size_t)NP * 8);
  L.table_v = off; off += al256((size_t)NP * 8);
  L.slot_of_page = off; off += al256((size_t)NP * 4);
  L.page_of_slot = off; off += al256((size_t)S * 4);
  L.stamp = off; off += al256((size_t)S * 4);
  L.copy_list = off; off += al256((size_t)S * 8);
  L.total = off;
  return L;
}

struct StoreView {
  int* hdr;  // [0] tick, [1] n_copy
  unsigned long long* table_k;
  unsigned long long* table_v;
  int* slot_of_page;
  int* page_of_slot;
  int* stamp;
  int2* copy_list;
};

StoreView view_of(const StoreDesc& st) {
  const StoreLayout L = store_layout(st.NP, st.S);
  StoreView v;
  v.hdr = reinterpret_cast<int*>(st.state);
  v.table_k = reinterpret_cast<unsigned long long*>(st.state + L.table_k);
  v.table_v = reinterpret_cast<unsigned long long*>(st.state + L.table_v);
  v.slot_of_page = reinterpret_cast<int*>(st.state + L.slot_of_page);
  v.page_of_slot = reinterpret_cast<int*>(st.state + L.page_of_slot);
  v.stamp = reinterpret_cast<int*>(st.state + L.stamp);
  v.copy_list = reinterpret_cast<int2*>(st.state + L.copy_list);
  return v;
}

__device__ __forceinline__ unsigned long long page_addr(const uint16_t* base, long long page, long long page_elems) {
  return reinterpret_cast<unsigned long long>(base + page * page_elems);
}

__global__ void store_init_kernel(const StoreDesc st, const StoreView v) {
  const long long pe = st.P_tok * st.C;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i == 0) {
    v.hdr[0] = 0;
    v.hdr[1] = 0;
  }
  if (i < st.NP) {
    v.table_k[i] = page_addr(st.host_k, i, pe);
    v.table_v[i] = page_addr(st.host_v, i, pe);
    v.slot_of_page[i] = -1;
  }
  if (i < st.S) {
    v.page_of_slot[i] = -1;
    v.stamp[i] = 0;
  }
}

// Make page p resident in `slot`, demoting the slot's previous page.
__device__ void assign_slot(const StoreDesc& st, const StoreView& v, int p, int slot, int tick, int& n_copy) {
  const long long pe = st.P_tok * st.C;
  const int q = v.page_of_slot[slot];
  if (q >= 0) {  // demote: the gather reads q from the host tier again
    v.slot_of_page[q] = -1;
    v.table_k[q] = page_addr(st.host_k, q, pe);
    v.table_v[q] = page_addr(st.host_v, q, pe);
  }
  v.page_of_slot[slot] = p;
  v.slot_of_page[p] = slot;
  v.stamp[slot] = tick;
  v.table_k[p] = page_addr(st.slot_k, slot, pe);
  v.table_v[p] = page_addr(st.slot_v, slot, pe);
  v.copy_list[n_copy++] = make_int2(p, slot);
}

// Lowest free slot, else the least recently used slot that `evictable` allows
// (ties -> lower slot); -1 if none.
template <typename F>
__device__ int pick_victim(const StoreDesc& st, const StoreView& v, F evictable) {
  for (int s = 0; s < st.S; ++s)
    if (v.page_of_slot[s] < 0) return s;
  int best = -1;
  for (int s = 0; s < st.S; ++s)
    if (evictable(s) && (best < 0 || v.stamp[s] < v.stamp[best])) best = s;
  return best;
}

__global__ void store_fetch_kernel(const StoreDesc st, const StoreView v, const int32_t* __restrict__ sel, int Kp,
                                   int* status) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  const int tick = v.hdr[0] + 1;
  v.hdr[0] = tick;
  int n_copy = 0;
  for (int i = 0; i < Kp; ++i) {  // touch the resident selected pages first
    const int p = sel[i];
    if (p < 0 || p >= st.NP) {
      set_status(status, HSA_ERR_DEVICE);
      continue;
    }
    const int s = v.slot_of_page[p];
    if (s >= 0) v.stamp[s] = tick;
  }
  for (int i = 0; i < Kp; ++i) {
    const int p = sel[i];
    if (p < 0 || p >= st.NP || v.slot_of_page[p] >= 0) continue;
    // a slot touched or filled by this fetch holds a selected page: not evictable
    const int slot = pick_victim(st, v, [&](int s) { return v.stamp[s] < tick; });
    if (slot < 0) {  // fewer slots than selected pages: p stays on the host tier
      set_status(status, HSA_ERR_DEVICE);
      continue;
    }
    assign_slot(st, v, p, slot, tick, n_copy);
  }
  v.hdr[1] = n_copy;
}

__global__ void store_prefetch_kernel(const StoreDesc st, const StoreView v, const float* __restrict__ scores,
                                      const int32_t* __restrict__ protect, int n_protect, int m, int* status) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  const int tick = v.hdr[0] + 1;
  v.hdr[0] = tick;
  int n_copy = 0;
  auto is_protected = [&](int p) {
    for (int k = 0; k < n_protect; ++k)
      if (protect[k] == p) return true;
    return false;
  };
  // the m best-scoring unprotected pages, in score order (ties -> lower page);
  // pages with a non-finite score (outside the candidate range) are never taken
  float last_s = INFINITY;
  int last_p = -1;
  for (int k = 0; k < m; ++k) {
    int bp = -1;
    float bs = -INFINITY;
    for (int p = 0; p < st.NP; ++p) {
      const float sp = scores[p];
      if (!isfinite(sp) || is_protected(p)) continue;
      const bool after_last = sp < last_s || (sp == last_s && p > last_p);  // strictly after the previous pick
      if (!after_last) continue;
      if (bp < 0 || sp > bs) {
        bp = p;
        bs = sp;
      }
    }
    if (bp < 0) break;
    last_s = bs;
    last_p = bp;
    const int cur = v.slot_of_page[bp];
    if (cur >= 0) {
      v.stamp[cur] = tick;
      continue;
    }
    const int slot = pick_victim(st, v, [&](int s) {
      return v.stamp[s] < tick && !is_protected(v.page_of_slot[s]);
    });
    if (slot < 0) break;  // every slot is protected or already prefetched
    assign_slot(st, v, bp, slot, tick, n_copy);
  }
  v.hdr[1] = n_copy;
  (void)status;
}

// Copy the pages of copy_list[0 .. n_copy) from the host tier into their slots:
// blockIdx.y = list entry, blockIdx.x = 64-row block of the page; each thread moves
// 16-byte vectors, 8 in flight.
constexpr int kCopyRows = 64;
constexpr int kCopyThreads = 256;

__global__ void __launch_bounds__(kCopyThreads) store_copy_kernel(const StoreDesc st, const StoreView v) {
  const int e = blockIdx.y;
  if (e >= v.hdr[1]) return;
  const int2 ps = v.copy_list[e];
  const long long pe = st.P_tok * st.C;
  const long long r0 = (long long)blockIdx.x * kCopyRows;
  const long long r1 = min(st.P_tok, r0 + kCopyRows);
  if (r0 >= r1) return;
  const long long nvec = (r1 - r0) * st.C / 8;  // 16-byte vectors of this row block, per tensor
  for (int kv = 0; kv < 2; ++kv) {
    const uint16_t* src = (kv ? st.host_v : st.host_k) + ps.x * pe + r0 * st.C;
    uint16_t* dst = (kv ? st.slot_v : st.slot_k) + ps.y * pe + r0 * st.C;
    for (long long i0 = threadIdx.x; i0 < nvec; i0 += 8LL * kCopyThreads) {
      uint4 w[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const long long i = i0 + (long long)u * kCopyThreads;
        if (i < nvec) w[u] = ld_nc_v4(src + i * 8);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const long long i = i0 + (long long)u * kCopyThreads;
        if (i < nvec) *reinterpret_cast<uint4*>(dst + i * 8) = w[u];
      }
    }
  }
}

__global__ void store_slots_kernel(const StoreDesc st, const StoreView v, int32_t* slot_of_page,
                                   int32_t* page_of_slot) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (slot_of_page && i < st.NP) slot_of_page[i] = v.slot_of_page[i];
  if (page_of_slot && i < st.S) page_of_slot[i] = v.page_of_slot[i];
}

cudaError_t launch_copies(const StoreDesc& st, const StoreView& v, int max_copies, cudaStream_t s) {
  const long long blocks = (st.P_tok + kCopyRows - 1) / kCopyRows;
  store_copy_kernel<<<dim3((unsigned)blocks, (unsigned)max_copies), kCopyThreads, 0, s>>>(st, v);
  return cudaGetLastError();
}

}  // namespace

size_t store_state_bytes(int NP, int S) { return store_layout(NP, S).total; }

size_t store_table_offset(int NP, int kv) {
  const StoreLayout L = store_layout(NP, 1);
  return kv ? L.table_v : L.table_k;
}

cudaError_t launch_store_init(const StoreDesc& st, cudaStream_t s) {
  const int n = st.NP > st.S ? st.NP : st.S;
  store_init_kernel<<<(n + 255) / 256, 256, 0, s>>>(st, view_of(st));
  return cudaGetLastError();
}

cudaError_t launch_store_fetch(const StoreDesc& st, const int32_t* sel, int Kp, int* status, cudaStream_t s) {
  const StoreView v = view_of(st);
  store_fetch_kernel<<<1, 32, 0, s>>>(st, v, sel, Kp, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_copies(st, v, Kp < st.S ? Kp : st.S, s);
}

cudaError_t launch_store_prefetch(const StoreDesc& st, const float* scores, const int32_t* protect, int n_protect,
                                  int m, int* status, cudaStream_t s) {
  const StoreView v = view_of(st);
  store_prefetch_kernel<<<1, 32, 0, s>>>(st, v, scores, protect, n_protect, m, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || m == 0) return e;
  return launch_copies(st, v, m < st.S ? m : st.S, s);
}

cudaError_t launch_store_slots(const StoreDesc& st, int32_t* slot_of_page, int32_t* page_of_slot, cudaStream_t s) {
  const int n = st.NP > st.S ? st.NP : st.S;
  store_slots_kernel<<<(n + 255) / 256, 256, 0, s>>>(st, view_of(st), slot_of_page, page_of_slot);
  return cudaGetLastError();
}

}  // namespace hsa
