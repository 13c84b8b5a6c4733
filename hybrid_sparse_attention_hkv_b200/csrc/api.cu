// C-ABI entry points of the HKV + HSA library: host-side argument checks,
// workspace layout, per-kernel trace events and the launch sequence of each call.
// Nothing here allocates device memory, frees or synchronises (hsa_status_read and
// hsa_thread_release excepted); hsa_forward creates, on its first call on a thread
// and device, one side stream (for the projection, beside the block selection) and
// two events that it keeps for that thread until hsa_thread_release.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"

namespace {

thread_local char t_detail[512] = "";
thread_local cudaEvent_t* t_events = nullptr;
thread_local const char** t_names = nullptr;
thread_local int t_pairs = 0;
thread_local int t_count = 0;
thread_local int t_fault = HSA_FAULT_NONE;  // hsa_inject_fault

hsa_status_t fail(hsa_status_t code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_detail, sizeof(t_detail), fmt, ap);
  va_end(ap);
  return code;
}

// Records an event pair around one kernel launch when tracing is on.
struct TraceScope {
  cudaStream_t s;
  int k = -1;
  TraceScope(const char* name, cudaStream_t s_) : s(s_) {
    if (t_events && t_count < t_pairs) {
      k = t_count++;
      cudaEventRecord(t_events[2 * k], s);
      if (t_names) t_names[k] = name;
    }
  }
  ~TraceScope() {
    if (k >= 0) cudaEventRecord(t_events[2 * k + 1], s);
  }
};

#define HSA_LAUNCH(name, call)                                                   \
  do {                                                                           \
    if (t_fault == HSA_FAULT_LAUNCH) return fail(HSA_ERR_CUDA, "%s: injected launch failure", name); \
    cudaError_t _e;                                                              \
    {                                                                            \
      TraceScope _tr(name, stream);                                              \
      _e = (call);                                                               \
    }                                                                            \
    if (_e != cudaSuccess) return fail(HSA_ERR_CUDA, "%s: %s", name, cudaGetErrorString(_e)); \
  } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// `fn` is the name of the entry point being checked (each entry point defines it).
#define REQUIRE_PTR(p)                                                                  \
  do {                                                                                  \
    if ((p) == nullptr) return fail(HSA_ERR_INVALID_ARG, "%s: " #p " is NULL", fn);     \
    if (!aligned16(p)) return fail(HSA_ERR_INVALID_ARG, "%s: " #p " is not 16-byte aligned", fn); \
  } while (0)
#define OPTIONAL_PTR(p)                                                                 \
  do {                                                                                  \
    if ((p) != nullptr && !aligned16(p))                                                \
      return fail(HSA_ERR_INVALID_ARG, "%s: " #p " is not 16-byte aligned", fn);        \
  } while (0)

#define OPTIONAL_PTR8(p)                                                                \
  do {                                                                                  \
    if ((p) != nullptr && (reinterpret_cast<uintptr_t>(p) & 7u) != 0)                   \
      return fail(HSA_ERR_INVALID_ARG, "%s: " #p " is not 8-byte aligned", __func__);   \
  } while (0)

// Workspace layout shared by every entry point (offsets in bytes).
struct Layout {
  size_t status = 0, colpart = 0, q128 = 0, q64 = 0, kq64 = 0, kc128 = 0, bscores = 0;
  size_t inter_idx = 0, inter_cnt = 0, intra_idx = 0, intra_cnt = 0;
  size_t units = 0, n_units = 0, tile_done = 0, part_o = 0, part_ml = 0, part_lin = 0, attn_end = 0;
  int max_units = 0, max_slots = 0;
  size_t ekhi = 0, eklo = 0, fvhi = 0, fvlo = 0, projpart = 0, ekfv_hist = 0;
  size_t pages_end = 0;  // bytes needed by the page (HKV) calls
  size_t total = 0;
  int splits = 0;
};

Layout make_layout(int H, int d, int Lq, long long Lc, int r) {
  Layout L;
  size_t off = 256;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += align256(bytes);
    return o;
  };
  const size_t hd = (size_t)H * d;
  L.colpart = take((size_t)hsa::kColMaxSplits * hd * 4);
  L.pages_end = off;
  const size_t nQ128 = (Lq + 127) / 128, nQ64 = (Lq + 63) / 64, nKc = (size_t)((Lc + 127) / 128);
  L.q128 = take(nQ128 * hd * 4);
  L.q64 = take(nQ64 * hd * 4);
  L.kq64 = take(nQ64 * hd * 4);
  L.kc128 = take(nKc * hd * 4);
  L.bscores = take(hsa::block_scores_floats(H, Lq, Lc) * 4);
  L.inter_idx = take((size_t)H * nQ64 * nKc * 4);  // nQ64 rows: room for the joint mode's per-64-row lists
  L.inter_cnt = take((size_t)H * nQ64 * 4);
  L.intra_idx = take((size_t)H * nQ64 * nQ64 * 4);
  L.intra_cnt = take((size_t)H * nQ64 * 4);
  // attention work plan and the partial results of split lists
  L.max_units = hsa::plan_max_units(H, (int)nQ128);
  L.max_slots = hsa::plan_max_slots();
  L.units = take((size_t)L.max_units * 16);
  L.n_units = take(16);
  L.tile_done = take((size_t)H * nQ128 * 4);
  L.part_o = take((size_t)L.max_slots * 128 * d * 4);
  L.part_ml = take((size_t)L.max_slots * 128 * 8);
  L.part_lin = take((size_t)L.max_slots * 128 * d * 4);
  L.attn_end = off;
  const size_t hrd = (size_t)H * r * d;
  L.ekhi = take(hrd * 2);
  L.eklo = take(hrd * 2);
  L.fvhi = take(hrd * 2);
  L.fvlo = take(hrd * 2);
  L.splits = r > 0 ? hsa::proj_tc_splits(H, d, r, Lc, Lq, hsa::kProjAll) : 0;
  L.projpart = take((size_t)L.splits * 2 * hrd * 4);
  L.ekfv_hist = take(2 * hrd * 4);  // E Kc and F Vc (fp32), kept over a chunk's denoising steps
  L.total = off;
  return L;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}
inline int* status_of(void* ws) { return static_cast<int*>(ws); }

hsa_status_t check_heads(const char* fn, int H, int d) {
  if (H < 1) return fail(HSA_ERR_INVALID_ARG, "%s: H = %d must be >= 1", fn, H);
  if (d <= 0) return fail(HSA_ERR_INVALID_ARG, "%s: d = %d must be positive", fn, d);
  if (d != 64 && d != 128) return fail(HSA_ERR_UNSUPPORTED, "%s: d = %d (supported: 64, 128)", fn, d);
  return HSA_OK;
}

hsa_status_t check_cfg(const char* fn, const hsa_config_t* c, bool need_rank) {
  if (t_fault == HSA_FAULT_ARG) return fail(HSA_ERR_INVALID_ARG, "%s: injected argument failure", fn);
  if (!c) return fail(HSA_ERR_INVALID_ARG, "%s: cfg is NULL", fn);
  hsa_status_t st = check_heads(fn, c->H, c->d);
  if (st != HSA_OK) return st;
  if (c->Lq < 1) return fail(HSA_ERR_INVALID_ARG, "%s: Lq = %d must be >= 1", fn, c->Lq);
  if (c->Lc < 0) return fail(HSA_ERR_INVALID_ARG, "%s: Lc = %d must be >= 0", fn, c->Lc);
  if (c->block_inter != 128 || c->block_intra != 64)
    return fail(HSA_ERR_UNSUPPORTED, "%s: block sizes %d/%d (supported: 128/64)", fn, c->block_inter, c->block_intra);
  if (c->Lc % 8 != 0 || c->Lq % 8 != 0)
    return fail(HSA_ERR_UNSUPPORTED, "%s: Lc = %d and Lq = %d must be multiples of 8", fn, c->Lc, c->Lq);
  if ((c->Lc + 127) / 128 > hsa::kMaxSelBlocks || (c->Lq + 63) / 64 > hsa::kMaxSelBlocks)
    return fail(HSA_ERR_UNSUPPORTED, "%s: more than %d blocks in a selection row", fn, hsa::kMaxSelBlocks);
  if (!(c->scale >= 0.f) || isinf(c->scale)) return fail(HSA_ERR_INVALID_ARG, "%s: scale must be finite and >= 0", fn);
  if (c->select_mode != HSA_SELECT_SEPARATE && c->select_mode != HSA_SELECT_JOINT)
    return fail(HSA_ERR_INVALID_ARG, "%s: select_mode = %d", fn, c->select_mode);
  if (c->select_mode == HSA_SELECT_JOINT && (c->Lc + 127) / 128 + (c->Lq + 63) / 64 > 2 * hsa::kMaxSelBlocks)
    return fail(HSA_ERR_UNSUPPORTED, "%s: more than %d blocks in a joint selection row", fn, 2 * hsa::kMaxSelBlocks);
  if (need_rank && (c->rank < 64 || c->rank > 1024 || c->rank % 64 != 0))
    return fail(HSA_ERR_UNSUPPORTED, "%s: rank = %d (supported: multiples of 64 in [64, 1024])", fn, c->rank);
  return HSA_OK;
}

inline float scale_of(const hsa_config_t* c) { return c->scale > 0.f ? c->scale : 1.0f / sqrtf((float)c->d); }

// A non-blocking side stream and a fork / join event pair per device for this thread.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
constexpr int kMaxDevices = 64;
thread_local SideStream t_side[kMaxDevices];

cudaError_t side_stream(SideStream** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  SideStream& ss = t_side[dev];
  if (!ss.s) {
    // the highest priority: the projection's CTAs are dispatched ahead of the selection's.
    // All three objects are created before any is kept, so a failure leaves none behind.
    int least = 0, greatest = 0;
    SideStream n;
    e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
    if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&n.s, cudaStreamNonBlocking, greatest);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&n.fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&n.join, cudaEventDisableTiming);
    if (e != cudaSuccess) {
      if (n.join) cudaEventDestroy(n.join);
      if (n.fork) cudaEventDestroy(n.fork);
      if (n.s) cudaStreamDestroy(n.s);
      return e;
    }
    ss = n;
  }
  *out = &ss;
  return cudaSuccess;
}

hsa_status_t check_ws(const char* fn, const void* ws, size_t ws_bytes, size_t need) {
  if (t_fault == HSA_FAULT_WORKSPACE) return fail(HSA_ERR_WORKSPACE, "%s: injected workspace failure", fn);
  if (!ws) return fail(HSA_ERR_WORKSPACE, "%s: workspace is NULL", fn);
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(HSA_ERR_WORKSPACE, "%s: workspace not 256-byte aligned", fn);
  if (ws_bytes < need) return fail(HSA_ERR_WORKSPACE, "%s: workspace %zu bytes < %zu needed", fn, ws_bytes, need);
  return HSA_OK;
}

hsa_status_t check_sel(const char* fn, const hsa_selection_t& s) {
  if (!s.inter_idx || !s.inter_cnt || !s.intra_idx || !s.intra_cnt)
    return fail(HSA_ERR_INVALID_ARG, "%s: selection has a NULL array", fn);
  if (!aligned16(s.inter_idx) || !aligned16(s.inter_cnt) || !aligned16(s.intra_idx) || !aligned16(s.intra_cnt))
    return fail(HSA_ERR_INVALID_ARG, "%s: selection arrays must be 16-byte aligned", fn);
  return HSA_OK;
}

#define TRY(x)                          \
  do {                                  \
    hsa_status_t _s = (x);              \
    if (_s != HSA_OK) return _s;        \
  } while (0)

}  // namespace

namespace hsa {
int injected_fault() { return t_fault; }

hsa_status_t api_fail(hsa_status_t code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_detail, sizeof(t_detail), fmt, ap);
  va_end(ap);
  return code;
}
}  // namespace hsa

extern "C" {

hsa_status_t hsa_inject_fault(int kind) {
  if (kind < HSA_FAULT_NONE || kind > HSA_FAULT_LAUNCH) return fail(HSA_ERR_INVALID_ARG, "hsa_inject_fault: kind = %d", kind);
  t_fault = kind;
  return HSA_OK;
}

const char* hsa_status_string(hsa_status_t s) {
  switch (s) {
    case HSA_OK: return "HSA_OK";
    case HSA_ERR_INVALID_ARG: return "HSA_ERR_INVALID_ARG";
    case HSA_ERR_UNSUPPORTED: return "HSA_ERR_UNSUPPORTED";
    case HSA_ERR_WORKSPACE: return "HSA_ERR_WORKSPACE";
    case HSA_ERR_CUDA: return "HSA_ERR_CUDA";
    case HSA_ERR_TIMEOUT: return "HSA_ERR_TIMEOUT";
    case HSA_ERR_DEVICE: return "HSA_ERR_DEVICE";
  }
  return "HSA_ERR_UNKNOWN";
}

const char* hsa_last_error_detail(void) { return t_detail; }

hsa_status_t hsa_workspace_size(const hsa_config_t* cfg, int NP, int P_tok, size_t* bytes) {
  (void)NP;
  (void)P_tok;
  if (!bytes) return fail(HSA_ERR_INVALID_ARG, "hsa_workspace_size: bytes is NULL");
  TRY(check_cfg("hsa_workspace_size", cfg, false));
  *bytes = make_layout(cfg->H, cfg->d, cfg->Lq, cfg->Lc, cfg->rank > 0 ? cfg->rank : 0).total;
  return HSA_OK;
}

hsa_status_t hsa_status_clear(void* ws, hsa_stream_t stream) {
  if (!ws) return fail(HSA_ERR_WORKSPACE, "hsa_status_clear: workspace is NULL");
  // the status, the ran-out flag and the first ran-out site (the wait limit stays)
  cudaError_t e = cudaMemsetAsync(ws, 0, 2 * sizeof(int), stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(static_cast<char*>(ws) + 4 * sizeof(int), 0, 2 * sizeof(int), stream);
  return e == cudaSuccess ? HSA_OK : fail(HSA_ERR_CUDA, "hsa_status_clear: %s", cudaGetErrorString(e));
}

hsa_status_t hsa_set_wait_limit(void* ws, unsigned int limit_us, hsa_stream_t stream) {
  if (!ws) return fail(HSA_ERR_WORKSPACE, "hsa_set_wait_limit: workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return fail(HSA_ERR_WORKSPACE, "hsa_set_wait_limit: workspace not 256-byte aligned");
  if (t_fault == HSA_FAULT_LAUNCH) return fail(HSA_ERR_CUDA, "hsa_set_wait_limit: injected launch failure");
  cudaError_t e = hsa::launch_set_wait_limit(status_of(ws), limit_us, stream);
  return e == cudaSuccess ? HSA_OK : fail(HSA_ERR_CUDA, "hsa_set_wait_limit: %s", cudaGetErrorString(e));
}

hsa_status_t hsa_selftest_wait(void* ws, unsigned long long* waited_ns, hsa_stream_t stream) {
  if (!ws) return fail(HSA_ERR_WORKSPACE, "hsa_selftest_wait: workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return fail(HSA_ERR_WORKSPACE, "hsa_selftest_wait: workspace not 256-byte aligned");
  OPTIONAL_PTR8(waited_ns);
  if (t_fault == HSA_FAULT_LAUNCH) return fail(HSA_ERR_CUDA, "hsa_selftest_wait: injected launch failure");
  cudaError_t e = hsa::launch_wait_selftest(status_of(ws), waited_ns, stream);
  return e == cudaSuccess ? HSA_OK : fail(HSA_ERR_CUDA, "hsa_selftest_wait: %s", cudaGetErrorString(e));
}

hsa_status_t hsa_status_read(const void* ws, hsa_stream_t stream, int* status) {
  if (!ws || !status) return fail(HSA_ERR_INVALID_ARG, "hsa_status_read: NULL argument");
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e == cudaSuccess) e = cudaMemcpy(status, ws, sizeof(int), cudaMemcpyDeviceToHost);
  return e == cudaSuccess ? HSA_OK : fail(HSA_ERR_CUDA, "hsa_status_read: %s", cudaGetErrorString(e));
}

hsa_status_t hsa_trace_begin(void* const* events, int n_pairs, const char** names) {
  if (events && n_pairs < 0) return fail(HSA_ERR_INVALID_ARG, "hsa_trace_begin: n_pairs < 0");
  t_events = reinterpret_cast<cudaEvent_t*>(const_cast<void**>(events));
  t_pairs = events ? n_pairs : 0;
  t_names = names;
  t_count = 0;
  return HSA_OK;
}
int hsa_trace_count(void) { return t_count; }
hsa_status_t hsa_trace_end(void) {
  t_events = nullptr;
  t_names = nullptr;
  t_pairs = 0;
  return HSA_OK;
}

hsa_status_t hsa_thread_release(void) {
  int cur = -1;
  cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return fail(HSA_ERR_CUDA, "hsa_thread_release: %s", cudaGetErrorString(e));
  cudaError_t first = cudaSuccess;
  for (int dev = 0; dev < kMaxDevices; ++dev) {
    SideStream& ss = t_side[dev];
    if (!ss.s) continue;
    cudaError_t r = cudaSetDevice(dev);
    if (r == cudaSuccess) r = cudaStreamSynchronize(ss.s);
    if (r == cudaSuccess) r = cudaEventDestroy(ss.join);
    if (r == cudaSuccess) r = cudaEventDestroy(ss.fork);
    if (r == cudaSuccess) r = cudaStreamDestroy(ss.s);
    if (r == cudaSuccess) ss = SideStream();
    else if (first == cudaSuccess) first = r;
  }
  cudaSetDevice(cur);
  return first == cudaSuccess ? HSA_OK : fail(HSA_ERR_CUDA, "hsa_thread_release: %s", cudaGetErrorString(first));
}

// ------------------------------------------------------------------ HKV

hsa_status_t hkv_page_summary(const hsa_bf16* K_page, int P_tok, int H, int d, float* kbar, void* ws,
                              size_t ws_bytes, hsa_stream_t stream) {
  const char* fn = __func__;
  TRY(check_heads(fn, H, d));
  if (P_tok < 1) return fail(HSA_ERR_INVALID_ARG, "%s: P_tok = %d must be >= 1", fn, P_tok);
  REQUIRE_PTR(K_page);
  REQUIRE_PTR(kbar);
  const Layout L = make_layout(H, d, 1, 0, 0);
  TRY(check_ws(fn, ws, ws_bytes, L.pages_end));
  float* part = at<float>(ws, L.colpart);
  HSA_LAUNCH("colsum_partial", hsa::launch_colsum_partial(K_page, P_tok, H * d, part, nullptr, stream));
  HSA_LAUNCH("page_summary_final", hsa::launch_page_summary_final(part, P_tok, H * d, kbar, stream));
  return HSA_OK;
}

hsa_status_t hkv_select_prompt(const float* e_cur, const float* e_seg, int n_seg, int dim, const int32_t* seg_begin,
                               int32_t* seg_out, int32_t* cand_range_out, hsa_stream_t stream) {
  const char* fn = __func__;
  if (n_seg < 1 || dim < 1) return fail(HSA_ERR_INVALID_ARG, "%s: n_seg = %d, dim = %d must be >= 1", fn, n_seg, dim);
  REQUIRE_PTR(e_cur);
  REQUIRE_PTR(e_seg);
  REQUIRE_PTR(seg_begin);
  if (!seg_out || !cand_range_out) return fail(HSA_ERR_INVALID_ARG, "%s: NULL output", fn);
  HSA_LAUNCH("select_prompt", hsa::launch_select_prompt(e_cur, e_seg, n_seg, dim, seg_begin, seg_out, cand_range_out, stream));
  return HSA_OK;
}

hsa_status_t hkv_select_pages(const float* kbar_pages, int NP, const int32_t* cand_range, const hsa_bf16* Q, int Lq,
                              int H, int d, int Kp, int32_t* sel_out, float* scores_out, void* ws, size_t ws_bytes,
                              hsa_stream_t stream) {
  const char* fn = __func__;
  TRY(check_heads(fn, H, d));
  if (NP < 1 || Lq < 1) return fail(HSA_ERR_INVALID_ARG, "%s: NP = %d, Lq = %d must be >= 1", fn, NP, Lq);
  if (Kp < 1 || Kp > NP || Kp > 64) return fail(HSA_ERR_INVALID_ARG, "%s: Kp = %d must be in [1, min(NP, 64)]", fn, Kp);
  if ((size_t)H * d * 8 + (size_t)NP * 8 > 200 * 1024)
    return fail(HSA_ERR_UNSUPPORTED, "%s: H*d*8 + NP*8 bytes exceed the shared-memory budget", fn);
  if (NP > H * d) return fail(HSA_ERR_UNSUPPORTED, "%s: NP = %d pages exceed H*d = %d", fn, NP, H * d);
  REQUIRE_PTR(kbar_pages);
  REQUIRE_PTR(Q);
  if (!sel_out) return fail(HSA_ERR_INVALID_ARG, "%s: sel_out is NULL", fn);
  const Layout L = make_layout(H, d, 1, 0, 0);
  TRY(check_ws(fn, ws, ws_bytes, L.pages_end));
  float* part = at<float>(ws, L.colpart);
  HSA_LAUNCH("page_scores_partial", hsa::launch_page_scores_partial(Q, Lq, H * d, kbar_pages, NP, cand_range, part,
                                                                    stream));
  HSA_LAUNCH("select_pages_final", hsa::launch_select_pages_final(part, Lq, NP, cand_range, Kp, sel_out, scores_out,
                                                                  status_of(ws), stream));
  return HSA_OK;
}

hsa_status_t hkv_page_scores(const float* kbar_pages, int NP, const int32_t* cand_range, const hsa_bf16* Q, int Lq,
                             int H, int d, float* scores_out, void* ws, size_t ws_bytes, hsa_stream_t stream) {
  const char* fn = __func__;
  TRY(check_heads(fn, H, d));
  if (NP < 1 || Lq < 1) return fail(HSA_ERR_INVALID_ARG, "%s: NP = %d, Lq = %d must be >= 1", fn, NP, Lq);
  if ((size_t)H * d * 4 > 200 * 1024) return fail(HSA_ERR_UNSUPPORTED, "%s: H*d*4 bytes exceed shared memory", fn);
  REQUIRE_PTR(kbar_pages);
  REQUIRE_PTR(Q);
  if (!scores_out) return fail(HSA_ERR_INVALID_ARG, "%s: scores_out is NULL", fn);
  const Layout L = make_layout(H, d, 1, 0, 0);
  const size_t need = 256 + align256((size_t)hsa::page_score_splits(Lq) * NP * 4);
  TRY(check_ws(fn, ws, ws_bytes, need > L.pages_end ? need : L.pages_end));
  float* part = at<float>(ws, 256);
  HSA_LAUNCH("page_scores_partial", hsa::launch_page_scores_partial(Q, Lq, H * d, kbar_pages, NP, cand_range, part,
                                                                    stream));
  HSA_LAUNCH("page_scores_sum", hsa::launch_page_scores_sum(part, Lq, NP, cand_range, scores_out, stream));
  return HSA_OK;
}

hsa_status_t hkv_select_top(const float* scores, int NP, const int32_t* cand_range, int Kp, int32_t* sel_out,
                            void* ws, size_t ws_bytes, hsa_stream_t stream) {
  const char* fn = __func__;
  if (NP < 1) return fail(HSA_ERR_INVALID_ARG, "%s: NP = %d must be >= 1", fn, NP);
  if (Kp < 1 || Kp > NP || Kp > 64) return fail(HSA_ERR_INVALID_ARG, "%s: Kp = %d must be in [1, min(NP, 64)]", fn, Kp);
  REQUIRE_PTR(scores);
  if (!sel_out) return fail(HSA_ERR_INVALID_ARG, "%s: sel_out is NULL", fn);
  TRY(check_ws(fn, ws, ws_bytes, 256));
  // the scores as one split of partial scores with "Lq" = 1: ranked as they are
  HSA_LAUNCH("select_pages_final", hsa::launch_select_pages_final(scores, 1, NP, cand_range, Kp, sel_out, nullptr,
                                                                  status_of(ws), stream));
  return HSA_OK;
}

hsa_status_t hkv_select_pages_policy(int policy, const float* kbar_pages, int NP, const int32_t* cand_range,
                                     const hsa_bf16* Q, int Lq, int H, int d, int Kp, const float* rand_keys,
                                     int32_t* sel_out, float* scores_out, void* ws, size_t ws_bytes,
                                     hsa_stream_t stream) {
  const char* fn = __func__;
  if (policy == hsa::kPolicyScore)
    return hkv_select_pages(kbar_pages, NP, cand_range, Q, Lq, H, d, Kp, sel_out, scores_out, ws, ws_bytes, stream);
  if (policy != hsa::kPolicyRecent && policy != hsa::kPolicyRandom)
    return fail(HSA_ERR_INVALID_ARG, "%s: unknown policy %d", fn, policy);
  if (NP < 1) return fail(HSA_ERR_INVALID_ARG, "%s: NP = %d must be >= 1", fn, NP);
  if (Kp < 1 || Kp > NP || Kp > 64) return fail(HSA_ERR_INVALID_ARG, "%s: Kp = %d must be in [1, min(NP, 64)]", fn, Kp);
  if (NP > (1 << 24)) return fail(HSA_ERR_UNSUPPORTED, "%s: NP = %d beyond 2^24 pages", fn, NP);
  if (policy == hsa::kPolicyRandom) REQUIRE_PTR(rand_keys);
  if (!sel_out) return fail(HSA_ERR_INVALID_ARG, "%s: sel_out is NULL", fn);
  TRY(check_ws(fn, ws, ws_bytes, 256 + align256((size_t)NP * 4)));
  float* part = at<float>(ws, 256);
  HSA_LAUNCH("policy_keys", hsa::launch_policy_keys(policy, rand_keys, NP, part, stream));
  // one split of keys, "Lq" = 1: the final pass ranks the keys as they are
  HSA_LAUNCH("select_pages_final", hsa::launch_select_pages_final(part, 1, NP, cand_range, Kp, sel_out, scores_out,
                                                                  status_of(ws), stream));
  return HSA_OK;
}

hsa_status_t hkv_gather(const hsa_bf16* const* page_k, const hsa_bf16* const* page_v, int NP, const int32_t* sel,
                        int Kp, int P_tok, int H, int d, hsa_bf16* Kc, hsa_bf16* Vc, float* kbar128, void* ws,
                        size_t ws_bytes, hsa_stream_t stream) {
  const char* fn = __func__;
  TRY(check_heads(fn, H, d));
  if (NP < 1 || P_tok < 1) return fail(HSA_ERR_INVALID_ARG, "%s: NP = %d, P_tok = %d must be >= 1", fn, NP, P_tok);
  if (Kp < 1 || Kp > NP) return fail(HSA_ERR_INVALID_ARG, "%s: Kp = %d must be in [1, NP]", fn, Kp);
  if (!page_k || !page_v || !sel) return fail(HSA_ERR_INVALID_ARG, "%s: NULL page table or selection", fn);
  REQUIRE_PTR(Kc);
  REQUIRE_PTR(Vc);
  OPTIONAL_PTR(kbar128);
  TRY(check_ws(fn, ws, ws_bytes, 256));
  HSA_LAUNCH("gather", hsa::launch_gather(reinterpret_cast<const uint16_t* const*>(page_k),
                                          reinterpret_cast<const uint16_t* const*>(page_v), NP, sel, Kp, P_tok, H, d,
                                          Kc, Vc, kbar128, status_of(ws), stream));
  return HSA_OK;
}

hsa_status_t hkv_page_block_sums(const hsa_bf16* K_page, int P_tok, int H, int d, float* sums64, hsa_stream_t stream) {
  const char* fn = __func__;
  TRY(check_heads(fn, H, d));
  if (P_tok < 1) return fail(HSA_ERR_INVALID_ARG, "%s: P_tok = %d must be >= 1", fn, P_tok);
  REQUIRE_PTR(K_page);
  REQUIRE_PTR(sums64);
  HSA_LAUNCH("block_sums64", hsa::launch_block_sums64(K_page, P_tok, H * d, sums64, stream));
  return HSA_OK;
}

hsa_status_t hkv_block_means_from_pages(const float* sums64_pages, int NP, const int32_t* sel, int Kp, int P_tok,
                                        int H, int d, float* kbar128, void* ws, size_t ws_bytes, hsa_stream_t stream) {
  const char* fn = __func__;
  TRY(check_heads(fn, H, d));
  if (NP < 1 || P_tok < 1) return fail(HSA_ERR_INVALID_ARG, "%s: NP = %d, P_tok = %d must be >= 1", fn, NP, P_tok);
  if (P_tok % 64 != 0) return fail(HSA_ERR_UNSUPPORTED, "%s: P_tok = %d is not a multiple of 64", fn, P_tok);
  if (Kp < 1 || Kp > NP) return fail(HSA_ERR_INVALID_ARG, "%s: Kp = %d must be in [1, NP]", fn, Kp);
  REQUIRE_PTR(sums64_pages);
  REQUIRE_PTR(kbar128);
  if (!sel) return fail(HSA_ERR_INVALID_ARG, "%s: sel is NULL", fn);
  TRY(check_ws(fn, ws, ws_bytes, 256));
  HSA_LAUNCH("kc128_from_pages", hsa::launch_kc128_from_pages(sums64_pages, NP, P_tok, sel, Kp, H * d, kbar128,
                                                              status_of(ws), stream));
  return HSA_OK;
}

// ------------------------------------------------------------------ tiered page store

static hsa_status_t store_desc(const char* fn, const hkv_store_t* st, hsa::StoreDesc* out) {
  if (!st) return fail(HSA_ERR_INVALID_ARG, "%s: store is NULL", fn);
  TRY(check_heads(fn, st->H, st->d));
  if (st->NP < 1 || st->S < 1 || st->P_tok < 1)
    return fail(HSA_ERR_INVALID_ARG, "%s: NP = %d, S = %d, P_tok = %d must be >= 1", fn, st->NP, st->S, st->P_tok);
  REQUIRE_PTR(st->host_k);
  REQUIRE_PTR(st->host_v);
  REQUIRE_PTR(st->slot_k);
  REQUIRE_PTR(st->slot_v);
  if (!st->state || (reinterpret_cast<uintptr_t>(st->state) & 255u) != 0)
    return fail(HSA_ERR_INVALID_ARG, "%s: state must be non-NULL and 256-byte aligned", fn);
  out->NP = st->NP;
  out->S = st->S;
  out->P_tok = st->P_tok;
  out->C = st->H * st->d;
  out->host_k = st->host_k;
  out->host_v = st->host_v;
  out->slot_k = st->slot_k;
  out->slot_v = st->slot_v;
  out->state = static_cast<unsigned char*>(st->state);
  return HSA_OK;
}

size_t hkv_store_state_size(int NP, int S) {
  if (NP < 1 || S < 1) return 0;
  return hsa::store_state_bytes(NP, S);
}

hsa_status_t hkv_store_init(const hkv_store_t* st, hsa_stream_t stream) {
  const char* fn = __func__;
  hsa::StoreDesc sd;
  TRY(store_desc(fn, st, &sd));
  HSA_LAUNCH("store_init", hsa::launch_store_init(sd, stream));
  return HSA_OK;
}

hsa_status_t hkv_store_tables(const hkv_store_t* st, const hsa_bf16* const** table_k,
                              const hsa_bf16* const** table_v) {
  const char* fn = __func__;
  hsa::StoreDesc sd;
  TRY(store_desc(fn, st, &sd));
  if (!table_k || !table_v) return fail(HSA_ERR_INVALID_ARG, "%s: NULL output", fn);
  unsigned char* base = static_cast<unsigned char*>(st->state);
  *table_k = reinterpret_cast<const hsa_bf16* const*>(base + hsa::store_table_offset(st->NP, 0));
  *table_v = reinterpret_cast<const hsa_bf16* const*>(base + hsa::store_table_offset(st->NP, 1));
  return HSA_OK;
}

hsa_status_t hkv_store_seal(const hkv_store_t* st, int page, const hsa_bf16* K_rows, const hsa_bf16* V_rows,
                            float* kbar_out, void* ws, size_t ws_bytes, hsa_stream_t stream) {
  const char* fn = __func__;
  hsa::StoreDesc sd;
  TRY(store_desc(fn, st, &sd));
  if (page < 0 || page >= st->NP) return fail(HSA_ERR_INVALID_ARG, "%s: page %d outside [0, %d)", fn, page, st->NP);
  REQUIRE_PTR(K_rows);
  REQUIRE_PTR(V_rows);
  REQUIRE_PTR(kbar_out);
  const Layout L = make_layout(st->H, st->d, 1, 0, 0);
  TRY(check_ws(fn, ws, ws_bytes, L.pages_end));
  const long long pe = (long long)st->P_tok * sd.C;
  float* part = at<float>(ws, L.colpart);
  // K: the copy into the host tier and the page summary in one pass; V: a plain copy
  HSA_LAUNCH("seal_colsum", hsa::launch_colsum_partial(K_rows, st->P_tok, sd.C, part, st->host_k + page * pe, stream));
  HSA_LAUNCH("page_summary_final", hsa::launch_page_summary_final(part, st->P_tok, sd.C, kbar_out, stream));
  cudaError_t e = cudaMemcpyAsync(st->host_v + page * pe, V_rows, (size_t)pe * 2, cudaMemcpyDefault, stream);
  if (e != cudaSuccess) return fail(HSA_ERR_CUDA, "%s: %s", fn, cudaGetErrorString(e));
  return HSA_OK;
}

hsa_status_t hkv_store_fetch(const hkv_store_t* st, const int32_t* sel, int Kp, void* ws, size_t ws_bytes,
                             hsa_stream_t stream) {
  const char* fn = __func__;
  hsa::StoreDesc sd;
  TRY(store_desc(fn, st, &sd));
  if (Kp < 1 || Kp > st->NP) return fail(HSA_ERR_INVALID_ARG, "%s: Kp = %d must be in [1, NP]", fn, Kp);
  if (!sel) return fail(HSA_ERR_INVALID_ARG, "%s: sel is NULL", fn);
  TRY(check_ws(fn, ws, ws_bytes, 256));
  HSA_LAUNCH("store_fetch", hsa::launch_store_fetch(sd, sel, Kp, status_of(ws), stream));
  return HSA_OK;
}

hsa_status_t hkv_store_prefetch(const hkv_store_t* st, const float* scores, const int32_t* protect, int n_protect,
                                int m, void* ws, size_t ws_bytes, hsa_stream_t stream) {
  const char* fn = __func__;
  hsa::StoreDesc sd;
  TRY(store_desc(fn, st, &sd));
  if (!scores) return fail(HSA_ERR_INVALID_ARG, "%s: scores is NULL", fn);
  if (n_protect < 0 || (n_protect > 0 && !protect)) return fail(HSA_ERR_INVALID_ARG, "%s: bad protect list", fn);
  if (m < 0) return fail(HSA_ERR_INVALID_ARG, "%s: m = %d must be >= 0", fn, m);
  TRY(check_ws(fn, ws, ws_bytes, 256));
  HSA_LAUNCH("store_prefetch", hsa::launch_store_prefetch(sd, scores, protect, n_protect, m, status_of(ws), stream));
  return HSA_OK;
}

hsa_status_t hkv_store_residency(const hkv_store_t* st, int32_t* slot_of_page, int32_t* page_of_slot,
                                 hsa_stream_t stream) {
  const char* fn = __func__;
  hsa::StoreDesc sd;
  TRY(store_desc(fn, st, &sd));
  if (!slot_of_page && !page_of_slot) return fail(HSA_ERR_INVALID_ARG, "%s: no output", fn);
  HSA_LAUNCH("store_slots", hsa::launch_store_slots(sd, slot_of_page, page_of_slot, stream));
  return HSA_OK;
}

// ------------------------------------------------------------------ HSA

static hsa_status_t run_block_select(const hsa_config_t* cfg, const Layout& L, const hsa_bf16* Q, const hsa_bf16* Kc,
                                     const hsa_bf16* Kq, const float* kbar128, const float* tau,
                                     const hsa_selection_t& sel, void* ws, hsa_stream_t stream) {
  float* q128 = at<float>(ws, L.q128);
  float* q64 = at<float>(ws, L.q64);
  float* kq64 = at<float>(ws, L.kq64);
  float* kc128 = kbar128 ? const_cast<float*>(kbar128) : at<float>(ws, L.kc128);
  HSA_LAUNCH("pool", hsa::launch_pool(Q, Kq, Kc, cfg->H, cfg->d, cfg->Lq, cfg->Lc, q128, q64, kq64,
                                      kbar128 ? nullptr : kc128, stream));
  HSA_LAUNCH("block_select", hsa::launch_block_select(q128, kc128, q64, kq64, tau, cfg->H, cfg->d, cfg->Lq, cfg->Lc,
                                                      scale_of(cfg), cfg->select_mode == HSA_SELECT_JOINT,
                                                      at<float>(ws, L.bscores), sel.inter_idx, sel.inter_cnt,
                                                      sel.intra_idx, sel.intra_cnt, stream));
  return HSA_OK;
}

static hsa::AttnArgs attn_args(const hsa_config_t* cfg, const Layout& L, void* ws, const hsa_bf16* Q,
                               const hsa_bf16* Kc, const hsa_bf16* Vc, const hsa_bf16* Kq, const hsa_bf16* Vq) {
  hsa::AttnArgs a;
  memset(&a, 0, sizeof(a));
  a.Q = Q; a.Kc = Kc; a.Vc = Vc; a.Kq = Kq; a.Vq = Vq;
  a.H = cfg->H; a.d = cfg->d; a.Lq = cfg->Lq; a.Lc = cfg->Lc;
  a.scale = scale_of(cfg);
  a.joint = cfg->select_mode == HSA_SELECT_JOINT;
  a.r = cfg->rank;
  a.status = status_of(ws);
  a.max_units = L.max_units;
  a.max_slots = L.max_slots;
  return a;
}

// Sparse-branch inputs of `a` and the work plan over them.
static hsa_status_t run_plan(const Layout& L, const hsa_selection_t& sel, void* ws, hsa::AttnArgs& a,
                             hsa_stream_t stream) {
  a.inter_idx = sel.inter_idx; a.inter_cnt = sel.inter_cnt; a.intra_idx = sel.intra_idx; a.intra_cnt = sel.intra_cnt;
  a.units = at<int4>(ws, L.units);
  a.n_units = at<int>(ws, L.n_units);
  a.tile_done = at<int>(ws, L.tile_done);
  a.part_o = at<float>(ws, L.part_o);
  a.part_ml = at<float2>(ws, L.part_ml);
  a.part_lin = at<float>(ws, L.part_lin);
  HSA_LAUNCH("attn_plan", hsa::launch_attn_plan(a, stream));
  return HSA_OK;
}

// Linformer projection (EK, FV as split-bf16 pairs in the workspace); sets the
// linear-branch fields of `a`.  which_part = kProjAll projects the whole active KV;
// kProjChunk projects only the current chunk's KV and adds the cached KV's products
// that hsa_prepare_history left in the workspace.
static hsa_status_t run_projection(const hsa_config_t* cfg, const Layout& L, const hsa_bf16* Kc, const hsa_bf16* Vc,
                                   const hsa_bf16* Kq, const hsa_bf16* Vq, const hsa_bf16* E, const hsa_bf16* F,
                                   long long ef_head_stride, void* ws, hsa::AttnArgs& a, int which_part,
                                   hsa_stream_t stream) {
  float* part = at<float>(ws, L.projpart);
  uint16_t* ekhi = at<uint16_t>(ws, L.ekhi);
  uint16_t* eklo = at<uint16_t>(ws, L.eklo);
  uint16_t* fvhi = at<uint16_t>(ws, L.fvhi);
  uint16_t* fvlo = at<uint16_t>(ws, L.fvlo);
  int splits = hsa::proj_tc_splits(cfg->H, cfg->d, cfg->rank, cfg->Lc, cfg->Lq, which_part);
  if (splits > L.splits) splits = L.splits;
  HSA_LAUNCH("linformer_proj", hsa::launch_proj_tc(E, F, ef_head_stride, Kc, Kq, Vc, Vq, cfg->H, cfg->d, cfg->rank,
                                                   cfg->Lc, cfg->Lq, which_part, splits, part, status_of(ws),
                                                   stream));
  const float* add = which_part == hsa::kProjChunk ? at<float>(ws, L.ekfv_hist) : nullptr;
  HSA_LAUNCH("linformer_reduce", hsa::launch_proj_reduce(part, splits, cfg->H, cfg->d, cfg->rank, add, nullptr, ekhi,
                                                         eklo, fvhi, fvlo, stream));
  a.EKhi = ekhi; a.EKlo = eklo; a.FVhi = fvhi; a.FVlo = fvlo;
  return HSA_OK;
}

static hsa_status_t check_tensors(const char* fn, const hsa_config_t* cfg, const hsa_bf16* Q, const hsa_bf16* Kc,
                                  const hsa_bf16* Vc, const hsa_bf16* Kq, const hsa_bf16* Vq, bool needV) {
  REQUIRE_PTR(Q);
  REQUIRE_PTR(Kq);
  if (needV) REQUIRE_PTR(Vq);
  if (cfg->Lc > 0) {
    REQUIRE_PTR(Kc);
    if (needV) REQUIRE_PTR(Vc);
  }
  return HSA_OK;
}

hsa_status_t hsa_block_select(const hsa_config_t* cfg, const hsa_bf16* Q, const hsa_bf16* Kc, const hsa_bf16* Kq,
                              const float* kbar128, const float* tau, hsa_selection_t sel, void* ws, size_t ws_bytes,
                              hsa_stream_t stream) {
  const char* fn = __func__;
  TRY(check_cfg(fn, cfg, false));
  TRY(check_tensors(fn, cfg, Q, Kc, nullptr, Kq, nullptr, false));
  OPTIONAL_PTR(kbar128);
  if (!tau) return fail(HSA_ERR_INVALID_ARG, "%s: tau is NULL", fn);
  TRY(check_sel(fn, sel));
  const Layout L = make_layout(cfg->H, cfg->d, cfg->Lq, cfg->Lc, 0);
  TRY(check_ws(fn, ws, ws_bytes, L.inter_idx));
  return run_block_select(cfg, L, Q, Kc, Kq, kbar128, tau, sel, ws, stream);
}

hsa_status_t hsa_sparse_attn(const hsa_config_t* cfg, const hsa_bf16* Q, const hsa_bf16* Kc, const hsa_bf16* Vc,
                             const hsa_bf16* Kq, const hsa_bf16* Vq, hsa_selection_t sel, float* o_sparse, void* ws,
                             size_t ws_bytes, hsa_stream_t stream) {
  const char* fn = __func__;
  TRY(check_cfg(fn, cfg, false));
  TRY(check_tensors(fn, cfg, Q, Kc, Vc, Kq, Vq, true));
  TRY(check_sel(fn, sel));
  REQUIRE_PTR(o_sparse);
  const Layout L = make_layout(cfg->H, cfg->d, cfg->Lq, cfg->Lc, 0);
  TRY(check_ws(fn, ws, ws_bytes, L.attn_end));
  hsa::AttnArgs a = attn_args(cfg, L, ws, Q, Kc, Vc, Kq, Vq);
  TRY(run_plan(L, sel, ws, a, stream));
  a.out_f32 = o_sparse;
  HSA_LAUNCH("attention", hsa::launch_attn_tc(a, stream));
  return HSA_OK;
}

hsa_status_t hsa_sparse_attn_lse(const hsa_config_t* cfg, const hsa_bf16* Q, const hsa_bf16* Kc, const hsa_bf16* Vc,
                                 const hsa_bf16* Kq, const hsa_bf16* Vq, hsa_selection_t sel, float* o_sparse,
                                 float* lse_out, void* ws, size_t ws_bytes, hsa_stream_t stream) {
  const char* fn = __func__;
  TRY(check_cfg(fn, cfg, false));
  TRY(check_tensors(fn, cfg, Q, Kc, Vc, Kq, Vq, true));
  TRY(check_sel(fn, sel));
  REQUIRE_PTR(o_sparse);
  REQUIRE_PTR(lse_out);
  const Layout L = make_layout(cfg->H, cfg->d, cfg->Lq, cfg->Lc, 0);
  TRY(check_ws(fn, ws, ws_bytes, L.attn_end));
  hsa::AttnArgs a = attn_args(cfg, L, ws, Q, Kc, Vc, Kq, Vq);
  TRY(run_plan(L, sel, ws, a, stream));
  a.out_f32 = o_sparse;
  a.lse_out = lse_out;
  HSA_LAUNCH("attention", hsa::launch_attn_tc(a, stream));
  return HSA_OK;
}

hsa_status_t hsa_fidelity(const hsa_config_t* cfg, const float* o_ref, const float* lse_ref, const float* o_sparse,
                          const float* lse_sparse, const float* o_linear, double* report, void* ws, size_t ws_bytes,
                          hsa_stream_t stream) {
  const char* fn = __func__;
  TRY(check_cfg(fn, cfg, false));
  REQUIRE_PTR(o_ref);
  REQUIRE_PTR(lse_ref);
  REQUIRE_PTR(o_sparse);
  REQUIRE_PTR(lse_sparse);
  REQUIRE_PTR(o_linear);
  REQUIRE_PTR(report);
  const size_t need = 256 + (size_t)cfg->H * hsa::kFidelitySplits * 8 * sizeof(double);
  TRY(check_ws(fn, ws, ws_bytes, need));
  HSA_LAUNCH("fidelity", hsa::launch_fidelity(o_ref, lse_ref, o_sparse, lse_sparse, o_linear, cfg->Lq, cfg->H, cfg->d,
                                              at<double>(ws, 256), report, stream));
  return HSA_OK;
}

hsa_status_t hsa_linear_attn(const hsa_config_t* cfg, const hsa_bf16* Q, const hsa_bf16* Kc, const hsa_bf16* Vc,
                             const hsa_bf16* Kq, const hsa_bf16* Vq, const hsa_bf16* E, const hsa_bf16* F,
                             long long ef_head_stride, float* o_linear, void* ws, size_t ws_bytes,
                             hsa_stream_t stream) {
  const char* fn = __func__;
  TRY(check_cfg(fn, cfg, true));
  TRY(check_tensors(fn, cfg, Q, Kc, Vc, Kq, Vq, true));
  REQUIRE_PTR(E);
  REQUIRE_PTR(F);
  REQUIRE_PTR(o_linear);
  if (ef_head_stride != 0 && ef_head_stride != (long long)cfg->rank * (cfg->Lc + cfg->Lq))
    return fail(HSA_ERR_UNSUPPORTED, "%s: ef_head_stride must be 0 (shared) or r * (Lc + Lq) (stacked per head)", fn);
  const Layout L = make_layout(cfg->H, cfg->d, cfg->Lq, cfg->Lc, cfg->rank);
  TRY(check_ws(fn, ws, ws_bytes, L.total));
  hsa::AttnArgs a = attn_args(cfg, L, ws, Q, Kc, Vc, Kq, Vq);
  TRY(run_projection(cfg, L, Kc, Vc, Kq, Vq, E, F, ef_head_stride, ws, a, hsa::kProjAll, stream));
  a.out_f32 = o_linear;
  HSA_LAUNCH("attention", hsa::launch_attn_tc(a, stream));
  return HSA_OK;
}

static hsa_status_t forward_impl(const char* fn, const hsa_config_t* cfg, const hsa_bf16* Q, const hsa_bf16* Kc,
                                 const hsa_bf16* Vc, const hsa_bf16* Kq, const hsa_bf16* Vq, const float* kbar128,
                                 const float* tau, const float* gate_logit, const hsa_bf16* E, const hsa_bf16* F,
                                 long long ef_head_stride, void* out, int out_is_bf16,
                                 const hsa_selection_t* sel_out, void* ws, size_t ws_bytes, int which_part,
                                 bool selected, hsa_stream_t stream) {
  TRY(check_cfg(fn, cfg, true));
  TRY(check_tensors(fn, cfg, Q, Kc, Vc, Kq, Vq, true));
  OPTIONAL_PTR(kbar128);
  if ((!selected && !tau) || !gate_logit) return fail(HSA_ERR_INVALID_ARG, "%s: tau / gate_logit is NULL", fn);
  if (selected && !sel_out) return fail(HSA_ERR_INVALID_ARG, "%s: the selection is NULL", fn);
  REQUIRE_PTR(E);
  REQUIRE_PTR(F);
  REQUIRE_PTR(out);
  if (ef_head_stride != 0 && ef_head_stride != (long long)cfg->rank * (cfg->Lc + cfg->Lq))
    return fail(HSA_ERR_UNSUPPORTED, "%s: ef_head_stride must be 0 (shared) or r * (Lc + Lq) (stacked per head)", fn);
  if (sel_out) TRY(check_sel(fn, *sel_out));
  const Layout L = make_layout(cfg->H, cfg->d, cfg->Lq, cfg->Lc, cfg->rank);
  TRY(check_ws(fn, ws, ws_bytes, L.total));

  hsa_selection_t sel;
  if (sel_out) {
    sel = *sel_out;
  } else {
    sel.inter_idx = at<int32_t>(ws, L.inter_idx);
    sel.inter_cnt = at<int32_t>(ws, L.inter_cnt);
    sel.intra_idx = at<int32_t>(ws, L.intra_idx);
    sel.intra_cnt = at<int32_t>(ws, L.intra_cnt);
  }
  // The Linformer projection does not depend on the block selection: it runs on a
  // side stream while this stream pools, selects and plans; the attention waits for
  // both.
  hsa::AttnArgs a = attn_args(cfg, L, ws, Q, Kc, Vc, Kq, Vq);
  SideStream* side = nullptr;
  cudaError_t e = side_stream(&side);
  if (e == cudaSuccess) e = cudaEventRecord(side->fork, stream);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(side->s, side->fork, 0);
  if (e != cudaSuccess) return fail(HSA_ERR_CUDA, "%s: side stream: %s", fn, cudaGetErrorString(e));
  TRY(run_projection(cfg, L, Kc, Vc, Kq, Vq, E, F, ef_head_stride, ws, a, which_part, side->s));
  if ((e = cudaEventRecord(side->join, side->s)) != cudaSuccess)
    return fail(HSA_ERR_CUDA, "%s: side stream: %s", fn, cudaGetErrorString(e));
  if (!selected) TRY(run_block_select(cfg, L, Q, Kc, Kq, kbar128, tau, sel, ws, stream));
  TRY(run_plan(L, sel, ws, a, stream));
  if ((e = cudaStreamWaitEvent(stream, side->join, 0)) != cudaSuccess)
    return fail(HSA_ERR_CUDA, "%s: side stream: %s", fn, cudaGetErrorString(e));
  a.gate_logit = gate_logit;
  if (out_is_bf16) a.out_bf16 = static_cast<uint16_t*>(out);
  else a.out_f32 = static_cast<float*>(out);
  HSA_LAUNCH("attention_merge", hsa::launch_attn_tc(a, stream));
  return HSA_OK;
}

hsa_status_t hsa_forward(const hsa_config_t* cfg, const hsa_bf16* Q, const hsa_bf16* Kc, const hsa_bf16* Vc,
                         const hsa_bf16* Kq, const hsa_bf16* Vq, const float* kbar128, const float* tau,
                         const float* gate_logit, const hsa_bf16* E, const hsa_bf16* F, long long ef_head_stride,
                         void* out, int out_is_bf16, const hsa_selection_t* sel_out, void* ws, size_t ws_bytes,
                         hsa_stream_t stream) {
  return forward_impl(__func__, cfg, Q, Kc, Vc, Kq, Vq, kbar128, tau, gate_logit, E, F, ef_head_stride, out,
                      out_is_bf16, sel_out, ws, ws_bytes, hsa::kProjAll, false, stream);
}

hsa_status_t hsa_forward_selected(const hsa_config_t* cfg, const hsa_bf16* Q, const hsa_bf16* Kc, const hsa_bf16* Vc,
                                  const hsa_bf16* Kq, const hsa_bf16* Vq, const float* gate_logit, const hsa_bf16* E,
                                  const hsa_bf16* F, long long ef_head_stride, const hsa_selection_t* sel, void* out,
                                  int out_is_bf16, void* ws, size_t ws_bytes, hsa_stream_t stream) {
  return forward_impl(__func__, cfg, Q, Kc, Vc, Kq, Vq, nullptr, nullptr, gate_logit, E, F, ef_head_stride, out,
                      out_is_bf16, sel, ws, ws_bytes, hsa::kProjAll, true, stream);
}

// The cached KV's Linformer products (E Kc, F Vc; fp32) into the workspace, on `stream`.
static hsa_status_t project_history(const hsa_config_t* cfg, const Layout& L, const hsa_bf16* Kc, const hsa_bf16* Vc,
                                    const hsa_bf16* E, const hsa_bf16* F, long long ef_head_stride, void* ws,
                                    hsa_stream_t stream) {
  float* part = at<float>(ws, L.projpart);
  int splits = hsa::proj_tc_splits(cfg->H, cfg->d, cfg->rank, cfg->Lc, cfg->Lq, hsa::kProjCached);
  if (splits > L.splits) splits = L.splits;
  // the chunk tensors are not read by this launch; their maps point at the history
  const hsa_bf16* Kq = cfg->Lc > 0 ? Kc : E;
  const hsa_bf16* Vq = cfg->Lc > 0 ? Vc : F;
  HSA_LAUNCH("linformer_proj_history",
             hsa::launch_proj_tc(E, F, ef_head_stride, Kc, Kq, Vc, Vq, cfg->H, cfg->d, cfg->rank, cfg->Lc, cfg->Lq,
                                 hsa::kProjCached, splits, part, status_of(ws), stream));
  HSA_LAUNCH("linformer_reduce_history",
             hsa::launch_proj_reduce(part, splits, cfg->H, cfg->d, cfg->rank, nullptr, at<float>(ws, L.ekfv_hist),
                                     nullptr, nullptr, nullptr, nullptr, stream));
  return HSA_OK;
}

hsa_status_t hsa_prepare_history(const hsa_config_t* cfg, const hsa_bf16* Kc, const hsa_bf16* Vc, const hsa_bf16* E,
                                 const hsa_bf16* F, long long ef_head_stride, void* ws, size_t ws_bytes,
                                 hsa_stream_t stream) {
  const char* fn = __func__;
  TRY(check_cfg(fn, cfg, true));
  if (cfg->Lc > 0) {
    REQUIRE_PTR(Kc);
    REQUIRE_PTR(Vc);
  }
  REQUIRE_PTR(E);
  REQUIRE_PTR(F);
  if (ef_head_stride != 0 && ef_head_stride != (long long)cfg->rank * (cfg->Lc + cfg->Lq))
    return fail(HSA_ERR_UNSUPPORTED, "%s: ef_head_stride must be 0 (shared) or r * (Lc + Lq) (stacked per head)", fn);
  const Layout L = make_layout(cfg->H, cfg->d, cfg->Lq, cfg->Lc, cfg->rank);
  TRY(check_ws(fn, ws, ws_bytes, L.total));
  return project_history(cfg, L, Kc, Vc, E, F, ef_head_stride, ws, stream);
}

hsa_status_t hsa_forward_ex(const hsa_config_t* cfg, const hsa_bf16* Q, const hsa_bf16* Kc, const hsa_bf16* Vc,
                            const hsa_bf16* Kq, const hsa_bf16* Vq, const float* kbar128, const float* tau,
                            const float* gate_logit, const hsa_bf16* E, const hsa_bf16* F, long long ef_head_stride,
                            void* out, int out_is_bf16, const hsa_selection_t* sel, unsigned flags, void* ws,
                            size_t ws_bytes, hsa_stream_t stream) {
  if (flags & ~(unsigned)(HSA_FWD_SELECTED | HSA_FWD_HISTORY))
    return fail(HSA_ERR_INVALID_ARG, "hsa_forward_ex: unknown flags 0x%x", flags);
  return forward_impl(__func__, cfg, Q, Kc, Vc, Kq, Vq, kbar128, tau, gate_logit, E, F, ef_head_stride, out,
                      out_is_bf16, sel, ws, ws_bytes, (flags & HSA_FWD_HISTORY) ? hsa::kProjChunk : hsa::kProjAll,
                      (flags & HSA_FWD_SELECTED) != 0, stream);
}

hsa_status_t hkv_gather_project(const hsa_config_t* cfg, const hsa_bf16* const* page_k, const hsa_bf16* const* page_v,
                                int NP, const int32_t* sel, int Kp, int P_tok, const hsa_bf16* E, const hsa_bf16* F,
                                long long ef_head_stride, hsa_bf16* Kc, hsa_bf16* Vc, void* ws, size_t ws_bytes,
                                hsa_stream_t stream) {
  const char* fn = __func__;
  TRY(check_cfg(fn, cfg, true));
  if (NP < 1 || P_tok < 1) return fail(HSA_ERR_INVALID_ARG, "%s: NP = %d, P_tok = %d must be >= 1", fn, NP, P_tok);
  if (Kp < 1 || Kp > NP) return fail(HSA_ERR_INVALID_ARG, "%s: Kp = %d must be in [1, NP]", fn, Kp);
  if ((long long)Kp * P_tok != cfg->Lc)
    return fail(HSA_ERR_INVALID_ARG, "%s: Kp * P_tok = %lld differs from cfg->Lc = %d", fn, (long long)Kp * P_tok,
                cfg->Lc);
  if (!page_k || !page_v || !sel) return fail(HSA_ERR_INVALID_ARG, "%s: NULL page table or selection", fn);
  REQUIRE_PTR(Kc);
  REQUIRE_PTR(Vc);
  REQUIRE_PTR(E);
  REQUIRE_PTR(F);
  if (ef_head_stride != 0 && ef_head_stride != (long long)cfg->rank * (cfg->Lc + cfg->Lq))
    return fail(HSA_ERR_UNSUPPORTED, "%s: ef_head_stride must be 0 (shared) or r * (Lc + Lq) (stacked per head)", fn);
  const Layout L = make_layout(cfg->H, cfg->d, cfg->Lq, cfg->Lc, cfg->rank);
  TRY(check_ws(fn, ws, ws_bytes, L.total));
  // The gather, then the history's products on the same stream.  (Two overlaps of
  // the HBM-bound copy with the tensor-bound projection measured slower on B200: one
  // kernel copying the pages into the projection's operand ring, and stages of whole
  // pages gathered on this stream while a side stream projected the previous stage.)
  HSA_LAUNCH("gather", hsa::launch_gather(reinterpret_cast<const uint16_t* const*>(page_k),
                                          reinterpret_cast<const uint16_t* const*>(page_v), NP, sel, Kp, P_tok,
                                          cfg->H, cfg->d, Kc, Vc, nullptr, status_of(ws), stream));
  return project_history(cfg, L, Kc, Vc, E, F, ef_head_stride, ws, stream);
}

hsa_status_t hsa_forward_reuse(const hsa_config_t* cfg, const hsa_bf16* Q, const hsa_bf16* Kc, const hsa_bf16* Vc,
                               const hsa_bf16* Kq, const hsa_bf16* Vq, const float* kbar128, const float* tau,
                               const float* gate_logit, const hsa_bf16* E, const hsa_bf16* F,
                               long long ef_head_stride, void* out, int out_is_bf16, const hsa_selection_t* sel_out,
                               void* ws, size_t ws_bytes, hsa_stream_t stream) {
  return forward_impl(__func__, cfg, Q, Kc, Vc, Kq, Vq, kbar128, tau, gate_logit, E, F, ef_head_stride, out,
                      out_is_bf16, sel_out, ws, ws_bytes, hsa::kProjChunk, false, stream);
}

}  // extern "C"
