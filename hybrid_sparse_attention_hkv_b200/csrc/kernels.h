// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
// Every launcher enqueues on `stream` and returns cudaGetLastError().
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hsa.h"

namespace hsa {

// Dynamic shared memory above this asks for the opt-in attribute first: a launch may
// use 48 KB without it, and the kernel's static shared memory (under 1 KB in every
// kernel that checks this) counts toward the same 48 KB.
constexpr size_t kDefaultSmemOptIn = 47 * 1024;

// ---------------------------------------------------------------- api.cu
// Record the text returned by hsa_last_error_detail() and return `code`.
hsa_status_t api_fail(hsa_status_t code, const char* fmt, ...);
// The calling thread's injected fault kind (HSA_FAULT_*; hsa_inject_fault).
int injected_fault();

// ---------------------------------------------------------------- hkv.cu
constexpr int kColMaxSplits = 296;  // 2 CTAs per SM for the column-sum partial pass

int colsum_splits(long long n);  // number of row splits used for n rows
cudaError_t launch_colsum_partial(const uint16_t* X, long long n, int C, float* part, uint16_t* copy_dst,
                                  cudaStream_t s);
cudaError_t launch_page_summary_final(const float* part, long long n, int C, float* kbar, cudaStream_t s);
// Page-level retrieval: partial scores per row split of Q (pass 1), then one CTA
// adds them, ranks the candidates and writes the top Kp ascending (pass 2).
int page_score_splits(long long Lq);  // row splits of pass 1 (<= kColMaxSplits)
cudaError_t launch_page_scores_partial(const uint16_t* Q, long long Lq, int C, const float* kbar_pages, int NP,
                                       const int32_t* cand_range, float* part, cudaStream_t s);
cudaError_t launch_page_scores_sum(const float* part, long long Lq, int NP, const int32_t* cand_range, float* scores,
                                   cudaStream_t s);
cudaError_t launch_select_pages_final(const float* part, long long Lq, int NP, const int32_t* cand_range, int Kp,
                                      int32_t* sel_out, float* scores_out, int* status, cudaStream_t s);
// Retrieval policies other than the mean-key score (hkv_select_pages_policy).
constexpr int kPolicyScore = 0;
constexpr int kPolicyRecent = 1;
constexpr int kPolicyRandom = 2;
// part[p] = the policy's ranking key of page p (its id, or rand_keys[p]); one split.
cudaError_t launch_policy_keys(int policy, const float* rand_keys, int NP, float* part, cudaStream_t s);
cudaError_t launch_select_prompt(const float* e_cur, const float* e_seg, int n_seg, int dim,
                                 const int32_t* seg_begin, int32_t* seg_out, int32_t* cand_range_out,
                                 cudaStream_t s);
// 64-row key sums of a page ([ceil(n/64)][C] fp32) and the active cache's 128-row
// key means from them (P_tok % 64 == 0).
cudaError_t launch_block_sums64(const uint16_t* X, long long n, int C, float* sums, cudaStream_t s);
cudaError_t launch_kc128_from_pages(const float* sums, int NP, long long P_tok, const int32_t* sel, int Kp, int C,
                                    float* kbar128, int* status, cudaStream_t s);
cudaError_t launch_gather(const uint16_t* const* page_k, const uint16_t* const* page_v, int NP,
                          const int32_t* sel, int Kp, long long P_tok, int H, int d, uint16_t* Kc,
                          uint16_t* Vc, float* kbar128, int* status, cudaStream_t s);

// ---------------------------------------------------------------- store.cu
// Tiered page store: device-side residency state (layout in store.cu).
struct StoreDesc {
  int NP, S;
  long long P_tok;
  int C;                   // H * d
  const uint16_t* host_k;  // [NP][P_tok][C] (device view of mapped page-locked host memory)
  const uint16_t* host_v;
  uint16_t* slot_k;        // [S][P_tok][C] device memory
  uint16_t* slot_v;
  unsigned char* state;
};
size_t store_state_bytes(int NP, int S);
size_t store_table_offset(int NP, int kv);  // byte offset of the K (kv = 0) or V page table
cudaError_t launch_store_init(const StoreDesc& st, cudaStream_t s);
cudaError_t launch_store_fetch(const StoreDesc& st, const int32_t* sel, int Kp, int* status, cudaStream_t s);
cudaError_t launch_store_prefetch(const StoreDesc& st, const float* scores, const int32_t* protect, int n_protect,
                                  int m, int* status, cudaStream_t s);
cudaError_t launch_store_slots(const StoreDesc& st, int32_t* slot_of_page, int32_t* page_of_slot, cudaStream_t s);

// ---------------------------------------------------------------- select.cu
constexpr int kMaxSelBlocks = 8192;  // blocks per selection row (inter: ceil(Lc/128), intra: ceil(Lq/64))

cudaError_t launch_pool(const uint16_t* Q, const uint16_t* Kq, const uint16_t* Kc, int H, int d, int Lq,
                        long long Lc, float* q128, float* q64, float* kq64, float* kc128, cudaStream_t s);
// joint: one softmax per 64-row query block over its Kc and Kq blocks (inter rows per
// 64-row query block); else the two maps separately.  scores: block_scores_floats()
// floats of scratch for the rows' block scores.
size_t block_scores_floats(int H, int Lq, long long Lc);
cudaError_t launch_block_select(const float* q128, const float* kc128, const float* q64, const float* kq64,
                                const float* tau, int H, int d, int Lq, long long Lc, float scale, bool joint,
                                float* scores, int32_t* inter_idx, int32_t* inter_cnt, int32_t* intra_idx,
                                int32_t* intra_cnt, cudaStream_t s);

// ---------------------------------------------------------------- attn_tc.cu / plan.cu
// The attention kernel runs one CTA per work unit: a segment of the key-tile list
// of one (head, 128-query tile).  Lists longer than a segment length are cut into
// segments of similar length; the CTA that finishes a list's last segment merges
// the segments' partial results (plan.cu chooses the segments).
constexpr int kPlanSMs = 148;        // units are sized for this many SMs ...
constexpr int kPlanUnitsPerSM = 1;   // ... and lists above the cost per SM are split
constexpr int kPlanMinSegment = 16;  // shortest segment worth a unit of its own

struct AttnArgs {
  const uint16_t* Q;
  const uint16_t* Kc;
  const uint16_t* Vc;
  const uint16_t* Kq;
  const uint16_t* Vq;
  int H, d, Lq;
  long long Lc;
  float scale;
  bool joint;  // inter lists per 64-row query block (joint block selection)
  // sparse branch (runs when inter_cnt != NULL)
  const int32_t* inter_idx;
  const int32_t* inter_cnt;
  const int32_t* intra_idx;
  const int32_t* intra_cnt;
  // linear branch (runs when EKhi != NULL): split-bf16 projections, [H][r][d]
  const uint16_t* EKhi;
  const uint16_t* EKlo;
  const uint16_t* FVhi;
  const uint16_t* FVlo;
  int r;
  // both branches: out = g o_s + (1 - g) o_l, g = sigmoid(gate_logit[h]) (NULL -> g = 1)
  const float* gate_logit;
  // output [Lq, H, d]: fp32 (out_f32) or bf16 (out_bf16)
  float* out_f32;
  uint16_t* out_bf16;
  int* status;  // workspace status word (may be NULL)
  float* lse_out;  // optional [Lq][H]: natural-log log-sum-exp of the sparse branch's scaled scores
  // work plan (workspace; sparse branch only -- without it, unit u is query tile u whole)
  int max_units;     // capacity of units (grid size of the attention launch)
  int max_slots;     // capacity of the partial-result slots
  int4* units;       // [max_units] (head * nQ128 + query tile, segment, segments, first slot)
  int* n_units;      // number of units
  int* tile_done;    // [H * nQ128] segments finished (zeroed by the plan)
  float* part_o;     // [max_slots][128][d] unnormalised O_s of a segment
  float2* part_ml;   // [max_slots][128] running max (log2 units) and sum of a segment
  float* part_lin;   // [max_slots][128][d] weighted linear branch of a split list (at its first slot)
};
// Sparse and/or linear branch with the gated merge, on tcgen05 / TMEM / TMA.
cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t s);
// The work plan over the selection (plan.cu): one CTA.
cudaError_t launch_attn_plan(const AttnArgs& a, cudaStream_t s);
// Capacities used by the workspace layout.
inline int plan_max_units(int H, int nQ128) { return H * nQ128 + kPlanSMs * kPlanUnitsPerSM + 1; }
inline int plan_max_slots() { return 2 * kPlanSMs * kPlanUnitsPerSM + 2; }

// ---------------------------------------------------------------- proj.cu
// tcgen05 / TMEM / TMA projection (proj_tc.cu): partial sums [splits][2][H][r][d] fp32
// (EK then FV), reduced by launch_proj_reduce (proj.cu).  A launch covers the rows of
// the whole active KV (kProjAll), of the cached KV only (kProjCached: the part that
// stays fixed over a chunk's denoising steps) or of the current chunk only (kProjChunk).
constexpr int kProjAll = 0;
constexpr int kProjCached = 1;
constexpr int kProjChunk = 2;
int proj_tc_splits(int H, int d, int r, long long Lc, int Lq, int which_part);
cudaError_t launch_proj_tc(const uint16_t* E, const uint16_t* F, long long ef_head_stride, const uint16_t* Kc,
                           const uint16_t* Kq, const uint16_t* Vc, const uint16_t* Vq, int H, int d, int r,
                           long long Lc, int Lq, int which_part, int splits, float* part, int* status,
                           cudaStream_t s);
// Sum the split partials in a fixed order, plus `add` ([2][H][r][d] fp32, nullable):
// into fp32 sums `sum_out` when it is given, else into the split-bf16 pairs.
cudaError_t launch_proj_reduce(const float* part, int splits, int H, int d, int r, const float* add,
                               float* sum_out, uint16_t* EKhi, uint16_t* EKlo, uint16_t* FVhi, uint16_t* FVlo,
                               cudaStream_t s);

// ---------------------------------------------------------------- fidelity.cu
// Per-head comparison of the two branches with dense attention (fp64 sums, fixed
// order): report[h][0..5) = cos(o_lin, o_ref), cos(o_sp, o_ref), mean kept mass
// exp(lse_sp - lse_ref), |o_lin - o_ref| / |o_ref|, |o_sp - o_ref| / |o_ref|.
constexpr int kFidelitySplits = 64;
cudaError_t launch_fidelity(const float* o_ref, const float* lse_ref, const float* o_sp, const float* lse_sp,
                            const float* o_lin, int Lq, int H, int d, double* part, double* report, cudaStream_t s);

// ---------------------------------------------------------------- waits.cu
// Write the wait limit (microseconds; 0 = the 2 s default) into a workspace header.
cudaError_t launch_set_wait_limit(int* header, uint32_t limit_us, cudaStream_t s);
// One thread waits on an mbarrier nothing arrives at; the bounded wait must give up
// after the header's limit and record HSA_ERR_TIMEOUT.  waited_ns (optional) gets
// the time the wait took.
cudaError_t launch_wait_selftest(int* status, unsigned long long* waited_ns, cudaStream_t s);

}  // namespace hsa
