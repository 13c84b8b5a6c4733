/*
 * hsa.h -- C ABI of the WorldAttention per-layer attention step on NVIDIA B200
 * (sm_100a): Hierarchical KV Cache (HKV) retrieval + Hybrid Sparse Attention
 * (HSA).
 *
 * Method sources (cited by short name below):
 *   [NEWS] "WorldAttention pairs hierarchical KV caching with hybrid sparse
 *          attention to reach 22 FPS on a single H100 and 0.9472 subject
 *          consistency on VBench-Long" (English news summary of the paper):
 *          HKV paragraph, HSA paragraph, kernel paragraph, open-questions
 *          paragraph.
 *   [PROJ] WorldAttention project page, Method figures ("Overall architecture
 *          of WorldAttention"; "three-tier hierarchical KV cache with
 *          prompt-level and page-level retrieval").
 *
 * Conventions shared by every entry point
 *   - bf16 tensors are passed as hsa_bf16 (the 16-bit pattern).  Token-major
 *     tensors are [tokens, H, d], row stride H*d elements, densely packed.
 *     A history page is K_p, V_p in [P_tok, H, d].
 *   - Every pointer argument is a DEVICE pointer (or, where stated, a pointer
 *     to page-locked host memory mapped into the device address space), 16-byte
 *     aligned.  The caller owns all memory: the library never allocates or
 *     frees device memory and never synchronises a caller's stream
 *     (hsa_status_read and hsa_thread_release are the documented exceptions).
 *     hsa_forward keeps, per host thread and device, one side stream and two
 *     events that it creates on its first call; hsa_thread_release destroys them.
 *   - All work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream).
 *   - Arguments are validated on the host before anything is launched; a
 *     failed check returns HSA_ERR_INVALID_ARG / HSA_ERR_UNSUPPORTED /
 *     HSA_ERR_WORKSPACE and launches nothing.  hsa_last_error_detail() then
 *     describes the check (thread-local text).
 *   - A launch failure returns HSA_ERR_CUDA.  Conditions only the device can
 *     see (for example a candidate page range shorter than Kp, or a bounded
 *     device wait that ran out) are written as an hsa_status_t code into the
 *     status word at the start of the workspace; read it with hsa_status_read
 *     after the stream has reached the call.
 *   - Workspace: one caller-allocated device buffer of hsa_workspace_size()
 *     bytes (256-byte aligned) serves every entry point of a configuration.
 *     Its 256-byte header (status word, ran-out flag, wait limit) must be zero
 *     before first use: allocate it zeroed, or call hsa_status_clear.
 *     Calls that share a workspace must be ordered on one stream.
 *   - Supported shapes: d in {64, 128}; H >= 1; block_inter = 128;
 *     block_intra = 64; rank a multiple of 64 in [64, 1024]; Lc and Lq
 *     multiples of 8; Lq >= 1.  Lc may be 0 (no retrieved history) and need not
 *     be a multiple of 128 (a partial last inter block is the mean of its rows).
 */
#ifndef HSA_H_
#define HSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t hsa_bf16;                  /* bfloat16 bit pattern */
typedef struct CUstream_st* hsa_stream_t;   /* == cudaStream_t */

typedef enum {
  HSA_OK = 0,
  HSA_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad size */
  HSA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. d = 96) */
  HSA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than hsa_workspace_size() */
  HSA_ERR_CUDA = 4,          /* a CUDA launch or API call failed */
  HSA_ERR_TIMEOUT = 5,       /* (device status) a bounded device wait ran out */
  HSA_ERR_DEVICE = 6         /* (device status) a device-side check failed */
} hsa_status_t;

/* Human-readable name of a status code (static storage). */
const char* hsa_status_string(hsa_status_t s);

/* Text of the last failing host-side check on this thread ("" if none). */
const char* hsa_last_error_detail(void);

/* Shape of one HSA call.  [NEWS] HSA paragraph: Binter = 128 against the cached
 * KV, Bintra = 64 inside the current chunk, Linformer rank r. */
typedef struct {
  int H;             /* heads */
  int d;             /* head dim: 64 or 128 */
  int Lq;            /* queries (= chunk tokens = chunk keys) */
  int Lc;            /* cached (retrieved) KV tokens */
  int block_inter;   /* must be 128 */
  int block_intra;   /* must be 64 */
  int rank;          /* Linformer r */
  float scale;       /* softmax scale; 0 means 1/sqrt(d) */
  int select_mode;   /* HSA_SELECT_SEPARATE (0) or HSA_SELECT_JOINT (1), see below */
} hsa_config_t;

/* Block-selection modes ([NEWS] HSA paragraph; the pages do not say whether the
 * cached-KV and in-chunk block masses share one softmax):
 *   HSA_SELECT_SEPARATE  the inter map (128-row query blocks x 128-row Kc blocks)
 *                        and the intra map (64-row query blocks x 64-row Kq blocks)
 *                        are softmaxed and thresholded separately (default);
 *   HSA_SELECT_JOINT     per 64-row query block, its mean query against both the
 *                        Kc 128-row block means and the Kq 64-row block means, one
 *                        softmax and one tau_h threshold over the union; the kept
 *                        Kc blocks then form an inter list per 64-row query block
 *                        (inter_idx [H][nQ64][nKc], inter_cnt [H][nQ64]). */
#define HSA_SELECT_SEPARATE 0
#define HSA_SELECT_JOINT 1

/* Per-head block selections (device buffers, written by hsa_block_select).
 * nQ128 = ceil(Lq/128), nKc = ceil(Lc/128), nQ64 = ceil(Lq/64), nKq = ceil(Lq/64).
 * Row (h, i) of inter_idx holds inter_cnt[h*nQ128+i] ascending block ids of Kc,
 * the rest of the row is unspecified; likewise for intra.  In HSA_SELECT_JOINT
 * mode the inter rows are per 64-row query block (nQ64 rows per head). */
typedef struct {
  int32_t* inter_idx;   /* [H][nQ128][nKc] (joint: [H][nQ64][nKc]) */
  int32_t* inter_cnt;   /* [H][nQ128]      (joint: [H][nQ64])      */
  int32_t* intra_idx;   /* [H][nQ64][nKq]  */
  int32_t* intra_cnt;   /* [H][nQ64]       */
} hsa_selection_t;

/* Bytes of workspace every entry point below needs for `cfg` with NP history
 * pages of P_tok tokens (NP, P_tok may be 0 when only hsa_* calls are used).
 * The size includes the 256-byte status header. */
hsa_status_t hsa_workspace_size(const hsa_config_t* cfg, int NP, int P_tok, size_t* bytes);

/* Clear the device status word of `ws` and its ran-out flag (enqueued on
 * `stream`). */
hsa_status_t hsa_status_clear(void* ws, hsa_stream_t stream);

/* Synchronise `stream`, then copy the device status word of `ws` into *status
 * (an hsa_status_t value).  Synchronises. */
hsa_status_t hsa_status_read(const void* ws, hsa_stream_t stream, int* status);

/* Limit of every bounded device wait of the kernels that use `ws` (mbarrier
 * waits of the tensor-core kernels), in microseconds; 0 restores the 2 s
 * default.  Enqueued on `stream`; kept in the workspace header until changed
 * (hsa_status_clear leaves it).  A wait that runs out records HSA_ERR_TIMEOUT in
 * the status word, sets the workspace's ran-out flag, and its kernel drains its
 * copies and MMAs and exits.  While the flag is set (until hsa_status_clear),
 * every other wait of a kernel using `ws` gives up once it has waited 50 us,
 * so a stalled launch ends after one wait limit rather than one per CTA. */
hsa_status_t hsa_set_wait_limit(void* ws, unsigned int limit_us, hsa_stream_t stream);

/* Self-test of the timeout path (failure detection; the paper has no
 * counterpart): one thread waits on an mbarrier that nothing arrives at, with no
 * copy or MMA in flight.  The wait gives up after the workspace's wait limit and
 * sets HSA_ERR_TIMEOUT in its status word; the context stays usable.
 * waited_ns: optional device uint64 that receives the time the wait took. */
hsa_status_t hsa_selftest_wait(void* ws, unsigned long long* waited_ns, hsa_stream_t stream);

/* Destroy the side stream and events hsa_forward created for this host thread
 * (on every device it ran on), after waiting for the work queued on them.  Call
 * it before a thread that used hsa_forward exits, or to release the handles. */
hsa_status_t hsa_thread_release(void);

/* Host-side fault injection, for tests of a caller's error handling that fault no
 * GPU (failure detection; the pages have no counterpart).  Sets the calling
 * thread's fault kind until it is set back to HSA_FAULT_NONE:
 *   HSA_FAULT_ARG        the configuration check of every entry point that takes
 *                        an hsa_config_t fails: HSA_ERR_INVALID_ARG;
 *   HSA_FAULT_WORKSPACE  the workspace check of every entry point that takes a
 *                        workspace fails: HSA_ERR_WORKSPACE;
 *   HSA_FAULT_LAUNCH     every entry point that launches kernels fails at its
 *                        first launch, before it: HSA_ERR_CUDA.
 * A failing call enqueues no kernel (hsa_forward may already have ordered its
 * side stream after `stream`) and leaves its outputs and the workspace as they
 * were; hsa_last_error_detail() says "injected".  Other threads are not affected.
 * HSA_ERR_INVALID_ARG for an unknown kind. */
#define HSA_FAULT_NONE 0
#define HSA_FAULT_ARG 1
#define HSA_FAULT_WORKSPACE 2
#define HSA_FAULT_LAUNCH 3
hsa_status_t hsa_inject_fault(int kind);

/* ---------------------------------------------------------------- HKV ---- */

/* Page descriptor ([NEWS] HKV paragraph; reading: the mean key of the page per
 * head, computed once when the page is sealed):
 *   kbar[h*d + c] = (1/P_tok) * sum_t K_page[t, h, c]            (fp32 out)
 * K_page: [P_tok, H, d] bf16 (device or mapped pinned host).  kbar: [H*d] fp32.
 * Deterministic (fixed reduction order).  Uses the workspace. */
hsa_status_t hkv_page_summary(const hsa_bf16* K_page, int P_tok, int H, int d, float* kbar,
                              void* ws, size_t ws_bytes, hsa_stream_t stream);

/* 64-row key sums of a page, computed once when it is sealed (reading: the block
 * pooling of the cached KV in [NEWS] HSA paragraph, Binter = 128, can then be done
 * from the page store before the active cache is gathered):
 *   sums64[b * H*d + c] = sum over rows [64 b, min(64 b + 64, P_tok)) of K_page[row, c]
 * K_page: [P_tok, H, d] bf16 (device or mapped pinned host); sums64: fp32
 * [ceil(P_tok/64), H, d].  Fixed order. */
hsa_status_t hkv_page_block_sums(const hsa_bf16* K_page, int P_tok, int H, int d, float* sums64, hsa_stream_t stream);

/* The 128-row key block means of the active cache that the pages sel[0..Kp) would
 * gather to, from their 64-row sums (sums64_pages: [NP, P_tok/64, H, d] fp32, from
 * hkv_page_block_sums), without the gathered copy:
 *   kbar128[j] = (sum of the two 64-row halves of rows [128 j, 128 j + 128)) / rows
 * P_tok must be a multiple of 64 (each half then lies in one page), else
 * HSA_ERR_UNSUPPORTED.  Pass kbar128 to hsa_block_select while hkv_gather copies.
 * An out-of-range page id sets HSA_ERR_DEVICE.  Uses the workspace (status). */
hsa_status_t hkv_block_means_from_pages(const float* sums64_pages, int NP, const int32_t* sel, int Kp, int P_tok,
                                        int H, int d, float* kbar128, void* ws, size_t ws_bytes,
                                        hsa_stream_t stream);

/* Stage 1, prompt-level retrieval ([NEWS] HKV and open-questions paragraphs:
 * Top-1): s* = argmax_s cos(e_cur, e_seg[s]) (ties -> lowest s); then
 *   seg_out[0] = s*,  cand_range_out = { seg_begin[s*], seg_begin[s*+1] }.
 * e_cur: [dim] fp32; e_seg: [n_seg, dim] fp32; seg_begin: [n_seg+1] int32
 * (segment s owns pages [seg_begin[s], seg_begin[s+1])).  All device. */
hsa_status_t hkv_select_prompt(const float* e_cur, const float* e_seg, int n_seg, int dim,
                               const int32_t* seg_begin, int32_t* seg_out, int32_t* cand_range_out,
                               hsa_stream_t stream);

/* Stage 2, page-level retrieval ([NEWS] HKV paragraph, Table 5: Kp = 4):
 *   qbar[h] = mean_t Q[t, h, :];   s_p = sum_h qbar[h] . kbar_pages[p, h, :]
 * keeps the Kp candidates with the largest s_p (ties -> lower p) and writes
 * them to sel_out[0..Kp) in ascending page order.
 * kbar_pages: [NP, H, d] fp32 (from hkv_page_summary).  cand_range: device
 * int32[2] {first, end} or NULL for all NP pages; a range with fewer than Kp
 * pages sets HSA_ERR_DEVICE in the workspace status and writes -1s.
 * scores_out: optional [NP] fp32 (entries outside the range are -inf).
 * Q: [Lq, H, d] bf16.  Uses the workspace. */
hsa_status_t hkv_select_pages(const float* kbar_pages, int NP, const int32_t* cand_range,
                              const hsa_bf16* Q, int Lq, int H, int d, int Kp,
                              int32_t* sel_out, float* scores_out,
                              void* ws, size_t ws_bytes, hsa_stream_t stream);

/* Page-level retrieval in two calls, for a step whose heads are spread over
 * several GPUs (the page score is a sum over heads, the only quantity of the step
 * that mixes heads):
 *   hkv_page_scores  scores_out[p] = sum over the heads of this call of
 *                    qbar[h] . kbar_pages[p, h, :] (as hkv_select_pages), -inf
 *                    outside cand_range; Q, kbar_pages hold these heads only;
 *   (the caller adds the scores of all head groups: an all-reduce)
 *   hkv_select_top   the Kp largest of scores[NP] within cand_range (ties -> lower
 *                    page id), ascending, as hkv_select_pages ranks them.
 * With one head group the two calls select exactly what hkv_select_pages
 * selects.  Both use the workspace. */
hsa_status_t hkv_page_scores(const float* kbar_pages, int NP, const int32_t* cand_range, const hsa_bf16* Q, int Lq,
                             int H, int d, float* scores_out, void* ws, size_t ws_bytes, hsa_stream_t stream);
hsa_status_t hkv_select_top(const float* scores, int NP, const int32_t* cand_range, int Kp, int32_t* sel_out,
                            void* ws, size_t ws_bytes, hsa_stream_t stream);

/* Retrieval policies of the method's retrieval ablations ([NEWS] HKV paragraph,
 * Table 6: page-only, prompt-only, recent-page and random-page retrieval under the
 * same budget of Kp pages; Table 5: the sliding-window cache):
 *   HKV_POLICY_SCORE   the mean-key score of hkv_select_pages (page-only retrieval
 *                      with cand_range NULL, two-stage with the prompt stage's range)
 *   HKV_POLICY_RECENT  the Kp most recent candidates (largest page ids): over all
 *                      pages the sliding window over the history, within the prompt
 *                      stage's range prompt-only retrieval
 *   HKV_POLICY_RANDOM  the Kp candidates with the largest rand_keys[p] (device fp32
 *                      [NP], drawn by the caller, e.g. uniform): a uniform random
 *                      subset; ties -> lower page id
 * Output as hkv_select_pages: sel_out[0..Kp) ascending; scores_out (optional) gets
 * each candidate's ranking key (score, page id or random key), -inf outside the
 * range.  Q is read only by HKV_POLICY_SCORE.  Uses the workspace. */
#define HKV_POLICY_SCORE 0
#define HKV_POLICY_RECENT 1
#define HKV_POLICY_RANDOM 2
hsa_status_t hkv_select_pages_policy(int policy, const float* kbar_pages, int NP, const int32_t* cand_range,
                                     const hsa_bf16* Q, int Lq, int H, int d, int Kp, const float* rand_keys,
                                     int32_t* sel_out, float* scores_out, void* ws, size_t ws_bytes,
                                     hsa_stream_t stream);

/* Active-cache assembly ([NEWS] HKV and kernel paragraphs: KV-cache
 * reorganisation into contiguous memory): for i < Kp,
 *   Kc[i*P_tok + t] = page_k[sel[i]][t],  Vc[i*P_tok + t] = page_v[sel[i]][t]
 * (bitwise copies).  page_k/page_v: device arrays of NP page pointers; a page
 * may live in device memory or in mapped page-locked host memory (the lower
 * tier), read directly by the copy kernel.  sel: device int32[Kp], values
 * checked on the device (out of range -> HSA_ERR_DEVICE status, row skipped).
 * Kc, Vc: [Kp*P_tok, H, d] bf16.  kbar128 (optional): [ceil(Lc/128), H, d]
 * fp32 block means of Kc, fused into the copy (pass it to hsa_block_select). */
hsa_status_t hkv_gather(const hsa_bf16* const* page_k, const hsa_bf16* const* page_v, int NP,
                        const int32_t* sel, int Kp, int P_tok, int H, int d,
                        hsa_bf16* Kc, hsa_bf16* Vc, float* kbar128,
                        void* ws, size_t ws_bytes, hsa_stream_t stream);

/* Allocation-free variant of hkv_select_pages.  The paper has no counterpart:
 * this exists for callers that may not allocate device memory at all -- a host
 * framework that owns every device buffer and passes a plugin only the tensors
 * of the call, a runtime whose memory plan is fixed before it serves, or a loop
 * where an allocation could stall the device -- and so cannot provide the
 * workspace hkv_select_pages uses for its column-sum partials.
 * Same inputs, outputs and results as hkv_select_pages; the scratch (the partial
 * page scores, 256 + 296 * NP * 4 bytes at most) lives in a static device array
 * of 2.3 MiB inside the library, held by every GPU that loads the library until
 * the process exits: NP <= 2048 pages, else HSA_ERR_UNSUPPORTED.  Calls no
 * allocator.
 * status_out: optional device int32 that receives the device status
 * (HSA_ERR_DEVICE for a candidate range shorter than Kp); cleared by the call.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it with the
 * device's current context (a new context, after cudaDeviceReset, looks it up
 * again): make that first call before any stream capture.  Every call on a device shares the
 * array: calls whose kernels could overlap on the GPU race and must be ordered
 * (one stream, or events). */
hsa_status_t hkv_select_pages_noalloc(const float* kbar_pages, int NP, const int32_t* cand_range,
                                      const hsa_bf16* Q, int Lq, int H, int d, int Kp,
                                      int32_t* sel_out, float* scores_out, int32_t* status_out,
                                      hsa_stream_t stream);

/* ------------------------------------------------- tiered page store ---- */

/* Hierarchical KV page store ([NEWS] HKV paragraph: pages live in a hierarchy of
 * memories ranked by cost, unselected pages are demoted to cheaper memory and GPU
 * occupancy stays bounded; [PROJ] "three-tier hierarchical KV cache").  Two tiers:
 * every sealed page in page-locked host memory mapped into the device address
 * space (its authoritative copy: pages do not change once sealed), and up to S
 * pages also in an HBM slot pool.  The store keeps, on the device, a page table
 * (per page, the address hkv_gather reads: its slot when resident, else its host
 * copy) and the residency state; every decision is made on the device from the
 * device-side selection, in a fixed order, so no call waits for the host.
 * The caller allocates all memory:
 *   host_k, host_v  device view of mapped page-locked host memory, [NP][P_tok][H][d]
 *   slot_k, slot_v  device memory, [S][P_tok][H][d]
 *   state           device memory of hkv_store_state_size(NP, S) bytes, 256-aligned
 * Calls on one store must be ordered (one stream, or events). */
typedef struct {
  int NP;            /* pages of the host tier */
  int S;             /* HBM slots */
  int P_tok, H, d;   /* page geometry */
  hsa_bf16* host_k;
  hsa_bf16* host_v;
  hsa_bf16* slot_k;
  hsa_bf16* slot_v;
  void* state;
} hkv_store_t;

/* Bytes of the state buffer (0 for NP < 1 or S < 1). */
size_t hkv_store_state_size(int NP, int S);

/* Every page on the host tier, every slot free (enqueued on `stream`). */
hsa_status_t hkv_store_init(const hkv_store_t* st, hsa_stream_t stream);

/* Device addresses of the store's K and V page tables (arrays of NP page
 * pointers inside `state`), to pass to hkv_gather.  Host-only, launches nothing. */
hsa_status_t hkv_store_tables(const hkv_store_t* st, const hsa_bf16* const** table_k,
                              const hsa_bf16* const** table_v);

/* Seal page `page` ([NEWS] HKV paragraph: pages of Psize frames): copy its P_tok
 * rows K_rows, V_rows ([P_tok, H, d] bf16, device) into the host tier and write
 * its summary kbar_out[H*d] (the mean key per head, as hkv_page_summary) in the
 * same pass over K.  Uses the workspace (hsa_workspace_size with any cfg of these
 * H, d). */
hsa_status_t hkv_store_seal(const hkv_store_t* st, int page, const hsa_bf16* K_rows, const hsa_bf16* V_rows,
                            float* kbar_out, void* ws, size_t ws_bytes, hsa_stream_t stream);

/* Promotion on demand: make the Kp selected pages sel[0..Kp) (device int32, e.g.
 * from hkv_select_pages) resident.  A resident page is touched (its slot's
 * last-use tick set to this call's); a missing page takes the lowest free slot,
 * else the least recently used slot whose page is not selected (ties -> lower
 * slot), whose page is demoted to the host tier; the page is then copied from the
 * host tier into the slot over the host link.  Fewer slots than missing pages, or
 * an out-of-range page id, set HSA_ERR_DEVICE in the workspace status (such a
 * page stays on the host tier and hkv_gather still reads it there). */
hsa_status_t hkv_store_fetch(const hkv_store_t* st, const int32_t* sel, int Kp, void* ws, size_t ws_bytes,
                             hsa_stream_t stream);

/* Speculative promotion: of the pages outside protect[0..n_protect) (device
 * int32; typically the current selection) with a finite score in scores[NP]
 * (device fp32, e.g. hkv_select_pages' scores_out), the m best (score descending,
 * ties -> lower page) are made resident in that order, as hkv_store_fetch would,
 * but never evicting a protected page or one made resident by this call; stops
 * when no slot is left.  Meant for a side stream while a chunk's denoising steps
 * run, so that the next chunk's fetch finds its pages in HBM. */
hsa_status_t hkv_store_prefetch(const hkv_store_t* st, const float* scores, const int32_t* protect, int n_protect,
                                int m, void* ws, size_t ws_bytes, hsa_stream_t stream);

/* Copy the residency state out: slot_of_page[NP] (-1 = host tier only) and
 * page_of_slot[S] (-1 = free); either may be NULL.  Device int32 buffers. */
hsa_status_t hkv_store_residency(const hkv_store_t* st, int32_t* slot_of_page, int32_t* page_of_slot,
                                 hsa_stream_t stream);

/* ---------------------------------------------------------------- HSA ---- */

/* Head-adaptive block selection ([NEWS] HSA paragraph).  Pools Q and Kc into
 * 128-row block means and Q and Kq into 64-row block means (a partial block is
 * the mean of its real rows), scores S = qbar . kbar * scale per head, softmaxes
 * each row, ranks blocks by mass (ties -> lower index) and keeps the shortest
 * prefix whose cumulative mass is >= tau[h] (tau >= 1 keeps all; at least one
 * block).  The inter map (128-query blocks x Kc blocks) and the intra map
 * (64-query blocks x Kq blocks) are thresholded separately.
 * Q, Kq: [Lq, H, d]; Kc: [Lc, H, d] bf16; kbar128: optional fp32 block means of
 * Kc from hkv_gather (NULL -> pooled here); tau: [H] fp32.
 * Masses are accumulated in fp64; scores are fp32. */
hsa_status_t hsa_block_select(const hsa_config_t* cfg, const hsa_bf16* Q, const hsa_bf16* Kc,
                              const hsa_bf16* Kq, const float* kbar128, const float* tau,
                              hsa_selection_t sel, void* ws, size_t ws_bytes, hsa_stream_t stream);

/* Sparse branch ([NEWS] HSA paragraph): for query t of head h, exact softmax
 * attention over the tokens of the Kc blocks sel.inter(h, t/128) together with
 * the Kq blocks sel.intra(h, t/64), one joint softmax, no causal mask:
 *   o_sparse[t, h, :] = sum_k softmax_k(q_t . k * scale) v_k        (fp32 out)
 * Q, Kq, Vq: [Lq, H, d]; Kc, Vc: [Lc, H, d] bf16; o_sparse: [Lq, H, d] fp32. */
hsa_status_t hsa_sparse_attn(const hsa_config_t* cfg, const hsa_bf16* Q, const hsa_bf16* Kc,
                             const hsa_bf16* Vc, const hsa_bf16* Kq, const hsa_bf16* Vq,
                             hsa_selection_t sel, float* o_sparse,
                             void* ws, size_t ws_bytes, hsa_stream_t stream);

/* hsa_sparse_attn that also writes, per query row and head, the natural-log
 * log-sum-exp of the scaled scores over the keys the row attends to:
 *   lse_out[t * H + h] = ln sum_k exp(q_t . k * scale)                  (fp32 [Lq, H])
 * With a selection that keeps every block this is dense attention's, and
 * exp(lse_sparse - lse_dense) is the share of dense attention's softmax mass that
 * falls inside the kept blocks. */
hsa_status_t hsa_sparse_attn_lse(const hsa_config_t* cfg, const hsa_bf16* Q, const hsa_bf16* Kc,
                                 const hsa_bf16* Vc, const hsa_bf16* Kq, const hsa_bf16* Vq,
                                 hsa_selection_t sel, float* o_sparse, float* lse_out,
                                 void* ws, size_t ws_bytes, hsa_stream_t stream);

/* Fidelity of the two branches against dense attention ([NEWS] HSA paragraph,
 * Figure 6: how much of full attention's global mass and output the linear branch
 * keeps), a diagnostic on any inputs.  o_ref / lse_ref: dense attention (the
 * sparse branch with every block kept), o_sparse / lse_sparse: the sparse branch,
 * o_linear: the linear branch, all [Lq, H, d] fp32 (lse [Lq, H]).  Writes, per head
 * h, report[5h + k] (device fp64):
 *   k = 0  cos(o_linear, o_ref)   over the head's rows and columns
 *   k = 1  cos(o_sparse, o_ref)
 *   k = 2  mean over rows of exp(lse_sparse - lse_ref): dense mass kept by the blocks
 *   k = 3  |o_linear - o_ref| / |o_ref|
 *   k = 4  |o_sparse - o_ref| / |o_ref|
 * fp64 sums in a fixed order.  Uses the workspace. */
hsa_status_t hsa_fidelity(const hsa_config_t* cfg, const float* o_ref, const float* lse_ref, const float* o_sparse,
                          const float* lse_sparse, const float* o_linear, double* report,
                          void* ws, size_t ws_bytes, hsa_stream_t stream);

/* Linear branch ([NEWS] HSA paragraph, Linformer-style low rank):
 *   EK_h = E_h [Kc; Kq]_h,  FV_h = F_h [Vc; Vq]_h   (E_h, F_h: [r, L], L = Lc+Lq)
 *   o_linear[t, h, :] = softmax_j(q_t . EK_h[j] * scale) FV_h        (fp32 out)
 * E, F: bf16 [r, L] row-major; head h reads E + h*ef_head_stride, where
 * ef_head_stride is 0 (one matrix shared by all heads) or r*L (H matrices
 * stacked).  EK/FV are accumulated in fp32 and applied with split-bf16 (hi + lo)
 * operands.  Uses the workspace. */
hsa_status_t hsa_linear_attn(const hsa_config_t* cfg, const hsa_bf16* Q, const hsa_bf16* Kc,
                             const hsa_bf16* Vc, const hsa_bf16* Kq, const hsa_bf16* Vq,
                             const hsa_bf16* E, const hsa_bf16* F, long long ef_head_stride,
                             float* o_linear, void* ws, size_t ws_bytes, hsa_stream_t stream);

/* Whole HSA step ([PROJ] overall architecture): block selection, linear branch,
 * sparse branch and the gated merge ([NEWS] HSA paragraph, learned gates;
 * reading: one sigmoid gate per head)
 *   g_h = 1 / (1 + exp(-gate_logit[h]));  out = g_h * o_sparse + (1 - g_h) * o_linear
 * kbar128: optional Kc block means from hkv_gather (NULL -> pooled here).
 * gate_logit may be +-inf (g exactly 1 or 0).  out: [Lq, H, d], fp32 when
 * out_is_bf16 == 0, else bf16.  sel_out: optional; when given, the selection
 * is written there (otherwise kept in the workspace).  Uses the workspace. */
hsa_status_t hsa_forward(const hsa_config_t* cfg, const hsa_bf16* Q, const hsa_bf16* Kc,
                         const hsa_bf16* Vc, const hsa_bf16* Kq, const hsa_bf16* Vq,
                         const float* kbar128, const float* tau, const float* gate_logit,
                         const hsa_bf16* E, const hsa_bf16* F, long long ef_head_stride,
                         void* out, int out_is_bf16, const hsa_selection_t* sel_out,
                         void* ws, size_t ws_bytes, hsa_stream_t stream);

/* hsa_forward with the block selection already made (sel, input: from
 * hsa_block_select): the Linformer branch, the sparse branch and the gated merge.
 * Lets a caller select blocks while the active cache is still being gathered
 * (kbar128 from hkv_block_means_from_pages), then run the rest once it is. */
hsa_status_t hsa_forward_selected(const hsa_config_t* cfg, const hsa_bf16* Q, const hsa_bf16* Kc,
                                  const hsa_bf16* Vc, const hsa_bf16* Kq, const hsa_bf16* Vq,
                                  const float* gate_logit, const hsa_bf16* E, const hsa_bf16* F,
                                  long long ef_head_stride, const hsa_selection_t* sel, void* out,
                                  int out_is_bf16, void* ws, size_t ws_bytes, hsa_stream_t stream);

/* hsa_forward with options (flags, OR-ed):
 *   HSA_FWD_SELECTED  sel is an input (the block selection already made); tau and
 *                     kbar128 are not read
 *   HSA_FWD_HISTORY   the cached KV's Linformer products are in the workspace
 *                     (hsa_prepare_history or hkv_gather_project): only the chunk's
 *                     own keys and values are projected, as hsa_forward_reuse
 * flags = 0 is hsa_forward. */
#define HSA_FWD_SELECTED 1u
#define HSA_FWD_HISTORY 2u
hsa_status_t hsa_forward_ex(const hsa_config_t* cfg, const hsa_bf16* Q, const hsa_bf16* Kc, const hsa_bf16* Vc,
                            const hsa_bf16* Kq, const hsa_bf16* Vq, const float* kbar128, const float* tau,
                            const float* gate_logit, const hsa_bf16* E, const hsa_bf16* F, long long ef_head_stride,
                            void* out, int out_is_bf16, const hsa_selection_t* sel, unsigned flags,
                            void* ws, size_t ws_bytes, hsa_stream_t stream);

/* The active-cache gather and the history's Linformer products in one call
 * ([NEWS] kernel paragraph: the KV copies dominate the preprocessing):
 *   Kc, Vc                as hkv_gather (bitwise copies of pages sel[0..Kp));
 *   history products      as hsa_prepare_history (E_h[:, 0:Lc] Kc_h, F_h[:, 0:Lc] Vc_h,
 *                         fp32 in the workspace), for hsa_forward_reuse /
 *                         hsa_forward_ex(HSA_FWD_HISTORY).
 * Enqueues the gather, then the projection, on `stream`.  Requires Kp * P_tok ==
 * cfg->Lc.  Page tables as hkv_gather; an out-of-range page id sets HSA_ERR_DEVICE.
 * Uses the workspace. */
hsa_status_t hkv_gather_project(const hsa_config_t* cfg, const hsa_bf16* const* page_k, const hsa_bf16* const* page_v,
                                int NP, const int32_t* sel, int Kp, int P_tok, const hsa_bf16* E, const hsa_bf16* F,
                                long long ef_head_stride, hsa_bf16* Kc, hsa_bf16* Vc,
                                void* ws, size_t ws_bytes, hsa_stream_t stream);

/* Multi-step reuse ([NEWS] HKV paragraph: retrieval assembles the active cache of
 * the current chunk; kernel paragraph: KV reorganisation and copies dominate the
 * preprocessing; reading: a chunk is denoised over several steps against one
 * retrieval, so the history part of the step is done once per chunk).
 *
 * hsa_prepare_history projects the cached KV once per chunk:
 *   EKc_h = E_h[:, 0:Lc] Kc_h,   FVc_h = F_h[:, 0:Lc] Vc_h        (fp32, kept in ws)
 * hsa_forward_reuse is hsa_forward for one denoising step of that chunk: it
 * projects only the chunk's own keys and values and adds the kept products,
 *   EK_h = EKc_h + E_h[:, Lc:L] Kq_h,   FV_h = FVc_h + F_h[:, Lc:L] Vq_h,
 * then selects blocks, runs both branches and merges exactly as hsa_forward (same
 * arguments and results).  Kc, Vc, E, F and the workspace must be the ones given
 * to the last hsa_prepare_history of this workspace; Q, Kq, Vq, tau and the gate
 * logits may change from step to step.  kbar128 from hkv_gather stays valid for
 * the chunk.  Both use the workspace; the kept products live in it (2 H r d fp32). */
hsa_status_t hsa_prepare_history(const hsa_config_t* cfg, const hsa_bf16* Kc, const hsa_bf16* Vc,
                                 const hsa_bf16* E, const hsa_bf16* F, long long ef_head_stride,
                                 void* ws, size_t ws_bytes, hsa_stream_t stream);
hsa_status_t hsa_forward_reuse(const hsa_config_t* cfg, const hsa_bf16* Q, const hsa_bf16* Kc,
                               const hsa_bf16* Vc, const hsa_bf16* Kq, const hsa_bf16* Vq,
                               const float* kbar128, const float* tau, const float* gate_logit,
                               const hsa_bf16* E, const hsa_bf16* F, long long ef_head_stride,
                               void* out, int out_is_bf16, const hsa_selection_t* sel_out,
                               void* ws, size_t ws_bytes, hsa_stream_t stream);

/* Optional per-kernel timing hook (tracing).  When `events` is non-NULL, the
 * next entry-point calls on this thread record events[2*k] before and
 * events[2*k+1] after their k-th kernel launch, for k < n_pairs, and store the
 * kernel's name pointer in names[k] (may be NULL).  hsa_trace_count() returns
 * how many pairs were recorded since the last hsa_trace_begin(). */
hsa_status_t hsa_trace_begin(void* const* events, int n_pairs, const char** names);
int hsa_trace_count(void);
hsa_status_t hsa_trace_end(void);

#ifdef __cplusplus
}
#endif

#endif /* HSA_H_ */
