"""One per-layer HKV + HSA step over a page store, through the C ABI.

``HkvHsaStep`` owns the device buffers of a step (selected page ids, the
contiguous active cache, block selections, workspace, output) and issues the
C-ABI calls in the order of the method's overall architecture (WorldAttention
project page, figure "Overall architecture of WorldAttention"): optional
prompt-level Top-1, page-level top-Kp retrieval, gather, HSA forward.  All
arithmetic happens in the library's kernels.
"""
from __future__ import annotations

import torch

from . import (FWD_SELECTED, SelectionBuffers, hkv_block_means_from_pages, hkv_gather,
               hkv_page_block_sums, hkv_page_summary, hkv_select_pages, hkv_select_prompt,
               hsa_block_select, hsa_forward, hsa_forward_ex, hsa_forward_reuse, hsa_prepare_history,
               hsa_workspace_size, make_config)


def page_pointers(pages: torch.Tensor) -> torch.Tensor:
    """Device int64 tensor of the base addresses of pages[p] for a [NP, P_tok, H, d] store
    (device memory or page-locked host memory)."""
    NP = pages.shape[0]
    stride = pages.stride(0) * pages.element_size()
    base = pages.data_ptr()
    return torch.tensor([base + p * stride for p in range(NP)], dtype=torch.int64, device="cuda")


class HkvHsaStep:
    def __init__(self, H, d, Lq, P_tok, NP, Kp, rank, page_k_ptrs, page_v_ptrs, out_dtype=torch.float32,
                 scale=0.0, device="cuda", store=None):
        """page_k_ptrs / page_v_ptrs: device int64 page tables read by the gather.  With a
        tiered page store (`store`, a PageStore), pass its tables: every retrieval is
        then followed by the store's fetch (the selected pages made resident in HBM)."""
        self.H, self.d, self.Lq, self.P_tok, self.NP, self.Kp, self.rank = H, d, Lq, P_tok, NP, Kp, rank
        self.store = store
        self.Lc = Kp * P_tok
        self.cfg = make_config(H, d, Lq, self.Lc, rank, scale)
        dev = torch.device(device)
        self.page_k_ptrs, self.page_v_ptrs = page_k_ptrs, page_v_ptrs
        self.kbar_pages = torch.zeros(NP, H, d, dtype=torch.float32, device=dev)
        self.sel = torch.zeros(Kp, dtype=torch.int32, device=dev)
        self.scores = torch.zeros(NP, dtype=torch.float32, device=dev)
        self.cand_range = torch.zeros(2, dtype=torch.int32, device=dev)
        self.seg = torch.zeros(1, dtype=torch.int32, device=dev)
        self.Kc = torch.empty(self.Lc, H, d, dtype=torch.bfloat16, device=dev)
        self.Vc = torch.empty(self.Lc, H, d, dtype=torch.bfloat16, device=dev)
        self.kbar128 = torch.zeros(-(-self.Lc // 128), H, d, dtype=torch.float32, device=dev)
        self.selection = SelectionBuffers.empty(self.cfg, dev)
        self.ws = torch.zeros(hsa_workspace_size(self.cfg, NP, P_tok), dtype=torch.uint8, device=dev)
        self.out = torch.empty(Lq, H, d, dtype=out_dtype, device=dev)
        # Pages of a multiple of 64 rows keep their 64-row key sums (from the seal): the
        # block selection then runs from them while the gather copies, on its own stream.
        self.early = P_tok % 64 == 0
        self.sums64 = torch.zeros(NP, P_tok // 64, H, d, dtype=torch.float32, device=dev) if self.early else None
        self.gather_stream = torch.cuda.Stream(device=dev) if self.early else None
        self.ev_sel = torch.cuda.Event()
        self.ev_gathered = torch.cuda.Event()

    def seal_pages(self, pages_k):
        """Page summaries (mean key per head) and, when kept, 64-row key sums of every
        page, computed once.  pages_k: [NP, P_tok, H, d] tensor or a list of pages."""
        for p in range(self.NP):
            hkv_page_summary(pages_k[p], self.kbar_pages[p], self.ws)
            if self.early:
                hkv_page_block_sums(pages_k[p], self.sums64[p])

    def _retrieve(self, Q, cand):
        """Page-level retrieval into self.sel (self.scores: the page scores)."""
        hkv_select_pages(self.kbar_pages, Q, self.Kp, self.sel, self.ws, self.scores, cand)
        return self.sel

    def __call__(self, Q, Kq, Vq, tau, gate_logit, E, F, e_cur=None, e_seg=None, seg_begin=None,
                 ef_head_stride=0, out=None):
        """One step on the current stream; the result goes to `out` (same shape and
        dtype as self.out) when given, else to self.out."""
        dst = self.out if out is None else out
        cand = None
        if e_cur is not None:
            hkv_select_prompt(e_cur, e_seg, seg_begin, self.seg, self.cand_range)
            cand = self.cand_range
        self._retrieve(Q, cand)
        if self.store is not None:
            self.store.fetch(self.sel, self.ws)
        if not self.early:
            hkv_gather(self.page_k_ptrs, self.page_v_ptrs, self.sel, self.Kp, self.P_tok, self.H, self.d,
                       self.Kc, self.Vc, self.ws, self.kbar128)
            hsa_forward(self.cfg, Q, self.Kc, self.Vc, Kq, Vq, tau, gate_logit, E, F, dst, self.ws,
                        self.kbar128, self.selection, ef_head_stride)
            return dst
        # the cache's block means from the pages' sums; then, on its own stream, the
        # gather (HBM-bound) while this stream pools the chunk and selects blocks; then
        # the Linformer projection (beside the plan) and the attention
        main = torch.cuda.current_stream()
        hkv_block_means_from_pages(self.sums64, self.sel, self.Kp, self.P_tok, self.H, self.d, self.kbar128, self.ws)
        self.ev_sel.record(main)
        self.gather_stream.wait_event(self.ev_sel)
        hkv_gather(self.page_k_ptrs, self.page_v_ptrs, self.sel, self.Kp, self.P_tok, self.H, self.d,
                   self.Kc, self.Vc, self.ws, stream=self.gather_stream)
        self.ev_gathered.record(self.gather_stream)
        hsa_block_select(self.cfg, Q, self.Kc, Kq, tau, self.selection, self.ws, self.kbar128)
        main.wait_event(self.ev_gathered)
        hsa_forward_ex(self.cfg, Q, self.Kc, self.Vc, Kq, Vq, tau, gate_logit, E, F, dst, self.ws, self.selection,
                       FWD_SELECTED, ef_head_stride=ef_head_stride)
        return dst

    # ------------------------------------------------------------ multi-step reuse
    def prepare_chunk(self, Q, E, F, e_cur=None, e_seg=None, seg_begin=None, ef_head_stride=0):
        """Once per chunk: retrieval (prompt-level, page-level) with the chunk's queries,
        the gather of the active cache, and the cached KV's Linformer products."""
        cand = None
        if e_cur is not None:
            hkv_select_prompt(e_cur, e_seg, seg_begin, self.seg, self.cand_range)
            cand = self.cand_range
        self._retrieve(Q, cand)
        if self.store is not None:
            self.store.fetch(self.sel, self.ws)
        hkv_gather(self.page_k_ptrs, self.page_v_ptrs, self.sel, self.Kp, self.P_tok, self.H, self.d,
                   self.Kc, self.Vc, self.ws, self.kbar128)
        hsa_prepare_history(self.cfg, self.Kc, self.Vc, E, F, self.ws, ef_head_stride)

    def denoise_step(self, Q, Kq, Vq, tau, gate_logit, E, F, ef_head_stride=0, out=None):
        """One denoising step of the prepared chunk (block selection, both branches, merge)."""
        dst = self.out if out is None else out
        hsa_forward_reuse(self.cfg, Q, self.Kc, self.Vc, Kq, Vq, tau, gate_logit, E, F, dst, self.ws,
                          self.kbar128, self.selection, ef_head_stride)
        return dst

    def prefetch(self, m, ws, stream=None):
        """Speculative promotion of the m best-scoring pages not selected by the last
        retrieval (its scores), e.g. on a side stream during the chunk's denoising
        steps.  `ws` is a workspace of its own (its status word), so that it does not
        race with the steps' use of self.ws."""
        if self.store is not None:
            self.store.prefetch(self.scores, self.sel, m, ws, stream)
