"""Python binding of ``libhsa.so``: the WorldAttention HKV + HSA attention step on B200.

Argument marshalling only.  Every step of the computation runs in the library's
CUDA kernels; torch supplies device memory, streams and events.  If the native
library is missing this module raises on first use -- there is no fallback.

The function names and argument orders mirror ``include/hsa.h``.
"""
from __future__ import annotations

import ctypes
import os
from contextlib import contextmanager
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhsa.so")

HSA_STATUS = {0: "HSA_OK", 1: "HSA_ERR_INVALID_ARG", 2: "HSA_ERR_UNSUPPORTED", 3: "HSA_ERR_WORKSPACE",
              4: "HSA_ERR_CUDA", 5: "HSA_ERR_TIMEOUT", 6: "HSA_ERR_DEVICE"}

EXPORTED = [
    "hsa_status_string", "hsa_last_error_detail", "hsa_workspace_size", "hsa_status_clear", "hsa_status_read",
    "hkv_page_summary", "hkv_select_prompt", "hkv_select_pages", "hkv_select_pages_noalloc", "hkv_gather",
    "hsa_block_select", "hsa_sparse_attn", "hsa_linear_attn", "hsa_forward",
    "hsa_trace_begin", "hsa_trace_count", "hsa_trace_end", "hsa_set_wait_limit", "hsa_selftest_wait",
    "hsa_thread_release", "hsa_prepare_history", "hsa_forward_reuse",
    "hkv_store_state_size", "hkv_store_init", "hkv_store_tables", "hkv_store_seal", "hkv_store_fetch",
    "hkv_store_prefetch", "hkv_store_residency", "hkv_select_pages_policy", "hkv_page_scores", "hkv_select_top",
    "hsa_sparse_attn_lse", "hsa_fidelity", "hkv_page_block_sums", "hkv_block_means_from_pages",
    "hsa_forward_selected", "hsa_forward_ex", "hkv_gather_project", "hsa_inject_fault",
]

FWD_SELECTED, FWD_HISTORY = 1, 2

POLICY_SCORE, POLICY_RECENT, POLICY_RANDOM = 0, 1, 2


class HsaError(RuntimeError):
    def __init__(self, code: int, where: str, detail: str):
        super().__init__(f"{where}: {HSA_STATUS.get(code, code)}: {detail}")
        self.code = code


class Config(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int), ("d", ctypes.c_int), ("Lq", ctypes.c_int), ("Lc", ctypes.c_int),
                ("block_inter", ctypes.c_int), ("block_intra", ctypes.c_int), ("rank", ctypes.c_int),
                ("scale", ctypes.c_float), ("select_mode", ctypes.c_int)]


SELECT_SEPARATE, SELECT_JOINT = 0, 1


class StoreDesc(ctypes.Structure):
    """hkv_store_t: the memories of a tiered page store (all device addresses)."""
    _fields_ = [("NP", ctypes.c_int), ("S", ctypes.c_int), ("P_tok", ctypes.c_int), ("H", ctypes.c_int),
                ("d", ctypes.c_int), ("host_k", ctypes.c_void_p), ("host_v", ctypes.c_void_p),
                ("slot_k", ctypes.c_void_p), ("slot_v", ctypes.c_void_p), ("state", ctypes.c_void_p)]


class _Selection(ctypes.Structure):
    _fields_ = [("inter_idx", ctypes.c_void_p), ("inter_cnt", ctypes.c_void_p),
                ("intra_idx", ctypes.c_void_p), ("intra_cnt", ctypes.c_void_p)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load the native library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m hybrid_sparse_attention_hkv_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, L, S, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t, ctypes.c_float
    CP = ctypes.POINTER(Config)
    sig = {
        "hsa_status_string": (ctypes.c_char_p, [I]),
        "hsa_last_error_detail": (ctypes.c_char_p, []),
        "hsa_workspace_size": (I, [CP, I, I, ctypes.POINTER(S)]),
        "hsa_status_clear": (I, [P, P]),
        "hsa_status_read": (I, [P, P, ctypes.POINTER(I)]),
        "hkv_page_summary": (I, [P, I, I, I, P, P, S, P]),
        "hkv_select_prompt": (I, [P, P, I, I, P, P, P, P]),
        "hkv_select_pages": (I, [P, I, P, P, I, I, I, I, P, P, P, S, P]),
        "hkv_select_pages_noalloc": (I, [P, I, P, P, I, I, I, I, P, P, P, P]),
        "hkv_gather": (I, [P, P, I, P, I, I, I, I, P, P, P, P, S, P]),
        "hsa_block_select": (I, [CP, P, P, P, P, P, _Selection, P, S, P]),
        "hsa_sparse_attn": (I, [CP, P, P, P, P, P, _Selection, P, P, S, P]),
        "hsa_linear_attn": (I, [CP, P, P, P, P, P, P, P, L, P, P, S, P]),
        "hsa_forward": (I, [CP, P, P, P, P, P, P, P, P, P, P, L, P, I, ctypes.POINTER(_Selection), P, S, P]),
        "hsa_trace_begin": (I, [P, I, P]),
        "hsa_trace_count": (I, []),
        "hsa_trace_end": (I, []),
        "hsa_prepare_history": (I, [CP, P, P, P, P, L, P, S, P]),
        "hsa_forward_reuse": (I, [CP, P, P, P, P, P, P, P, P, P, P, L, P, I, ctypes.POINTER(_Selection), P, S,
                                  P]),
        "hkv_select_pages_policy": (I, [I, P, I, P, P, I, I, I, I, P, P, P, P, S, P]),
        "hkv_page_scores": (I, [P, I, P, P, I, I, I, P, P, S, P]),
        "hsa_sparse_attn_lse": (I, [CP, P, P, P, P, P, _Selection, P, P, P, S, P]),
        "hkv_page_block_sums": (I, [P, I, I, I, P, P]),
        "hkv_block_means_from_pages": (I, [P, I, P, I, I, I, I, P, P, S, P]),
        "hsa_forward_selected": (I, [CP, P, P, P, P, P, P, P, P, L, ctypes.POINTER(_Selection), P, I, P, S, P]),
        "hsa_forward_ex": (I, [CP, P, P, P, P, P, P, P, P, P, P, L, P, I, ctypes.POINTER(_Selection), ctypes.c_uint,
                               P, S, P]),
        "hkv_gather_project": (I, [CP, P, P, I, P, I, I, P, P, L, P, P, P, S, P]),
        "hsa_fidelity": (I, [CP, P, P, P, P, P, P, P, S, P]),
        "hkv_select_top": (I, [P, I, P, I, P, P, S, P]),
        "hkv_store_state_size": (S, [I, I]),
        "hkv_store_init": (I, [ctypes.POINTER(StoreDesc), P]),
        "hkv_store_tables": (I, [ctypes.POINTER(StoreDesc), ctypes.POINTER(P), ctypes.POINTER(P)]),
        "hkv_store_seal": (I, [ctypes.POINTER(StoreDesc), I, P, P, P, P, S, P]),
        "hkv_store_fetch": (I, [ctypes.POINTER(StoreDesc), P, I, P, S, P]),
        "hkv_store_prefetch": (I, [ctypes.POINTER(StoreDesc), P, P, I, I, P, S, P]),
        "hkv_store_residency": (I, [ctypes.POINTER(StoreDesc), P, P, P]),
        "hsa_set_wait_limit": (I, [P, ctypes.c_uint, P]),
        "hsa_selftest_wait": (I, [P, P, P]),
        "hsa_thread_release": (I, []),
        "hsa_inject_fault": (I, [I]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(code: int, where: str):
    if code != 0:
        detail = load_library().hsa_last_error_detail().decode()
        raise HsaError(code, where, detail)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def make_config(H, d, Lq, Lc, rank=0, scale=0.0, block_inter=128, block_intra=64, select_mode=0) -> Config:
    return Config(H, d, Lq, Lc, block_inter, block_intra, rank, scale, select_mode)


def hsa_workspace_size(cfg: Config, NP: int = 0, P_tok: int = 0) -> int:
    n = ctypes.c_size_t(0)
    _check(load_library().hsa_workspace_size(ctypes.byref(cfg), NP, P_tok, ctypes.byref(n)), "hsa_workspace_size")
    return n.value


def workspace(cfg: Config, device="cuda") -> torch.Tensor:
    """A zeroed device workspace of hsa_workspace_size(cfg) bytes (256-byte aligned by torch)."""
    return torch.zeros(hsa_workspace_size(cfg), dtype=torch.uint8, device=device)


def hsa_status_clear(ws, stream=None):
    _check(load_library().hsa_status_clear(_p(ws), _stream(stream)), "hsa_status_clear")


def wait_report(ws) -> dict:
    """The workspace header's record of a bounded wait that ran out: the status word,
    the ran-out flag, and the site (kind << 24 | warp << 16 | tile, 0 if none) and CTA
    of the first such wait.  Reads the header after synchronising the device."""
    torch.cuda.synchronize(ws.device)
    w = ws[:24].view(torch.int32).cpu().tolist()
    site = w[4]
    return {"status": w[0], "ran_out": w[1], "site": site, "kind": site >> 24, "warp": (site >> 16) & 0xFF,
            "tile": site & 0xFFFF, "cta": w[5]}


def hsa_status_read(ws, stream=None) -> int:
    st = ctypes.c_int(0)
    _check(load_library().hsa_status_read(_p(ws), _stream(stream), ctypes.byref(st)), "hsa_status_read")
    return st.value


def hsa_set_wait_limit(ws, limit_us: int, stream=None):
    """Limit of the bounded device waits of kernels using `ws` (microseconds; 0 = 2 s default)."""
    _check(load_library().hsa_set_wait_limit(_p(ws), int(limit_us), _stream(stream)), "hsa_set_wait_limit")


def hsa_selftest_wait(ws, waited_ns=None, stream=None):
    """Run the timeout self-test kernel (an mbarrier wait nothing completes)."""
    _check(load_library().hsa_selftest_wait(_p(ws), _p(waited_ns), _stream(stream)), "hsa_selftest_wait")


def hsa_thread_release():
    _check(load_library().hsa_thread_release(), "hsa_thread_release")


FAULT_NONE, FAULT_ARG, FAULT_WORKSPACE, FAULT_LAUNCH = 0, 1, 2, 3


def hsa_inject_fault(kind: int):
    """Make this thread's library calls fail at their configuration check
    (FAULT_ARG), workspace check (FAULT_WORKSPACE) or first kernel launch
    (FAULT_LAUNCH) until FAULT_NONE is set again."""
    _check(load_library().hsa_inject_fault(int(kind)), "hsa_inject_fault")


@contextmanager
def injected_fault(kind: int):
    """hsa_inject_fault(kind) for the duration of a with-block."""
    hsa_inject_fault(kind)
    try:
        yield
    finally:
        hsa_inject_fault(FAULT_NONE)


@dataclass
class SelectionBuffers:
    """Device buffers of one hsa_selection_t for a configuration."""
    inter_idx: torch.Tensor
    inter_cnt: torch.Tensor
    intra_idx: torch.Tensor
    intra_cnt: torch.Tensor

    @staticmethod
    def empty(cfg: Config, device="cuda") -> "SelectionBuffers":
        """Buffers of one selection; in joint mode the inter rows are per 64-row query block."""
        nQ128, nQ64 = -(-cfg.Lq // 128), -(-cfg.Lq // 64)
        if cfg.select_mode == SELECT_JOINT:
            nQ128 = nQ64
        nKc = -(-cfg.Lc // 128)
        i32 = dict(dtype=torch.int32, device=device)
        return SelectionBuffers(torch.zeros(cfg.H, nQ128, max(nKc, 1), **i32), torch.zeros(cfg.H, nQ128, **i32),
                                torch.zeros(cfg.H, nQ64, nQ64, **i32), torch.zeros(cfg.H, nQ64, **i32))

    def c(self) -> _Selection:
        return _Selection(self.inter_idx.data_ptr(), self.inter_cnt.data_ptr(),
                          self.intra_idx.data_ptr(), self.intra_cnt.data_ptr())


# ---------------------------------------------------------------- HKV

def hkv_page_summary(K_page, kbar, ws, stream=None):
    P_tok, H, d = K_page.shape
    _check(load_library().hkv_page_summary(_p(K_page), P_tok, H, d, _p(kbar), _p(ws), ws.numel(), _stream(stream)),
           "hkv_page_summary")


def hkv_select_prompt(e_cur, e_seg, seg_begin, seg_out, cand_range_out, stream=None):
    n_seg, dim = e_seg.shape
    _check(load_library().hkv_select_prompt(_p(e_cur), _p(e_seg), n_seg, dim, _p(seg_begin), _p(seg_out),
                                            _p(cand_range_out), _stream(stream)), "hkv_select_prompt")


def hkv_select_pages(kbar_pages, Q, Kp, sel_out, ws, scores_out=None, cand_range=None, stream=None):
    NP = kbar_pages.shape[0]
    Lq, H, d = Q.shape
    _check(load_library().hkv_select_pages(_p(kbar_pages), NP, _p(cand_range), _p(Q), Lq, H, d, Kp, _p(sel_out),
                                           _p(scores_out), _p(ws), ws.numel(), _stream(stream)), "hkv_select_pages")


def hkv_page_scores(kbar_pages, Q, scores_out, ws, cand_range=None, stream=None):
    """Page scores summed over the heads of Q / kbar_pages (one head group)."""
    NP = kbar_pages.shape[0]
    Lq, H, d = Q.shape
    _check(load_library().hkv_page_scores(_p(kbar_pages), NP, _p(cand_range), _p(Q), Lq, H, d, _p(scores_out), _p(ws),
                                          ws.numel(), _stream(stream)), "hkv_page_scores")


def hkv_select_top(scores, Kp, sel_out, ws, cand_range=None, stream=None):
    """Top-Kp pages of the (all-reduced) page scores, ascending."""
    _check(load_library().hkv_select_top(_p(scores), scores.numel(), _p(cand_range), Kp, _p(sel_out), _p(ws),
                                         ws.numel(), _stream(stream)), "hkv_select_top")


def hkv_select_pages_policy(policy, kbar_pages, Q, Kp, sel_out, ws, scores_out=None, cand_range=None,
                            rand_keys=None, stream=None):
    """Page retrieval by policy: POLICY_SCORE (mean-key score), POLICY_RECENT, POLICY_RANDOM."""
    NP = kbar_pages.shape[0]
    Lq, H, d = Q.shape
    _check(load_library().hkv_select_pages_policy(policy, _p(kbar_pages), NP, _p(cand_range), _p(Q), Lq, H, d, Kp,
                                                  _p(rand_keys), _p(sel_out), _p(scores_out), _p(ws), ws.numel(),
                                                  _stream(stream)), "hkv_select_pages_policy")


def hkv_select_pages_noalloc(kbar_pages, Q, Kp, sel_out, scores_out=None, cand_range=None, status_out=None,
                             stream=None):
    """hkv_select_pages without a workspace (scratch in a static device array)."""
    NP = kbar_pages.shape[0]
    Lq, H, d = Q.shape
    _check(load_library().hkv_select_pages_noalloc(_p(kbar_pages), NP, _p(cand_range), _p(Q), Lq, H, d, Kp,
                                                   _p(sel_out), _p(scores_out), _p(status_out), _stream(stream)),
           "hkv_select_pages_noalloc")


def hkv_page_block_sums(K_page, sums64, stream=None):
    """64-row key sums of one page ([ceil(P_tok/64), H, d] fp32)."""
    P_tok, H, d = K_page.shape
    _check(load_library().hkv_page_block_sums(_p(K_page), P_tok, H, d, _p(sums64), _stream(stream)),
           "hkv_page_block_sums")


def hkv_block_means_from_pages(sums64_pages, sel, Kp, P_tok, H, d, kbar128, ws, stream=None):
    NP = sums64_pages.shape[0]
    _check(load_library().hkv_block_means_from_pages(_p(sums64_pages), NP, _p(sel), Kp, P_tok, H, d, _p(kbar128),
                                                     _p(ws), ws.numel(), _stream(stream)),
           "hkv_block_means_from_pages")


def hkv_gather(page_k_ptrs, page_v_ptrs, sel, Kp, P_tok, H, d, Kc, Vc, ws, kbar128=None, stream=None):
    """page_k_ptrs / page_v_ptrs: device int64 tensors [NP] of page base addresses."""
    NP = page_k_ptrs.numel()
    _check(load_library().hkv_gather(_p(page_k_ptrs), _p(page_v_ptrs), NP, _p(sel), Kp, P_tok, H, d, _p(Kc), _p(Vc),
                                     _p(kbar128), _p(ws), ws.numel(), _stream(stream)), "hkv_gather")


# ---------------------------------------------------------------- HSA

def hsa_block_select(cfg, Q, Kc, Kq, tau, sel: SelectionBuffers, ws, kbar128=None, stream=None):
    _check(load_library().hsa_block_select(ctypes.byref(cfg), _p(Q), _p(Kc), _p(Kq), _p(kbar128), _p(tau), sel.c(),
                                           _p(ws), ws.numel(), _stream(stream)), "hsa_block_select")


def hsa_sparse_attn(cfg, Q, Kc, Vc, Kq, Vq, sel: SelectionBuffers, o_sparse, ws, stream=None):
    _check(load_library().hsa_sparse_attn(ctypes.byref(cfg), _p(Q), _p(Kc), _p(Vc), _p(Kq), _p(Vq), sel.c(),
                                          _p(o_sparse), _p(ws), ws.numel(), _stream(stream)), "hsa_sparse_attn")


def hsa_sparse_attn_lse(cfg, Q, Kc, Vc, Kq, Vq, sel: SelectionBuffers, o_sparse, lse, ws, stream=None):
    _check(load_library().hsa_sparse_attn_lse(ctypes.byref(cfg), _p(Q), _p(Kc), _p(Vc), _p(Kq), _p(Vq), sel.c(),
                                              _p(o_sparse), _p(lse), _p(ws), ws.numel(), _stream(stream)),
           "hsa_sparse_attn_lse")


def hsa_fidelity(cfg, o_ref, lse_ref, o_sparse, lse_sparse, o_linear, report, ws, stream=None):
    """report: device float64 [H, 5] (see include/hsa.h)."""
    _check(load_library().hsa_fidelity(ctypes.byref(cfg), _p(o_ref), _p(lse_ref), _p(o_sparse), _p(lse_sparse),
                                       _p(o_linear), _p(report), _p(ws), ws.numel(), _stream(stream)), "hsa_fidelity")


def fidelity_report(cfg, Q, Kc, Vc, Kq, Vq, E, F, sel: SelectionBuffers, ws, ef_head_stride=0):
    """Both branches of one step against dense attention (the sparse branch with every
    block kept): float64 [H, 5] on the device (include/hsa.h, hsa_fidelity)."""
    dense = SelectionBuffers.empty(cfg)
    ones = torch.ones(cfg.H, dtype=torch.float32, device=Q.device)
    hsa_block_select(cfg, Q, Kc, Kq, ones, dense, ws)
    shape = (cfg.Lq, cfg.H, cfg.d)
    o_ref, o_sp, o_lin = (torch.empty(shape, dtype=torch.float32, device=Q.device) for _ in range(3))
    lse_ref = torch.empty(cfg.Lq, cfg.H, dtype=torch.float32, device=Q.device)
    lse_sp = torch.empty_like(lse_ref)
    hsa_sparse_attn_lse(cfg, Q, Kc, Vc, Kq, Vq, dense, o_ref, lse_ref, ws)
    hsa_sparse_attn_lse(cfg, Q, Kc, Vc, Kq, Vq, sel, o_sp, lse_sp, ws)
    hsa_linear_attn(cfg, Q, Kc, Vc, Kq, Vq, E, F, o_lin, ws, ef_head_stride)
    report = torch.empty(cfg.H, 5, dtype=torch.float64, device=Q.device)
    hsa_fidelity(cfg, o_ref, lse_ref, o_sp, lse_sp, o_lin, report, ws)
    return report


def hsa_linear_attn(cfg, Q, Kc, Vc, Kq, Vq, E, F, o_linear, ws, ef_head_stride=0, stream=None):
    _check(load_library().hsa_linear_attn(ctypes.byref(cfg), _p(Q), _p(Kc), _p(Vc), _p(Kq), _p(Vq), _p(E), _p(F),
                                          ef_head_stride, _p(o_linear), _p(ws), ws.numel(), _stream(stream)),
           "hsa_linear_attn")


def hsa_forward(cfg, Q, Kc, Vc, Kq, Vq, tau, gate_logit, E, F, out, ws, kbar128=None, sel=None,
                ef_head_stride=0, stream=None):
    """out: [Lq, H, d] float32 or bfloat16 tensor."""
    csel = ctypes.byref(sel.c()) if sel is not None else None
    _check(load_library().hsa_forward(ctypes.byref(cfg), _p(Q), _p(Kc), _p(Vc), _p(Kq), _p(Vq), _p(kbar128),
                                      _p(tau), _p(gate_logit), _p(E), _p(F), ef_head_stride, _p(out),
                                      1 if out.dtype == torch.bfloat16 else 0, csel, _p(ws), ws.numel(),
                                      _stream(stream)), "hsa_forward")


def hsa_forward_selected(cfg, Q, Kc, Vc, Kq, Vq, gate_logit, E, F, sel: SelectionBuffers, out, ws, ef_head_stride=0,
                         stream=None):
    """hsa_forward with the selection `sel` already made (input)."""
    _check(load_library().hsa_forward_selected(ctypes.byref(cfg), _p(Q), _p(Kc), _p(Vc), _p(Kq), _p(Vq),
                                               _p(gate_logit), _p(E), _p(F), ef_head_stride, ctypes.byref(sel.c()),
                                               _p(out), 1 if out.dtype == torch.bfloat16 else 0, _p(ws), ws.numel(),
                                               _stream(stream)), "hsa_forward_selected")


def hsa_forward_ex(cfg, Q, Kc, Vc, Kq, Vq, tau, gate_logit, E, F, out, ws, sel: SelectionBuffers, flags=0,
                   kbar128=None, ef_head_stride=0, stream=None):
    """hsa_forward with FWD_SELECTED (sel is an input) and/or FWD_HISTORY (prepared history)."""
    _check(load_library().hsa_forward_ex(ctypes.byref(cfg), _p(Q), _p(Kc), _p(Vc), _p(Kq), _p(Vq), _p(kbar128),
                                         _p(tau), _p(gate_logit), _p(E), _p(F), ef_head_stride, _p(out),
                                         1 if out.dtype == torch.bfloat16 else 0, ctypes.byref(sel.c()), flags, _p(ws),
                                         ws.numel(), _stream(stream)), "hsa_forward_ex")


def hkv_gather_project(cfg, page_k_ptrs, page_v_ptrs, sel, Kp, P_tok, E, F, Kc, Vc, ws, ef_head_stride=0,
                       stream=None):
    """Gather of the selected pages + the history's Linformer products, one pass."""
    NP = page_k_ptrs.numel()
    _check(load_library().hkv_gather_project(ctypes.byref(cfg), _p(page_k_ptrs), _p(page_v_ptrs), NP, _p(sel), Kp,
                                             P_tok, _p(E), _p(F), ef_head_stride, _p(Kc), _p(Vc), _p(ws), ws.numel(),
                                             _stream(stream)), "hkv_gather_project")


def hsa_prepare_history(cfg, Kc, Vc, E, F, ws, ef_head_stride=0, stream=None):
    """Once per chunk: project the cached KV (E Kc, F Vc) into the workspace."""
    _check(load_library().hsa_prepare_history(ctypes.byref(cfg), _p(Kc), _p(Vc), _p(E), _p(F), ef_head_stride,
                                              _p(ws), ws.numel(), _stream(stream)), "hsa_prepare_history")


def hsa_forward_reuse(cfg, Q, Kc, Vc, Kq, Vq, tau, gate_logit, E, F, out, ws, kbar128=None, sel=None,
                      ef_head_stride=0, stream=None):
    """One denoising step against the history prepared by hsa_prepare_history."""
    csel = ctypes.byref(sel.c()) if sel is not None else None
    _check(load_library().hsa_forward_reuse(ctypes.byref(cfg), _p(Q), _p(Kc), _p(Vc), _p(Kq), _p(Vq), _p(kbar128),
                                            _p(tau), _p(gate_logit), _p(E), _p(F), ef_head_stride, _p(out),
                                            1 if out.dtype == torch.bfloat16 else 0, csel, _p(ws), ws.numel(),
                                            _stream(stream)), "hsa_forward_reuse")


# ---------------------------------------------------------------- tracing

class KernelTrace:
    """Per-kernel CUDA-event timing of the library's launches on this thread."""

    def __init__(self, max_kernels: int = 64):
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * max_kernels)]
        s = torch.cuda.current_stream()
        for e in self.events:  # materialise the event handles
            e.record(s)
        self._handles = (ctypes.c_void_p * len(self.events))(*[e.cuda_event for e in self.events])
        self._names = (ctypes.c_char_p * max_kernels)()
        self.max = max_kernels

    def __enter__(self):
        _check(load_library().hsa_trace_begin(self._handles, self.max, self._names), "hsa_trace_begin")
        return self

    def __exit__(self, *exc):
        self.count = load_library().hsa_trace_count()
        load_library().hsa_trace_end()

    def results(self):
        """[(kernel name, ms)] for the launches recorded (call after synchronising)."""
        return [(self._names[k].decode(), self.events[2 * k].elapsed_time(self.events[2 * k + 1]))
                for k in range(self.count)]
