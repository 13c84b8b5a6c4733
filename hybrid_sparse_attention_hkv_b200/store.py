"""Tiered page store of the hierarchical KV cache, through the C ABI (hkv_store_*).

The memories of the store are allocated here (plumbing): the host tier in
page-locked host memory mapped into the device address space, the HBM slot pool
and the residency state with torch.  Every decision and copy runs in the library's
kernels; this class only marshals arguments.
"""
from __future__ import annotations

import ctypes

import torch

from . import StoreDesc, _check, _p, _stream, load_library


class MappedHostMemory:
    """Page-locked host memory mapped into the device address space
    (cudaHostAlloc with the mapped and portable flags), freed by close()."""

    def __init__(self, nbytes: int):
        from cuda.bindings import runtime as rt
        self._rt = rt
        err, ptr = rt.cudaHostAlloc(nbytes, rt.cudaHostAllocMapped | rt.cudaHostAllocPortable)
        if err != rt.cudaError_t.cudaSuccess:
            raise RuntimeError(f"cudaHostAlloc({nbytes}): {err}")
        self.host_ptr = int(ptr)
        err, dptr = rt.cudaHostGetDevicePointer(self.host_ptr, 0)
        if err != rt.cudaError_t.cudaSuccess:
            rt.cudaFreeHost(self.host_ptr)
            raise RuntimeError(f"cudaHostGetDevicePointer: {err}")
        self.dev_ptr = int(dptr)
        self.nbytes = nbytes

    def close(self):
        if self.host_ptr:
            self._rt.cudaFreeHost(self.host_ptr)
            self.host_ptr = 0


class PageStore:
    """NP pages of [P_tok, H, d] bf16 K and V on the host tier, S of them in HBM slots."""

    def __init__(self, NP: int, S: int, P_tok: int, H: int, d: int, host=None, stream=None):
        """host: optional (K, V) objects with a `dev_ptr` attribute that already hold
        the host tier (e.g. pages written by the caller); else it is allocated here."""
        self.NP, self.S, self.P_tok, self.H, self.d = NP, S, P_tok, H, d
        page_bytes = P_tok * H * d * 2
        self._own = host is None
        self.host = host if host is not None else (MappedHostMemory(NP * page_bytes), MappedHostMemory(NP * page_bytes))
        self.slot_k = torch.empty(S, P_tok, H, d, dtype=torch.bfloat16, device="cuda")
        self.slot_v = torch.empty(S, P_tok, H, d, dtype=torch.bfloat16, device="cuda")
        lib = load_library()
        self.state = torch.zeros(lib.hkv_store_state_size(NP, S), dtype=torch.uint8, device="cuda")
        self.desc = StoreDesc(NP, S, P_tok, H, d, self.host[0].dev_ptr, self.host[1].dev_ptr,
                              self.slot_k.data_ptr(), self.slot_v.data_ptr(), self.state.data_ptr())
        _check(lib.hkv_store_init(ctypes.byref(self.desc), _stream(stream)), "hkv_store_init")
        tk, tv = ctypes.c_void_p(), ctypes.c_void_p()
        _check(lib.hkv_store_tables(ctypes.byref(self.desc), ctypes.byref(tk), ctypes.byref(tv)), "hkv_store_tables")
        self.table_k, self.table_v = tk.value, tv.value

    def page_tables(self):
        """(K, V) device page tables as int64 tensor views (for hkv_gather)."""
        n = self.NP
        off_k = self.table_k - self.state.data_ptr()
        off_v = self.table_v - self.state.data_ptr()
        return (self.state[off_k:off_k + 8 * n].view(torch.int64), self.state[off_v:off_v + 8 * n].view(torch.int64))

    def seal(self, page: int, K_rows, V_rows, kbar_out, ws, stream=None):
        _check(load_library().hkv_store_seal(ctypes.byref(self.desc), page, _p(K_rows), _p(V_rows), _p(kbar_out),
                                             _p(ws), ws.numel(), _stream(stream)), "hkv_store_seal")

    def fetch(self, sel, ws, stream=None):
        _check(load_library().hkv_store_fetch(ctypes.byref(self.desc), _p(sel), sel.numel(), _p(ws), ws.numel(),
                                              _stream(stream)), "hkv_store_fetch")

    def prefetch(self, scores, protect, m: int, ws, stream=None):
        n = 0 if protect is None else protect.numel()
        _check(load_library().hkv_store_prefetch(ctypes.byref(self.desc), _p(scores), _p(protect), n, m, _p(ws),
                                                 ws.numel(), _stream(stream)), "hkv_store_prefetch")

    def residency(self, stream=None):
        """(slot_of_page [NP], page_of_slot [S]) as device int32 tensors."""
        sp = torch.empty(self.NP, dtype=torch.int32, device="cuda")
        ps = torch.empty(self.S, dtype=torch.int32, device="cuda")
        _check(load_library().hkv_store_residency(ctypes.byref(self.desc), _p(sp), _p(ps), _stream(stream)),
               "hkv_store_residency")
        return sp, ps

    def close(self):
        if self._own:
            for h in self.host:
                h.close()
        self.host = None
