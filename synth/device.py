"""Upload seeded step inputs to the GPU for the C-ABI path (tests and benchmark).

Plumbing only: allocation, host-to-device copies and the page tables a step
needs.  Imports neither the oracle nor any of the method's arithmetic.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import StepShape, make_inputs


def to_dev(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def bits_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class MappedHostBuffer:
    """Page-locked host memory mapped into the device address space
    (cudaHostAlloc with cudaHostAllocMapped; device address from cudaHostGetDevicePointer)."""

    def __init__(self, nbytes: int):
        from cuda.bindings import runtime as rt
        self._rt = rt
        err, ptr = rt.cudaHostAlloc(nbytes, rt.cudaHostAllocMapped | rt.cudaHostAllocPortable)
        assert err == rt.cudaError_t.cudaSuccess, err
        self.host_ptr = int(ptr)
        err, dptr = rt.cudaHostGetDevicePointer(self.host_ptr, 0)
        assert err == rt.cudaError_t.cudaSuccess, err
        self.dev_ptr = int(dptr)
        self.nbytes = nbytes

    def numpy(self, dtype, shape):
        buf = (ctypes.c_char * self.nbytes).from_address(self.host_ptr)
        return np.frombuffer(buf, dtype=dtype, count=int(np.prod(shape))).reshape(shape)

    def free(self):
        if self.host_ptr:
            self._rt.cudaFreeHost(self.host_ptr)
            self.host_ptr = 0


class DeviceStep:
    """Seeded inputs of one step uploaded for the GPU path, plus its HkvHsaStep."""

    def __init__(self, shape: StepShape, seed: int, out_dtype=torch.float32, x=None, store_slots=0):
        """store_slots > 0 (host-pinned workloads): the pages are read through a tiered
        page store with that many HBM slots instead of straight from the host tier."""
        from hybrid_sparse_attention_hkv_b200.step import HkvHsaStep, page_pointers
        self.shape = shape
        NP, P, H, d = shape.NP, shape.P_tok, shape.H, shape.d
        self.host = None
        if x is None and shape.host_pages:
            nb = NP * P * H * d * 2
            self.host = (MappedHostBuffer(nb), MappedHostBuffer(nb))
            pk = self.host[0].numpy(np.uint16, (NP, P, H, d))
            pv = self.host[1].numpy(np.uint16, (NP, P, H, d))
            x = make_inputs(shape, seed, pages_out=(pk, pv))
        elif x is None:
            x = make_inputs(shape, seed)
        self.x = x
        self.Q, self.Kq, self.Vq = to_dev(x.Q), to_dev(x.Kq), to_dev(x.Vq)
        self.E, self.F = to_dev(x.E), to_dev(x.F)
        self.tau = torch.from_numpy(x.tau).cuda()
        self.z = torch.from_numpy(x.z).cuda()
        stride = P * H * d * 2
        self.store = None
        if self.host:
            kp = torch.tensor([self.host[0].dev_ptr + p * stride for p in range(NP)], dtype=torch.int64, device="cuda")
            vp = torch.tensor([self.host[1].dev_ptr + p * stride for p in range(NP)], dtype=torch.int64, device="cuda")
            self.host_tables = (kp, vp)  # straight from the host tier (zero-copy gather)
            self.pages_k = self.pages_v = None
            if store_slots:
                from hybrid_sparse_attention_hkv_b200.store import PageStore
                self.store = PageStore(NP, store_slots, P, H, d, host=self.host)
                kp, vp = self.store.page_tables()
        else:
            self.pages_k, self.pages_v = to_dev(x.pages_k), to_dev(x.pages_v)
            kp, vp = page_pointers(self.pages_k), page_pointers(self.pages_v)
        self.step = HkvHsaStep(H, d, shape.Lq, P, NP, shape.Kp, shape.r, kp, vp, out_dtype, store=self.store)
        if self.host:
            # summaries read the mapped host pages directly
            self.step.seal_pages([_HostPageView(self.host[0].dev_ptr + p * stride, P, H, d) for p in range(NP)])
        else:
            self.step.seal_pages(self.pages_k)
        self.e_cur = self.e_seg = self.seg_begin = None
        if shape.n_segments:
            self.e_cur = torch.from_numpy(x.e_cur).cuda()
            self.e_seg = torch.from_numpy(x.e_seg).cuda()
            self.seg_begin = torch.from_numpy(x.seg_begin).cuda()

    def run(self, tau=None, z=None):
        return self.step(self.Q, self.Kq, self.Vq, self.tau if tau is None else tau, self.z if z is None else z,
                         self.E, self.F, self.e_cur, self.e_seg, self.seg_begin)

    def close(self):
        if self.store is not None:
            self.store.close()  # the host tier belongs to this object: freed below
            self.store = None
        if self.host:
            for b in self.host:
                b.free()
            self.host = None


class _HostPageView:
    """Minimal tensor-like view (shape + data_ptr) of one mapped host page."""

    def __init__(self, ptr, P, H, d):
        self._ptr = ptr
        self.shape = (P, H, d)

    def data_ptr(self):
        return self._ptr
