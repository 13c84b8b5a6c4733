"""Seeded synthetic inputs for the HKV + HSA attention step.

This module is shared by the tests, the benchmark and the oracle checks.  It
only draws numbers (a counter-based SplitMix64 + Box-Muller generator in
``synth.c``) and lays them out in the shapes of the workloads; none of the
attention method's arithmetic lives here.

Workloads follow the shapes of the WorldAttention evaluation ("WorldAttention
pairs hierarchical KV caching with hybrid sparse attention..." news summary,
HKV paragraph: pages of Psize = 8 latent frames, Kp = 4 pages kept; HSA
paragraph: Binter = 128, Bintra = 64, tau from 1.00 down to 0.35), on Wan
480p / 720p latent geometry (1560 / 3600 tokens per latent frame).  The video
benchmarks the pages evaluate on are replaced by these synthetic tensors.

Recipe (per workload, seed fixed):
  * Q, K, V ~ N(0, 1), rounded to bf16.
  * each history page p has a key offset mu_p ~ N(0, 0.5^2 I) in R^{H x d},
    added to every key row of that page.
  * E, F ~ N(0, 1/r), shape [r, L] with L = Kp * P_tok + Lq, bf16.
  * gate logits z_h ~ N(0, 1); tau_h linear from 1.00 (head 0) to 0.35.
  * for the large workloads, 3 distinct seed-chosen pages c_0..c_2; the query
    rows of latent frame f get + mu_{c_f} (queries biased toward those pages).
  * the host-pinned workload groups the 48 pages into 9 prompt segments of
    contiguous pages, draws a 4096-d embedding per segment ~ N(0, I) and a
    current embedding = e_{s*} + 0.5 N(0, I); c_0..c_2 are drawn inside s*.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the generator into ``synth/libsynth.so`` (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, u64, dbl = ctypes.c_int64, ctypes.c_uint64, ctypes.c_double
        lib.synth_normal_bf16.argtypes = [ctypes.c_void_p, i64, u64, u64, i64, dbl, ctypes.c_void_p, i64]
        lib.synth_normal_bf16.restype = None
        lib.synth_normal_f32.argtypes = [ctypes.c_void_p, i64, u64, u64, i64, dbl]
        lib.synth_normal_f32.restype = None
        lib.synth_uniform_int.argtypes = [u64, u64, i64, i64]
        lib.synth_uniform_int.restype = i64
        _lib = lib
    return _lib


def normal_bf16(shape, seed, stream, sigma=1.0, offset=None, start=0, out=None):
    """bf16 bit patterns (uint16) of sigma * N(0,1) (+ offset repeated along the last axes)."""
    lib = _load()
    if out is None:
        out = np.empty(shape, dtype=np.uint16)
    assert out.dtype == np.uint16 and out.flags.c_contiguous
    off_ptr, period = None, 1
    if offset is not None:
        offset = np.ascontiguousarray(offset, dtype=np.float32)
        off_ptr, period = offset.ctypes.data, offset.size
    lib.synth_normal_bf16(out.ctypes.data, out.size, seed, stream, start, float(sigma), off_ptr, period)
    return out


def normal_f32(shape, seed, stream, sigma=1.0, start=0):
    lib = _load()
    out = np.empty(shape, dtype=np.float32)
    lib.synth_normal_f32(out.ctypes.data, out.size, seed, stream, start, float(sigma))
    return out


def uniform_int(seed, stream, i, m) -> int:
    return int(_load().synth_uniform_int(seed, stream, i, m))


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 bit patterns (nearest even)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


@dataclass(frozen=True)
class StepShape:
    """Sizes of one per-layer attention step."""
    name: str
    H: int                 # heads
    d: int                 # head dim
    frames: int            # latent frames in the current chunk
    F_tok: int             # tokens per latent frame
    page_frames: int       # Psize: latent frames per page
    NP: int                # history pages
    Kp: int                # pages retrieved
    r: int                 # Linformer rank
    n_biased: int = 0      # pages the queries are biased toward (0 or 3)
    host_pages: bool = False
    n_segments: int = 0
    emb_dim: int = 0
    page_tok: int = 0      # tokens per page when not page_frames * F_tok
    block_inter: int = 128
    block_intra: int = 64
    tau_max: float = 1.00
    tau_min: float = 0.35

    @property
    def Lq(self) -> int:
        return self.frames * self.F_tok

    @property
    def P_tok(self) -> int:
        return self.page_tok or self.page_frames * self.F_tok

    @property
    def Lc(self) -> int:
        return self.Kp * self.P_tok

    @property
    def L(self) -> int:
        return self.Lc + self.Lq

    def replace(self, **kw) -> "StepShape":
        d = dict(self.__dict__)
        d.update(kw)
        return StepShape(**d)


# The five workloads.  Index i uses seed 1000 + i.
SHAPES = [
    # tiny step: 2 heads, d=64, one 256-token latent frame as the chunk,
    # 8 pages of 8 frames x 32 tokens (256 tokens), Kp = 2, r = 64
    StepShape("tiny_h2_d64_lq256", H=2, d=64, frames=1, F_tok=256, page_frames=8, page_tok=256,
              NP=8, Kp=2, r=64),
    # Wan-1.3B-shaped 480p: 12 heads, 3 x 1560 queries, 16 pages of 8 x 1560 tokens, Kp = 4, r = 256
    StepShape("wan1.3b_480p_h12_lq4680", H=12, d=128, frames=3, F_tok=1560, page_frames=8,
              NP=16, Kp=4, r=256, n_biased=3),
    # 14B-shaped 480p: 40 heads, same token geometry
    StepShape("wan14b_480p_h40_lq4680", H=40, d=128, frames=3, F_tok=1560, page_frames=8,
              NP=16, Kp=4, r=256, n_biased=3),
    # 14B-shaped 720p: 40 heads, 3 x 3600 queries, 12 pages of 8 x 3600 tokens, r = 512
    StepShape("wan14b_720p_h40_lq10800", H=40, d=128, frames=3, F_tok=3600, page_frames=8,
              NP=12, Kp=4, r=512, n_biased=3),
    # 90-second horizon: 48 host-pinned pages in 9 prompt segments, two-stage retrieval
    StepShape("wan1.3b_480p_90s_host48_h12_lq4680", H=12, d=128, frames=3, F_tok=1560,
              page_frames=8, NP=48, Kp=4, r=256, n_biased=3, host_pages=True,
              n_segments=9, emb_dim=4096),
]


def seed_of(index: int) -> int:
    return 1000 + index


# stream ids (one per tensor)
S_Q, S_KQ, S_VQ, S_E, S_F, S_Z = 1, 2, 3, 4, 5, 6
S_PAGE_K, S_PAGE_V, S_MU = 100_000, 200_000, 300_000
S_PICK_PAGES, S_PICK_SEGMENT = 400_000, 400_001
S_EMB, S_EMB_NOISE = 500_000, 600_000


def segment_bounds(NP: int, S: int) -> np.ndarray:
    """Segment s holds pages [b[s], b[s+1]) with b[s] = floor(NP * s / S)."""
    return np.array([(NP * s) // S for s in range(S + 1)], dtype=np.int32)


def tau_schedule(H: int, tau_max=1.00, tau_min=0.35) -> np.ndarray:
    """tau_h linear from tau_max at head 0 to tau_min at head H-1."""
    if H == 1:
        return np.array([tau_max], dtype=np.float32)
    h = np.arange(H, dtype=np.float64)
    return (tau_max - (tau_max - tau_min) * h / (H - 1)).astype(np.float32)


def _distinct_pages(seed, lo, hi, count):
    picked, i = [], 0
    while len(picked) < count:
        p = lo + uniform_int(seed, S_PICK_PAGES, i, hi - lo)
        i += 1
        if p not in picked:
            picked.append(p)
    return picked


@dataclass
class StepInputs:
    shape: StepShape
    seed: int
    Q: np.ndarray          # uint16 [Lq, H, d]   (bf16 bits)
    Kq: np.ndarray         # uint16 [Lq, H, d]
    Vq: np.ndarray         # uint16 [Lq, H, d]
    pages_k: np.ndarray    # uint16 [NP, P_tok, H, d]
    pages_v: np.ndarray    # uint16 [NP, P_tok, H, d]
    E: np.ndarray          # uint16 [r, L]
    F: np.ndarray          # uint16 [r, L]
    z: np.ndarray          # float32 [H] gate logits
    tau: np.ndarray        # float32 [H]
    mu: np.ndarray         # float32 [NP, H, d] page key offsets (recipe metadata)
    biased: list = field(default_factory=list)
    e_seg: np.ndarray | None = None      # float32 [S, D]
    e_cur: np.ndarray | None = None      # float32 [D]
    seg_begin: np.ndarray | None = None  # int32 [S + 1]
    s_star: int = -1


def make_inputs(shape: StepShape, seed: int, pages_out=None) -> StepInputs:
    """Draw every input of one step.  ``pages_out`` = optional (K, V) uint16 arrays
    of shape [NP, P_tok, H, d] to fill in place (e.g. pinned host buffers)."""
    H, d, Lq, P, NP, r, L = shape.H, shape.d, shape.Lq, shape.P_tok, shape.NP, shape.r, shape.L
    hd = H * d
    mu = np.stack([normal_f32((H, d), seed, S_MU + p, sigma=0.5) for p in range(NP)])

    e_seg = e_cur = seg_begin = None
    s_star = -1
    biased = []
    if shape.n_segments:
        seg_begin = segment_bounds(NP, shape.n_segments)
        s_star = uniform_int(seed, S_PICK_SEGMENT, 0, shape.n_segments)
        e_seg = np.stack([normal_f32((shape.emb_dim,), seed, S_EMB + s) for s in range(shape.n_segments)])
        e_cur = (e_seg[s_star] + normal_f32((shape.emb_dim,), seed, S_EMB_NOISE, sigma=0.5)).astype(np.float32)
        if shape.n_biased:
            biased = _distinct_pages(seed, int(seg_begin[s_star]), int(seg_begin[s_star + 1]), shape.n_biased)
    elif shape.n_biased:
        biased = _distinct_pages(seed, 0, NP, shape.n_biased)

    Q = np.empty((Lq, H, d), dtype=np.uint16)
    if biased:
        assert shape.frames == len(biased)
        ft = shape.F_tok * hd
        flat = Q.reshape(-1)
        for f, c in enumerate(biased):
            seg = flat[f * ft:(f + 1) * ft]
            normal_bf16(None, seed, S_Q, offset=mu[c], start=f * ft, out=seg)
    else:
        normal_bf16(None, seed, S_Q, out=Q)
    Kq = normal_bf16((Lq, H, d), seed, S_KQ)
    Vq = normal_bf16((Lq, H, d), seed, S_VQ)

    if pages_out is None:
        pk = np.empty((NP, P, H, d), dtype=np.uint16)
        pv = np.empty((NP, P, H, d), dtype=np.uint16)
    else:
        pk, pv = pages_out
    for p in range(NP):
        normal_bf16(None, seed, S_PAGE_K + p, offset=mu[p], out=pk[p])
        normal_bf16(None, seed, S_PAGE_V + p, out=pv[p])

    sig = 1.0 / np.sqrt(r)
    E = normal_bf16((r, L), seed, S_E, sigma=sig)
    Fm = normal_bf16((r, L), seed, S_F, sigma=sig)
    z = normal_f32((H,), seed, S_Z)
    tau = tau_schedule(H, shape.tau_max, shape.tau_min)
    return StepInputs(shape, seed, Q, Kq, Vq, pk, pv, E, Fm, z, tau, mu, biased,
                      e_seg, e_cur, seg_begin, s_star)
