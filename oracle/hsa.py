"""fp64 reference of the WorldAttention per-layer attention step (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` may
use this module.  It is the plain definition of each step, written with numpy in
float64 from the pages' description; a matmul, a sort, a sum or an exp from numpy
stands in for a step where convenient, with no blocking, fusion or reordering.

Sources, cited below by short name:
  [NEWS]  "WorldAttention pairs hierarchical KV caching with hybrid sparse attention
          to reach 22 FPS on a single H100 and 0.9472 subject consistency on
          VBench-Long" (English news summary of the paper):
            - HKV paragraph (pages of Psize = 8 frames, two-stage prompt-level and
              page-level retrieval of a top-Kp active cache, Table 5: Kp = 4);
            - HSA paragraph (Linformer-style low-rank linear branch, per-head
              minimal block set whose cumulative attention mass reaches tau_h,
              Binter = 128 / Bintra = 64, Table 4: tau from 1.00 to 0.35, learned
              gates merging the two branches);
            - kernel paragraph (KV-cache reorganisation into contiguous memory);
            - open-questions paragraph (Top-1 prompt retrieval).
  [PROJ]  WorldAttention project page, Method figures "Overall architecture of
          WorldAttention" and "three-tier hierarchical KV cache with prompt-level
          and page-level retrieval".

Readings taken where the pages are silent (each restated at its function):
  * page descriptor = mean key per head; page score = sum over heads of
    (mean query) . (mean key); one page selection per layer, shared by all heads;
    top-Kp ties go to the lower page id; gathered pages are laid out in ascending
    page-id order.
  * queries are pooled with the block size of the keys they are scored against
    (128 against the cached KV, 64 inside the chunk); a partial last block is the
    mean of its real rows; inter and intra maps are softmaxed and thresholded
    separately; the attention itself is one joint softmax over the union.
  * threshold test is "cumulative mass >= tau_h"; tau_h >= 1 keeps every block;
    at least one block is kept; blocks are ranked by mass, ties to lower index.
  * no causal mask inside the chunk; scale 1/sqrt(d) everywhere.
  * E, F in R^{r x L} span the active KV (L = Lc + Lq) and are shared by the heads
    unless a per-head stack [H, r, L] is given.
  * gate g_h = sigmoid(z_h), one scalar per head.

Precision: inputs are bf16 bit patterns (uint16), widened exactly to float64.
The selection functions take ``dtype``: the block means and scores that decide
an integer result are rounded to that type (float32 = the GPU kernels' choice;
float64 for the pins); masses and attention are always float64.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

__all__ = [
    "widen", "prompt_top1", "page_summary", "pooled_query", "page_scores", "select_pages", "select_pages_policy",
    "gather_pages", "block_means", "block_probs", "keep_blocks", "Selection", "block_select",
    "sparse_attention", "linear_projection", "linear_attention", "fidelity", "gate", "gated_merge",
    "hsa_step", "hkv_hsa_step",
]


def widen(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly."""
    b = np.asarray(bits)
    if b.dtype != np.uint16:
        return b.astype(np.float64)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _as(x, dtype):
    return np.asarray(x, dtype=np.float64).astype(dtype).astype(np.float64)


# --------------------------------------------------------------------------- HKV

def prompt_top1(e_cur, e_seg) -> int:
    """Stage 1 of the two-stage retrieval ([NEWS] HKV paragraph; [NEWS] open-questions
    paragraph: Top-1 is used): the prompt segment whose embedding has the largest
    cosine similarity with the current prompt embedding.  Ties -> lowest index."""
    e = np.asarray(e_cur, dtype=np.float64)
    S = np.asarray(e_seg, dtype=np.float64)
    cos = (S @ e) / (np.linalg.norm(S, axis=1) * np.linalg.norm(e))
    return int(np.argmax(cos))  # argmax returns the first maximum


def page_summary(K_page, dtype=np.float64) -> np.ndarray:
    """Descriptor of one KV page ([NEWS] HKV paragraph; reading: mean key per head):
    kbar[h, :] = (1 / P_tok) * sum_t K_page[t, h, :].  K_page: [P_tok, H, d]."""
    K = widen(K_page)
    return _as(K.sum(axis=0) / K.shape[0], dtype)


def pooled_query(Q, dtype=np.float64) -> np.ndarray:
    """qbar[h, :] = mean over the chunk's Lq query rows of Q[t, h, :]."""
    Qf = widen(Q)
    return _as(Qf.sum(axis=0) / Qf.shape[0], dtype)


def page_scores(kbar_pages, qbar, dtype=np.float64) -> np.ndarray:
    """s_p = sum_h qbar[h] . kbar_p[h]  (reading: one score per page, summed over heads)."""
    kb = np.asarray(kbar_pages, dtype=np.float64)
    qb = np.asarray(qbar, dtype=np.float64)
    return _as(np.einsum("phc,hc->p", kb, qb), dtype)


def select_pages(kbar_pages, Q, Kp, cand=None, dtype=np.float32):
    """Stage 2, page-level retrieval ([NEWS] HKV paragraph, Table 5: Kp = 4): keep the
    Kp candidate pages with the largest score; ties -> lower page id.  Returns
    (page ids ascending, scores of every page)."""
    kb = np.asarray(kbar_pages, dtype=np.float64)
    s = page_scores(kb, pooled_query(Q, dtype), dtype)
    cand = list(range(kb.shape[0])) if cand is None else [int(c) for c in cand]
    if not 1 <= Kp <= len(cand):
        raise ValueError("need 1 <= Kp <= number of candidates")
    ranked = sorted(cand, key=lambda p: (-s[p], p))
    return np.array(sorted(ranked[:Kp]), dtype=np.int32), s


def select_pages_policy(policy, kbar_pages, Q, Kp, cand=None, rand_keys=None, dtype=np.float32):
    """The retrieval ablations ([NEWS] HKV paragraph, Table 6: page-only, prompt-only,
    recent-page and random-page retrieval under one budget of Kp pages; Table 5: the
    sliding window).  "score": the mean-key score (select_pages); "recent": the Kp
    candidates with the largest page ids (the most recent pages); "random": the Kp
    candidates with the largest caller-drawn keys rand_keys[p], ties -> lower page id.
    Returns the kept page ids ascending."""
    if policy == "score":
        return select_pages(kbar_pages, Q, Kp, cand, dtype)[0]
    NP = np.asarray(kbar_pages).shape[0]
    cand = list(range(NP)) if cand is None else [int(c) for c in cand]
    if not 1 <= Kp <= len(cand):
        raise ValueError("need 1 <= Kp <= number of candidates")
    if policy == "recent":
        return np.array(sorted(cand)[-Kp:], dtype=np.int32)
    if policy == "random":
        keys = np.asarray(rand_keys, dtype=np.float64)
        ranked = sorted(cand, key=lambda p: (-keys[p], p))
        return np.array(sorted(ranked[:Kp]), dtype=np.int32)
    raise ValueError(f"unknown policy {policy!r}")


def gather_pages(pages, sel) -> np.ndarray:
    """Active-cache assembly ([NEWS] HKV and kernel paragraphs): the selected pages
    concatenated along the token axis in the given (ascending) order.
    pages: [NP, P_tok, H, d] (any dtype; bf16 bits stay bits)."""
    return np.concatenate([np.asarray(pages[int(p)]) for p in sel], axis=0)


# --------------------------------------------------------------------------- HSA, sparse branch

def block_means(X, B, dtype=np.float64) -> np.ndarray:
    """Mean pooling of token rows into blocks of B ([NEWS] HSA paragraph):
    out[j] = mean of X[j*B : min((j+1)*B, n)] (a partial last block averages its
    real rows).  X: [n, H, d] -> [ceil(n/B), H, d]."""
    n = X.shape[0]
    nb = -(-n // B)
    out = np.empty((nb,) + tuple(X.shape[1:]), dtype=np.float64)
    for j in range(nb):
        rows = widen(X[j * B:min((j + 1) * B, n)])
        out[j] = rows.sum(axis=0) / rows.shape[0]
    return _as(out, dtype)


def block_probs(qbar, kbar, scale, dtype=np.float64) -> np.ndarray:
    """Block attention mass: per head, row i of softmax_j(qbar_i . kbar_j * scale).
    qbar: [nQ, H, d], kbar: [nK, H, d] -> [H, nQ, nK] (float64)."""
    s = _as(np.einsum("ihc,jhc->hij", np.asarray(qbar, np.float64), np.asarray(kbar, np.float64)) * scale, dtype)
    if s.shape[2] == 0:  # no retrieved history: an empty map, nothing to keep
        return s
    s = s - s.max(axis=2, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=2, keepdims=True)


def keep_blocks(p_row, tau) -> np.ndarray:
    """The smallest block set whose cumulative mass reaches tau ([NEWS] HSA paragraph).
    Blocks are ranked by mass, descending (ties -> lower index); the shortest ranked
    prefix with mass >= tau is kept (at least one block; tau >= 1 keeps every block).
    Returns the kept block indices ascending."""
    p = np.asarray(p_row, dtype=np.float64)
    n = p.shape[0]
    if tau >= 1.0:
        return np.arange(n, dtype=np.int32)
    order = sorted(range(n), key=lambda j: (-p[j], j))
    mass, k = 0.0, 0
    while k < n:
        mass += p[order[k]]
        k += 1
        if mass >= tau:
            break
    return np.array(sorted(order[:k]), dtype=np.int32)


@dataclass
class Selection:
    inter: list      # inter[h][i] = ascending Kc-block ids kept for 128-query block i
    intra: list      # intra[h][i] = ascending Kq-block ids kept for 64-query block i
    p_inter: np.ndarray  # [H, nQ128, nKc128]
    p_intra: np.ndarray  # [H, nQ64, nKq64]


def block_select(Q, Kc, Kq, tau, scale=None, Binter=128, Bintra=64, dtype=np.float32, joint=False) -> Selection:
    """Head-adaptive block selection ([NEWS] HSA paragraph).

    Inter map: 128-row query blocks against 128-row blocks of the cached KV Kc.
    Intra map: 64-row query blocks against 64-row blocks of the chunk's own keys Kq.
    Each map row is softmaxed and thresholded at tau_h separately.

    joint=True (the other reading of the pages): per 64-row query block, its mean
    query scored against the Kc blocks followed by the Kq blocks, one softmax and one
    threshold over that whole row; the kept ids below nKc form the row's inter list,
    the others (minus nKc) its intra list.  p_inter then holds the joint masses
    [H, nQ64, nKc + nKq] and p_intra is None."""
    H, d = Q.shape[1], Q.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if joint:
        q64 = block_means(Q, Bintra, dtype)
        kc, kq = block_means(Kc, Binter, dtype), block_means(Kq, Bintra, dtype)
        nKc = kc.shape[0]
        p = block_probs(q64, np.concatenate([kc, kq], axis=0), scale, dtype)
        inter, intra = [], []
        for h in range(H):
            kept = [keep_blocks(p[h, i], float(tau[h])) for i in range(p.shape[1])]
            inter.append([k[k < nKc].astype(np.int32) for k in kept])
            intra.append([(k[k >= nKc] - nKc).astype(np.int32) for k in kept])
        return Selection(inter, intra, p, None)
    p_inter = block_probs(block_means(Q, Binter, dtype), block_means(Kc, Binter, dtype), scale, dtype)
    p_intra = block_probs(block_means(Q, Bintra, dtype), block_means(Kq, Bintra, dtype), scale, dtype)
    inter = [[keep_blocks(p_inter[h, i], float(tau[h])) for i in range(p_inter.shape[1])] for h in range(H)]
    intra = [[keep_blocks(p_intra[h, i], float(tau[h])) for i in range(p_intra.shape[1])] for h in range(H)]
    return Selection(inter, intra, p_inter, p_intra)


def _block_rows(blocks, B, n) -> np.ndarray:
    if len(blocks) == 0:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate([np.arange(j * B, min((j + 1) * B, n)) for j in blocks]).astype(np.int64)


def sparse_attention(Q, Kc, Vc, Kq, Vq, inter, intra, scale=None, Binter=128, Bintra=64, rows=None,
                     inter_rows=None):
    """Exact attention over the selected blocks only ([NEWS] HSA paragraph).

    For query t of head h the key set is the tokens of Kc blocks inter[h][t // inter_rows]
    together with the tokens of Kq blocks intra[h][t // Bintra]; one softmax over
    that whole set:  o[t, h] = sum_k softmax_k(q_t . k * scale) v_k.
    inter_rows = the query rows an inter list serves: Binter (default), or Bintra for
    the joint selection's per-64-row inter lists.
    ``rows`` (optional) = query rows to compute; returns [len(rows), H, d] float64."""
    Lq, H, d = Q.shape
    Lc, Lk = Kc.shape[0], Kq.shape[0]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    inter_rows = Binter if inter_rows is None else inter_rows
    rows = np.arange(Lq) if rows is None else np.asarray(rows)
    out = np.zeros((len(rows), H, d), dtype=np.float64)
    groups = {}
    for n, t in enumerate(rows):
        groups.setdefault((int(t) // inter_rows, int(t) // Bintra), []).append(n)
    for h in range(H):
        for (i128, i64), ns in groups.items():
            kc = _block_rows(inter[h][i128], Binter, Lc)
            kq = _block_rows(intra[h][i64], Bintra, Lk)
            K = np.concatenate([widen(Kc[kc, h]), widen(Kq[kq, h])], axis=0)
            V = np.concatenate([widen(Vc[kc, h]), widen(Vq[kq, h])], axis=0)
            q = widen(Q[rows[ns], h])
            s = (q @ K.T) * scale
            s -= s.max(axis=1, keepdims=True)
            w = np.exp(s)
            out[ns, h] = (w @ V) / w.sum(axis=1, keepdims=True)
    return out


# --------------------------------------------------------------------------- HSA, linear branch

def linear_projection(E, F, Kc, Kq, Vc, Vq):
    """Linformer-style low-rank projection ([NEWS] HSA paragraph; Linformer):
    EK_h = E_h [Kc; Kq]_h and FV_h = F_h [Vc; Vq]_h, E_h, F_h in R^{r x L}.
    E, F: [r, L] shared by all heads or [H, r, L] per head.
    Returns EK, FV: [H, r, d] float64."""
    H, d = Kc.shape[1], Kc.shape[2]
    Ef, Ff = widen(E), widen(F)
    r = Ef.shape[-2]
    EK = np.empty((H, r, d))
    FV = np.empty((H, r, d))
    for h in range(H):
        Kh = np.concatenate([widen(Kc[:, h]), widen(Kq[:, h])], axis=0)
        Vh = np.concatenate([widen(Vc[:, h]), widen(Vq[:, h])], axis=0)
        EK[h] = (Ef[h] if Ef.ndim == 3 else Ef) @ Kh
        FV[h] = (Ff[h] if Ff.ndim == 3 else Ff) @ Vh
    return EK, FV


def linear_attention(Q, EK, FV, scale=None, rows=None):
    """o_l[t, h] = softmax_j(q_t . EK_h[j] * scale) FV_h  ([NEWS] HSA paragraph).
    Returns [len(rows), H, d] float64."""
    Lq, H, d = Q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    rows = np.arange(Lq) if rows is None else np.asarray(rows)
    out = np.empty((len(rows), H, d))
    for h in range(H):
        q = widen(Q[rows, h])
        s = (q @ EK[h].T) * scale
        s -= s.max(axis=1, keepdims=True)
        w = np.exp(s)
        out[:, h] = (w @ FV[h]) / w.sum(axis=1, keepdims=True)
    return out


# --------------------------------------------------------------------------- fidelity diagnostic

def fidelity(Q, Kc, Vc, Kq, Vq, inter, intra, EK, FV, scale=None, Binter=128, Bintra=64):
    """How close each branch comes to dense attention ([NEWS] HSA paragraph, Figure 6:
    the linear branch's fidelity to full attention in global mass and in output).
    Per head h, over all rows t and columns:
      [0] cos(o_lin, o_dense), [1] cos(o_sparse, o_dense),
      [2] mean over t of the dense softmax mass of the keys the sparse branch keeps,
      [3] |o_lin - o_dense| / |o_dense|, [4] |o_sparse - o_dense| / |o_dense|.
    Dense attention = every key of [Kc; Kq].  Returns [H, 5] float64."""
    Lq, H, d = Q.shape
    Lc, Lk = Kc.shape[0], Kq.shape[0]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    all_inter = [[np.arange(-(-Lc // Binter))] * (-(-Lq // Binter))] * H
    all_intra = [[np.arange(-(-Lk // Bintra))] * (-(-Lq // Bintra))] * H
    o_ref = sparse_attention(Q, Kc, Vc, Kq, Vq, all_inter, all_intra, scale, Binter, Bintra)
    o_sp = sparse_attention(Q, Kc, Vc, Kq, Vq, inter, intra, scale, Binter, Bintra)
    o_lin = linear_attention(Q, EK, FV, scale)
    out = np.zeros((H, 5))
    for h in range(H):
        K = np.concatenate([widen(Kc[:, h]), widen(Kq[:, h])], axis=0)
        s = (widen(Q[:, h]) @ K.T) * scale
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        mass = np.empty(Lq)
        for t in range(Lq):
            kept = np.concatenate([_block_rows(inter[h][t // Binter], Binter, Lc),
                                   Lc + _block_rows(intra[h][t // Bintra], Bintra, Lk)])
            mass[t] = p[t, kept].sum()
        r, sp, li = o_ref[:, h].ravel(), o_sp[:, h].ravel(), o_lin[:, h].ravel()
        out[h] = [li @ r / np.sqrt((li @ li) * (r @ r)), sp @ r / np.sqrt((sp @ sp) * (r @ r)), mass.mean(),
                  np.linalg.norm(li - r) / np.linalg.norm(r), np.linalg.norm(sp - r) / np.linalg.norm(r)]
    return out


# --------------------------------------------------------------------------- merge and full step

def gate(z) -> np.ndarray:
    """g_h = 1 / (1 + exp(-z_h)); z = +inf gives exactly 1, z = -inf exactly 0."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def gated_merge(o_s, o_l, z) -> np.ndarray:
    """Gated merge of the two branches ([NEWS] HSA paragraph, learned gates; reading:
    one sigmoid gate per head): out = g_h o_s + (1 - g_h) o_l."""
    g = gate(z)[None, :, None]
    return g * o_s + (1.0 - g) * o_l


def hsa_step(Q, Kc, Vc, Kq, Vq, tau, z, E, F, scale=None, Binter=128, Bintra=64,
             rows=None, selection=None, dtype=np.float32, joint=False):
    """HSA over the active cache plus the current chunk ([PROJ] overall architecture):
    block selection, sparse branch, linear branch, gated merge.  ``selection`` may be
    passed in (e.g. a GPU selection already verified against this oracle); joint =
    the joint block selection (inter lists per 64-row query block)."""
    sel = block_select(Q, Kc, Kq, tau, scale, Binter, Bintra, dtype, joint) if selection is None else selection
    o_s = sparse_attention(Q, Kc, Vc, Kq, Vq, sel.inter, sel.intra, scale, Binter, Bintra, rows,
                           inter_rows=Bintra if joint else Binter)
    EK, FV = linear_projection(E, F, Kc, Kq, Vc, Vq)
    o_l = linear_attention(Q, EK, FV, scale, rows)
    return {"selection": sel, "o_s": o_s, "o_l": o_l, "out": gated_merge(o_s, o_l, z), "EK": EK, "FV": FV}


def hkv_hsa_step(pages_k, pages_v, Q, Kq, Vq, Kp, tau, z, E, F, scale=None, Binter=128, Bintra=64,
                 e_cur=None, e_seg=None, seg_begin=None, rows=None, dtype=np.float32):
    """The whole per-layer step ([PROJ] overall architecture): optional prompt-level
    Top-1 segment, page-level top-Kp retrieval, gather, then HSA."""
    NP = pages_k.shape[0]
    cand, s_star = None, -1
    if e_cur is not None:
        s_star = prompt_top1(e_cur, e_seg)
        cand = list(range(int(seg_begin[s_star]), int(seg_begin[s_star + 1])))
    kbar = np.stack([page_summary(pages_k[p], dtype) for p in range(NP)])
    sel, scores = select_pages(kbar, Q, Kp, cand, dtype)
    Kc = gather_pages(pages_k, sel)
    Vc = gather_pages(pages_v, sel)
    res = hsa_step(Q, Kc, Vc, Kq, Vq, tau, z, E, F, scale, Binter, Bintra, rows, None, dtype)
    res.update({"s_star": s_star, "pages": sel, "page_scores": scores, "kbar": kbar, "Kc": Kc, "Vc": Vc})
    return res
