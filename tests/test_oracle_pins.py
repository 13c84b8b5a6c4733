"""Pins for the fp64 oracle, against things other than itself.

* dense softmax attention from a library routine (torch SDPA, float64, CPU);
* closed forms and hand-derived fixtures (tests/golden/*.json);
* brute-force subset enumeration for the block-selection rule;
* invariants the method fixes (tau = 1 keeps everything, E = F = I, gates at +-inf).

Each test targets a plausible mistake: a dropped scale, a wrong comparison at the
threshold, a wrong tie order, a block index computed at the wrong granularity, E and
F swapped or transposed, a gate applied the wrong way round.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth


def bf16(x):
    return synth.f32_to_bf16(np.asarray(x, dtype=np.float32))


def rand_bf16(shape, seed, stream, sigma=1.0):
    return synth.normal_bf16(shape, seed, stream, sigma=sigma)


def sdpa(q, k, v, scale, mask=None):
    """Library dense attention, float64: q [Lq,H,d], k/v [Lk,H,d] -> [Lq,H,d]."""
    tq = torch.from_numpy(np.ascontiguousarray(q, dtype=np.float64)).permute(1, 0, 2)
    tk = torch.from_numpy(np.ascontiguousarray(k, dtype=np.float64)).permute(1, 0, 2)
    tv = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float64)).permute(1, 0, 2)
    m = None if mask is None else torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=m, scale=scale)
    return o.permute(1, 0, 2).numpy()


def load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------- block selection rule

def test_keep_blocks_golden(golden_dir):
    g = load(golden_dir, "keep_blocks.json")
    for c in g["cases"]:
        got = oracle.keep_blocks(np.array(c["p"]), c["tau"]).tolist()
        assert got == c["keep"], c


def test_keep_blocks_bruteforce():
    """The greedy prefix equals the minimum-cardinality subset with mass >= tau, and among
    subsets of that size it has the largest mass (enumerating every subset, n <= 12)."""
    rng = np.random.default_rng(7)
    for trial in range(400):
        n = int(rng.integers(1, 13))
        p = rng.dirichlet(np.full(n, rng.choice([0.2, 1.0, 5.0])))
        if trial % 5 == 0:  # quantised masses create exact ties
            p = np.round(p * 16) / 16
            if p.sum() == 0:
                p[0] = 1.0
            p = p / p.sum()
        tau = float(rng.choice([rng.uniform(0, 1), 0.35, 0.5, 0.9, 1.0, 0.0]))
        got = oracle.keep_blocks(p, tau)
        if tau >= 1.0:
            assert got.tolist() == list(range(n))
            continue
        best_k = None
        for k in range(1, n + 1):
            masses = [sum(p[list(s)]) for s in itertools.combinations(range(n), k)]
            if max(masses) >= tau:
                best_k, best_mass = k, max(masses)
                break
        if best_k is None:  # rounding left the total just below tau: everything is kept
            assert len(got) == n
            continue
        assert len(got) == best_k, (p, tau, got)
        assert math.isclose(p[got].sum(), best_mass, rel_tol=0, abs_tol=1e-12)
        assert np.all(np.diff(got) > 0)


def test_keep_blocks_invariants():
    rng = np.random.default_rng(11)
    for _ in range(200):
        n = int(rng.integers(2, 60))
        p = rng.dirichlet(np.full(n, 0.5))
        prev = 0
        for tau in np.linspace(0.0, 0.999, 25):
            kept = oracle.keep_blocks(p, tau)
            m = p[kept].sum()
            assert m >= tau - 1e-15
            assert m - p[kept].min() < tau or len(kept) == 1
            assert len(kept) >= prev  # monotone in tau
            prev = len(kept)


# ----------------------------------------------------------------- pages

def test_page_select_golden(golden_dir):
    g = load(golden_dir, "page_select.json")
    Q = bf16(g["Q"])
    kbar = np.array(g["kbar"], dtype=np.float64)
    for c in g["cases"]:
        sel, s = oracle.select_pages(kbar, Q, c["Kp"], c["cand"], dtype=np.float64)
        assert sel.tolist() == c["sel"], c
        assert s.tolist() == g["scores"]


def test_page_summary_and_scores_closed_form():
    # K_page[t, h, c] = t (P_tok rows) -> mean (P_tok - 1) / 2 everywhere
    P, H, d = 100, 3, 4
    K = bf16(np.broadcast_to(np.arange(P, dtype=np.float32)[:, None, None], (P, H, d)))
    kb = oracle.page_summary(K)
    assert np.all(kb == 49.5)
    Q = bf16(np.ones((7, H, d)))
    assert oracle.page_scores(kb[None], oracle.pooled_query(Q))[0] == 49.5 * H * d


def test_page_select_full_sort_and_plant():
    rng = np.random.default_rng(3)
    for trial in range(50):
        NP, H, d, Kp = int(rng.integers(2, 20)), 2, 8, 0
        Kp = int(rng.integers(1, NP + 1))
        kbar = rng.standard_normal((NP, H, d))
        Q = rand_bf16((33, H, d), 5 + trial, 1)
        sel, s = oracle.select_pages(kbar, Q, Kp, dtype=np.float64)
        qbar = synth.bf16_to_f32(Q).astype(np.float64).mean(axis=0)
        ref = np.array([(kbar[p] * qbar).sum() for p in range(NP)])
        np.testing.assert_allclose(s, ref, rtol=1e-12, atol=1e-12)
        top = np.argsort(-ref, kind="stable")[:Kp]
        assert sel.tolist() == sorted(top.tolist())
    # planted: queries carry the offset of pages 2 and 5 -> those two are retrieved
    H, d, NP = 4, 16, 8
    mu = rng.standard_normal((NP, H, d)) * 0.5
    pages = np.stack([bf16(rng.standard_normal((64, H, d)) + mu[p]) for p in range(NP)])
    Q = bf16(rng.standard_normal((64, H, d)) + np.concatenate([np.repeat(mu[2][None], 32, 0), np.repeat(mu[5][None], 32, 0)]))
    kbar = np.stack([oracle.page_summary(pages[p]) for p in range(NP)])
    sel, _ = oracle.select_pages(kbar, Q, 2)
    assert sel.tolist() == [2, 5]


def test_prompt_top1():
    rng = np.random.default_rng(5)
    S, D = 9, 256
    e = rng.standard_normal((S, D))
    for s in range(S):
        cur = e[s] + 0.5 * rng.standard_normal(D)
        assert oracle.prompt_top1(cur, e) == s
        # cosine: positive row scaling changes nothing
        assert oracle.prompt_top1(cur, e * rng.uniform(0.1, 10, (S, 1))) == s
    e2 = e.copy()
    e2[6] = e2[2] * 2.0  # same direction (power-of-two scale keeps the tie exact)
    assert oracle.prompt_top1(e2[2], e2) == 2
    e2[1] = e2[2]        # exact duplicate at a lower index wins
    assert oracle.prompt_top1(e2[2], e2) == 1


def test_gather_is_index_copy():
    pages = rand_bf16((6, 10, 2, 4), 9, 1)
    sel = [1, 3, 4]
    Kc = oracle.gather_pages(pages, sel)
    assert Kc.dtype == np.uint16 and Kc.shape == (30, 2, 4)
    ref = torch.from_numpy(pages.astype(np.int32)).index_select(0, torch.tensor(sel)).reshape(30, 2, 4).numpy()
    assert np.array_equal(Kc.astype(np.int32), ref)


# ----------------------------------------------------------------- pooling and block masses

def test_block_means_closed_form():
    # X[t] = t for t < 200 (exact in bf16), B = 64: blocks [0,64) [64,128) [128,192) [192,200)
    X = bf16(np.broadcast_to(np.arange(200, dtype=np.float32)[:, None, None], (200, 2, 3)))
    m = oracle.block_means(X, 64)
    assert m.shape == (4, 2, 3)
    assert m[:, 0, 0].tolist() == [31.5, 95.5, 159.5, 195.5]
    m128 = oracle.block_means(X, 128)
    assert m128[:, 1, 2].tolist() == [63.5, 163.5]


def test_block_probs_block_size_one_are_attention_weights():
    """With blocks of one token the block masses are the dense attention weights, which
    the library routine returns when V is the identity."""
    H, d, Lq, Lk = 2, 16, 12, 20
    Q = rand_bf16((Lq, H, d), 21, 1)
    K = rand_bf16((Lk, H, d), 21, 2)
    scale = 1 / math.sqrt(d)
    p = oracle.block_probs(oracle.block_means(Q, 1), oracle.block_means(K, 1), scale)
    eye = np.broadcast_to(np.eye(Lk)[:, None, :], (Lk, H, Lk))
    w = sdpa(oracle.widen(Q), oracle.widen(K), eye, scale)  # [Lq, H, Lk]
    np.testing.assert_allclose(p, w.transpose(1, 0, 2), rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------- sparse branch

def _tiny(seed, Lq=100, Lc=96, H=2, d=16):
    Q = rand_bf16((Lq, H, d), seed, 1)
    Kc = rand_bf16((Lc, H, d), seed, 2)
    Vc = rand_bf16((Lc, H, d), seed, 3)
    Kq = rand_bf16((Lq, H, d), seed, 4)
    Vq = rand_bf16((Lq, H, d), seed, 5)
    return Q, Kc, Vc, Kq, Vq


@pytest.mark.parametrize("Bi,Bq", [(16, 8), (32, 16), (128, 64)])
def test_tau_one_sparse_branch_is_dense_attention(Bi, Bq):
    Q, Kc, Vc, Kq, Vq = _tiny(31, Lq=100, Lc=256)  # ragged Lq tail
    H, d = Q.shape[1], Q.shape[2]
    tau = np.ones(H)
    sel = oracle.block_select(Q, Kc, Kq, tau, None, Bi, Bq, dtype=np.float64)
    assert all(len(b) == -(-256 // Bi) for rows in sel.inter for b in rows)
    o = oracle.sparse_attention(Q, Kc, Vc, Kq, Vq, sel.inter, sel.intra, None, Bi, Bq)
    ref = sdpa(oracle.widen(Q), np.concatenate([oracle.widen(Kc), oracle.widen(Kq)]),
               np.concatenate([oracle.widen(Vc), oracle.widen(Vq)]), 1 / math.sqrt(d))
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-12)


def test_sparse_branch_equals_masked_dense_attention():
    """Random selections; the key set of each query is written out as an explicit token
    mask and handed to the library routine."""
    rng = np.random.default_rng(17)
    Bi, Bq = 16, 8
    Q, Kc, Vc, Kq, Vq = _tiny(41, Lq=45, Lc=80)
    Lq, H, d = Q.shape
    Lc = Kc.shape[0]
    nQi, nKi, nQq, nKq = -(-Lq // Bi), Lc // Bi, -(-Lq // Bq), -(-Lq // Bq)
    inter = [[np.sort(rng.choice(nKi, int(rng.integers(1, nKi + 1)), replace=False)) for _ in range(nQi)] for _ in range(H)]
    intra = [[np.sort(rng.choice(nKq, int(rng.integers(0, nKq + 1)), replace=False)) for _ in range(nQq)] for _ in range(H)]
    o = oracle.sparse_attention(Q, Kc, Vc, Kq, Vq, inter, intra, None, Bi, Bq)
    Kall = np.concatenate([oracle.widen(Kc), oracle.widen(Kq)])
    Vall = np.concatenate([oracle.widen(Vc), oracle.widen(Vq)])
    for h in range(H):
        mask = np.zeros((1, Lq, Lc + Lq), dtype=bool)
        for t in range(Lq):
            for key in range(Lc):
                mask[0, t, key] = (key // Bi) in set(inter[h][t // Bi].tolist())
            for key in range(Lq):
                mask[0, t, Lc + key] = (key // Bq) in set(intra[h][t // Bq].tolist())
        ref = sdpa(oracle.widen(Q[:, h:h + 1]), Kall[:, h:h + 1], Vall[:, h:h + 1], 1 / math.sqrt(d), mask)
        np.testing.assert_allclose(o[:, h:h + 1], ref, rtol=1e-11, atol=1e-12)


def test_sparse_branch_uniform_keys_average_selected_values():
    """Identical keys give uniform weights: the output is the mean of the selected value rows."""
    Bi, Bq, H, d, Lq, Lc = 16, 8, 1, 8, 20, 48
    Q = rand_bf16((Lq, H, d), 2, 1)
    Kc = bf16(np.ones((Lc, H, d)))
    Kq = bf16(np.ones((Lq, H, d)))
    Vc = bf16(np.arange(Lc, dtype=np.float32)[:, None, None] * np.ones((1, H, d)))
    Vq = bf16(200 + np.arange(Lq, dtype=np.float32)[:, None, None] * np.ones((1, H, d)))
    inter = [[np.array([0, 2]), np.array([1])]]
    intra = [[np.array([0]), np.array([1, 2]), np.array([2])]]
    o = oracle.sparse_attention(Q, Kc, Vc, Kq, Vq, inter, intra, None, Bi, Bq)
    # query 0..7: Kc blocks 0,2 (rows 0-15, 32-47) + Kq block 0 (rows 0-7)
    exp0 = np.mean(list(range(16)) + list(range(32, 48)) + [200 + i for i in range(8)])
    # values 0..47 and 200..219 are exact in bf16
    # query 16..19: Kc block 1 (16-31) + Kq block 2 (rows 16-19, a partial block)
    exp2 = np.mean(list(range(16, 32)) + [200 + i for i in range(16, 20)])
    assert np.allclose(o[0:8, 0, :], exp0, rtol=0, atol=1e-9)
    assert np.allclose(o[16:20, 0, :], exp2, rtol=0, atol=1e-9)


def test_attention_closed_forms(golden_dir):
    g = load(golden_dir, "attention_closed_form.json")
    arr = {k: bf16(g[k]) for k in ("Q", "Kc", "Vc", "Kq", "Vq")}
    for c in g["sparse_cases"]:
        o = oracle.sparse_attention(arr["Q"], arr["Kc"], arr["Vc"], arr["Kq"], arr["Vq"],
                                    [[np.array(c["inter"])]], [[np.array(c["intra"], dtype=np.int64)]], 1.0, 1, 1)
        assert math.isclose(o[0, 0, 0], c["out"], rel_tol=1e-15), c
    for c in g["linear_cases"]:
        EK, FV = oracle.linear_projection(bf16(c["E"]), bf16(c["F"]), arr["Kc"], arr["Kq"], arr["Vc"], arr["Vq"])
        o = oracle.linear_attention(arr["Q"], EK, FV, 1.0)
        assert math.isclose(o[0, 0, 0], c["out"], rel_tol=1e-15), c
    for c in g["gate_cases"]:
        z = float(c["z"])
        assert math.isclose(float(oracle.gate(np.array([z]))[0]), c["g"], rel_tol=1e-15), c


# ----------------------------------------------------------------- linear branch

def test_linear_branch_identity_is_dense_attention():
    Q, Kc, Vc, Kq, Vq = _tiny(51, Lq=37, Lc=64, d=8)
    L = Kc.shape[0] + Q.shape[0]
    I = bf16(np.eye(L))
    EK, FV = oracle.linear_projection(I, I, Kc, Kq, Vc, Vq)
    o = oracle.linear_attention(Q, EK, FV)
    ref = sdpa(oracle.widen(Q), np.concatenate([oracle.widen(Kc), oracle.widen(Kq)]),
               np.concatenate([oracle.widen(Vc), oracle.widen(Vq)]), 1 / math.sqrt(Q.shape[2]))
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-12)


def test_linear_branch_permutations_pin_E_and_F_roles():
    Q, Kc, Vc, Kq, Vq = _tiny(61, Lq=20, Lc=32, d=8)
    L = 52
    rng = np.random.default_rng(0)
    P1, P2 = np.eye(L)[rng.permutation(L)], np.eye(L)[rng.permutation(L)]
    Kall = np.concatenate([oracle.widen(Kc), oracle.widen(Kq)])
    Vall = np.concatenate([oracle.widen(Vc), oracle.widen(Vq)])
    sc = 1 / math.sqrt(8)
    EK, FV = oracle.linear_projection(bf16(P1), bf16(P1), Kc, Kq, Vc, Vq)
    np.testing.assert_allclose(oracle.linear_attention(Q, EK, FV), sdpa(oracle.widen(Q), Kall, Vall, sc), rtol=1e-11, atol=1e-12)
    # different permutations: keys follow E, values follow F
    EK, FV = oracle.linear_projection(bf16(P1), bf16(P2), Kc, Kq, Vc, Vq)
    Vperm = np.einsum("ij,jhc->ihc", P1.T @ P2, Vall)
    np.testing.assert_allclose(oracle.linear_attention(Q, EK, FV), sdpa(oracle.widen(Q), Kall, Vperm, sc), rtol=1e-11, atol=1e-12)


def test_linear_branch_per_head_matrices():
    Q, Kc, Vc, Kq, Vq = _tiny(71, Lq=16, Lc=16, H=2, d=8)
    L = 32
    E = np.stack([np.eye(L), np.eye(L)[::-1]])
    F = np.stack([np.eye(L)[::-1], np.eye(L)])
    EK, FV = oracle.linear_projection(bf16(E), bf16(F), Kc, Kq, Vc, Vq)
    Kall = np.concatenate([oracle.widen(Kc), oracle.widen(Kq)])
    Vall = np.concatenate([oracle.widen(Vc), oracle.widen(Vq)])
    np.testing.assert_array_equal(EK[0], Kall[:, 0])
    np.testing.assert_array_equal(EK[1], Kall[::-1, 1])
    np.testing.assert_array_equal(FV[0], Vall[::-1, 0])
    np.testing.assert_array_equal(FV[1], Vall[:, 1])


def test_linear_projection_is_matrix_product():
    Q, Kc, Vc, Kq, Vq = _tiny(81, Lq=10, Lc=16, H=2, d=4)
    E = rand_bf16((3, 26), 81, 9)
    EK, _ = oracle.linear_projection(E, E, Kc, Kq, Vc, Vq)
    Kall = np.concatenate([oracle.widen(Kc), oracle.widen(Kq)])
    for h in range(2):
        for j in range(3):
            for c in range(4):
                ref = math.fsum(oracle.widen(E)[j, t] * Kall[t, h, c] for t in range(26))
                assert math.isclose(EK[h, j, c], ref, rel_tol=1e-13, abs_tol=1e-13)


# ----------------------------------------------------------------- merge and full step

def test_gates_isolate_each_branch_exactly():
    Q, Kc, Vc, Kq, Vq = _tiny(91, Lq=70, Lc=128, d=16)
    H = Q.shape[1]
    L = 198
    E = rand_bf16((32, L), 91, 7, 1 / math.sqrt(32))
    F = rand_bf16((32, L), 91, 8, 1 / math.sqrt(32))
    tau = np.array([0.9, 0.35])
    for z, which in ((np.full(H, np.inf), "o_s"), (np.full(H, -np.inf), "o_l")):
        r = oracle.hsa_step(Q, Kc, Vc, Kq, Vq, tau, z, E, F, None, 32, 16)
        assert np.array_equal(r["out"], r[which])
    r = oracle.hsa_step(Q, Kc, Vc, Kq, Vq, tau, np.array([0.0, np.log(3.0)]), E, F, None, 32, 16)
    np.testing.assert_allclose(r["out"][:, 0], 0.5 * (r["o_s"][:, 0] + r["o_l"][:, 0]), rtol=1e-15)
    np.testing.assert_allclose(r["out"][:, 1], 0.75 * r["o_s"][:, 1] + 0.25 * r["o_l"][:, 1], rtol=1e-14)


def test_full_step_tau_one_gate_one_is_dense_over_retrieved_pages():
    shape = synth.SHAPES[0]
    x = synth.make_inputs(shape, synth.seed_of(0))
    H = shape.H
    r = oracle.hkv_hsa_step(x.pages_k, x.pages_v, x.Q, x.Kq, x.Vq, shape.Kp, np.ones(H), np.full(H, np.inf),
                            x.E, x.F, dtype=np.float64)
    assert len(r["pages"]) == shape.Kp and np.all(np.diff(r["pages"]) > 0)
    Kall = np.concatenate([oracle.widen(r["Kc"]), oracle.widen(x.Kq)])
    Vall = np.concatenate([oracle.widen(r["Vc"]), oracle.widen(x.Vq)])
    ref = sdpa(oracle.widen(x.Q), Kall, Vall, 1 / math.sqrt(shape.d))
    np.testing.assert_allclose(r["out"], ref, rtol=1e-10, atol=1e-11)


def test_rows_subset_matches_full():
    Q, Kc, Vc, Kq, Vq = _tiny(101, Lq=90, Lc=64, d=16)
    sel = oracle.block_select(Q, Kc, Kq, np.array([0.6, 0.4]), None, 32, 16)
    full = oracle.sparse_attention(Q, Kc, Vc, Kq, Vq, sel.inter, sel.intra, None, 32, 16)
    rows = np.array([0, 17, 33, 64, 89])
    part = oracle.sparse_attention(Q, Kc, Vc, Kq, Vq, sel.inter, sel.intra, None, 32, 16, rows=rows)
    np.testing.assert_allclose(part, full[rows], rtol=1e-13, atol=1e-14)  # BLAS blocking may differ


def test_biased_workload_retrieves_the_planted_pages():
    """Structure of the large workloads at reduced token counts: the three pages the
    queries are biased toward are among the retrieved ones, in every configuration."""
    for i in (1, 3, 4):
        shape = synth.SHAPES[i].replace(F_tok=96, page_tok=0, H=4)
        x = synth.make_inputs(shape, synth.seed_of(i))
        kbar = np.stack([oracle.page_summary(x.pages_k[p], np.float32) for p in range(shape.NP)])
        cand = None
        if shape.n_segments:
            s = oracle.prompt_top1(x.e_cur, x.e_seg)
            assert s == x.s_star
            cand = range(int(x.seg_begin[s]), int(x.seg_begin[s + 1]))
        sel, _ = oracle.select_pages(kbar, x.Q, shape.Kp, cand)
        assert set(x.biased) <= set(sel.tolist()), (i, x.biased, sel)


def test_no_history_reduces_to_chunk_attention():
    """Lc = 0: the inter map is empty and, with tau = 1, the sparse branch is dense
    attention over the chunk's own keys (library routine)."""
    Q, _, _, Kq, Vq = _tiny(111, Lq=40, Lc=8, d=16)
    H, d = Q.shape[1], Q.shape[2]
    empty = np.zeros((0, H, d), dtype=np.uint16)
    sel = oracle.block_select(Q, empty, Kq, np.ones(H), None, 16, 8, dtype=np.float64)
    assert all(len(b) == 0 for rows in sel.inter for b in rows)
    o = oracle.sparse_attention(Q, empty, empty, Kq, Vq, sel.inter, sel.intra, None, 16, 8)
    ref = sdpa(oracle.widen(Q), oracle.widen(Kq), oracle.widen(Vq), 1 / math.sqrt(d))
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-12)


def _frac(s):
    n, d = s.split("/")
    return int(n) / int(d)


def test_block_select_golden(golden_dir):
    """Block pooling + block scores + per-map softmax + per-head threshold, composed, at
    tau < 1, against hand-derived masses and kept lists.  The fixture is built so that
    pooling Q at the wrong block size, one joint inter+intra softmax, a swapped head
    index or the wrong head's tau each changes a kept list."""
    g = load(golden_dir, "block_select.json")
    Q64 = np.asarray(g["Q64_blocks"], dtype=np.float32)     # [H][4][d]
    Kc128 = np.asarray(g["Kc128_blocks"], dtype=np.float32)  # [H][4][d]
    Kq64 = np.asarray(g["Kq64_blocks"], dtype=np.float32)    # [H][4][d]
    Q = bf16(np.repeat(Q64.transpose(1, 0, 2), 64, axis=0))    # [256, H, d]
    Kc = bf16(np.repeat(Kc128.transpose(1, 0, 2), 128, axis=0))  # [512, H, d]
    Kq = bf16(np.repeat(Kq64.transpose(1, 0, 2), 64, axis=0))  # [256, H, d]
    tau = np.asarray(g["tau"], dtype=np.float32)
    sel = oracle.block_select(Q, Kc, Kq, tau, scale=math.log(2.0), dtype=np.float64)
    want_pi = np.array([[[_frac(x) for x in row] for row in head] for head in g["p_inter"]])
    want_pq = np.array([[[_frac(x) for x in row] for row in head] for head in g["p_intra"]])
    np.testing.assert_allclose(sel.p_inter, want_pi, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(sel.p_intra, want_pq, rtol=1e-12, atol=1e-15)
    assert [[r.tolist() for r in h] for h in sel.inter] == g["keep_inter"]
    assert [[r.tolist() for r in h] for h in sel.intra] == g["keep_intra"]
    # the fp32 decision precision gives the same lists here (no mass within 1e-5 of a threshold)
    sel32 = oracle.block_select(Q, Kc, Kq, tau, scale=math.log(2.0), dtype=np.float32)
    assert [[r.tolist() for r in h] for h in sel32.inter] == g["keep_inter"]
    assert [[r.tolist() for r in h] for h in sel32.intra] == g["keep_intra"]


def test_block_select_golden_rejects_plausible_mistakes(golden_dir):
    """Planted mistakes (built on the CPU from the oracle's own parts) disagree with the
    golden lists: queries pooled at 64 for the inter map, at 128 for the intra map, one
    joint softmax over the inter and intra rows of a query, the wrong head's keys."""
    g = load(golden_dir, "block_select.json")
    Q = bf16(np.repeat(np.asarray(g["Q64_blocks"], np.float32).transpose(1, 0, 2), 64, axis=0))
    Kc = bf16(np.repeat(np.asarray(g["Kc128_blocks"], np.float32).transpose(1, 0, 2), 128, axis=0))
    Kq = bf16(np.repeat(np.asarray(g["Kq64_blocks"], np.float32).transpose(1, 0, 2), 64, axis=0))
    tau = np.asarray(g["tau"])
    sc = math.log(2.0)
    want_inter, want_intra = g["keep_inter"], g["keep_intra"]

    def keep(p, h):
        return [oracle.keep_blocks(p[h, i], tau[h]).tolist() for i in range(p.shape[1])]

    kc128 = oracle.block_means(Kc, 128)
    kq64 = oracle.block_means(Kq, 64)
    # inter map scored with 64-row query means (rows 0 and 2 stand for the two 128-row blocks)
    p_bad = oracle.block_probs(oracle.block_means(Q, 64)[::2], kc128, sc)
    assert [keep(p_bad, h) for h in range(2)] != want_inter
    # intra map scored with 128-row query means (each used for both of its 64-row halves)
    p_bad = oracle.block_probs(np.repeat(oracle.block_means(Q, 128), 2, axis=0), kq64, sc)
    assert [keep(p_bad, h) for h in range(2)] != want_intra
    # one joint softmax over [inter row of the 128-block | intra row of the 64-block]
    q128, q64 = oracle.block_means(Q, 128), oracle.block_means(Q, 64)
    joint_intra = []
    for h in range(2):
        rows = []
        for i in range(4):
            s = np.concatenate([q128[i // 2, h] @ kc128[:, h].T, q64[i, h] @ kq64[:, h].T]) * sc
            w = np.exp(s - s.max())
            kept = oracle.keep_blocks(w / w.sum(), tau[h])
            rows.append([int(j) - 4 for j in kept if j >= 4])
        joint_intra.append(rows)
    assert joint_intra != want_intra
    # head 1 scored against head 0's keys
    swapped = Kc.copy()
    swapped[:, 1] = Kc[:, 0]
    assert [r.tolist() for r in oracle.block_select(Q, swapped, Kq, tau, scale=sc, dtype=np.float64).inter[1]] \
        != want_inter[1]


def test_retrieval_policies_closed_forms():
    """Recent pages are the last Kp candidates; random pages are the Kp largest keys
    (ties -> lower page id), checked against a plain stable sort; 'score' is select_pages."""
    rng = np.random.default_rng(11)
    kb = rng.normal(size=(12, 2, 8))
    Q = bf16(rng.normal(size=(16, 2, 8)))
    assert oracle.select_pages_policy("recent", kb, Q, 3).tolist() == [9, 10, 11]
    assert oracle.select_pages_policy("recent", kb, Q, 2, cand=range(3, 7)).tolist() == [5, 6]
    keys = np.array([0.5, 0.9, 0.1, 0.9, 0.3, 0.7, 0.2, 0.0, 0.8, 0.6, 0.4, 0.95])
    # ranked: 11 (.95), 1 and 3 tie at .9 (1 first), 8 (.8) ...
    assert oracle.select_pages_policy("random", kb, Q, 3, rand_keys=keys).tolist() == [1, 3, 11]
    assert oracle.select_pages_policy("random", kb, Q, 2, cand=[0, 2, 4, 6], rand_keys=keys).tolist() == [0, 4]
    for _ in range(50):
        k = rng.integers(0, 5, size=12).astype(float)  # many ties
        Kp = int(rng.integers(1, 12))
        order = np.argsort(-k, kind="stable")  # stable: ties keep the lower index first
        assert oracle.select_pages_policy("random", kb, Q, Kp, rand_keys=k).tolist() == sorted(order[:Kp].tolist())
    assert np.array_equal(oracle.select_pages_policy("score", kb, Q, 3), oracle.select_pages(kb, Q, 3)[0])


def test_fidelity_closed_forms():
    """Keeping every block: the sparse branch is dense attention (cos 1, error 0, mass 1);
    E = F = I with r = L: the linear branch is dense attention too; the kept mass equals
    exp(lse_kept - lse_all) computed with a library log-sum-exp."""
    from scipy.special import logsumexp
    H, d, Lq, Lc = 2, 8, 128, 256
    L = Lq + Lc
    Q = rand_bf16((Lq, H, d), 31, 1)
    Kc, Vc = rand_bf16((Lc, H, d), 31, 2), rand_bf16((Lc, H, d), 31, 3)
    Kq, Vq = rand_bf16((Lq, H, d), 31, 4), rand_bf16((Lq, H, d), 31, 5)
    I = bf16(np.eye(L))
    EK, FV = oracle.linear_projection(I, I, Kc, Kq, Vc, Vq)
    full_i = [[np.arange(2)] * 1] * H
    full_q = [[np.arange(2)] * 2] * H
    rep = oracle.fidelity(Q, Kc, Vc, Kq, Vq, full_i, full_q, EK, FV)
    np.testing.assert_allclose(rep[:, [0, 1, 2]], 1.0, atol=1e-12)
    np.testing.assert_allclose(rep[:, [3, 4]], 0.0, atol=1e-12)
    inter = [[np.array([1])], [np.array([0])]]
    intra = [[np.array([0]), np.array([0, 1])], [np.array([1]), np.array([1])]]
    rep = oracle.fidelity(Q, Kc, Vc, Kq, Vq, inter, intra, EK, FV)
    scale = 1 / math.sqrt(d)
    for h in range(H):
        K = np.concatenate([oracle.widen(Kc[:, h]), oracle.widen(Kq[:, h])])
        s = oracle.widen(Q[:, h]) @ K.T * scale
        m = []
        for t in range(Lq):
            kept = [k for k in range(L) if (k < Lc and k // 128 in inter[h][0]) or
                    (k >= Lc and (k - Lc) // 64 in intra[h][t // 64])]
            m.append(np.exp(logsumexp(s[t, kept]) - logsumexp(s[t])))
        assert abs(rep[h, 2] - np.mean(m)) < 1e-12
        assert 0 < rep[h, 2] < 1 and rep[h, 1] < 1 and rep[h, 4] > 0


def test_block_select_joint_golden(golden_dir):
    """The joint selection (one softmax per 64-row query block over the cached and the
    chunk blocks) against hand-derived lists, some of them empty, on the separate
    mode's fixture; the lists are also the minimum-cardinality subsets found by
    enumeration over the joint masses computed here with numpy."""
    g = load(golden_dir, "block_select.json")
    Q = bf16(np.repeat(np.asarray(g["Q64_blocks"], np.float32).transpose(1, 0, 2), 64, axis=0))
    Kc = bf16(np.repeat(np.asarray(g["Kc128_blocks"], np.float32).transpose(1, 0, 2), 128, axis=0))
    Kq = bf16(np.repeat(np.asarray(g["Kq64_blocks"], np.float32).transpose(1, 0, 2), 64, axis=0))
    tau = np.asarray(g["tau"], dtype=np.float32)
    sel = oracle.block_select(Q, Kc, Kq, tau, scale=math.log(2.0), dtype=np.float64, joint=True)
    assert [[r.tolist() for r in h] for h in sel.inter] == g["joint"]["keep_inter"]
    assert [[r.tolist() for r in h] for h in sel.intra] == g["joint"]["keep_intra"]
    q64 = np.asarray(g["Q64_blocks"], np.float64)
    keys = np.concatenate([np.asarray(g["Kc128_blocks"], np.float64), np.asarray(g["Kq64_blocks"], np.float64)], axis=1)
    for h in range(2):
        for i in range(4):
            w = 2.0 ** (keys[h] @ q64[h, i])
            p = w / w.sum()
            kept = g["joint"]["keep_inter"][h][i] + [4 + j for j in g["joint"]["keep_intra"][h][i]]
            assert p[kept].sum() >= tau[h]
            smaller = [sum(p[list(c)]) for c in itertools.combinations(range(8), len(kept) - 1)] if len(kept) > 1 else []
            assert all(m < tau[h] for m in smaller)  # no fewer blocks reach tau


def test_sparse_attention_joint_rows_use_64_row_inter_lists():
    """With inter_rows = 64 each 64-row query block uses its own inter list: equal to
    masked dense attention with the per-64-row key sets."""
    H, d, Lq, Lc = 1, 8, 128, 256
    Q, Kc, Vc = rand_bf16((Lq, H, d), 41, 1), rand_bf16((Lc, H, d), 41, 2), rand_bf16((Lc, H, d), 41, 3)
    Kq, Vq = rand_bf16((Lq, H, d), 41, 4), rand_bf16((Lq, H, d), 41, 5)
    inter = [[np.array([0]), np.array([1])]]
    intra = [[np.array([1]), np.array([0])]]
    got = oracle.sparse_attention(Q, Kc, Vc, Kq, Vq, inter, intra, inter_rows=64)
    K = np.concatenate([oracle.widen(Kc), oracle.widen(Kq)])
    V = np.concatenate([oracle.widen(Vc), oracle.widen(Vq)])
    mask = np.full((1, Lq, Lc + Lq), -np.inf)
    mask[0, :64, 0:128] = 0
    mask[0, :64, Lc + 64:Lc + 128] = 0
    mask[0, 64:, 128:256] = 0
    mask[0, 64:, Lc:Lc + 64] = 0
    want = sdpa(oracle.widen(Q), K, V, 1 / math.sqrt(d), mask)
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)
