"""Tiered page store on the GPU (hkv_store_*), against the oracle: page seal (copy into
the host tier + summary), residency decisions after every fetch / prefetch equal to
the plain model's (integer state, bit-exact), slot contents equal to the pages, and
the gather through the store's page table equal to the plain gather (bitwise)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from hsa_testlib import bits_of, to_dev
from oracle.store import PageStoreModel

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import hybrid_sparse_attention_hkv_b200 as hsa
    from hybrid_sparse_attention_hkv_b200.store import PageStore


def _host_pages(store, kv):
    mem = store.host[kv]
    n = store.NP * store.P_tok * store.H * store.d
    buf = (ctypes.c_uint16 * n).from_address(mem.host_ptr)
    return np.frombuffer(buf, dtype=np.uint16).reshape(store.NP, store.P_tok, store.H, store.d)


def _sealed_store(NP, S, P_tok, H, d, seed):
    store = PageStore(NP, S, P_tok, H, d)
    ws = hsa.workspace(hsa.make_config(H, d, 8, 0, 64))
    kbar = torch.zeros(NP, H, d, dtype=torch.float32, device="cuda")
    pk = synth.normal_bf16((NP, P_tok, H, d), seed, 1)
    pv = synth.normal_bf16((NP, P_tok, H, d), seed, 2)
    for p in range(NP):
        store.seal(p, to_dev(pk[p]), to_dev(pv[p]), kbar[p], ws)
    torch.cuda.synchronize()
    return store, ws, kbar, pk, pv


def _check_state(store, model, pk, pv):
    sp, ps = store.residency()
    assert sp.cpu().tolist() == model.slot_of_page
    assert ps.cpu().tolist() == model.page_of_slot
    sk, sv = bits_of(store.slot_k), bits_of(store.slot_v)
    for s, p in enumerate(model.page_of_slot):
        if p >= 0:
            assert np.array_equal(sk[s], pk[p]) and np.array_equal(sv[s], pv[p]), (s, p)


def test_seal_writes_host_tier_and_summary():
    NP, S, P_tok, H, d = 5, 2, 200, 3, 128
    store, ws, kbar, pk, pv = _sealed_store(NP, S, P_tok, H, d, 41)
    try:
        assert np.array_equal(_host_pages(store, 0), pk)
        assert np.array_equal(_host_pages(store, 1), pv)
        ref = np.stack([oracle.page_summary(pk[p]) for p in range(NP)])
        np.testing.assert_allclose(kbar.cpu().numpy(), ref, rtol=1e-5, atol=1e-6)
        assert hsa.hsa_status_read(ws) == 0
    finally:
        store.close()


def test_residency_matches_model_over_a_random_sequence():
    NP, S, P_tok, H, d = 9, 4, 136, 2, 64
    store, ws, kbar, pk, pv = _sealed_store(NP, S, P_tok, H, d, 42)
    try:
        model = PageStoreModel(NP, S)
        rng = np.random.default_rng(5)
        _check_state(store, model, pk, pv)
        for step in range(24):
            if step % 3 != 2:
                Kp = int(rng.integers(1, S + 1))
                sel = sorted(rng.choice(NP, Kp, replace=False).tolist())
                model.fetch(sel)
                store.fetch(torch.tensor(sel, dtype=torch.int32, device="cuda"), ws)
            else:
                scores = rng.normal(size=NP).astype(np.float32)
                scores[rng.random(NP) < 0.25] = -np.inf
                protect = sorted(rng.choice(NP, int(rng.integers(0, 3)), replace=False).tolist())
                m = int(rng.integers(0, S + 2))
                model.prefetch(scores.astype(np.float64), protect, m)
                store.prefetch(torch.from_numpy(scores).cuda(), torch.tensor(protect, dtype=torch.int32, device="cuda"),
                               m, ws)
            torch.cuda.synchronize()
            _check_state(store, model, pk, pv)
        assert hsa.hsa_status_read(ws) == 0
    finally:
        store.close()


def test_gather_through_the_store_is_bitwise():
    NP, S, P_tok, H, d, Kp = 6, 3, 200, 3, 128, 3
    store, ws, kbar, pk, pv = _sealed_store(NP, S, P_tok, H, d, 43)
    try:
        tk, tv = store.page_tables()
        Lc = Kp * P_tok
        for sel in ([0, 2, 5], [1, 2, 3], [0, 4, 5]):
            st_sel = torch.tensor(sel, dtype=torch.int32, device="cuda")
            Kc = torch.empty(Lc, H, d, dtype=torch.bfloat16, device="cuda")
            Vc = torch.empty_like(Kc)
            kb128 = torch.empty(-(-Lc // 128), H, d, dtype=torch.float32, device="cuda")
            # before the fetch the gather reads the missing pages from the host tier
            hsa.hkv_gather(tk, tv, st_sel, Kp, P_tok, H, d, Kc, Vc, ws, kb128)
            torch.cuda.synchronize()
            assert np.array_equal(bits_of(Kc), oracle.gather_pages(pk, sel))
            store.fetch(st_sel, ws)
            Kc.zero_()
            Vc.zero_()
            hsa.hkv_gather(tk, tv, st_sel, Kp, P_tok, H, d, Kc, Vc, ws, kb128)
            torch.cuda.synchronize()
            sp, _ = store.residency()
            assert all(sp.cpu().numpy()[sel] >= 0)  # read from HBM slots this time
            assert np.array_equal(bits_of(Kc), oracle.gather_pages(pk, sel))
            assert np.array_equal(bits_of(Vc), oracle.gather_pages(pv, sel))
            np.testing.assert_allclose(kb128.cpu().numpy(), oracle.block_means(bits_of(Kc), 128), rtol=1e-5,
                                       atol=1e-6)
        assert hsa.hsa_status_read(ws) == 0
    finally:
        store.close()


def test_fewer_slots_than_selected_pages_reads_the_rest_from_the_host_tier():
    NP, S, P_tok, H, d, Kp = 5, 2, 136, 2, 64, 3
    store, ws, kbar, pk, pv = _sealed_store(NP, S, P_tok, H, d, 44)
    try:
        sel = [0, 1, 4]
        st_sel = torch.tensor(sel, dtype=torch.int32, device="cuda")
        hsa.hsa_status_clear(ws)
        store.fetch(st_sel, ws)
        assert hsa.hsa_status_read(ws) == 6  # HSA_ERR_DEVICE: one page stays on the host tier
        model = PageStoreModel(NP, S)
        model.fetch(sel)
        _check_state(store, model, pk, pv)
        tk, tv = store.page_tables()
        Kc = torch.empty(Kp * P_tok, H, d, dtype=torch.bfloat16, device="cuda")
        Vc = torch.empty_like(Kc)
        hsa.hsa_status_clear(ws)
        hsa.hkv_gather(tk, tv, st_sel, Kp, P_tok, H, d, Kc, Vc, ws)
        assert hsa.hsa_status_read(ws) == 0
        assert np.array_equal(bits_of(Kc), oracle.gather_pages(pk, sel))
        assert np.array_equal(bits_of(Vc), oracle.gather_pages(pv, sel))
    finally:
        store.close()
