"""Full-size parity on the five workloads, in the launch configuration bench.py
times (HkvHsaStep: select pages -> gather -> hsa_forward).

Compared in full: page summaries of sampled pages, prompt segment, page
selection, the gathered active cache (bitwise), block selections of the sampled
heads.  Compared on samples the oracle computes one by one: the output rows of
sampled heads (all Lq-tail and block-boundary rows included)."""
import gc

import numpy as np
import pytest
import torch

import hybrid_sparse_attention_hkv_b200 as hsa
import oracle
import synth
from hsa_testlib import (DeviceStep, assert_close, bits_of, check_pages, check_selection_both, sample_rows,
                         selection_lists)

pytestmark = pytest.mark.gpu


def sampled_heads(H):
    return sorted({0, H // 2, H - 1}) if H > 4 else list(range(H))


@pytest.fixture(scope="module", params=range(len(synth.SHAPES)), ids=[s.name for s in synth.SHAPES])
def run(request):
    i = request.param
    shape = synth.SHAPES[i]
    ds = DeviceStep(shape, synth.seed_of(i))
    ds.run()
    torch.cuda.synchronize()
    assert hsa.hsa_status_read(ds.step.ws) == 0, hsa.wait_report(ds.step.ws)
    yield i, ds
    ds.close()
    del ds
    gc.collect()
    torch.cuda.empty_cache()


def test_retrieval(run):
    i, ds = run
    x, st, shape = ds.x, ds.step, ds.shape
    kbar = st.kbar_pages.cpu().numpy()
    for p in sorted({0, shape.NP - 1}):
        np.testing.assert_allclose(kbar[p], oracle.page_summary(x.pages_k[p]), rtol=1e-5, atol=1e-6)
    cand = None
    if shape.n_segments:
        s = oracle.prompt_top1(x.e_cur, x.e_seg)
        assert int(st.seg.item()) == s == x.s_star
        cand = range(int(x.seg_begin[s]), int(x.seg_begin[s + 1]))
        assert st.cand_range.cpu().tolist() == [cand.start, cand.stop]
    sel_ref, scores = oracle.select_pages(kbar, x.Q, shape.Kp, cand)
    gsel = st.sel.cpu().numpy()
    check_pages(gsel, sel_ref, scores, shape.Kp)
    if x.biased:
        assert set(x.biased) <= set(gsel.tolist())


def test_gather_bitwise(run):
    i, ds = run
    x, st = ds.x, ds.step
    sel = st.sel.cpu().numpy()
    assert np.array_equal(bits_of(st.Kc), oracle.gather_pages(x.pages_k, sel))
    assert np.array_equal(bits_of(st.Vc), oracle.gather_pages(x.pages_v, sel))


def test_selection_and_output(run):
    i, ds = run
    x, st, shape = ds.x, ds.step, ds.shape
    hs = sampled_heads(shape.H)
    Kc, Vc = bits_of(st.Kc)[:, hs], bits_of(st.Vc)[:, hs]
    Q, Kq, Vq = x.Q[:, hs], x.Kq[:, hs], x.Vq[:, hs]
    tau, z = x.tau[hs], x.z[hs]
    sb = st.selection
    gi = selection_lists(sb.inter_idx.cpu().numpy()[hs], sb.inter_cnt.cpu().numpy()[hs])
    gq = selection_lists(sb.intra_idx.cpu().numpy()[hs], sb.intra_cnt.cpu().numpy()[hs])
    check_selection_both(gi, gq, Q, Kc, Kq, tau, f"{shape.name} heads {hs}")
    rows = sample_rows(shape.Lq, 40, seed=i)
    res = oracle.hsa_step(Q, Kc, Vc, Kq, Vq, tau, z, x.E, x.F, rows=rows,
                          selection=oracle.Selection(gi, gq, None, None))
    got = st.out.cpu().numpy()[rows][:, hs]
    assert_close(got, res["out"], f"{shape.name} output (heads {hs}, {len(rows)} rows)")
