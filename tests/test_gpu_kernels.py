"""GPU parity of every step of the path against the fp64 oracle, on shapes the
oracle finishes in seconds that still span several tiles and a ragged tail, plus
edge cases and the invariants the method fixes.  All calls go through the C ABI."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from hsa_testlib import (DeviceStep, assert_close, bits_of, check_pages, check_selection, check_selection_both,
                         errors, selection_lists, to_dev)

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import hybrid_sparse_attention_hkv_b200 as hsa
    from hybrid_sparse_attention_hkv_b200 import SelectionBuffers, make_config

# several 128-query tiles, a ragged query tail, pages not a multiple of 128 tokens
SMALL = [
    synth.StepShape("h3_d128_lq296_p200", H=3, d=128, frames=1, F_tok=296, page_frames=1, page_tok=200,
                    NP=6, Kp=3, r=128),
    synth.StepShape("h2_d64_lq200_p136", H=2, d=64, frames=1, F_tok=200, page_frames=1, page_tok=136,
                    NP=5, Kp=2, r=64),
    synth.StepShape("h4_d128_lq520_p384_biased", H=4, d=128, frames=2, F_tok=260, page_frames=1, page_tok=384,
                    NP=8, Kp=2, r=192, n_biased=2),
]


def _ids(s):
    return s.name


@pytest.fixture(scope="module", params=SMALL, ids=_ids)
def small(request):
    ds = DeviceStep(request.param, 77)
    ds.run()
    torch.cuda.synchronize()
    yield ds
    ds.close()


def test_page_summaries(small):
    x = small.x
    ref = np.stack([oracle.page_summary(x.pages_k[p]) for p in range(small.shape.NP)])
    got = small.step.kbar_pages.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-6)


def test_page_selection(small):
    x, st = small.x, small.step
    kbar = st.kbar_pages.cpu().numpy()
    sel_ref, scores_ref = oracle.select_pages(kbar, x.Q, small.shape.Kp)
    scores = st.scores.cpu().numpy()
    np.testing.assert_allclose(scores, scores_ref, rtol=1e-5, atol=1e-5 * np.abs(scores_ref).max())
    check_pages(st.sel.cpu().numpy(), sel_ref, scores_ref, small.shape.Kp)
    assert np.all(np.diff(st.sel.cpu().numpy()) > 0)
    if x.biased:
        assert set(x.biased) <= set(st.sel.cpu().numpy().tolist())


def test_gather_bitwise_and_fused_pooling(small):
    x, st = small.x, small.step
    sel = st.sel.cpu().numpy()
    assert np.array_equal(bits_of(st.Kc), oracle.gather_pages(x.pages_k, sel))
    assert np.array_equal(bits_of(st.Vc), oracle.gather_pages(x.pages_v, sel))
    ref = oracle.block_means(bits_of(st.Kc), 128)
    np.testing.assert_allclose(st.kbar128.cpu().numpy(), ref, rtol=1e-5, atol=1e-6)


def test_block_selection(small):
    x, st = small.x, small.step
    Kc = bits_of(st.Kc)
    sb = st.selection
    gi = selection_lists(sb.inter_idx.cpu().numpy(), sb.inter_cnt.cpu().numpy())
    gq = selection_lists(sb.intra_idx.cpu().numpy(), sb.intra_cnt.cpu().numpy())
    check_selection_both(gi, gq, x.Q, Kc, x.Kq, x.tau, small.shape.name)


def test_forward_output(small):
    x, st = small.x, small.step
    Kc, Vc = bits_of(st.Kc), bits_of(st.Vc)
    sb = st.selection
    sel = oracle.Selection(selection_lists(sb.inter_idx.cpu().numpy(), sb.inter_cnt.cpu().numpy()),
                           selection_lists(sb.intra_idx.cpu().numpy(), sb.intra_cnt.cpu().numpy()), None, None)
    ref = oracle.hsa_step(x.Q, Kc, Vc, x.Kq, x.Vq, x.tau, x.z, x.E, x.F, selection=sel)
    assert_close(st.out.cpu().numpy(), ref["out"], "hsa_forward out")


def test_end_to_end_against_the_oracle_pipeline(small):
    """The whole step from the page store, GPU against the oracle's own pipeline in fp64
    (its own page retrieval, gather, selection, both branches and merge): same pages,
    and the output of every (query row, head) whose two kept block lists agree with
    the oracle's is within the tolerance; disagreeing lists are rare exempt rows."""
    x, st, shape = small.x, small.step, small.shape
    res = oracle.hkv_hsa_step(x.pages_k, x.pages_v, x.Q, x.Kq, x.Vq, shape.Kp, x.tau, x.z, x.E, x.F,
                              dtype=np.float64)
    assert st.sel.cpu().numpy().tolist() == res["pages"].tolist()
    sb = st.selection
    gi = selection_lists(sb.inter_idx.cpu().numpy(), sb.inter_cnt.cpu().numpy())
    gq = selection_lists(sb.intra_idx.cpu().numpy(), sb.intra_cnt.cpu().numpy())
    ref_sel = res["selection"]
    Lq, H = shape.Lq, shape.H
    agree = np.zeros((Lq, H), dtype=bool)
    for h in range(H):
        for t in range(Lq):
            agree[t, h] = (np.array_equal(gi[h][t // 128], ref_sel.inter[h][t // 128])
                           and np.array_equal(gq[h][t // 64], ref_sel.intra[h][t // 64]))
    assert agree.mean() >= 0.99, agree.mean()
    got = st.out.cpu().numpy()
    assert_close(got[agree], res["out"][agree], "end-to-end output on agreeing rows")


def test_branches_standalone(small):
    x, st = small.x, small.step
    cfg = st.cfg
    Kc, Vc = bits_of(st.Kc), bits_of(st.Vc)
    o_s = torch.empty_like(st.out)
    o_l = torch.empty_like(st.out)
    hsa.hsa_sparse_attn(cfg, small.Q, st.Kc, st.Vc, small.Kq, small.Vq, st.selection, o_s, st.ws)
    hsa.hsa_linear_attn(cfg, small.Q, st.Kc, st.Vc, small.Kq, small.Vq, small.E, small.F, o_l, st.ws)
    torch.cuda.synchronize()
    sb = st.selection
    inter = selection_lists(sb.inter_idx.cpu().numpy(), sb.inter_cnt.cpu().numpy())
    intra = selection_lists(sb.intra_idx.cpu().numpy(), sb.intra_cnt.cpu().numpy())
    ref_s = oracle.sparse_attention(x.Q, Kc, Vc, x.Kq, x.Vq, inter, intra)
    assert_close(o_s.cpu().numpy(), ref_s, "sparse branch")
    EK, FV = oracle.linear_projection(x.E, x.F, Kc, x.Kq, Vc, x.Vq)
    ref_l = oracle.linear_attention(x.Q, EK, FV)
    assert_close(o_l.cpu().numpy(), ref_l, "linear branch")
    # the gates isolate each branch exactly (g = 1 or 0 in the merge): the output is
    # then that branch bit for bit
    H = small.shape.H
    for z, want in ((float("inf"), o_s), (float("-inf"), o_l)):
        zz = torch.full((H,), z, dtype=torch.float32, device="cuda")
        out = torch.empty_like(st.out)
        hsa.hsa_forward(cfg, small.Q, st.Kc, st.Vc, small.Kq, small.Vq, small.tau, zz, small.E, small.F, out, st.ws,
                        st.kbar128)
        torch.cuda.synchronize()
        assert torch.equal(out, want), z


def test_deterministic(small):
    first = small.step.out.clone()
    small.run()
    torch.cuda.synchronize()
    assert torch.equal(first, small.step.out)


def test_bf16_output(small):
    """The bf16 output is the fp32 output of the same call rounded to bf16."""
    st = small.step
    out = torch.empty(st.out.shape, dtype=torch.bfloat16, device="cuda")
    ref = torch.empty(st.out.shape, dtype=torch.float32, device="cuda")
    for o in (out, ref):
        hsa.hsa_forward(st.cfg, small.Q, st.Kc, st.Vc, small.Kq, small.Vq, small.tau, small.z, small.E, small.F, o,
                        st.ws, st.kbar128)
    torch.cuda.synchronize()
    assert torch.equal(out, ref.to(torch.bfloat16))


# ----------------------------------------------------------------- invariants on the GPU path

def _sdpa64(q, k, v, scale):
    tq = torch.from_numpy(q).permute(1, 0, 2)
    tk = torch.from_numpy(k).permute(1, 0, 2)
    tv = torch.from_numpy(v).permute(1, 0, 2)
    return torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=scale).permute(1, 0, 2).numpy()


def test_tau_one_is_dense_attention():
    shape = SMALL[0]
    ds = DeviceStep(shape, 5)
    H = shape.H
    ones = torch.ones(H, dtype=torch.float32, device="cuda")
    inf = torch.full((H,), float("inf"), dtype=torch.float32, device="cuda")
    out = ds.run(tau=ones, z=inf).cpu().numpy()
    st = ds.step
    assert np.all(st.selection.inter_cnt.cpu().numpy() == -(-st.Lc // 128))
    K = np.concatenate([oracle.widen(bits_of(st.Kc)), oracle.widen(ds.x.Kq)])
    V = np.concatenate([oracle.widen(bits_of(st.Vc)), oracle.widen(ds.x.Vq)])
    ref = _sdpa64(oracle.widen(ds.x.Q), K, V, 1 / math.sqrt(shape.d))
    assert_close(out, ref, "tau = 1 vs dense attention")


def test_tau_zero_keeps_one_block_per_row():
    shape = SMALL[0]
    ds = DeviceStep(shape, 6)
    zeros = torch.zeros(shape.H, dtype=torch.float32, device="cuda")
    ds.run(tau=zeros)
    torch.cuda.synchronize()
    assert np.all(ds.step.selection.inter_cnt.cpu().numpy() == 1)
    assert np.all(ds.step.selection.intra_cnt.cpu().numpy() == 1)


def test_linear_identity_is_dense_attention():
    H, d, Lq, Lc = 2, 128, 256, 256
    L = Lq + Lc
    x = synth.make_inputs(synth.StepShape("id", H=H, d=d, frames=1, F_tok=Lq, page_frames=1, page_tok=Lc,
                                          NP=1, Kp=1, r=L), 9)
    I = synth.f32_to_bf16(np.eye(L, dtype=np.float32))
    cfg = make_config(H, d, Lq, Lc, L)
    ws = hsa.workspace(cfg)
    out = torch.empty(Lq, H, d, dtype=torch.float32, device="cuda")
    Kc, Vc = to_dev(x.pages_k[0]), to_dev(x.pages_v[0])
    hsa.hsa_linear_attn(cfg, to_dev(x.Q), Kc, Vc, to_dev(x.Kq), to_dev(x.Vq), to_dev(I), to_dev(I), out, ws)
    torch.cuda.synchronize()
    K = np.concatenate([oracle.widen(x.pages_k[0]), oracle.widen(x.Kq)])
    V = np.concatenate([oracle.widen(x.pages_v[0]), oracle.widen(x.Vq)])
    assert_close(out.cpu().numpy(), _sdpa64(oracle.widen(x.Q), K, V, 1 / math.sqrt(d)), "E = F = I")


def test_per_head_projection_matrices():
    shape = SMALL[1]
    x = synth.make_inputs(shape, 12)
    H, r, L = shape.H, shape.r, shape.L
    E = synth.normal_bf16((H, r, L), 12, 901, sigma=1 / math.sqrt(r))
    F = synth.normal_bf16((H, r, L), 12, 902, sigma=1 / math.sqrt(r))
    Kc = oracle.gather_pages(x.pages_k, [0, 1])
    Vc = oracle.gather_pages(x.pages_v, [0, 1])
    cfg = make_config(H, shape.d, shape.Lq, shape.Lc, r)
    ws = hsa.workspace(cfg)
    out = torch.empty(shape.Lq, H, shape.d, dtype=torch.float32, device="cuda")
    hsa.hsa_linear_attn(cfg, to_dev(x.Q), to_dev(Kc), to_dev(Vc), to_dev(x.Kq), to_dev(x.Vq), to_dev(E), to_dev(F),
                        out, ws, ef_head_stride=r * L)
    torch.cuda.synchronize()
    EK, FV = oracle.linear_projection(E, F, Kc, x.Kq, Vc, x.Vq)
    assert_close(out.cpu().numpy(), oracle.linear_attention(x.Q, EK, FV), "per-head E, F")


@pytest.mark.parametrize("Lq,d,H", [(8, 64, 1), (64, 128, 2), (136, 128, 3)])
def test_no_history(Lq, d, H):
    """Lc = 0: no retrieved pages; the sparse branch runs over the chunk's own blocks."""
    shape = synth.StepShape("nohist", H=H, d=d, frames=1, F_tok=Lq, page_frames=1, page_tok=8, NP=1, Kp=1, r=64)
    x = synth.make_inputs(shape, 21)
    E = x.E[:, shape.page_tok:].copy()  # columns of the chunk only
    F = x.F[:, shape.page_tok:].copy()
    cfg = make_config(H, d, Lq, 0, 64)
    ws = hsa.workspace(cfg)
    sel = SelectionBuffers.empty(cfg)
    out = torch.empty(Lq, H, d, dtype=torch.float32, device="cuda")
    hsa.hsa_forward(cfg, to_dev(x.Q), None, None, to_dev(x.Kq), to_dev(x.Vq), torch.from_numpy(x.tau).cuda(),
                    torch.from_numpy(x.z).cuda(), to_dev(E), to_dev(F), out, ws, sel=sel)
    torch.cuda.synchronize()
    assert np.all(sel.inter_cnt.cpu().numpy() == 0)
    empty = np.zeros((0, H, d), dtype=np.uint16)
    ref = oracle.hsa_step(x.Q, empty, empty, x.Kq, x.Vq, x.tau, x.z, E, F)
    gq = selection_lists(sel.intra_idx.cpu().numpy(), sel.intra_cnt.cpu().numpy())
    check_selection(gq, ref["selection"].intra, ref["selection"].p_intra, x.tau, "intra")
    ref = oracle.hsa_step(x.Q, empty, empty, x.Kq, x.Vq, x.tau, x.z, E, F,
                          selection=oracle.Selection([[np.zeros(0, np.int64)] * -(-Lq // 128)] * H, gq, None, None))
    assert_close(out.cpu().numpy(), ref["out"], "Lc = 0")


@pytest.mark.parametrize("Lq,d,H", [(64, 128, 2), (64, 64, 3), (192, 128, 2)])
def test_fused_merge_short_lists(Lq, d, H):
    """Units with two or three key tiles (one linear tile, one or two chunk tiles): the
    fused output is repeatable and equals the gated merge of the two branches run
    alone.  With so few tiles the P.V product of the next-to-last tile can still be
    running when the softmax ends, so the epilogue must wait for both last products."""
    shape = synth.StepShape("short", H=H, d=d, frames=1, F_tok=Lq, page_frames=1, page_tok=8, NP=1, Kp=1, r=64)
    x = synth.make_inputs(shape, 21)
    E = to_dev(x.E[:, shape.page_tok:].copy())
    F = to_dev(x.F[:, shape.page_tok:].copy())
    cfg = make_config(H, d, Lq, 0, 64)
    ws = hsa.workspace(cfg)
    sel = SelectionBuffers.empty(cfg)
    Q, Kq, Vq = to_dev(x.Q), to_dev(x.Kq), to_dev(x.Vq)
    tau = torch.from_numpy(x.tau).cuda()
    z = torch.from_numpy(x.z).cuda()
    outs = []
    for _ in range(3):
        out = torch.empty(Lq, H, d, dtype=torch.float32, device="cuda")
        hsa.hsa_forward(cfg, Q, None, None, Kq, Vq, tau, z, E, F, out, ws, sel=sel)
        outs.append(out)
    o_s = torch.empty_like(outs[0])
    o_l = torch.empty_like(outs[0])
    hsa.hsa_sparse_attn(cfg, Q, None, None, Kq, Vq, sel, o_s, ws)
    hsa.hsa_linear_attn(cfg, Q, None, None, Kq, Vq, E, F, o_l, ws)
    torch.cuda.synchronize()
    assert hsa.hsa_status_read(ws) == 0
    for out in outs[1:]:
        assert torch.equal(out, outs[0])
    g = torch.sigmoid(z).view(1, H, 1)
    merged = g * o_s + (1 - g) * o_l
    assert float((outs[0] - merged).abs().max()) <= 1e-5


# ----------------------------------------------------------------- device-side status and argument checks

def test_device_status_short_candidate_range():
    shape = SMALL[0]
    ds = DeviceStep(shape, 3)
    st = ds.step
    hsa.hsa_status_clear(st.ws)
    rng = torch.tensor([2, 3], dtype=torch.int32, device="cuda")  # one page < Kp = 3
    hsa.hkv_select_pages(st.kbar_pages, ds.Q, shape.Kp, st.sel, st.ws, st.scores, rng)
    assert hsa.hsa_status_read(st.ws) == 6  # HSA_ERR_DEVICE
    assert np.all(st.sel.cpu().numpy() == -1)
    hsa.hsa_status_clear(st.ws)
    assert hsa.hsa_status_read(st.ws) == 0


def test_device_status_bad_page_id():
    shape = SMALL[0]
    ds = DeviceStep(shape, 4)
    st = ds.step
    hsa.hsa_status_clear(st.ws)
    bad = torch.tensor([0, 99, 1], dtype=torch.int32, device="cuda")
    hsa.hkv_gather(st.page_k_ptrs, st.page_v_ptrs, bad, shape.Kp, shape.P_tok, shape.H, shape.d, st.Kc, st.Vc,
                   st.ws, st.kbar128)
    assert hsa.hsa_status_read(st.ws) == 6
    # rows of valid slots were still copied
    assert np.array_equal(bits_of(st.Kc)[:shape.P_tok], ds.x.pages_k[0])


def test_invalid_arguments_launch_nothing():
    cfg = make_config(2, 128, 256, 256, 64)
    ws = hsa.workspace(cfg)
    Q = torch.zeros(256, 2, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(256, 2, 128, dtype=torch.float32, device="cuda")
    tau = torch.ones(2, device="cuda")
    E = torch.zeros(64, 512, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(hsa.HsaError) as e:  # misaligned pointer
        hsa.hsa_forward(cfg, Q[:, :, 1:], Q, Q, Q, Q, tau, tau, E, E, out, ws)
    assert e.value.code == 1
    with pytest.raises(hsa.HsaError) as e:  # workspace too small
        hsa.hsa_forward(cfg, Q, Q, Q, Q, Q, tau, tau, E, E, out, ws[:1024])
    assert e.value.code == 3
    with pytest.raises(hsa.HsaError) as e:  # unsupported head dim
        hsa.hsa_forward(make_config(2, 96, 256, 256, 64), Q, Q, Q, Q, Q, tau, tau, E, E, out, ws)
    assert e.value.code == 2
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0


def test_forward_split_lists_merge():
    """Lists much longer than the step's cost per SM are cut into segments whose
    partial results are merged in segment order: same output as the oracle, and the
    same bits on a second run."""
    shape = synth.StepShape("h2_d128_lq200_lc8192", H=2, d=128, frames=1, F_tok=200, page_frames=1,
                            page_tok=1024, NP=10, Kp=8, r=64)
    ds = DeviceStep(shape, 91)
    try:
        hsa.hsa_status_clear(ds.step.ws)
        ds.run()
        torch.cuda.synchronize()
        x, st = ds.x, ds.step
        first = st.out.clone()
        ds.run()
        torch.cuda.synchronize()
        assert torch.equal(first, st.out)
        Kc, Vc = bits_of(st.Kc), bits_of(st.Vc)
        sb = st.selection
        inter_cnt = sb.inter_cnt.cpu().numpy()
        assert inter_cnt[0].min() == Kc.shape[0] // 128  # tau = 1 keeps every cached block: long lists
        sel = oracle.Selection(selection_lists(sb.inter_idx.cpu().numpy(), inter_cnt),
                               selection_lists(sb.intra_idx.cpu().numpy(), sb.intra_cnt.cpu().numpy()), None, None)
        ref = oracle.hsa_step(x.Q, Kc, Vc, x.Kq, x.Vq, x.tau, x.z, x.E, x.F, selection=sel)
        assert_close(st.out.cpu().numpy(), ref["out"], "hsa_forward out (split lists)")
        assert hsa.hsa_status_read(ds.step.ws) == 0
    finally:
        ds.close()


# ----------------------------------------------------------------- bounded device waits

def test_bounded_wait_times_out_and_context_stays_usable():
    """A wait nothing completes gives up after the workspace's limit, records
    HSA_ERR_TIMEOUT, and the next launches on the same context run normally."""
    Lq, d, H = 64, 128, 2
    cfg = make_config(H, d, Lq, 0, 64)
    ws = hsa.workspace(cfg)
    hsa.hsa_set_wait_limit(ws, 3000)  # 3 ms
    waited = torch.zeros(1, dtype=torch.int64, device="cuda")
    hsa.hsa_selftest_wait(ws, waited)
    assert hsa.hsa_status_read(ws) == 5  # HSA_ERR_TIMEOUT
    ns = int(waited.item())
    assert 3_000_000 <= ns < 500_000_000, ns
    rep = hsa.wait_report(ws)  # the self-test's wait names site kind 0x7E, CTA 0
    assert rep["ran_out"] == 1 and rep["kind"] == 0x7E and rep["cta"] == 0, rep
    # the ran-out flag is now set: under a 1 s limit, the next wait gives up after
    # 50 us instead of running out on its own
    hsa.hsa_set_wait_limit(ws, 1_000_000)
    hsa.hsa_selftest_wait(ws, waited)
    assert hsa.hsa_status_read(ws) == 5
    ns = int(waited.item())
    assert ns < 100_000_000, ns
    # the context is usable: a fused forward under a generous limit completes with status 0
    hsa.hsa_status_clear(ws)
    rep = hsa.wait_report(ws)
    assert rep["status"] == 0 and rep["ran_out"] == 0 and rep["site"] == 0, rep
    hsa.hsa_set_wait_limit(ws, 200_000)  # 200 ms
    shape = synth.StepShape("wait", H=H, d=d, frames=1, F_tok=Lq, page_frames=1, page_tok=8, NP=1, Kp=1, r=64)
    x = synth.make_inputs(shape, 33)
    E = to_dev(x.E[:, shape.page_tok:].copy())
    F = to_dev(x.F[:, shape.page_tok:].copy())
    sel = SelectionBuffers.empty(cfg)
    Q, Kq, Vq = to_dev(x.Q), to_dev(x.Kq), to_dev(x.Vq)
    tau = torch.from_numpy(x.tau).cuda()
    z = torch.from_numpy(x.z).cuda()
    out = torch.empty(Lq, H, d, dtype=torch.float32, device="cuda")
    hsa.hsa_forward(cfg, Q, None, None, Kq, Vq, tau, z, E, F, out, ws, sel=sel)
    assert hsa.hsa_status_read(ws) == 0
    empty = np.zeros((0, H, d), dtype=np.uint16)
    gq = selection_lists(sel.intra_idx.cpu().numpy(), sel.intra_cnt.cpu().numpy())
    ref = oracle.hsa_step(x.Q, empty, empty, x.Kq, x.Vq, x.tau, x.z, x.E[:, shape.page_tok:], x.F[:, shape.page_tok:],
                          selection=oracle.Selection([[np.zeros(0, np.int64)]] * H, gq, None, None))
    assert_close(out.cpu().numpy(), ref["out"], "forward after a timeout")
    hsa.hsa_set_wait_limit(ws, 0)  # back to the default
    hsa.hsa_selftest_wait(ws)  # default limit 2 s: still a timeout, bounded
    assert hsa.hsa_status_read(ws) == 5


# ----------------------------------------------------------------- multi-step reuse

@pytest.mark.parametrize("shape", SMALL, ids=_ids)
def test_multi_step_reuse(shape):
    """Retrieval, gather and the history's Linformer products once per chunk; three
    denoising steps with fresh chunk tensors.  Each step equals hsa_forward on the same
    inputs (same selections, outputs within fp32 summation-order differences) and the
    oracle's HSA step within the tolerance."""
    ds = DeviceStep(shape, 55)
    try:
        st, x = ds.step, ds.x
        st.prepare_chunk(ds.Q, ds.E, ds.F)
        Kc, Vc = bits_of(st.Kc), bits_of(st.Vc)
        Lq, H, d = shape.Lq, shape.H, shape.d
        for k in range(3):
            Qb = synth.normal_bf16((Lq, H, d), 600 + k, 1)
            Kqb = synth.normal_bf16((Lq, H, d), 600 + k, 2)
            Vqb = synth.normal_bf16((Lq, H, d), 600 + k, 3)
            Q, Kq, Vq = to_dev(Qb), to_dev(Kqb), to_dev(Vqb)
            out_r = st.denoise_step(Q, Kq, Vq, ds.tau, ds.z, ds.E, ds.F, out=torch.empty_like(st.out))
            sel_f = SelectionBuffers.empty(st.cfg)
            out_f = torch.empty_like(st.out)
            hsa.hsa_forward(st.cfg, Q, st.Kc, st.Vc, Kq, Vq, ds.tau, ds.z, ds.E, ds.F, out_f, st.ws, st.kbar128,
                            sel=sel_f)
            torch.cuda.synchronize()
            sb = st.selection
            for a, b in ((sb.inter_cnt, sel_f.inter_cnt), (sb.intra_cnt, sel_f.intra_cnt)):
                assert torch.equal(a, b)
            assert float((out_r - out_f).abs().max()) <= 1e-4
            sel = oracle.Selection(selection_lists(sb.inter_idx.cpu().numpy(), sb.inter_cnt.cpu().numpy()),
                                   selection_lists(sb.intra_idx.cpu().numpy(), sb.intra_cnt.cpu().numpy()), None, None)
            ref = oracle.hsa_step(Qb, Kc, Vc, Kqb, Vqb, x.tau, x.z, x.E, x.F, selection=sel)
            assert_close(out_r.cpu().numpy(), ref["out"], f"denoising step {k}")
        assert hsa.hsa_status_read(st.ws) == 0
    finally:
        ds.close()


# ----------------------------------------------------------------- retrieval policies

def test_retrieval_policies_match_the_oracle():
    """Page-only, prompt-only (recent pages of a candidate range), recent-page (sliding
    window) and random-page retrieval: the GPU's page ids equal the oracle's exactly."""
    H, d, Lq, NP, Kp = 4, 128, 520, 16, 4
    kbar = torch.from_numpy(synth.normal_f32((NP, H, d), 71, 1, sigma=0.5)).cuda()
    Qb = synth.normal_bf16((Lq, H, d), 71, 2)
    Q = to_dev(Qb)
    keys = synth.normal_f32((NP,), 71, 3)
    keys[5] = keys[9]  # a tie: the lower page id ranks first
    cfg = make_config(H, d, Lq, 0, 64)
    ws = hsa.workspace(cfg)
    kb = kbar.cpu().numpy()
    for cand in (None, (3, 11)):
        rng_t = None if cand is None else torch.tensor(cand, dtype=torch.int32, device="cuda")
        cl = None if cand is None else range(*cand)
        for pol, name in ((hsa.POLICY_SCORE, "score"), (hsa.POLICY_RECENT, "recent"), (hsa.POLICY_RANDOM, "random")):
            sel = torch.full((Kp,), -7, dtype=torch.int32, device="cuda")
            sc = torch.zeros(NP, dtype=torch.float32, device="cuda")
            hsa.hkv_select_pages_policy(pol, kbar, Q, Kp, sel, ws, sc, rng_t, torch.from_numpy(keys).cuda())
            torch.cuda.synchronize()
            want = oracle.select_pages_policy(name, kb, Qb, Kp, cand=cl, rand_keys=keys)
            if name == "score":
                _, scores = oracle.select_pages(kb, Qb, Kp, cl)
                check_pages(sel.cpu().numpy(), want, scores, Kp)
            else:
                assert sel.cpu().tolist() == want.tolist(), (name, cand)
    assert hsa.hsa_status_read(ws) == 0


# ----------------------------------------------------------------- head-sharded step

def test_head_groups_emulated_on_one_gpu():
    """The step of two head groups, one after the other on one GPU (no group waits for
    another): the partial page scores of the groups, added, select the pages the
    unsharded retrieval selects; each group's output equals the unsharded output of
    its heads."""
    from hybrid_sparse_attention_hkv_b200.sharded import head_range
    from hybrid_sparse_attention_hkv_b200.step import HkvHsaStep, page_pointers
    shape = SMALL[2]
    ds = DeviceStep(shape, 81)
    x, st = ds.x, ds.step
    H, Kp, NP = shape.H, shape.Kp, shape.NP
    full_out = ds.run().clone()
    torch.cuda.synchronize()
    total = torch.zeros(NP, dtype=torch.float32, device="cuda")
    groups = [head_range(H, r, 2) for r in range(2)]
    steps = []
    for h0, h1 in groups:
        pk = to_dev(np.ascontiguousarray(x.pages_k[:, :, h0:h1]))
        pv = to_dev(np.ascontiguousarray(x.pages_v[:, :, h0:h1]))
        g = HkvHsaStep(h1 - h0, shape.d, shape.Lq, shape.P_tok, NP, Kp, shape.r, page_pointers(pk),
                       page_pointers(pv))
        g.seal_pages(pk)
        Qg = to_dev(np.ascontiguousarray(x.Q[:, h0:h1]))
        hsa.hkv_page_scores(g.kbar_pages, Qg, g.scores, g.ws)
        total += g.scores
        steps.append((g, pk, pv, Qg))
    sel = torch.zeros(Kp, dtype=torch.int32, device="cuda")
    hsa.hkv_select_top(total, Kp, sel, steps[0][0].ws)
    torch.cuda.synchronize()
    check_pages(sel.cpu().numpy(), st.sel.cpu().numpy(), st.scores.cpu().numpy(), Kp)
    assert sel.cpu().tolist() == st.sel.cpu().tolist()
    for (h0, h1), (g, pk, pv, Qg) in zip(groups, steps):
        sl = slice(h0, h1)
        g.sel.copy_(sel)
        hsa.hkv_gather(g.page_k_ptrs, g.page_v_ptrs, g.sel, Kp, shape.P_tok, h1 - h0, shape.d, g.Kc, g.Vc, g.ws,
                       g.kbar128)
        hsa.hsa_forward(g.cfg, Qg, g.Kc, g.Vc, to_dev(np.ascontiguousarray(x.Kq[:, sl])),
                        to_dev(np.ascontiguousarray(x.Vq[:, sl])), ds.tau[sl].contiguous(), ds.z[sl].contiguous(),
                        ds.E, ds.F, g.out, g.ws, g.kbar128, g.selection)
        torch.cuda.synchronize()
        assert torch.equal(g.selection.inter_cnt, st.selection.inter_cnt[sl])
        assert torch.equal(g.selection.intra_cnt, st.selection.intra_cnt[sl])
        assert float((g.out - full_out[:, sl]).abs().max()) <= 1e-4


# ----------------------------------------------------------------- fidelity diagnostic

def test_fidelity_report_matches_the_oracle(small):
    """Per-head cosine and relative error of both branches against dense attention and
    the kept dense mass (through the kernel's log-sum-exp), against the oracle's
    definitions; and the lse of dense attention equals a library log-sum-exp."""
    x, st, shape = small.x, small.step, small.shape
    rep = hsa.fidelity_report(st.cfg, small.Q, st.Kc, st.Vc, small.Kq, small.Vq, small.E, small.F, st.selection,
                              st.ws).cpu().numpy()
    Kc, Vc = bits_of(st.Kc), bits_of(st.Vc)
    sb = st.selection
    inter = selection_lists(sb.inter_idx.cpu().numpy(), sb.inter_cnt.cpu().numpy())
    intra = selection_lists(sb.intra_idx.cpu().numpy(), sb.intra_cnt.cpu().numpy())
    EK, FV = oracle.linear_projection(x.E, x.F, Kc, x.Kq, Vc, x.Vq)
    ref = oracle.fidelity(x.Q, Kc, Vc, x.Kq, x.Vq, inter, intra, EK, FV)
    np.testing.assert_allclose(rep[:, [0, 1, 2]], ref[:, [0, 1, 2]], atol=2e-3)
    np.testing.assert_allclose(rep[:, [3, 4]], ref[:, [3, 4]], atol=5e-3, rtol=5e-2)
    # the dense log-sum-exp itself
    dense = SelectionBuffers.empty(st.cfg)
    hsa.hsa_block_select(st.cfg, small.Q, st.Kc, small.Kq, torch.ones(shape.H, device="cuda"), dense, st.ws)
    o = torch.empty_like(st.out)
    lse = torch.empty(shape.Lq, shape.H, dtype=torch.float32, device="cuda")
    hsa.hsa_sparse_attn_lse(st.cfg, small.Q, st.Kc, st.Vc, small.Kq, small.Vq, dense, o, lse, st.ws)
    torch.cuda.synchronize()
    K = torch.from_numpy(np.concatenate([oracle.widen(Kc), oracle.widen(x.Kq)]))
    s = torch.einsum("thc,khc->htk", torch.from_numpy(oracle.widen(x.Q)), K) / math.sqrt(shape.d)
    want = torch.logsumexp(s, dim=2).T.numpy()
    np.testing.assert_allclose(lse.cpu().numpy(), want, atol=2e-3)


def test_block_means_from_page_sums():
    """64-row key sums kept per page give the active cache's 128-row block means without
    the gathered copy: equal to the oracle's block means of the gathered cache."""
    shape = SMALL[2]  # pages of 384 rows
    ds = DeviceStep(shape, 19)
    x, st = ds.x, ds.step
    assert st.early
    ds.run()
    torch.cuda.synchronize()
    for p in range(shape.NP):
        want = oracle.block_means(x.pages_k[p], 64) * 64
        np.testing.assert_allclose(st.sums64[p].cpu().numpy(), want, rtol=1e-5, atol=1e-4)
    Kc = oracle.gather_pages(x.pages_k, st.sel.cpu().numpy())
    np.testing.assert_allclose(st.kbar128.cpu().numpy(), oracle.block_means(Kc, 128), rtol=1e-5, atol=1e-6)
    assert np.array_equal(bits_of(st.Kc), Kc)
    assert hsa.hsa_status_read(st.ws) == 0


# ----------------------------------------------------------------- joint block selection

def test_joint_selection_and_output(small):
    """HSA_SELECT_JOINT: one softmax per 64-row query block over its cached and chunk
    blocks.  The GPU's kept blocks (inter and intra together) equal the oracle's, with
    the same exemptions, and the output equals the oracle's HSA step on that selection
    (inter lists per 64-row query block)."""
    x, st, shape = small.x, small.step, small.shape
    cfg = make_config(shape.H, shape.d, shape.Lq, shape.Lc, shape.r, select_mode=hsa.SELECT_JOINT)
    sel = SelectionBuffers.empty(cfg)
    out = torch.empty_like(st.out)
    hsa.hsa_forward(cfg, small.Q, st.Kc, st.Vc, small.Kq, small.Vq, small.tau, small.z, small.E, small.F, out, st.ws,
                    st.kbar128, sel=sel)
    torch.cuda.synchronize()
    assert hsa.hsa_status_read(st.ws) == 0
    Kc, Vc = bits_of(st.Kc), bits_of(st.Vc)
    nKc = -(-shape.Lc // 128)
    gi = selection_lists(sel.inter_idx.cpu().numpy(), sel.inter_cnt.cpu().numpy())
    gq = selection_lists(sel.intra_idx.cpu().numpy(), sel.intra_cnt.cpu().numpy())
    assert len(gi[0]) == -(-shape.Lq // 64)
    combined = [[np.concatenate([gi[h][i], gq[h][i] + nKc]) for i in range(len(gi[h]))] for h in range(shape.H)]
    for dt in (np.float32, np.float64):
        ref = oracle.block_select(x.Q, Kc, x.Kq, x.tau, dtype=dt, joint=True)
        ref_c = [[np.concatenate([ref.inter[h][i], ref.intra[h][i] + nKc]) for i in range(len(ref.inter[h]))]
                 for h in range(shape.H)]
        n, e = check_selection(combined, ref_c, ref.p_inter, x.tau, f"joint {dt.__name__}")
        assert e <= max(1, n // 100)
    res = oracle.hsa_step(x.Q, Kc, Vc, x.Kq, x.Vq, x.tau, x.z, x.E, x.F, joint=True,
                          selection=oracle.Selection(gi, gq, None, None))
    assert_close(out.cpu().numpy(), res["out"], "joint selection output")


def test_gather_project_equals_gather_then_projection():
    """One pass over the selected pages: the same Kc / Vc bits as hkv_gather, and
    denoising steps on its history products equal to hsa_forward on the full KV."""
    shape = SMALL[2]  # pages of 384 rows (a multiple of 64)
    ds = DeviceStep(shape, 23)
    x, st = ds.x, ds.step
    hsa.hkv_select_pages(st.kbar_pages, ds.Q, shape.Kp, st.sel, st.ws, st.scores)
    hsa.hkv_gather_project(st.cfg, st.page_k_ptrs, st.page_v_ptrs, st.sel, shape.Kp, shape.P_tok, ds.E, ds.F,
                           st.Kc, st.Vc, st.ws)
    torch.cuda.synchronize()
    sel = st.sel.cpu().numpy()
    assert np.array_equal(bits_of(st.Kc), oracle.gather_pages(x.pages_k, sel))
    assert np.array_equal(bits_of(st.Vc), oracle.gather_pages(x.pages_v, sel))
    out_r = torch.empty_like(st.out)
    hsa.hsa_forward_reuse(st.cfg, ds.Q, st.Kc, st.Vc, ds.Kq, ds.Vq, ds.tau, ds.z, ds.E, ds.F, out_r, st.ws,
                          sel=st.selection)
    out_f = torch.empty_like(st.out)
    sel_f = SelectionBuffers.empty(st.cfg)
    hsa.hsa_forward(st.cfg, ds.Q, st.Kc, st.Vc, ds.Kq, ds.Vq, ds.tau, ds.z, ds.E, ds.F, out_f, st.ws, sel=sel_f)
    torch.cuda.synchronize()
    assert float((out_r - out_f).abs().max()) <= 1e-4
    assert hsa.hsa_status_read(st.ws) == 0


def test_thread_release_and_recreate():
    """hsa_thread_release destroys the side stream and events hsa_forward keeps for the
    thread; the next hsa_forward creates them again and gives the same output."""
    shape = SMALL[0]
    ds = DeviceStep(shape, 13)
    first = ds.run().clone()
    torch.cuda.synchronize()
    hsa.hsa_thread_release()
    hsa.hsa_thread_release()  # nothing left to release: still fine
    second = ds.run().clone()
    torch.cuda.synchronize()
    assert torch.equal(first, second)
    assert hsa.hsa_status_read(ds.step.ws) == 0


@pytest.mark.parametrize("nKc", [300, 1000, 2000, 3000, 4200])
def test_block_selection_row_lengths(nKc):
    """Selection rows of every length the ranking takes (register networks of 256 to
    4096 keys, and the shared-memory passes beyond) against the oracle."""
    H, d, Lq = 2, 64, 128
    Lc = nKc * 128 - 40  # a partial last block
    Lc -= Lc % 8
    cfg = make_config(H, d, Lq, Lc, 0)
    g = torch.Generator(device="cuda").manual_seed(nKc)
    Q = torch.randn(Lq, H, d, device="cuda", generator=g).to(torch.bfloat16)
    Kc = torch.randn(Lc, H, d, device="cuda", generator=g).to(torch.bfloat16)
    Kq = torch.randn(Lq, H, d, device="cuda", generator=g).to(torch.bfloat16)
    tau = torch.tensor([0.5, 0.8], dtype=torch.float32, device="cuda")
    sel = SelectionBuffers.empty(cfg)
    ws = hsa.workspace(cfg)
    hsa.hsa_block_select(cfg, Q, Kc, Kq, tau, sel, ws)
    torch.cuda.synchronize()
    assert hsa.hsa_status_read(ws) == 0
    gi = selection_lists(sel.inter_idx.cpu().numpy(), sel.inter_cnt.cpu().numpy())
    gq = selection_lists(sel.intra_idx.cpu().numpy(), sel.intra_cnt.cpu().numpy())
    check_selection_both(gi, gq, bits_of(Q), bits_of(Kc), bits_of(Kq), tau.cpu().numpy(), f"nKc {nKc}")


@pytest.mark.parametrize("joint", [False, True], ids=["separate", "joint"])
def test_block_selection_longest_rows(joint):
    """The longest selection rows the boundary accepts: 8192 cached blocks (the per-row
    maximum of a separate map), and in joint mode those plus the chunk's blocks in one
    row (16384 sort slots, the block-wide ranking), against the oracle."""
    H, d, Lq = 2, 64, 128
    nKc = 8192
    Lc = nKc * 128 - 40
    Lc -= Lc % 8
    cfg = make_config(H, d, Lq, Lc, 0, select_mode=hsa.SELECT_JOINT if joint else hsa.SELECT_SEPARATE)
    g = torch.Generator(device="cuda").manual_seed(8192 + joint)
    Q = torch.randn(Lq, H, d, device="cuda", generator=g).to(torch.bfloat16)
    Kc = torch.randn(Lc, H, d, device="cuda", generator=g).to(torch.bfloat16)
    Kq = torch.randn(Lq, H, d, device="cuda", generator=g).to(torch.bfloat16)
    tau = torch.tensor([0.5, 0.8], dtype=torch.float32, device="cuda")
    sel = SelectionBuffers.empty(cfg)
    ws = hsa.workspace(cfg)
    hsa.hsa_block_select(cfg, Q, Kc, Kq, tau, sel, ws)
    torch.cuda.synchronize()
    assert hsa.hsa_status_read(ws) == 0
    gi = selection_lists(sel.inter_idx.cpu().numpy(), sel.inter_cnt.cpu().numpy())
    gq = selection_lists(sel.intra_idx.cpu().numpy(), sel.intra_cnt.cpu().numpy())
    Qh, Kch, Kqh, t = bits_of(Q), bits_of(Kc), bits_of(Kq), tau.cpu().numpy()
    del Kc
    if not joint:
        check_selection_both(gi, gq, Qh, Kch, Kqh, t, "longest rows")
        return
    assert len(gi[0]) == Lq // 64
    combined = [[np.concatenate([gi[h][i], gq[h][i] + nKc]) for i in range(len(gi[h]))] for h in range(H)]
    for dt in (np.float32, np.float64):
        ref = oracle.block_select(Qh, Kch, Kqh, t, dtype=dt, joint=True)
        ref_c = [[np.concatenate([ref.inter[h][i], ref.intra[h][i] + nKc]) for i in range(len(ref.inter[h]))]
                 for h in range(H)]
        n, e = check_selection(combined, ref_c, ref.p_inter, t, f"longest joint rows {dt.__name__}")
        assert e <= max(1, n // 100)
