"""hkv_select_pages_noalloc: page-level retrieval without a caller workspace.

For callers that may not allocate device memory (a framework that owns every
device buffer, a runtime with a fixed memory plan, a loop where an allocation
could stall the device).  The entry point is called through the C ABI and its
output is checked against the workspace-based hkv_select_pages on two calls in a
row (the second with other queries and a candidate range), within the tolerance
the other page-selection tests use.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _c_call(lib, kbar, Q, Kp, sel, scores, cand, status):
    NP = kbar.shape[0]
    Lq, H, d = Q.shape
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return lib.hkv_select_pages_noalloc(p(kbar), NP, p(cand), p(Q), Lq, H, d, Kp, p(sel), p(scores), p(status),
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_page_selection_matches_workspace_version():
    import hybrid_sparse_attention_hkv_b200 as hsa
    from synth.device import to_dev
    lib = hsa.load_library()
    H, d, Lq, NP, Kp = 12, 128, 4680, 16, 4
    cfg = hsa.make_config(H, d, Lq, 49920, 256)
    ws = hsa.workspace(cfg)
    kbar = torch.from_numpy(synth.normal_f32((NP, H, d), 5, 77, sigma=0.5)).cuda()
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    cases = [(to_dev(synth.normal_bf16((Lq, H, d), 5, 78)), None),
             (to_dev(synth.normal_bf16((Lq, H, d), 6, 79, offset=synth.normal_f32((H, d), 6, 80))),
              torch.tensor([3, 11], dtype=torch.int32, device="cuda"))]
    for Q, cand in cases:  # two calls in a row
        sel_a = torch.full((Kp,), -7, dtype=torch.int32, device="cuda")
        sel_b = torch.full((Kp,), -7, dtype=torch.int32, device="cuda")
        sc_a = torch.zeros(NP, dtype=torch.float32, device="cuda")
        sc_b = torch.zeros(NP, dtype=torch.float32, device="cuda")
        hsa.hkv_select_pages(kbar, Q, Kp, sel_a, ws, sc_a, cand)
        assert _c_call(lib, kbar, Q, Kp, sel_b, sc_b, cand, status) == 0, lib.hsa_last_error_detail()
        torch.cuda.synchronize()
        assert status.item() == 0
        assert torch.equal(sel_a, sel_b)
        a, b = sc_a.cpu().numpy(), sc_b.cpu().numpy()
        fin = np.isfinite(a)
        assert np.array_equal(fin, np.isfinite(b))
        np.testing.assert_allclose(b[fin], a[fin], rtol=1e-5, atol=1e-5 * np.abs(a[fin]).max())
        if cand is not None:
            s = sel_b.cpu().numpy()
            assert np.all((s >= 3) & (s < 11)) and np.all(np.diff(s) > 0)


def test_noalloc_rejects_sizes_beyond_the_static_maximum():
    """The static scratch holds the partial page scores of at most 2048 pages; one page
    more is rejected on the host with a clear error and nothing is launched."""
    import hybrid_sparse_attention_hkv_b200 as hsa
    lib = hsa.load_library()
    H, d, NP = 40, 128, 2049  # NP <= H * d, so only the static maximum rejects it
    Q = torch.zeros(8, H, d, dtype=torch.bfloat16, device="cuda")
    kbar = torch.zeros(NP, H, d, dtype=torch.float32, device="cuda")
    sel = torch.full((2,), -7, dtype=torch.int32, device="cuda")
    assert _c_call(lib, kbar, Q, 2, sel, None, None, None) == 2
    assert b"static maximum" in lib.hsa_last_error_detail()
    torch.cuda.synchronize()
    assert torch.all(sel == -7)
    # the largest page count it serves still runs
    kbar = kbar[:2048].contiguous()
    assert _c_call(lib, kbar, Q, 2, sel, None, None, None) == 0, lib.hsa_last_error_detail()
    torch.cuda.synchronize()
    assert sel.cpu().tolist() == [0, 1]  # all scores tie at 0: the lowest page ids
