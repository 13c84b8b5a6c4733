"""The C-ABI library loads on a machine without a GPU, exports every entry point
include/hsa.h declares, and rejects bad arguments on the host before any launch
(none of these calls reach the CUDA runtime)."""
import ctypes
import os
import re

import pytest

import hybrid_sparse_attention_hkv_b200 as hsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "hsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b((?:hsa|hkv)_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from hybrid_sparse_attention_hkv_b200 import build
    build.build()
    return hsa.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 16
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(hsa.EXPORTED)


def test_status_strings(lib):
    for code, name in hsa.HSA_STATUS.items():
        assert lib.hsa_status_string(code).decode() == name


def test_workspace_size_and_shape_checks(lib):
    small = hsa.hsa_workspace_size(hsa.make_config(2, 64, 256, 512, 64))
    big = hsa.hsa_workspace_size(hsa.make_config(12, 128, 4680, 49920, 256))
    assert 0 < small < big
    assert big % 256 == 0
    cases = [
        (hsa.make_config(2, 96, 256, 512, 64), 2),              # head dim
        (hsa.make_config(0, 64, 256, 512, 64), 1),              # heads
        (hsa.make_config(2, 64, 0, 512, 64), 1),                # empty chunk
        (hsa.make_config(2, 64, 257, 512, 64), 2),              # Lq not a multiple of 8
        (hsa.make_config(2, 64, 260, 500, 64), 2),              # Lc, Lq not multiples of 8 (sum is)
        (hsa.make_config(2, 64, 256, -8, 64), 1),               # negative history
        (hsa.make_config(2, 64, 256, 512, 64, block_inter=64), 2),
        (hsa.make_config(2, 64, 256, 512, 64, scale=float("nan")), 1),
    ]
    for cfg, code in cases:
        with pytest.raises(hsa.HsaError) as e:
            hsa.hsa_workspace_size(cfg)
        assert e.value.code == code, (cfg.H, cfg.d, cfg.Lq, cfg.Lc)


def test_null_and_misaligned_pointers_rejected(lib):
    cfg = hsa.make_config(2, 64, 256, 512, 64)
    P = ctypes.c_void_p
    aligned = P(0x10000)
    mis = P(0x10002)
    ws = P(0x100000)
    # hsa_forward with a NULL query
    code = lib.hsa_forward(ctypes.byref(cfg), None, aligned, aligned, aligned, aligned, None, aligned, aligned,
                           aligned, aligned, 0, aligned, 0, None, ws, 1 << 30, None)
    assert code == 1 and b"Q is NULL" in lib.hsa_last_error_detail()
    # misaligned key pointer
    code = lib.hsa_forward(ctypes.byref(cfg), aligned, mis, aligned, aligned, aligned, None, aligned, aligned,
                           aligned, aligned, 0, aligned, 0, None, ws, 1 << 30, None)
    assert code == 1 and b"16-byte" in lib.hsa_last_error_detail()
    # too small a workspace
    code = lib.hsa_forward(ctypes.byref(cfg), aligned, aligned, aligned, aligned, aligned, None, aligned, aligned,
                           aligned, aligned, 0, aligned, 0, None, ws, 1024, None)
    assert code == 3
    # rank not supported
    cfg2 = hsa.make_config(2, 64, 256, 512, 96)
    code = lib.hsa_linear_attn(ctypes.byref(cfg2), aligned, aligned, aligned, aligned, aligned, aligned, aligned, 0,
                               aligned, ws, 1 << 30, None)
    assert code == 2
    # Kp out of range for the page calls
    code = lib.hkv_select_pages(aligned, 4, None, aligned, 256, 2, 64, 5, aligned, None, ws, 1 << 30, None)
    assert code == 1
    code = lib.hkv_gather(aligned, aligned, 4, aligned, 0, 256, 2, 64, aligned, aligned, None, ws, 1 << 30, None)
    assert code == 1


def test_injected_faults_fail_before_any_launch(lib):
    """Host-side fault injection: each kind fails its check with its code and an
    "injected" detail, before anything is launched; setting it back restores the
    ordinary checks; the kind belongs to the calling thread."""
    import threading
    cfg = hsa.make_config(2, 64, 256, 512, 64)
    P = ctypes.c_void_p
    a = P(0x10000)
    ws = P(0x100000)
    sel = hsa._Selection(0x20000, 0x30000, 0x40000, 0x50000)

    def block_select(ws_bytes):
        return lib.hsa_block_select(ctypes.byref(cfg), a, a, a, None, a, sel, ws, ws_bytes, None)

    def detail():
        return lib.hsa_last_error_detail().decode()

    with hsa.injected_fault(hsa.FAULT_ARG):
        with pytest.raises(hsa.HsaError) as e:
            hsa.hsa_workspace_size(cfg)
        assert e.value.code == 1 and "injected" in str(e.value)
    with hsa.injected_fault(hsa.FAULT_WORKSPACE):
        assert block_select(1 << 30) == 3 and "injected workspace" in detail()
    with hsa.injected_fault(hsa.FAULT_LAUNCH):
        # every check passes; the first launch (the pooling) fails before it is made
        assert block_select(1 << 30) == 4 and "pool: injected launch" in detail()
        code = lib.hkv_select_pages_noalloc(a, 4, None, a, 256, 2, 64, 2, a, None, None, None)
        assert code == 4 and "injected launch" in detail()
    # back to the ordinary checks
    assert hsa.hsa_workspace_size(cfg) > 0
    assert block_select(1024) == 3 and "injected" not in detail()
    with pytest.raises(hsa.HsaError) as e:
        hsa.hsa_inject_fault(7)
    assert e.value.code == 1
    # another thread's fault does not reach this one
    seen = {}

    def other():
        with hsa.injected_fault(hsa.FAULT_ARG):
            try:
                hsa.hsa_workspace_size(cfg)
                seen["other"] = 0
            except hsa.HsaError as err:
                seen["other"] = err.code

    t = threading.Thread(target=other)
    t.start()
    t.join()
    assert seen["other"] == 1
    assert hsa.hsa_workspace_size(cfg) > 0


def test_product_path_never_imports_the_oracle():
    """The package and its native sources carry no reference to the oracle."""
    pkg = os.path.join(ROOT, "hybrid_sparse_attention_hkv_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f


def test_missing_library_fails_loudly(tmp_path):
    import importlib
    mod = importlib.reload(hsa)
    saved = mod._lib
    mod._lib = None
    try:
        with pytest.raises(ImportError):
            mod.load_library(str(tmp_path / "nope.so"))
    finally:
        mod._lib = saved
