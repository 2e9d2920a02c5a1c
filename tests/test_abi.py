"""Host-side checks of the C ABI: the library loads, exports every entry point
the header declares, and rejects bad arguments before touching a GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

import self_referential_nested_b200 as S
from srnl_inputs import CONFIGS, make_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "srnl_scan.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"SRNL_API\s+[\w\s\*]+?\b(srnl_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from self_referential_nested_b200 import build
    build.build()
    return S.load_library()


def test_header_declares_the_bound_names():
    assert set(_declared()) == set(S.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings(lib):
    assert S.srnl_status_string(0) == "SRNL_OK"
    assert S.srnl_status_string(-1) == "SRNL_E_INVAL"
    assert S.srnl_status_string(-2) == "SRNL_E_UNSUPPORTED"
    assert S.srnl_status_string(-5) == "SRNL_E_TIMEOUT"
    assert S.srnl_status_string(7) == "SRNL_E_UNKNOWN"


def _cfg_dict(cfg, **kw):
    d = dict(B=cfg.B, H=cfg.H, W=cfg.W, C=cfg.C, heads=cfg.heads, d=cfg.d, alpha=cfg.alpha,
             eps=cfg.eps, chunk_row=cfg.chunk_row, chunk_col=cfg.chunk_col,
             act_dtype=cfg.act_dtype, gen_dtype=cfg.act_dtype)
    d.update(kw)
    return d


@pytest.mark.parametrize("bad,status", [
    (dict(B=0), S.SRNL_E_INVAL),
    (dict(H=-1), S.SRNL_E_INVAL),
    (dict(C=63), S.SRNL_E_INVAL),
    (dict(alpha=1.0), S.SRNL_E_INVAL),
    (dict(alpha=0.0), S.SRNL_E_INVAL),
    (dict(eps=0.0), S.SRNL_E_INVAL),
    (dict(eps=float("inf")), S.SRNL_E_INVAL),
    (dict(chunk_row=-2), S.SRNL_E_INVAL),
    (dict(act_dtype=7), S.SRNL_E_INVAL),
    (dict(C=256, heads=2, d=128), S.SRNL_E_UNSUPPORTED),
    (dict(C=24, heads=2, d=12), S.SRNL_E_UNSUPPORTED),
])
def test_create_rejects_bad_config_before_cuda(lib, bad, status):
    inp = make_inputs(CONFIGS["pr1_8x8"])
    with pytest.raises(S.SrnlError) as ei:
        S.srnl_scan_create(_cfg_dict(inp.cfg, **bad), inp.params())
    assert ei.value.status == status
    assert S.srnl_scan_last_error(None)


def test_create_rejects_null_params(lib):
    cfg = S._Config(B=1, H=2, W=2, C=32, heads=1, d=32, alpha=0.9, eps=1e-6)
    p = S._Params()
    h = ctypes.c_void_p()
    st = lib.srnl_scan_create(ctypes.byref(h), ctypes.byref(cfg), ctypes.byref(p))
    assert st == S.SRNL_E_INVAL and h.value is None
    assert b"NULL" in lib.srnl_scan_last_error(None)


def test_null_handle_calls_fail_cleanly(lib):
    assert lib.srnl_scan_forward(None, None, None, None, None) == S.SRNL_E_INVAL
    assert lib.srnl_scan_forward_host(None, None, None, None) == S.SRNL_E_INVAL
    assert lib.srnl_scan_route_index(None, 0, None, None) == S.SRNL_E_INVAL
    assert lib.srnl_scan_gather(None, 0, None, None, None) == S.SRNL_E_INVAL
    assert lib.srnl_scan_workspace_bytes(None) == 0
    lib.srnl_scan_destroy(None)  # accepted


def test_product_package_never_imports_oracle():
    pkg = os.path.join(ROOT, "self_referential_nested_b200")
    pat = re.compile(r"^\s*(import|from)\s+oracle\b|srnl_oracle", re.M)
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f), errors="ignore").read()
                assert not pat.search(src), f


# ------------------------------------------------ standalone sequence layer
def _seq_cfg(**kw):
    c = dict(B=2, T=257, D=64, heads=2, d=32, alpha=0.95, eps=1e-6, chunk=0, act_dtype="f32", gen_dtype="f32")
    c.update(kw)
    return c


@pytest.mark.parametrize("bad,status", [
    (dict(B=0), S.SRNL_E_INVAL),
    (dict(T=-1), S.SRNL_E_INVAL),
    (dict(D=63), S.SRNL_E_INVAL),
    (dict(alpha=1.0), S.SRNL_E_INVAL),
    (dict(eps=0.0), S.SRNL_E_INVAL),
    (dict(chunk=-1), S.SRNL_E_INVAL),
    (dict(gen_dtype=5), S.SRNL_E_INVAL),
    (dict(D=256, heads=2, d=128), S.SRNL_E_UNSUPPORTED),
])
def test_seq_create_rejects_bad_config_before_cuda(lib, bad, status):
    from srnl_inputs import make_seq_inputs
    inp = make_seq_inputs(1, 4, 64, 2)
    with pytest.raises(S.SrnlError) as e:
        S.srnl_seq_create(_seq_cfg(**bad), inp.params())
    assert e.value.status == status


def test_seq_null_handle_calls_fail_cleanly(lib):
    assert lib.srnl_seq_forward(None, None, None, None, None, None) == S.SRNL_E_INVAL
    assert lib.srnl_seq_device_status(None) == S.SRNL_E_INVAL
    lib.srnl_seq_destroy(None)
    assert isinstance(lib.srnl_seq_last_error(None), bytes)


def test_create_rejects_bad_injection_cap(lib):
    inp = make_inputs(CONFIGS["pr1_8x8"])
    with pytest.raises(S.SrnlError) as e:
        S.srnl_scan_create(_cfg_dict(inp.cfg, injection_cap=3), inp.params())
    assert e.value.status == S.SRNL_E_INVAL
    from srnl_inputs import make_seq_inputs
    sinp = make_seq_inputs(1, 4, 64, 2)
    with pytest.raises(S.SrnlError) as e:
        S.srnl_seq_create(_seq_cfg(injection_cap=-1), sinp.params())
    assert e.value.status == S.SRNL_E_INVAL
    assert lib.srnl_scan_cap_count(None, None) == S.SRNL_E_INVAL
    assert lib.srnl_seq_cap_count(None, None) == S.SRNL_E_INVAL


def test_selftest_rejects_out_of_range_limits_before_cuda(lib):
    for ms in (0, -1, 5001):
        assert lib.srnl_selftest_wait_timeout(ms) == S.SRNL_E_INVAL
        assert b"wait_ms" in lib.srnl_scan_last_error(None)


def test_backward_null_arguments_fail_cleanly(lib):
    assert lib.srnl_scan_backward(None, None, None, None, None, None) == S.SRNL_E_INVAL
    assert lib.srnl_seq_backward(None, None, None, None, None, None, None, None) == S.SRNL_E_INVAL


def test_committed_code_never_uses_the_scratch_directory():
    """Nothing in the product, the tests or the bench may read or run files from _work/."""
    pat = re.compile(r"\b_work/")
    for dirpath, dirnames, files in os.walk(ROOT):
        dirnames[:] = [d for d in dirnames if d not in ("_work", ".git", "gpurun_out", "__pycache__", ".pytest_cache")]
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".sh")):
                path = os.path.join(dirpath, f)
                if os.path.samefile(path, __file__):
                    continue
                assert not pat.search(open(path, errors="ignore").read()), path
