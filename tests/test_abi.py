"""The C-ABI library without a GPU: it loads, exports every symbol include/hs2.h
declares, and rejects bad arguments on the host before touching the device."""

import ctypes
import os
import re

import pytest

import long_context_hs2_b200 as hs2
from long_context_hs2_b200 import build as hs2_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    src = open(os.path.join(ROOT, "include", "hs2.h")).read()
    return sorted(set(re.findall(r"HS2_API\s+[\w\s\*]*?\b(hs2_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    hs2_build.build()
    return hs2.load_library()


def test_header_declares_entry_points():
    names = header_symbols()
    for n in ("hs2_bridge_kv", "hs2_full_attn_select", "hs2_full_attn_select_workspace",
              "hs2_sparse_attn", "hs2_last_device_status", "hs2_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in header_symbols():
        assert hasattr(lib, name), name
    assert set(hs2.EXPORTED) <= set(header_symbols())


def test_version_and_status_strings(lib):
    assert hs2.hs2_version() >= 100
    for st in range(7):
        assert hs2.hs2_status_string(st)
    assert hs2.hs2_status_string(0) == "ok"


def test_workspace_sizes(lib):
    n = hs2.hs2_full_attn_select_workspace(8, 1, 32768, 32, 128, 1024, 128, hs2.HS2_KV_BF16)
    # must at least hold the fp32 score rows and the level-1 histograms
    assert n >= 8 * 32768 * 4 + 8 * 2048 * 4
    assert hs2.hs2_full_attn_select_workspace(8, 1, 32768, 24, 128, 1024, 128, 0) == 0   # H
    assert hs2.hs2_full_attn_select_workspace(8, 1, 32768, 32, 96, 1024, 128, 0) == 0    # D
    assert hs2.hs2_full_attn_select_workspace(1, 10, 5, 32, 128, 1024, 128, 0) == 0      # T > L
    assert hs2.hs2_full_attn_select_workspace(1, 1, 5, 32, 128, 4000, 128, 0) == 0       # slots


def _call_full(lib, **kw):
    a = dict(Q=16, kv=hs2.hs2_kv_cache(16, 16, None, None), B=1, T=1, L=64, H=32, D=128,
             scale=0.1, topk=16, window=8, dt=0, O=16, lse=None, idx=16, n_sel=16, ws=16,
             ws_bytes=1 << 40, stream=None)
    a.update(kw)
    return lib.hs2_full_attn_select(a["Q"], ctypes.byref(a["kv"]), a["B"], a["T"], a["L"], a["H"],
                                    a["D"], a["scale"], a["topk"], a["window"], a["dt"], a["O"],
                                    a["lse"], a["idx"], a["n_sel"], a["ws"], a["ws_bytes"],
                                    a["stream"])


def test_full_attn_rejects_bad_arguments(lib):
    assert _call_full(lib, Q=None) == 1
    assert _call_full(lib, Q=8) == 1                                     # misaligned
    assert _call_full(lib, kv=hs2.hs2_kv_cache(None, 16, None, None)) == 1
    assert _call_full(lib, T=65) == 1                                    # T > L
    assert _call_full(lib, window=0) == 1
    assert _call_full(lib, topk=-1) == 1
    assert _call_full(lib, scale=float("nan")) == 1
    assert _call_full(lib, dt=1) == 1                                    # fp8 without scales
    assert _call_full(lib, H=12) == 2
    assert _call_full(lib, D=256) == 2
    assert _call_full(lib, ws=None) == 4
    assert _call_full(lib, ws_bytes=16) == 4


def test_sparse_attn_rejects_bad_arguments(lib):
    kv = hs2.hs2_kv_cache(16, 16, None, None)
    f = lib.hs2_sparse_attn
    assert f(None, ctypes.byref(kv), 1, 1, 64, 32, 128, 0.1, 16, 16, 8, 0, 16, None) == 1
    assert f(16, ctypes.byref(kv), 1, 1, 64, 32, 128, 0.1, None, 16, 8, 0, 16, None) == 1
    assert f(16, ctypes.byref(kv), 1, 1, 64, 32, 128, 0.1, 16, 16, 0, 0, 16, None) == 1
    assert f(16, ctypes.byref(kv), 1, 1, 64, 32, 128, 0.1, 16, 16, 5000, 0, 16, None) == 2
    assert f(16, ctypes.byref(kv), 1, 1, 64, 32, 64, 0.1, 16, 16, 8, 1, 16, None) == 1  # fp8, no scales
    kv8 = hs2.hs2_kv_cache(16, 16, 16, 16)
    assert f(16, ctypes.byref(kv8), 1, 1, 64, 32, 64, 0.1, 16, 16, 8, 1, 16, None) == 2  # fp8 needs D=128


def test_noalloc_checks_arguments_before_the_size(lib):
    # a request far beyond the built-in scratch, but with a null or misaligned
    # pointer: the argument error is reported first, and nothing is enqueued
    kv = hs2.hs2_kv_cache(16, 16, None, None)
    f = lib.hs2_full_attn_select_noalloc
    B, T, L, H, D = 64, 1, 65536, 32, 128
    assert f(None, ctypes.byref(kv), B, T, L, H, D, 0.1, 1024, 128, 0, 16, None, 16, 16, None) == 1
    assert f(16, ctypes.byref(kv), B, T, L, H, D, 0.1, 1024, 128, 0, 8, None, 16, 16, None) == 1
    assert f(16, ctypes.byref(kv), B, T, L, H, 96, 0.1, 1024, 128, 0, 16, None, 16, 16, None) == 2


def test_fault_injection_setter(lib):
    assert lib.hs2_set_fault_injection(1, 2000000) == 0
    assert lib.hs2_set_fault_injection(0, 0) == 0


def test_phase_stamps_setter(lib):
    # the setter only records the buffer for later calls: it checks its arguments
    assert lib.hs2_set_phase_stamps(ctypes.c_void_p(4096), 0) == 1
    assert lib.hs2_set_phase_stamps(ctypes.c_void_p(4100), 8) == 1
    assert lib.hs2_set_phase_stamps(None, 0) == 0


def test_stage_events_pairing(lib):
    assert lib.hs2_set_stage_events(ctypes.c_void_p(16), None) == 1
    assert lib.hs2_set_stage_events(None, ctypes.c_void_p(16)) == 1
    assert lib.hs2_set_stage_events(None, None) == 0


def test_kv_cache_keeps_its_tensors():
    # the struct holds raw pointers; it must keep the tensors behind them alive
    import gc
    import weakref
    import torch
    k, v = torch.zeros(8), torch.zeros(8)
    rk = weakref.ref(k)
    c = hs2.kv_cache(k, v)
    ptr = k.data_ptr()
    del k, v
    gc.collect()
    assert rk() is not None and c.k == ptr
    del c
    gc.collect()
    assert rk() is None


def test_product_path_does_not_import_oracle():
    pkg = os.path.join(ROOT, "long_context_hs2_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f
                assert "hs2_oracle" not in src, f
