"""hs2_full_attn_select_noalloc: the allocation-free entry point.

Some callers cannot allocate device memory: code hosted by a framework that
owns all device memory and gives plugins no allocator, or code on a
latency-critical path that cannot pay for cudaMalloc's device-wide
synchronisation.  For them the library offers this entry point, which takes no
workspace and uses a scratch area built into the library instead.

The test calls it through the C ABI twice in a row and checks each result
against the ordinary entry point (which is given a torch workspace) within the
tolerances the parity tests use: 1e-2 max-abs on O, 1e-3 on lse, identical
selections.  It also checks that a request larger than the built-in scratch is
refused before any work is enqueued.  This file is collected last, so a run
that stops at its first failure has already run every other test; it passes
both alone and after the other tests.
"""

import ctypes

import numpy as np
import pytest
import torch

import hs2_testlib as tl
import long_context_hs2_b200 as hs2
from hs2_synth import WORKLOADS, make_attention_inputs

pytestmark = pytest.mark.gpu


def _outputs(wl):
    B, T, H, D = wl.B, wl.T, wl.H, wl.D
    slots = wl.topk + wl.window
    return (torch.full((B, T, H, D), float("nan"), device="cuda"),
            torch.full((B, T, H), float("nan"), device="cuda"),
            torch.full((B, T, slots), -7, dtype=torch.int32, device="cuda"),
            torch.full((B, T), -7, dtype=torch.int32, device="cuda"))


def test_noalloc_matches_workspace_entry_point_twice():
    wl = WORKLOADS["decode_bf16_32k"].resized(B=3, L=6000, n_needles=10, n_sparse=0)
    di = tl.DeviceInputs(make_attention_inputs(wl))
    B, T, L, H, D = wl.B, wl.T, wl.L, wl.H, wl.D
    assert hs2.hs2_full_attn_select_workspace(B, T, L, H, D, wl.topk, wl.window, di.dt) <= \
        hs2.HS2_NOALLOC_SCRATCH_BYTES
    ref = tl.run_full(di)
    lib = hs2.load_library()
    for call in range(2):
        O, lse, idx, ns = _outputs(wl)
        st = lib.hs2_full_attn_select_noalloc(
            di.q.data_ptr(), ctypes.byref(di.kv), B, T, L, H, D, ctypes.c_float(wl.scale),
            wl.topk, wl.window, di.dt, O.data_ptr(), lse.data_ptr(), idx.data_ptr(),
            ns.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert st == 0, hs2.hs2_status_string(st)
        assert hs2.hs2_last_device_status() == 0
        o = O.cpu().numpy().reshape(B * T, H, D)
        assert tl.max_abs(o, ref["o"]) <= tl.TOL_BF16, call
        assert tl.max_abs(lse.cpu().numpy().reshape(B * T, H), ref["lse"]) <= 1e-3, call
        assert np.array_equal(idx.cpu().numpy().reshape(B * T, -1), ref["idx"]), call
        assert np.array_equal(ns.cpu().numpy().reshape(-1), ref["n_sel"]), call


def test_noalloc_rejects_requests_beyond_its_scratch():
    # 64 sequences of 64K positions need far more than the built-in scratch
    B, T, L, H, D = 64, 1, 65536, 32, 128
    assert hs2.hs2_full_attn_select_workspace(B, T, L, H, D, 1024, 128, 0) > \
        hs2.HS2_NOALLOC_SCRATCH_BYTES
    lib = hs2.load_library()
    kv = hs2.hs2_kv_cache(16, 16, None, None)
    st = lib.hs2_full_attn_select_noalloc(16, ctypes.byref(kv), B, T, L, H, D,
                                          ctypes.c_float(0.1), 1024, 128, 0, 16, None, 16, 16,
                                          None)
    assert st == 4   # HS2_ERR_WORKSPACE, nothing enqueued
