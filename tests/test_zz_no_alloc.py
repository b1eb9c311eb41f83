"""hs2_full_attn_select_noalloc: the allocation-free entry point.

Some callers cannot allocate device memory: code hosted by a framework that
owns all device memory and gives plugins no allocator, or code on a
latency-critical path that cannot pay for cudaMalloc's device-wide
synchronisation.  For them the library offers this entry point, which takes no
workspace and uses a scratch area built into the library instead.

The tests call it through the C ABI, twice in a row per shape, and check each
result against the ordinary entry point (which is given a torch workspace)
within the tolerances the parity tests use -- 1e-2 max-abs on O, 1e-3 on lse,
identical selections -- and against the oracle.  Two shapes take the two
paths the scratch serves: one decode query per sequence (the fused kernel:
arrival counters, per-split candidate lists) and a chunk of 8 queries per
sequence with 32 heads (separate partial, score and selection kernels: score
rows and histograms in the scratch); each runs on scratch the other left
dirty.  A request larger than the built-in scratch is refused before any work
is enqueued (checked with real, large enough buffers, so that even a wrongly
accepted call would only touch valid memory).  This file is collected last, so
a run that stops at its first failure has already run every other test; it
passes both alone and after the other tests.
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


def _noalloc(lib, di, O, lse, idx, ns):
    wl = di.wl
    return lib.hs2_full_attn_select_noalloc(
        di.q.data_ptr(), ctypes.byref(di.kv), wl.B, wl.T, wl.L, wl.H, wl.D,
        ctypes.c_float(wl.scale), wl.topk, wl.window, di.dt, O.data_ptr(), lse.data_ptr(),
        idx.data_ptr(), ns.data_ptr(), torch.cuda.current_stream().cuda_stream)


SHAPES = {
    # one query per sequence: the fused kernel
    "fused": WORKLOADS["decode_bf16_32k"].resized(B=3, L=6000, n_needles=10, n_sparse=0),
    # 8 queries per sequence, 32 heads: the separate partial / score / select kernels
    "chunk": WORKLOADS["decode_bf16_32k"].resized(B=2, T=8, L=7000, n_needles=10, n_sparse=0),
}


def _check_shape(lib, wl):
    di = tl.DeviceInputs(make_attention_inputs(wl))
    B, T, L, H, D = wl.B, wl.T, wl.L, wl.H, wl.D
    assert hs2.hs2_full_attn_select_workspace(B, T, L, H, D, wl.topk, wl.window, di.dt) <= \
        hs2.HS2_NOALLOC_SCRATCH_BYTES
    ref = tl.run_full(di)
    orc = tl.oracle_full(di.inp)
    for call in range(2):
        O, lse, idx, ns = _outputs(wl)
        st = _noalloc(lib, di, O, lse, idx, ns)
        assert st == 0, hs2.hs2_status_string(st)
        assert hs2.hs2_last_device_status() == 0
        o = O.cpu().numpy().reshape(B * T, H, D)
        g_lse = lse.cpu().numpy().reshape(B * T, H)
        g_idx = idx.cpu().numpy().reshape(B * T, -1)
        g_ns = ns.cpu().numpy().reshape(-1)
        # the ordinary entry point on the same inputs
        assert tl.max_abs(o, ref["o"]) <= tl.TOL_BF16, call
        assert tl.max_abs(g_lse, ref["lse"]) <= 1e-3, call
        assert np.array_equal(g_idx, ref["idx"]), call
        assert np.array_equal(g_ns, ref["n_sel"]), call
        # the oracle
        assert tl.max_abs(o, orc["o"]) <= tl.TOL_BF16, call
        tl.check_selection(g_idx, g_ns, orc, [L - T + t for _ in range(B) for t in range(T)],
                           wl.topk, wl.window)


@pytest.mark.parametrize("order", [("fused", "chunk"), ("chunk", "fused")])
def test_noalloc_matches_workspace_entry_point_twice(order):
    lib = hs2.load_library()
    for name in order:     # each shape runs on scratch the previous one left dirty
        _check_shape(lib, SHAPES[name])


def test_noalloc_rejects_requests_beyond_its_scratch():
    # one sequence of 4M positions needs more workspace than the built-in
    # scratch holds; the buffers are real and large enough for the request
    B, T, L, H, D = 1, 1, 1 << 22, 32, 128
    need = hs2.hs2_full_attn_select_workspace(B, T, L, H, D, 1024, 128, hs2.HS2_KV_BF16)
    assert need > hs2.HS2_NOALLOC_SCRATCH_BYTES
    lib = hs2.load_library()
    k = torch.zeros(B * L, D, dtype=torch.bfloat16, device="cuda")
    v = torch.zeros(B * L, D, dtype=torch.bfloat16, device="cuda")
    q = torch.zeros(B, T, H, D, dtype=torch.bfloat16, device="cuda")
    O = torch.zeros(B, T, H, D, device="cuda")
    idx = torch.full((B, T, 1152), -7, dtype=torch.int32, device="cuda")
    ns = torch.full((B, T), -7, dtype=torch.int32, device="cuda")
    kv = hs2.kv_cache(k, v)
    st = lib.hs2_full_attn_select_noalloc(q.data_ptr(), ctypes.byref(kv), B, T, L, H, D,
                                          ctypes.c_float(0.1), 1024, 128, hs2.HS2_KV_BF16,
                                          O.data_ptr(), None, idx.data_ptr(), ns.data_ptr(),
                                          torch.cuda.current_stream().cuda_stream)
    assert st == 4   # HS2_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert (ns.cpu() == -7).all() and (idx.cpu() == -7).all()   # nothing was enqueued
    del k, v
    torch.cuda.empty_cache()
