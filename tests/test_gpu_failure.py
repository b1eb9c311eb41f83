"""Failure detection on the GPU without a GPU fault.

The fused full-attention kernel's CTAs meet at group barriers through global
arrival counters, each wait bounded.  hs2_set_fault_injection makes those
barriers wait for one arrival more than the group has CTAs -- an arrival that
never comes -- with a 2 ms limit: every wait must give up, the call must report
HS2_ERR_TIMEOUT through hs2_last_device_status, and the kernel must return, so
that the context stays usable: the same call without the injected fault then
gives the oracle's results.
"""

import numpy as np
import pytest
import torch

import hs2_testlib as tl
import long_context_hs2_b200 as hs2
from hs2_synth import WORKLOADS, make_attention_inputs

pytestmark = pytest.mark.gpu

HS2_ERR_TIMEOUT = 5


def test_group_barrier_timeout_is_reported_and_the_kernel_returns():
    wl = WORKLOADS["decode_bf16_32k"].resized(B=2, L=6000, n_needles=4, n_sparse=0)
    inp = make_attention_inputs(wl)
    di = tl.DeviceInputs(inp)
    B, T, L, H, D = wl.B, wl.T, wl.L, wl.H, wl.D
    slots = wl.topk + wl.window
    ws_bytes = hs2.hs2_full_attn_select_workspace(B, T, L, H, D, wl.topk, wl.window, di.dt)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    O = torch.empty(B, T, H, D, device="cuda")
    idx = torch.empty(B, T, slots, dtype=torch.int32, device="cuda")
    ns = torch.empty(B, T, dtype=torch.int32, device="cuda")
    hs2.hs2_set_fault_injection(1, 2_000_000)
    try:
        hs2.hs2_full_attn_select(di.q, di.kv, B, T, L, H, D, wl.scale, wl.topk, wl.window, di.dt,
                                 O, None, idx, ns, ws, ws_bytes)
        assert hs2.hs2_last_device_status() == HS2_ERR_TIMEOUT
        assert hs2.hs2_last_device_status() == 0        # cleared by the read
    finally:
        hs2.hs2_set_fault_injection()
    # the context is still usable, and the same call is correct without the fault
    g = tl.run_full(di)
    orc = tl.oracle_full(inp)
    assert tl.max_abs(g["o"], orc["o"]) <= tl.TOL_BF16
    tl.check_selection(g["idx"], g["n_sel"], orc, [L - 1] * B, wl.topk, wl.window)
