"""GPU parity of the hybrid block replayed as one CUDA graph.

A decode loop runs the block once per generated token: the full-attention
layer with its selection, then the sparse layers that reuse its cache and
indices (IT Home announcement, "KV Reuse" paragraphs).  Here the block is
captured once -- hs2_full_attn_select (its arrival-counter memset node and the
fused kernel) followed by three hs2_sparse_attn launches, the first of them
launched programmatically behind the fused kernel, exactly as the benchmark's
step graph holds them -- and replayed with two different sets of queries
copied into the captured input buffers.  After each replay all outputs (O and
lse of the full layer, the indices and counts, and the three sparse layers'
outputs) are compared with the oracle on the same inputs.
"""

import numpy as np
import pytest
import torch

import hs2_testlib as tl
import long_context_hs2_b200 as hs2
from hs2_synth import WORKLOADS, make_attention_inputs

pytestmark = pytest.mark.gpu


def _queries(wl, seed):
    """The block's queries (full layer + sparse layers) of another seeded draw."""
    qi = make_attention_inputs(wl.resized(L=1, T=wl.T, seed=seed), needles=False)
    return [qi.q] + qi.q_sparse


@pytest.mark.parametrize("name,kw", [
    ("decode_bf16_32k", {}),
    ("decode_fp8_256k", {"B": 2, "L": 20000, "n_needles": 12, "fp8_scale": "mantissa"}),
])
def test_block_graph_replays_match_oracle(name, kw):
    wl = WORKLOADS[name].resized(**kw)
    inp = make_attention_inputs(wl)
    di = tl.DeviceInputs(inp)
    B, T, L, H, D = wl.B, wl.T, wl.L, wl.H, wl.D
    slots = wl.topk + wl.window
    n_layers = 1 + wl.n_sparse
    ws_bytes = hs2.hs2_full_attn_select_workspace(B, T, L, H, D, wl.topk, wl.window, di.dt)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    q_buf = [torch.empty(B, T, H, D, dtype=torch.bfloat16, device="cuda")
             for _ in range(n_layers)]
    outs = [torch.empty(B, T, H, D, device="cuda") for _ in range(n_layers)]
    lse = torch.empty(B, T, H, device="cuda")
    idx = torch.empty(B, T, slots, dtype=torch.int32, device="cuda")
    nsel = torch.empty(B, T, dtype=torch.int32, device="cuda")

    def block():
        hs2.hs2_full_attn_select(q_buf[0], di.kv, B, T, L, H, D, wl.scale, wl.topk, wl.window,
                                 di.dt, outs[0], lse, idx, nsel, ws, ws_bytes)
        for s in range(wl.n_sparse):
            hs2.hs2_sparse_attn(q_buf[1 + s], di.kv, B, T, L, H, D, wl.scale, idx, nsel, slots,
                                di.dt, outs[1 + s])

    for qb, q in zip(q_buf, [di.q] + di.q_sparse):
        qb.copy_(q)
    block()                       # loads the kernels before capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        block()

    draws = [[inp.q] + inp.q_sparse, _queries(wl, wl.seed + 77)]
    for qs in draws:
        for qb, q in zip(q_buf, qs):
            qb.copy_(tl.dev(q.view(np.int16)).view(torch.bfloat16))
        for o in outs:
            o.fill_(float("nan"))
        idx.fill_(-7)
        graph.replay()
        torch.cuda.synchronize()
        assert hs2.hs2_last_device_status() == 0
        case = type(inp)(wl, qs[0], qs[1:], inp.k, inp.v, inp.k_scale, inp.v_scale, inp.needles)
        orc = tl.oracle_full(case)
        tol = tl.TOL_FP8 if di.fp8 else tl.TOL_BF16
        g_o = outs[0].cpu().numpy().reshape(B * T, H, D)
        g_idx = idx.cpu().numpy().reshape(B * T, slots)
        g_ns = nsel.cpu().numpy().reshape(-1)
        assert tl.max_abs(g_o, orc["o"]) <= tol
        assert tl.max_abs(lse.cpu().numpy().reshape(B * T, H), orc["lse"]) <= 1e-3
        tl.check_selection(g_idx, g_ns, orc, [L - T + t for _ in range(B) for t in range(T)],
                           wl.topk, wl.window)
        same = [r for r in range(B * T) if np.array_equal(g_idx[r], orc["idx"][r])]
        assert len(same) >= B * T - max(1, B * T // 50)
        for s in range(wl.n_sparse):
            o_orc = tl.oracle_sparse(case, s, orc["idx"], orc["n_sel"], rows=np.asarray(same))
            g_s = outs[1 + s].cpu().numpy().reshape(B * T, H, D)
            assert tl.max_abs(g_s[same], o_orc) <= tol
    del graph
