"""GPU parity of the context-parallel steps (hs2_cp_*), ranks emulated on one GPU.

The G ranks' slices are processed one after another on this GPU; what NCCL
would do between them is done here with plain tensor operations (the
all-gathers are stacks, the all-reduce is a sum).  No rank waits on another,
so nothing needs more than one device.  Checked against the oracle:
  * each slice's partial O and lse (oracle.attn_slice), and its top-k list
    under the global normaliser (sets equal except swaps inside the tie band);
  * the merged layer: O and lse of the whole cache, and the selection of
    hs2_full_attn_select (sets equal except swaps among candidates whose oracle
    score lies within 1e-3 relative of the k-th score).
"""

import numpy as np
import pytest
import torch

import hs2_testlib as tl
import long_context_hs2_b200 as hs2
import oracle
from hs2_synth import WORKLOADS, make_attention_inputs

pytestmark = pytest.mark.gpu

CASES = {
    # name: (workload, resize, slice boundaries)
    "chunk_fp8_two_slices": ("chunk_fp8_1m", dict(T=200, L=20011, n_needles=30, n_sparse=0,
                                                  fp8_scale="mantissa"), [0, 9000, 20011]),
    "decode_bf16_four_slices": ("decode_bf16_32k", dict(B=4, L=30000, n_needles=16, n_sparse=0),
                                [0, 7000, 15000, 22500, 30000]),
    # the last slice is shorter than the chunk of queries, which span two slices
    "chunk_spans_slices": ("decode_bf16_32k", dict(B=1, T=300, L=1700, H=16, n_needles=6,
                                                   n_sparse=0, topk=512, window=64),
                           [0, 1500, 1700]),
}


def _slice(t, a, b):
    return None if t is None else t[:, a:b].contiguous()


@pytest.mark.parametrize("case", sorted(CASES))
def test_context_parallel_steps_match_oracle(case):
    name, kw, bounds = CASES[case]
    wl = WORKLOADS[name].resized(**kw)
    inp = make_attention_inputs(wl)
    fp8 = wl.kv_dtype == "fp8"
    dt = hs2.HS2_KV_FP8_E4M3 if fp8 else hs2.HS2_KV_BF16
    B, T, L, H, D, topk, window = wl.B, wl.T, wl.L, wl.H, wl.D, wl.topk, wl.window
    G = len(bounds) - 1
    tol = tl.TOL_FP8 if fp8 else tl.TOL_BF16
    di = tl.DeviceInputs(inp)
    k = di.k.view(B, L, D)
    v = di.v.view(B, L, D)
    ks = di.ks.view(B, L) if fp8 else None
    vs = di.vs.view(B, L) if fp8 else None
    q_pos0 = L - T
    kvs, o_parts, lse_parts = [], [], []
    for r in range(G):
        a, b = bounds[r], bounds[r + 1]
        ksl, vsl = _slice(k, a, b), _slice(v, a, b)
        kss, vss = _slice(ks, a, b), _slice(vs, a, b)
        kv = hs2.kv_cache(ksl, vsl, kss, vss)
        kvs.append((kv, ksl, vsl, kss, vss))
        nb = hs2.hs2_cp_workspace(B, T, b - a, H, D, topk, window, dt)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        o = torch.empty(B, T, H, D, device="cuda")
        lse = torch.empty(B, T, H, device="cuda")
        hs2.hs2_cp_attn_partial(di.q, kv, B, T, b - a, q_pos0 - a, H, D, wl.scale, dt, o, lse,
                                ws, nb)
        assert hs2.hs2_last_device_status() == 0
        # the slice's own partial against the oracle's slice function
        sl = oracle.attn_slice(inp.q, inp.k[:, a:b], inp.v[:, a:b],
                               None if not fp8 else inp.k_scale[:, a:b],
                               None if not fp8 else inp.v_scale[:, a:b],
                               qpos=q_pos0 - a, scale=wl.scale, window=window)
        g_lse = lse.cpu().numpy().reshape(B * T, H)
        assert np.array_equal(np.isneginf(g_lse), np.isneginf(sl["lse"]))
        fin = np.isfinite(sl["lse"])
        assert np.abs(g_lse[fin] - sl["lse"][fin]).max() <= 1e-3
        assert tl.max_abs(o.cpu().numpy().reshape(B * T, H, D), sl["o"]) <= tol
        o_parts.append(o)
        lse_parts.append(lse)
    lse_all = torch.stack(lse_parts)                     # the all-gather
    lse_g = torch.empty(B, T, H, device="cuda")
    hs2.hs2_cp_lse_combine(lse_all, G, B * T * H, lse_g)
    for r in range(G):
        hs2.hs2_cp_rescale(o_parts[r], lse_parts[r], lse_g, B * T * H, D)
    o_g = torch.stack(o_parts).sum(0)                    # the sum all-reduce
    cs_all, ci_all = [], []
    for r in range(G):
        a, b = bounds[r], bounds[r + 1]
        kv = kvs[r][0]
        nb = hs2.hs2_cp_workspace(B, T, b - a, H, D, topk, window, dt)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        cs = torch.full((B, T, topk), 7.0, device="cuda")
        ci = torch.full((B, T, topk), -7, dtype=torch.int32, device="cuda")
        hs2.hs2_cp_select_local(di.q, kv, B, T, b - a, q_pos0 - a, a, H, D, wl.scale, topk, window,
                                dt, lse_g, cs, ci, ws, nb)
        assert hs2.hs2_last_device_status() == 0
        cs_all.append(cs)
        ci_all.append(ci)
    idx = torch.full((B, T, topk + window), -7, dtype=torch.int32, device="cuda")
    ns = torch.full((B, T), -7, dtype=torch.int32, device="cuda")
    hs2.hs2_cp_merge_select(torch.stack(cs_all), torch.stack(ci_all), G, B, T, q_pos0, topk,
                            window, idx, ns)
    assert hs2.hs2_last_device_status() == 0

    orc = tl.oracle_full(inp)
    assert tl.max_abs(o_g.cpu().numpy().reshape(B * T, H, D), orc["o"]) <= tol
    assert tl.max_abs(lse_g.cpu().numpy().reshape(B * T, H), orc["lse"]) <= 1e-3
    positions = [q_pos0 + t for _ in range(B) for t in range(T)]
    differ = tl.check_selection(idx.cpu().numpy().reshape(B * T, -1), ns.cpu().numpy().reshape(-1),
                                orc, positions, topk, window)
    assert differ <= max(1, B * T // 50)
    # every slice's list: global positions inside the slice, ascending, scores
    # equal to the oracle's score of that position (same global normaliser)
    for r in range(G):
        a, b = bounds[r], bounds[r + 1]
        ci = ci_all[r].cpu().numpy().reshape(B * T, topk)
        cs = cs_all[r].cpu().numpy().reshape(B * T, topk)
        for row in range(B * T):
            n = int((ci[row] >= 0).sum())
            assert (ci[row, n:] == -1).all() and (cs[row, n:] == -1.0).all()
            lst = ci[row, :n]
            assert (np.diff(lst) > 0).all() and (lst >= a).all() and (lst < b).all()
            i = positions[row]
            assert (lst <= i - window).all()
            ncand = max(0, min(b, i - window + 1) - a)
            assert n == min(topk, ncand)
            ref = orc["score"][row, lst]
            assert np.allclose(cs[row, :n], ref, rtol=2e-3, atol=1e-7)
