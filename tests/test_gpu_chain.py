"""GPU parity of the hot path chained end to end on an E4M3 cache.

hs2_bridge_kv writes the target layers' caches as E4M3 codes with its own
per-token scales (max|y| / 448: arbitrary fp32 mantissas, unlike the
power-of-two scales of the generator's default packing).  hs2_full_attn_select
and three hs2_sparse_attn layers then run on one of those caches, as a decode
step of the hybrid block would (IT Home announcement, "KV Bridging" and "KV
Reuse" paragraphs: the bridged full layer builds its cache from the source
hidden state, and the sparse layers reuse that cache and its indices).

The oracle runs on the very cache bytes and scales the GPU wrote, so the
attention checks isolate the attention kernels' use of those scales; sampled
rows of the bridge itself are checked against the oracle's projection.  Keys
for planted needles are planted in X: the needle's hidden row is the
minimum-norm solution of Wk x = 4 sqrt(D) u, u the unit head-sum of the
decode query, so the bridged key points along the query.
"""

import numpy as np
import pytest
import torch

import hs2_testlib as tl
import long_context_hs2_b200 as hs2
import oracle
import oracle_pins as P
from hs2_synth import (WORKLOADS, AttnInputs, f32_to_bf16_bits, make_attention_inputs,
                       make_bridge_inputs, uniform_stream, stream_seed)

pytestmark = pytest.mark.gpu

B, L, H, D = 4, 8192, 32, 128
HIDDEN, N_LAYERS, LAYER = 1024, 2, 1    # the cache of bridged layer 1 is attended
N_NEEDLES = 16


class _Dev:
    """The attention-side view hs2_testlib's runners expect, over GPU-written caches."""

    def __init__(self, wl, q, q_sparse, k, v, ks, vs):
        self.wl, self.fp8, self.dt = wl, True, hs2.HS2_KV_FP8_E4M3
        self.q = tl.dev(q.view(np.int16)).view(torch.bfloat16)
        self.q_sparse = [tl.dev(x.view(np.int16)).view(torch.bfloat16) for x in q_sparse]
        self.kv = hs2.kv_cache(k, v, ks, vs)


def _plant_needles(bi, q_bits):
    """Rewrites rows of X so that the layer's bridged keys at the needle positions
    point along the decode query's head-sum; returns (b, j, t=0) triples."""
    wk = P.dec_bf16(bi.wt[LAYER * 2 * D: LAYER * 2 * D + D])          # [D, hidden]
    qf = P.dec_bf16(q_bits)                                              # [B, 1, H, D]
    seed = stream_seed(2026, "chain_needles")
    u = uniform_stream(seed, B * N_NEEDLES)
    planted = []
    for b in range(B):
        s = qf[b, 0].sum(axis=0)
        k_target = 4.0 * np.sqrt(D) * s / np.linalg.norm(s)
        x = wk.T @ np.linalg.solve(wk @ wk.T, k_target)
        js = set()
        for n in range(N_NEEDLES):
            j = int(u[b * N_NEEDLES + n] * (L - 128 - 1))
            if j in js:
                continue
            js.add(j)
            bi.x[b * L + j] = f32_to_bf16_bits(x)
            planted.append((b, j, 0))
    return np.asarray(planted, dtype=np.int64)


def test_bridge_e4m3_into_full_attention_and_three_sparse_layers():
    wl = WORKLOADS["decode_fp8_256k"].resized(B=B, L=L, n_needles=0, n_sparse=3)
    qin = make_attention_inputs(wl.resized(L=1, T=1), needles=False)   # queries only
    bwl = WORKLOADS["bridge_131k"].resized(T=B * L, hidden=HIDDEN, n_layers=N_LAYERS)
    bi = make_bridge_inputs(bwl)
    needles = _plant_needles(bi, qin.q)

    # ---- KV Bridging on the GPU: E4M3 caches of both target layers
    x = tl.dev(bi.x.view(np.int16)).view(torch.bfloat16)
    wt = tl.dev(bi.wt.view(np.int16)).view(torch.bfloat16)
    bufs = [(torch.empty(B * L, D, dtype=torch.uint8, device="cuda"),
             torch.empty(B * L, D, dtype=torch.uint8, device="cuda"),
             torch.empty(B * L, device="cuda"), torch.empty(B * L, device="cuda"))
            for _ in range(N_LAYERS)]
    hs2.hs2_bridge_kv(x, B * L, HIDDEN, wt, N_LAYERS, D, hs2.HS2_KV_FP8_E4M3,
                      [hs2.kv_cache(*b) for b in bufs], 0)
    assert hs2.hs2_last_device_status() == 0
    k, v, ks, vs = bufs[LAYER]
    kh, vh = k.cpu().numpy().reshape(B, L, D), v.cpu().numpy().reshape(B, L, D)
    ksh, vsh = ks.cpu().numpy().reshape(B, L), vs.cpu().numpy().reshape(B, L)
    mant, _ = np.frexp(ksh)
    assert (mant != 0.5).mean() > 0.99     # the bridge's scales are not powers of two

    # sampled bridge rows (needle rows included) against the oracle's projection
    rows = np.unique(np.r_[needles[:, 0] * L + needles[:, 1],
                           np.random.default_rng(3).integers(0, B * L, 48)])
    ob = oracle.bridge(bi.x, bi.wt, N_LAYERS, D, rows=rows)
    for kv_i, (codes, sc) in enumerate(((kh, ksh), (vh, vsh))):
        y = ob["y"][:, LAYER * 2 * D + kv_i * D: LAYER * 2 * D + (kv_i + 1) * D]
        s_orc = ob[("k" if kv_i == 0 else "v") + "_scale"][LAYER]
        s_gpu = sc.reshape(-1)[rows]
        assert np.allclose(s_gpu, s_orc, rtol=1e-5, atol=0)
        deq = P.dec_e4m3(codes.reshape(-1, D)[rows], s_gpu)
        # half an E4M3 step (2^-4 relative, 2^-10 * s for subnormal codes), doubled
        # for the fp32-vs-fp64 rounding decision
        assert (np.abs(deq - y) <= 2.0 ** -3 * np.abs(y) + 2.0 ** -9 * s_gpu[:, None]).all()

    # ---- full attention + selection, then three sparse layers, on the GPU
    di = _Dev(wl, qin.q, qin.q_sparse, k, v, ks, vs)
    g = tl.run_full(di)
    slots = wl.topk + wl.window
    o_sparse_gpu = [tl.run_sparse(di, layer, g["idx_dev"], g["nsel_dev"], slots)
                    for layer in range(3)]

    # ---- the oracle on the same cache bytes
    inp = AttnInputs(wl, qin.q, qin.q_sparse, kh, vh, ksh, vsh, needles)
    orc = tl.oracle_full(inp)
    assert tl.max_abs(g["o"], orc["o"]) <= tl.TOL_FP8
    assert tl.max_abs(g["lse"], orc["lse"]) <= 1e-3
    positions = [L - 1] * B
    tl.check_selection(g["idx"], g["n_sel"], orc, positions, wl.topk, wl.window)
    for b, j, _ in needles:
        assert j in g["idx"][b, : g["n_sel"][b]], ("needle not selected", b, j)
    same = [r for r in range(B) if np.array_equal(g["idx"][r], orc["idx"][r])]
    for layer in range(3):
        # on the oracle's indices (isolates the sparse kernel) ...
        o_iso = tl.run_sparse(di, layer, orc["idx"], orc["n_sel"], slots)
        o_orc = tl.oracle_sparse(inp, layer, orc["idx"], orc["n_sel"])
        assert tl.max_abs(o_iso, o_orc) <= tl.TOL_FP8
        # ... and end to end on the GPU's own indices where they equal the oracle's
        if same:
            assert tl.max_abs(o_sparse_gpu[layer][same], o_orc[same]) <= tl.TOL_FP8
