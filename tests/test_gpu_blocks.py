"""GPU parity of the block-level selection variant (hs2_full_attn_select_blocks).

The earlier HySparse chose history in blocks of 64 tokens; HySparse2 chooses
single tokens (dpshk.com explainer, section 03; cnyes.com article, section
"檢索精確到token").  The variant shares the attention pass and replaces the
selection.  Checks:
  * O and lse equal the oracle's, as for the token-level call;
  * selected sets equal the oracle's block-level selection on the oracle's
    scores, except swaps among blocks whose oracle block score lies within
    1e-3 (relative) of the last kept block's score; kept blocks are whole
    (clipped to the candidates), the window is present, indices ascend;
  * blocks of one position reproduce the GPU's token-level selection exactly
    (the same fp32 scores, the same order);
  * at the decode workload's full size, an A/B of needle recall: token-level
    selection keeps every planted needle; block-level selection, with the same
    1024-position budget in 16 blocks, cannot keep more needles than 16 blocks
    hold (the pages' motivation for token-level selection).
"""

import numpy as np
import pytest
import torch

import hs2_testlib as tl
import long_context_hs2_b200 as hs2
import oracle
from hs2_synth import WORKLOADS, make_attention_inputs

pytestmark = pytest.mark.gpu

BAND = 1e-3


def run_blocks(di, block, topk=None, window=None):
    wl = di.wl
    topk = wl.topk if topk is None else topk
    window = wl.window if window is None else window
    B, T, L, H, D = wl.B, wl.T, wl.L, wl.H, wl.D
    nb = hs2.hs2_full_attn_select_workspace(B, T, L, H, D, topk, window, di.dt)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    O = torch.empty(B, T, H, D, device="cuda")
    lse = torch.empty(B, T, H, device="cuda")
    idx = torch.full((B, T, topk + window), -7, dtype=torch.int32, device="cuda")
    ns = torch.full((B, T), -7, dtype=torch.int32, device="cuda")
    hs2.hs2_full_attn_select_blocks(di.q, di.kv, B, T, L, H, D, wl.scale, topk, window, block,
                                    di.dt, O, lse, idx, ns, ws, nb)
    assert hs2.hs2_last_device_status() == 0
    return dict(o=O.cpu().numpy().reshape(B * T, H, D), lse=lse.cpu().numpy().reshape(B * T, H),
                idx=idx.cpu().numpy().reshape(B * T, -1), n_sel=ns.cpu().numpy().reshape(-1))


def check_block_selection(g, orc, positions, topk, window, block):
    differ = 0
    for r, i in enumerate(positions):
        ref, ns = oracle.select_blocks(orc["score"][r], i, topk, window, block)
        assert int(g["n_sel"][r]) <= topk + window
        gs = g["idx"][r, : g["n_sel"][r]]
        assert (np.diff(gs) > 0).all()
        assert (g["idx"][r, g["n_sel"][r]:] == -1).all()
        assert np.isin(np.arange(max(0, i - window + 1), i + 1), gs).all()
        if int(g["n_sel"][r]) == ns and np.array_equal(gs, ref[:ns]):
            continue
        differ += 1
        last = i - window
        s = orc["score"][r, : last + 1]
        bsum = np.bincount(np.arange(last + 1) // block, weights=s)
        kept_o = np.unique(ref[:ns][ref[:ns] <= last] // block)
        kept_g = np.unique(gs[gs <= last] // block)
        # kept blocks are whole: every candidate position of a kept block is selected
        for b in kept_g:
            blk = np.arange(b * block, min((b + 1) * block, last + 1))
            assert np.isin(blk, gs).all(), ("partial block", r, b)
        assert len(kept_g) == len(kept_o)
        kth = bsum[kept_o].min()
        for b in np.setxor1d(kept_g, kept_o):
            assert abs(bsum[b] - kth) <= BAND * kth, (r, b, bsum[b], kth)
    return differ


@pytest.mark.parametrize("name,kw", [
    ("decode_bf16_32k", {"B": 3, "L": 9000, "n_needles": 12, "n_sparse": 0}),     # fused kernel
    ("decode_bf16_32k", {"B": 2, "T": 8, "L": 7000, "n_needles": 8, "n_sparse": 0}),  # separate kernels
    ("decode_fp8_256k", {"B": 2, "L": 20011, "n_needles": 10, "n_sparse": 0,
                         "fp8_scale": "mantissa"}),
    ("tiny", {"T": 200, "L": 2500, "n_needles": 8, "n_sparse": 0}),                 # head_dim 64
])
def test_blocks_of_64_match_oracle(name, kw):
    wl = WORKLOADS[name].resized(**kw)
    inp = make_attention_inputs(wl)
    di = tl.DeviceInputs(inp)
    g = run_blocks(di, 64)
    orc = tl.oracle_full(inp)
    tol = tl.TOL_FP8 if di.fp8 else tl.TOL_BF16
    assert tl.max_abs(g["o"], orc["o"]) <= tol
    assert tl.max_abs(g["lse"], orc["lse"]) <= 1e-3
    positions = [wl.L - wl.T + t for _ in range(wl.B) for t in range(wl.T)]
    differ = check_block_selection(g, orc, positions, wl.topk, wl.window, 64)
    assert differ <= max(1, len(positions) // 50)


def test_blocks_of_one_equal_token_level():
    wl = WORKLOADS["decode_bf16_32k"].resized(B=3, L=12000, n_needles=12, n_sparse=0)
    di = tl.DeviceInputs(make_attention_inputs(wl))
    tok = tl.run_full(di)
    blk = run_blocks(di, 1)
    assert np.array_equal(blk["n_sel"], tok["n_sel"])
    assert np.array_equal(blk["idx"], tok["idx"])


def test_blocks_edge_cases():
    wl = WORKLOADS["decode_bf16_32k"].resized(B=2, T=3, L=900, n_needles=0, n_sparse=0)
    inp = make_attention_inputs(wl, needles=False)
    di = tl.DeviceInputs(inp)
    orc = tl.oracle_full(inp)
    positions = [wl.L - wl.T + t for _ in range(wl.B) for t in range(wl.T)]
    # every candidate block fits the budget: all positions 0 .. i
    g = run_blocks(di, 64)
    for r, i in enumerate(positions):
        assert g["n_sel"][r] == i + 1 and np.array_equal(g["idx"][r, : i + 1], np.arange(i + 1))
    # a zero budget: the window alone; a budget of 2 blocks of 128 positions
    for topk, block in ((0, 64), (256, 128), (192, 64)):
        g = run_blocks(di, block, topk=topk)
        assert check_block_selection(g, orc, positions, topk, wl.window, block) <= 1


def test_needle_recall_token_versus_block_level():
    # the decode workload at full size: 64 needles per sequence, each in its own
    # region of the context; token-level keeps them all, block-level keeps at
    # most the needles of its 16 blocks
    wl = WORKLOADS["decode_bf16_32k"].resized(n_sparse=0)
    inp = make_attention_inputs(wl)
    di = tl.DeviceInputs(inp)
    tok = tl.run_full(di)
    blk = run_blocks(di, 64)

    def recall(res):
        hit = [int(j) in set(res["idx"][b, : res["n_sel"][b]].tolist()) for b, j, _ in inp.needles]
        return float(np.mean(hit))

    r_tok, r_blk = recall(tok), recall(blk)
    # most needles any 16 blocks of a sequence can hold
    bound = 0
    for b in range(wl.B):
        per_block = np.bincount(inp.needles[inp.needles[:, 0] == b, 1] // 64)
        bound += np.sort(per_block)[::-1][: wl.topk // 64].sum()
    assert r_tok == 1.0
    assert r_blk <= bound / len(inp.needles) + 1e-12
    assert r_blk < r_tok
