"""GPU parity: hs2_full_attn_select and hs2_sparse_attn against the CPU oracle.

Every case runs the CUDA path through the C ABI and the oracle on the same
seeded input bytes.  O and O' must be within the stated max-abs tolerance
(1e-2 bf16 cache, 3e-2 E4M3 cache); selected sets must match except for
swaps among candidates whose oracle score lies within 1e-3 (relative) of the
k-th score; the forced window and the planted needles must be selected.
"""

import numpy as np
import pytest
import torch

import hs2_testlib as tl
from hs2_synth import WORKLOADS, make_attention_inputs
import long_context_hs2_b200 as hs2

pytestmark = pytest.mark.gpu


def _positions(wl, rows):
    return [wl.L - wl.T + (r % wl.T) for r in rows]


def _check_block(wl, rows=None, sparse_layers=None, needles=True, inp=None):
    inp = make_attention_inputs(wl, needles=needles) if inp is None else inp
    di = tl.DeviceInputs(inp)
    g = tl.run_full(di)
    rows = np.arange(wl.B * wl.T) if rows is None else np.asarray(rows)
    orc = tl.oracle_full(inp, rows=rows)
    tol = tl.TOL_FP8 if di.fp8 else tl.TOL_BF16
    assert tl.max_abs(g["o"][rows], orc["o"]) <= tol
    assert tl.max_abs(g["lse"][rows], orc["lse"]) <= 1e-3
    differ = tl.check_selection(g["idx"][rows], g["n_sel"][rows], orc, _positions(wl, rows),
                                wl.topk, wl.window)
    assert differ <= max(1, len(rows) // 50)
    sel_rows = {int(r): k for k, r in enumerate(rows)}
    for b, j, t in inp.needles:
        r = int(b) * wl.T + int(t)
        if r in sel_rows:
            assert j in g["idx"][r, : g["n_sel"][r]], ("needle not selected", b, j, t)
    layers = range(wl.n_sparse) if sparse_layers is None else sparse_layers
    slots = wl.topk + wl.window
    # each sparse layer reuses the oracle's indices: isolates the sparse kernel
    full_idx = np.full((wl.B * wl.T, slots), -1, dtype=np.int32)
    full_ns = np.zeros(wl.B * wl.T, dtype=np.int32)
    full_idx[rows] = orc["idx"]
    full_ns[rows] = orc["n_sel"]
    for layer in layers:
        o_gpu = tl.run_sparse(di, layer, full_idx, full_ns, slots)
        o_orc = tl.oracle_sparse(inp, layer, full_idx, full_ns, rows=rows)
        assert tl.max_abs(o_gpu[rows], o_orc) <= tol
    # the GPU's own indices, end to end, on rows whose sets equal the oracle's
    same = [k for k, r in enumerate(rows)
            if np.array_equal(g["idx"][r], orc["idx"][k])]
    if layers and same:
        layer = list(layers)[0]
        o_gpu = tl.run_sparse(di, layer, g["idx_dev"], g["nsel_dev"], slots)
        o_orc = tl.oracle_sparse(inp, layer, full_idx, full_ns, rows=rows[same])
        assert tl.max_abs(o_gpu[rows[same]], o_orc) <= tol
    return g


def test_tiny_block():
    _check_block(WORKLOADS["tiny"])


def test_decode_bf16_ragged():
    _check_block(WORKLOADS["decode_bf16_32k"].resized(B=3, L=5003, n_needles=12))


def test_decode_bf16_32k():
    _check_block(WORKLOADS["decode_bf16_32k"])


@pytest.mark.parametrize("fp8_scale", ["pow2", "mantissa"])
def test_decode_fp8_ragged(fp8_scale):
    # "mantissa": per-token scales with random mantissa bits, so the kernels'
    # products with k_scale and v_scale are inexact at reduced precision
    _check_block(WORKLOADS["decode_fp8_256k"].resized(B=2, L=9007, n_needles=20,
                                                      fp8_scale=fp8_scale))


def test_decode_fp8_256k():
    _check_block(WORKLOADS["decode_fp8_256k"])


@pytest.mark.parametrize("fp8_scale", ["pow2", "mantissa"])
def test_chunk_fp8_small(fp8_scale):
    wl = WORKLOADS["chunk_fp8_1m"].resized(T=200, L=20011, n_needles=40, n_sparse=1,
                                           fp8_scale=fp8_scale)
    rows = np.unique(np.r_[0, 199, np.random.default_rng(1).integers(0, 200, 30)])
    _check_block(wl, rows=rows)


def test_chunk_bf16_heads8_d64():
    wl = WORKLOADS["tiny"].resized(T=300, L=3001, n_needles=10)
    _check_block(wl)


def test_heads16_bf16():
    wl = WORKLOADS["decode_bf16_32k"].resized(B=2, T=3, L=4000, H=16, n_needles=6)
    _check_block(wl)


def test_context_within_budget_sparse_equals_dense():
    # every position is selected, so a sparse layer with the full layer's own
    # queries must reproduce the full layer's output
    wl = WORKLOADS["decode_bf16_32k"].resized(B=2, T=5, L=1100, n_needles=0, n_sparse=1)
    inp = make_attention_inputs(wl, needles=False)
    inp.q_sparse[0] = inp.q
    di = tl.DeviceInputs(inp)
    g = tl.run_full(di)
    assert (g["n_sel"] == np.tile(wl.L - wl.T + np.arange(wl.T) + 1, wl.B)).all()
    o2 = tl.run_sparse(di, 0, g["idx_dev"], g["nsel_dev"], wl.topk + wl.window)
    assert tl.max_abs(o2, g["o"]) <= 2e-3


def test_short_context_and_zero_topk():
    wl = WORKLOADS["tiny"].resized(T=50, L=50, n_needles=0, topk=16, window=128)
    _check_block(wl, needles=False)
    wl = WORKLOADS["tiny"].resized(T=40, L=700, n_needles=0, topk=0, window=32)
    _check_block(wl, needles=False)


def test_sparse_empty_selection_gives_zero():
    wl = WORKLOADS["decode_bf16_32k"].resized(B=2, L=512, n_needles=0, n_sparse=1)
    di = tl.DeviceInputs(make_attention_inputs(wl, needles=False))
    idx = -np.ones((2, 16), dtype=np.int32)
    o = tl.run_sparse(di, 0, idx, np.zeros(2, dtype=np.int32), 16)
    assert np.all(o == 0)


def test_sparse_out_of_range_index_is_reported():
    wl = WORKLOADS["decode_bf16_32k"].resized(B=1, L=512, n_needles=0, n_sparse=1)
    di = tl.DeviceInputs(make_attention_inputs(wl, needles=False))
    idx = np.arange(16, dtype=np.int32)[None, :].copy()
    idx[0, 5] = 512 + 40   # past the cache: the kernel must skip it and report
    nsel = np.array([16], dtype=np.int32)
    O = torch.empty(1, 1, wl.H, wl.D, dtype=torch.float32, device="cuda")
    hs2.hs2_sparse_attn(di.q_sparse[0], di.kv, 1, 1, wl.L, wl.H, wl.D, wl.scale, tl.dev(idx),
                        tl.dev(nsel), 16, di.dt, O)
    assert hs2.hs2_last_device_status() == 6
    assert hs2.hs2_last_device_status() == 0   # cleared by the read


def test_chunk_bf16_h32_wide_groups():
    # several queries per sequence with 32 heads: groups of 4 queries x 32 heads
    wl = WORKLOADS["decode_bf16_32k"].resized(B=2, T=70, L=9000, n_needles=20, n_sparse=1)
    rows = np.unique(np.r_[0, 69, 70, 139, np.random.default_rng(2).integers(0, 140, 24)])
    _check_block(wl, rows=rows)


def test_fused_short_context_and_zero_topk():
    # head_dim 128 takes the fused kernel: contexts whose candidates all fit
    # the budget, and a zero budget (the window alone)
    wl = WORKLOADS["decode_bf16_32k"].resized(B=2, T=3, L=100, n_needles=0, topk=16, window=128)
    _check_block(wl, needles=False)
    wl = WORKLOADS["decode_bf16_32k"].resized(B=2, T=2, L=700, n_needles=0, topk=0, window=32)
    _check_block(wl, needles=False)


def test_all_scores_tied_large_context():
    # identical keys: every candidate score is the same pattern, so the
    # selection is decided by position alone (lowest positions first), and the
    # level-1 bin holds every candidate (more than the fused selection keeps
    # in shared memory)
    wl = WORKLOADS["decode_bf16_32k"].resized(B=1, L=65536, n_needles=0, n_sparse=1)
    inp = make_attention_inputs(wl, needles=False)
    inp.k[:] = inp.k[:, :1, :]
    di = tl.DeviceInputs(inp)
    g = tl.run_full(di)
    orc = tl.oracle_full(inp, rows=np.arange(1))
    i = wl.L - 1
    want = np.r_[np.arange(wl.topk), np.arange(i - wl.window + 1, i + 1)]
    assert np.array_equal(orc["idx"][0, : orc["n_sel"][0]], want)
    assert int(g["n_sel"][0]) == want.size
    assert np.array_equal(g["idx"][0, : want.size], want)
    assert tl.max_abs(g["o"][:1], orc["o"]) <= tl.TOL_BF16


def test_chunk_fp8_1m_sampled_rows():
    # the full 4096-query chunk over a 1M-token E4M3 cache (per-token scales with
    # random mantissas), in the launch configuration of that shape; the oracle
    # checks 64 query rows one by one -- the first, the last, 8 rows that own
    # planted needles, and the rest drawn from a seeded stream (they land in
    # different 128-row groups and key splits) -- and all three sparse layers on
    # those rows
    wl = WORKLOADS["chunk_fp8_1m"].resized(fp8_scale="mantissa")
    inp = make_attention_inputs(wl)
    rng = np.random.default_rng(2026)
    needle_rows = sorted({int(t) for _, _, t in inp.needles})
    rows = np.unique(np.r_[0, wl.T - 1, needle_rows[:: max(1, len(needle_rows) // 8)][:8]])
    while rows.size < 64:
        rows = np.unique(np.r_[rows, rng.integers(1, wl.T - 1, 64 - rows.size)])
    _check_block(wl, rows=rows, inp=inp)


def test_decode_bf16_64k_many_tiles_per_split():
    # 29 key tiles per split: more than tensor memory keeps, so the fused
    # kernel's score pass recomputes the logits from K (bf16 cache)
    _check_block(WORKLOADS["decode_bf16_32k"].resized(L=65536, n_needles=32), sparse_layers=[0])


def test_decode_bf16_unaligned_slot_shares():
    # 1000 + 100 slots over a cluster of 8 CTAs: each CTA's 138-slot share
    # starts inside a 16-key group and ends on a partly valid one
    _check_block(WORKLOADS["decode_bf16_32k"].resized(L=8192, topk=1000, window=100,
                                                      n_needles=16))


@pytest.mark.parametrize("H", [8, 16, 32])
@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_sparse_random_index_lists(H, kv):
    # each query gets its own random set of positions (unsorted, any size from
    # 0 to the full budget): tiles end anywhere, clusters split them anywhere,
    # and some queries have no position at all (O = 0)
    name = "decode_bf16_32k" if kv == "bf16" else "decode_fp8_256k"
    wl = WORKLOADS[name].resized(B=3, T=4, L=6000, H=H, n_needles=0, n_sparse=1,
                                 **({"fp8_scale": "mantissa"} if kv == "fp8" else {}))
    inp = make_attention_inputs(wl, needles=False)
    di = tl.DeviceInputs(inp)
    slots = wl.topk + wl.window
    rng = np.random.default_rng(7 + H)
    idx = -np.ones((wl.B * wl.T, slots), dtype=np.int32)
    nsel = np.zeros(wl.B * wl.T, dtype=np.int32)
    sizes = [0, 1, 127, 128, 129, 700, slots, slots - 1, 300, 16, 1000, 5]
    for r in range(wl.B * wl.T):
        n = sizes[r % len(sizes)]
        idx[r, :n] = rng.choice(wl.L, n, replace=False)
        nsel[r] = n
    o_gpu = tl.run_sparse(di, 0, idx, nsel, slots)
    o_orc = tl.oracle_sparse(inp, 0, idx, nsel)
    tol = tl.TOL_FP8 if kv == "fp8" else tl.TOL_BF16
    assert tl.max_abs(o_gpu, o_orc) <= tol
    assert np.all(o_gpu[nsel == 0] == 0)
