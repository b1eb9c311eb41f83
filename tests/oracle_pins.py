"""Checks that pin the CPU oracle to something other than itself.

Each check compares the oracle with an independent source of truth: torch's
CPU casts for the bf16/E4M3 codecs, numpy's float64 matmul for KV Bridging,
torch float64 softmax/logsumexp for attention, numpy's stable lexsort and a
brute-force rank count for the selection, closed forms (probabilities sum to
1 per head, sparse == dense when the context fits the budget, all-equal keys
tie down to the lowest indices), the selection's invariants on the seeded
workloads (planted needles and the forced window always selected) and a
hand-worked fixture under tests/golden.

The checks are plain functions so that the mutation test can run them against
deliberately broken copies of the oracle.
"""

import json
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# --------------------------------------------------- independent decoders --
def dec_bf16(bits) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16))
    return t.view(torch.bfloat16).double().numpy()


def dec_e4m3(codes, scale=None) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8))
    x = t.view(torch.float8_e4m3fn).double().numpy()
    if scale is not None:
        x = x * np.asarray(scale, dtype=np.float64)[..., None]
    return x


def rand_bf16(rng, shape, std=1.0) -> np.ndarray:
    x = torch.from_numpy((rng.standard_normal(shape) * std).astype(np.float32))
    return x.bfloat16().view(torch.int16).numpy().view(np.uint16)


def torch_attention(qf, kf, vf, scale):
    """Dense causal MQA attention in torch float64: queries are the last T positions."""
    q = torch.from_numpy(qf)
    k = torch.from_numpy(kf)
    v = torch.from_numpy(vf)
    B, T, H, D = q.shape
    L = k.shape[1]
    s = torch.einsum("bthd,bld->bthl", q, k) * scale
    pos = torch.arange(L)
    qpos = torch.arange(T) + (L - T)
    mask = pos[None, :] <= qpos[:, None]                      # [T, L]
    s = s.masked_fill(~mask[None, :, None, :], float("-inf"))
    p = torch.softmax(s, dim=-1)
    o = torch.einsum("bthl,bld->bthd", p, v)
    lse = torch.logsumexp(s, dim=-1)
    return o.numpy(), lse.numpy(), p.sum(dim=2).numpy()      # score [B, T, L]


# ----------------------------------------------------------------- codecs --
def check_e4m3_decode():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_f64(codes)
    ref = dec_e4m3(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def check_e4m3_encode():
    vals = dec_e4m3(np.arange(127, dtype=np.uint8))          # 0 .. 448
    mids = (vals[:-1] + vals[1:]) / 2                         # exact ties
    rng = np.random.default_rng(7)
    rnd = (np.exp(rng.uniform(np.log(2.0 ** -11), np.log(448.0), 3000))).astype(np.float32)
    x = np.concatenate([vals, mids, rnd.astype(np.float64), vals * 1.0001, mids * 0.9999])
    x = np.concatenate([x, -x])
    x = x[np.abs(x) <= 448.0].astype(np.float32).astype(np.float64)
    ours = oracle.f64_to_e4m3(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    # torch and the oracle may differ only in the sign of a zero result
    same = (ours == ref) | (((ours & 0x7F) == 0) & ((ref & 0x7F) == 0))
    assert same.all(), x[~same][:10]


def check_e4m3_saturation():
    x = np.array([448.0, 449.0, 464.0, 480.0, 1e6, -449.0, -1e9])
    assert list(oracle.f64_to_e4m3(x)) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]


def check_bf16_codec():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    sub = bits[::7]
    ref = dec_bf16(sub)
    fin = np.isfinite(ref)
    ours = oracle.bf16_to_f64(sub)
    assert np.array_equal(ours[fin], ref[fin])
    rng = np.random.default_rng(3)
    x = rng.standard_normal(2000).astype(np.float32) * np.exp2(rng.integers(-20, 20, 2000)).astype(np.float32)
    b = torch.from_numpy(x).bfloat16().view(torch.int16).numpy().view(np.uint16)
    exact = dec_bf16(b)
    # exact halfway points between neighbouring bf16 values (representable in fp32)
    nb = dec_bf16((b.astype(np.uint32) + 1).astype(np.uint16))
    half = ((exact + nb) / 2).astype(np.float32)
    xs = np.concatenate([x, half]).astype(np.float32)
    ref_b = torch.from_numpy(xs).bfloat16().view(torch.int16).numpy().view(np.uint16)
    ours_b = oracle.f64_to_bf16(xs.astype(np.float64))
    assert np.array_equal(ours_b, ref_b)


# ----------------------------------------------------------- KV Bridging --
def check_bridge_numpy():
    rng = np.random.default_rng(11)
    T, hidden, nl, D = 37, 96, 2, 16
    x = rand_bf16(rng, (T, hidden))
    wt = rand_bf16(rng, (nl * 2 * D, hidden), std=0.1)
    rows = np.array([0, 5, 36, 17, 17], dtype=np.int64)
    r = oracle.bridge(x, wt, nl, D, rows)
    y_ref = dec_bf16(x)[rows] @ dec_bf16(wt).T
    assert np.allclose(r["y"], y_ref, rtol=1e-12, atol=1e-14)
    for l in range(nl):
        for kv, name in ((0, "k"), (1, "v")):
            seg = y_ref[:, l * 2 * D + kv * D: l * 2 * D + (kv + 1) * D]
            # bf16: the nearest bf16 value to y (neighbours one code away are no closer)
            got = r[name + "_bf16"][l]
            g = dec_bf16(got)
            up = dec_bf16((got.astype(np.int32) + 1).astype(np.uint16))
            dn = dec_bf16((got.astype(np.int32) - 1).astype(np.uint16))
            assert (np.abs(g - seg) <= np.abs(up - seg) + 1e-300).all()
            assert (np.abs(g - seg) <= np.abs(dn - seg) + 1e-300).all()
            # fp8: scale = amax / 448 per token; the largest magnitude maps to code 448
            amax = np.abs(seg).max(axis=1)
            assert np.allclose(r[name + "_scale"][l], amax / 448.0, rtol=1e-14)
            codes = r[name + "_fp8"][l]
            ref = torch.from_numpy((seg / (amax / 448.0)[:, None]).astype(np.float32)).to(
                torch.float8_e4m3fn).view(torch.uint8).numpy()
            assert (codes == ref).mean() > 0.99
            deq = dec_e4m3(codes, r[name + "_scale"][l])
            assert np.allclose(deq, seg, rtol=2.0 ** -4, atol=amax[:, None] * 2.0 ** -10)
            assert (np.abs(dec_e4m3(codes)).max(axis=1) == 448.0).all()


def check_bridge_identity():
    rng = np.random.default_rng(12)
    T, hidden, nl, D = 9, 64, 3, 8
    x = rand_bf16(rng, (T, hidden))
    wt = np.zeros((nl * 2 * D, hidden), dtype=np.uint16)
    src = (np.arange(nl * 2 * D) * 5 + 3) % hidden
    wt[np.arange(nl * 2 * D), src] = 0x3F80                    # bf16 1.0
    r = oracle.bridge(x, wt, nl, D)
    for l in range(nl):
        assert np.array_equal(r["k_bf16"][l], x[:, src[l * 2 * D: l * 2 * D + D]])
        assert np.array_equal(r["v_bf16"][l], x[:, src[l * 2 * D + D: (l + 1) * 2 * D]])


# -------------------------------------------------------------- attention --
def _small_attn(rng, B, T, L, H, D, fp8):
    q = rand_bf16(rng, (B, T, H, D))
    if fp8:
        from hs2_synth import fp8_quantise_pow2
        k, ks = fp8_quantise_pow2(rng.standard_normal((B, L, D)))
        v, vs = fp8_quantise_pow2(rng.standard_normal((B, L, D)))
        kf, vf = dec_e4m3(k, ks), dec_e4m3(v, vs)
    else:
        k, v = rand_bf16(rng, (B, L, D)), rand_bf16(rng, (B, L, D))
        ks = vs = None
        kf, vf = dec_bf16(k), dec_bf16(v)
    return q, k, v, ks, vs, dec_bf16(q), kf, vf


def check_attention_vs_torch():
    rng = np.random.default_rng(21)
    for fp8 in (False, True):
        B, T, H, D, L = 2, 5, 4, 16, 300
        q, k, v, ks, vs, qf, kf, vf = _small_attn(rng, B, T, L, H, D, fp8)
        sc = 1 / np.sqrt(D)
        r = oracle.full_attn_select(q, k, v, ks, vs, scale=sc, topk=16, window=8, want_score=True)
        o_ref, lse_ref, score_ref = torch_attention(qf, kf, vf, sc)
        assert np.allclose(r["o"], o_ref.reshape(B * T, H, D), rtol=1e-11, atol=1e-13)
        assert np.allclose(r["lse"], lse_ref.reshape(B * T, H), rtol=1e-12, atol=1e-12)
        assert np.allclose(r["score"], score_ref.reshape(B * T, L), rtol=1e-11, atol=1e-15)


def check_scores_sum_to_heads():
    rng = np.random.default_rng(22)
    B, T, H, D, L = 1, 7, 8, 32, 500
    q, k, v, ks, vs, *_ = _small_attn(rng, B, T, L, H, D, False)
    r = oracle.full_attn_select(q, k, v, scale=0.3, topk=64, window=16, want_score=True)
    assert np.allclose(r["score"].sum(axis=1), H, rtol=0, atol=1e-12)


# -------------------------------------------------------------- selection --
def _lexsort_select(score, i, topk, window):
    cand = np.arange(0, max(0, i - window + 1))
    order = np.lexsort((cand, -score[cand]))                  # score desc, then index asc
    top = cand[order[:topk]]
    win = np.arange(max(0, i - window + 1), i + 1)
    return np.sort(np.concatenate([top, win]))


def check_select_vs_lexsort():
    rng = np.random.default_rng(31)
    for trial in range(60):
        n = int(rng.integers(1, 400))
        score = rng.integers(0, 6, n).astype(np.float64)      # many exact ties
        if trial % 2:
            score = rng.random(n)
        i = n - 1
        topk = int(rng.integers(0, 40))
        window = int(rng.integers(1, 20))
        idx, ns = oracle.select(score, i, topk, window)
        ref = _lexsort_select(score, i, topk, window)
        assert ns == len(ref)
        assert np.array_equal(idx[:ns], ref)
        assert (idx[ns:] == -1).all()


def check_select_bruteforce_rank():
    rng = np.random.default_rng(32)
    topk, window = 16, 8
    for L, H in ((300, 4), (64, 2), (20, 1)):
        B, T, D = 1, min(L, 12), 16
        q, k, v, ks, vs, qf, kf, vf = _small_attn(rng, B, T, L, H, D, False)
        r = oracle.full_attn_select(q, k, v, scale=0.25, topk=topk, window=window)
        _, _, score = torch_attention(qf, kf, vf, 0.25)
        for t in range(T):
            i = L - T + t
            s = score[0, t]
            cand = range(0, i - window + 1)
            chosen = set()
            for j in cand:
                rank = sum(1 for m in cand if s[m] > s[j] or (s[m] == s[j] and m < j))
                if rank < topk:
                    chosen.add(j)
            chosen |= set(range(max(0, i - window + 1), i + 1))
            ns = r["n_sel"][t]
            assert ns == len(chosen) == min(topk + window, i + 1)
            assert set(r["idx"][t, :ns].tolist()) == chosen


def check_all_equal_keys():
    D, H, L = 16, 4, 2000
    q = rand_bf16(np.random.default_rng(33), (1, 1, H, D))
    k = np.tile(rand_bf16(np.random.default_rng(34), (1, 1, D)), (1, L, 1))
    v = rand_bf16(np.random.default_rng(35), (1, L, D))
    r = oracle.full_attn_select(q, k, v, scale=0.25, topk=1024, window=128, want_score=True)
    assert np.allclose(r["score"][0], H / L, rtol=1e-12)
    expect = np.concatenate([np.arange(1024), np.arange(L - 128, L)])
    assert np.array_equal(r["idx"][0], expect)


# ------------------------------------------- context-parallel slice --
def check_slice_of_the_whole_cache_is_full_attention():
    rng = np.random.default_rng(61)
    for fp8 in (False, True):
        B, T, H, D, L = 2, 6, 4, 16, 260
        q, k, v, ks, vs, *_ = _small_attn(rng, B, T, L, H, D, fp8)
        r = oracle.full_attn_select(q, k, v, ks, vs, scale=0.3, topk=16, window=8, want_score=True)
        sl = oracle.attn_slice(q, k, v, ks, vs, qpos=L - T, scale=0.3, window=8, want_score=True)
        assert np.allclose(sl["o"], r["o"], rtol=1e-12, atol=1e-14)
        assert np.allclose(sl["lse"], r["lse"], rtol=1e-13, atol=1e-13)
        cand = np.arange(L)[None, :] <= (L - T + np.tile(np.arange(T), B))[:, None] - 8
        assert np.allclose(sl["score"], np.where(cand, r["score"], 0.0), rtol=1e-11, atol=1e-15)


def check_slice_vs_torch():
    # slices that lie before, around and after the queries, with a given
    # normaliser for the scores
    rng = np.random.default_rng(62)
    B, T, H, D, Ls, window = 1, 5, 3, 8, 40, 4
    q, k, v, ks, vs, qf, kf, vf = _small_attn(rng, B, T, Ls, H, D, False)
    lse_in = rng.normal(3.0, 1.0, (B * T, H))
    for qpos in (100, 38, 20, 2, -3):
        sl = oracle.attn_slice(q, k, v, qpos=qpos, scale=0.4, window=window, lse_in=lse_in,
                               want_score=True)
        s = torch.einsum("thd,ld->thl", torch.from_numpy(qf[0]), torch.from_numpy(kf[0])) * 0.4
        pos = torch.arange(Ls)
        i = qpos + torch.arange(T)
        vis = pos[None, :] <= i[:, None]                                    # [T, Ls]
        sm = s.masked_fill(~vis[:, None, :], float("-inf"))
        lse = torch.logsumexp(sm, -1)                                       # -inf: no key
        p = torch.where(vis[:, None, :], torch.exp(sm - lse[..., None]), torch.zeros(()))
        o = torch.einsum("thl,ld->thd", p, torch.from_numpy(vf[0]))
        cand = pos[None, :] <= (i - window)[:, None]
        sc = torch.exp(s - torch.from_numpy(lse_in)[..., None]).sum(1)
        sc = torch.where(cand, sc, torch.zeros(()))
        assert np.array_equal(np.isneginf(sl["lse"]), np.isneginf(lse.numpy()))
        fin = np.isfinite(lse.numpy())
        assert np.allclose(sl["lse"][fin], lse.numpy()[fin], rtol=1e-13)
        assert np.allclose(sl["o"], o.numpy(), rtol=1e-11, atol=1e-14)
        assert np.allclose(sl["score"], sc.numpy(), rtol=1e-11, atol=1e-15)


# -------------------------------------------------- block-level selection --
def check_select_blocks_of_one_are_token_level():
    # blocks of a single position are the token-level selection (pinned above
    # against numpy's lexsort; compared with it directly here)
    rng = np.random.default_rng(51)
    for trial in range(40):
        n = int(rng.integers(1, 300))
        score = rng.integers(0, 5, n).astype(np.float64) if trial % 2 else rng.random(n)
        topk, window = int(rng.integers(0, 40)), int(rng.integers(1, 20))
        idx, ns = oracle.select_blocks(score, n - 1, topk, window, block=1)
        ref = _lexsort_select(score, n - 1, topk, window)
        assert ns == len(ref) and np.array_equal(idx[:ns], ref)


def check_select_blocks_bruteforce_rank():
    # a block is kept iff fewer than topk/block candidate blocks outrank it
    # (larger summed score, or equal and lower index): pairwise counts, no sort
    rng = np.random.default_rng(52)
    for trial in range(60):
        n = int(rng.integers(1, 400))
        block = int(rng.choice([2, 3, 4, 8, 64]))
        score = rng.integers(0, 3, n).astype(np.float64) if trial % 3 == 0 else rng.random(n)
        window = int(rng.integers(1, 30))
        kb = int(rng.integers(0, 12))
        i = n - 1
        idx, ns = oracle.select_blocks(score, i, kb * block, window, block=block)
        last = i - window
        sums = {}
        for j in range(0, last + 1):
            sums[j // block] = sums.get(j // block, 0.0) + score[j]
        chosen = set()
        for b, sb in sums.items():
            rank = sum(1 for c, sc in sums.items() if sc > sb or (sc == sb and c < b))
            if rank < kb:
                chosen |= {j for j in range(b * block, (b + 1) * block) if j <= last}
        chosen |= set(range(max(0, i - window + 1), i + 1))
        assert ns == len(chosen)
        assert idx[:ns].tolist() == sorted(chosen) and (idx[ns:] == -1).all()


def check_golden_worked_block_selection():
    with open(os.path.join(GOLDEN, "worked_block_selection.json")) as f:
        g = json.load(f)
    score = np.array(g["score"], dtype=np.float64)
    for case in g["cases"]:
        idx, ns = oracle.select_blocks(score, g["i"], case["topk"], g["window"], g["block"])
        assert idx[:ns].tolist() == case["selected"]
    idx, ns = oracle.select(score, g["i"], 4, g["window"])
    assert idx[:ns].tolist() == g["token_level_topk4"]


def check_planted_needles_and_window():
    # invariants of the selection on the seeded workloads' own inputs: every
    # planted needle key (k = 4*sqrt(D) times the unit head-sum of a later
    # query, outside that query's window) is selected for its query, the last
    # `window` positions are always present, and the set holds min(i + 1,
    # topk + window) distinct positions <= i
    from hs2_synth import WORKLOADS, make_attention_inputs
    for name, kw in (("decode_bf16_32k", dict(B=2, L=2600, n_needles=6, n_sparse=0)),
                     ("decode_fp8_256k", dict(B=1, L=3100, n_needles=8, n_sparse=0,
                                              fp8_scale="mantissa")),
                     ("tiny", dict(T=300, L=1400, n_needles=5, n_sparse=0))):
        wl = WORKLOADS[name].resized(**kw)
        inp = make_attention_inputs(wl)
        assert len(inp.needles) == wl.B * wl.n_needles
        rows = np.unique([int(b) * wl.T + int(t) for b, _, t in inp.needles] + [0, wl.B * wl.T - 1])
        r = oracle.full_attn_select(inp.q, inp.k, inp.v, inp.k_scale, inp.v_scale, scale=wl.scale,
                                    topk=wl.topk, window=wl.window, rows=rows)
        for k_, row in enumerate(rows):
            i = wl.L - wl.T + int(row) % wl.T
            sel = r["idx"][k_, :r["n_sel"][k_]]
            assert r["n_sel"][k_] == min(i + 1, wl.topk + wl.window)
            assert len(set(sel.tolist())) == len(sel) and sel.min() >= 0 and sel.max() <= i
            assert set(range(max(0, i - wl.window + 1), i + 1)) <= set(sel.tolist())
        for b, j, t in inp.needles:
            k_ = int(np.searchsorted(rows, int(b) * wl.T + int(t)))
            assert int(j) in r["idx"][k_, :r["n_sel"][k_]], (name, b, j, t)


# ------------------------------------------------------------ sparse layer --
def check_sparse_equals_dense():
    rng = np.random.default_rng(41)
    for fp8 in (False, True):
        B, T, H, D, L = 2, 40, 4, 32, 1100                   # L <= 1024 + 128: all selected
        q, k, v, ks, vs, *_ = _small_attn(rng, B, T, L, H, D, fp8)
        r = oracle.full_attn_select(q, k, v, ks, vs, scale=0.17)
        assert (r["n_sel"] == L - T + np.tile(np.arange(T), B) + 1).all()
        o2 = oracle.sparse_attn(q, k, v, ks, vs, r["idx"], r["n_sel"], scale=0.17)
        assert np.array_equal(o2, r["o"])


def check_sparse_vs_torch():
    rng = np.random.default_rng(42)
    B, T, H, D, L, slots = 2, 3, 4, 16, 200, 40
    q, k, v, ks, vs, qf, kf, vf = _small_attn(rng, B, T, L, H, D, True)
    idx = -np.ones((B * T, slots), dtype=np.int32)
    nsel = np.zeros(B * T, dtype=np.int32)
    for r_ in range(B * T):
        n = int(rng.integers(1, slots + 1))
        idx[r_, :n] = np.sort(rng.choice(L, n, replace=False))
        nsel[r_] = n
    o = oracle.sparse_attn(q, k, v, ks, vs, idx, nsel, scale=0.2)
    for r_ in range(B * T):
        b, t = divmod(r_, T)
        sel = idx[r_, :nsel[r_]]
        s = torch.from_numpy(qf[b, t]) @ torch.from_numpy(kf[b, sel]).T * 0.2
        ref = torch.softmax(s, -1) @ torch.from_numpy(vf[b, sel])
        assert np.allclose(o[r_], ref.numpy(), rtol=1e-12, atol=1e-14)


# ------------------------------------------------------ hand-worked case --
def check_golden_worked_example():
    with open(os.path.join(GOLDEN, "worked_selection.json")) as f:
        g = json.load(f)
    q = oracle.f64_to_bf16(np.array(g["q"], dtype=np.float64)).reshape(1, 1, 1, -1)
    k = oracle.f64_to_bf16(np.array(g["k"], dtype=np.float64)).reshape(1, -1, len(g["q"]))
    v = oracle.f64_to_bf16(np.array(g["v"], dtype=np.float64)).reshape(1, -1, len(g["q"]))
    for case in g["cases"]:
        r = oracle.full_attn_select(q, k, v, scale=g["scale"], topk=case["topk"],
                                    window=case["window"])
        ns = r["n_sel"][0]
        assert r["idx"][0, :ns].tolist() == case["selected"]
        assert abs(r["lse"][0, 0] - g["lse"]) < 1e-12
        assert abs(r["o"][0, 0, 0] - g["o0"]) < 1e-12


ALL_CHECKS = [
    check_e4m3_decode, check_e4m3_encode, check_e4m3_saturation, check_bf16_codec,
    check_bridge_numpy, check_bridge_identity, check_attention_vs_torch,
    check_scores_sum_to_heads, check_select_vs_lexsort, check_select_bruteforce_rank,
    check_all_equal_keys, check_sparse_equals_dense, check_sparse_vs_torch,
    check_golden_worked_example, check_select_blocks_of_one_are_token_level,
    check_select_blocks_bruteforce_rank, check_golden_worked_block_selection,
    check_slice_of_the_whole_cache_is_full_attention, check_slice_vs_torch,
    check_planted_needles_and_window,
]
