"""Context-parallel full attention with selection, orchestrated across two
gloo ranks on CPU.

long_context_hs2_b200.cp runs one full-attention layer over a context split
into contiguous slices, one per rank: partial attention per slice, an
all-gather of the slices' normalisers and their log-sum-exp, a rescale and sum
all-reduce of the partial outputs, a per-slice top-k under the global
normaliser, an all-gather of the candidate lists and a merge.  Here its five
arithmetic steps are done on the host in float64 (the oracle's slice function
and numpy; the GPU kernels of the same steps have their own GPU test), so that
this test checks the decomposition and the orchestration -- slices, the order
of the collectives, the rank order of the gathered lists -- against the
oracle's single-device full attention and selection on the whole cache:
O and lse to 1e-9, selected sets equal except swaps among candidates whose
oracle score lies within 1e-9 (relative) of the k-th candidate score.
"""

import multiprocessing as mp
import os
import socket

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = {
    # name: (B, T, L, H, D, topk, window, slice boundaries)
    "even": (2, 24, 600, 4, 16, 64, 16, [0, 300, 600]),
    # the second slice is shorter than the chunk of queries and starts inside it
    "chunk_spans_slices": (1, 40, 100, 4, 16, 16, 8, [0, 70, 100]),
    # an uneven two-way split
    "uneven": (2, 3, 900, 8, 32, 128, 32, [0, 100, 900]),
}


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class HostOps:
    """The five steps of long_context_hs2_b200.cp on host tensors, float64."""

    def __init__(self, q_bits, k, v):
        import torch
        self.float_dtype = torch.float64
        self.q_bits, self.k, self.v = q_bits, k, v

    def partial(self, q, kv, s, o, lse):
        import oracle
        r = oracle.attn_slice(self.q_bits, self.k, self.v, qpos=s.q_pos0 - s.key_pos0,
                              scale=s.scale, window=s.window)
        o.copy_(_t(r["o"].reshape(o.shape)))
        lse.copy_(_t(r["lse"].reshape(lse.shape)))

    def lse_combine(self, lse_parts, lse):
        x = lse_parts.numpy()
        m = x.max(axis=0)
        with np.errstate(invalid="ignore"):
            acc = np.where(np.isneginf(m), 0.0, np.exp(x - np.where(np.isneginf(m), 0.0, m)).sum(0))
        lse.copy_(_t(np.where(np.isneginf(m), -np.inf, m + np.log(np.where(acc > 0, acc, 1.0)))))

    def rescale(self, o, lse_part, lse):
        lp, lg = lse_part.numpy(), lse.numpy()
        f = np.where(np.isneginf(lp), 0.0, np.exp(lp - np.where(np.isneginf(lp), 0.0, lg)))
        o.mul_(_t(f[..., None]))

    def select_local(self, q, kv, s, lse, cand_score, cand_idx):
        import oracle
        qloc = s.q_pos0 - s.key_pos0
        r = oracle.attn_slice(self.q_bits, self.k, self.v, qpos=qloc, scale=s.scale,
                              window=s.window, lse_in=lse.numpy().reshape(s.B * s.T, s.H),
                              want_score=True)
        cs = np.full((s.B * s.T, s.topk), -1.0)
        ci = np.full((s.B * s.T, s.topk), -1, dtype=np.int32)
        for row in range(s.B * s.T):
            t = row % s.T
            last = min(s.L_local - 1, qloc + t - s.window)
            cand = np.arange(0, last + 1)
            top = cand[np.lexsort((cand, -r["score"][row, cand]))[: s.topk]]
            top = np.sort(top)
            cs[row, : top.size] = r["score"][row, top]
            ci[row, : top.size] = top + s.key_pos0
        cand_score.copy_(_t(cs.reshape(cand_score.shape)))
        cand_idx.copy_(_t(ci.reshape(cand_idx.shape)))

    def merge_select(self, cand_scores, cand_idxs, s, idx, n_sel):
        sc = cand_scores.numpy().reshape(cand_scores.shape[0], s.B * s.T, s.topk)
        ci = cand_idxs.numpy().reshape(cand_idxs.shape[0], s.B * s.T, s.topk)
        out = np.full((s.B * s.T, s.topk + s.window), -1, dtype=np.int32)
        ns = np.zeros(s.B * s.T, dtype=np.int32)
        for row in range(s.B * s.T):
            i = s.q_pos0 + row % s.T
            v = ci[:, row].ravel() >= 0
            pos, score = ci[:, row].ravel()[v], sc[:, row].ravel()[v]
            top = pos[np.lexsort((pos, -score))[: s.topk]]
            sel = np.sort(np.r_[top, np.arange(max(0, i - s.window + 1), i + 1)])
            out[row, : sel.size] = sel
            ns[row] = sel.size
        idx.copy_(_t(out.reshape(idx.shape)))
        n_sel.copy_(_t(ns.reshape(n_sel.shape)))


def _t(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a))


def _worker(rank, world, port, case, out):
    import datetime
    import torch
    import torch.distributed as dist
    from hs2_synth import WORKLOADS, make_attention_inputs
    from long_context_hs2_b200 import cp

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        B, T, L, H, D, topk, window, bounds = CASES[case]
        wl = WORKLOADS["decode_bf16_32k"].resized(B=B, T=T, L=L, H=H, D=D, topk=topk,
                                                  window=window, n_needles=3, n_sparse=0)
        inp = make_attention_inputs(wl)
        a, b = bounds[rank], bounds[rank + 1]
        ops = HostOps(inp.q, np.ascontiguousarray(inp.k[:, a:b]), np.ascontiguousarray(inp.v[:, a:b]))
        s = cp.CpSlice(B=B, T=T, H=H, D=D, L_local=b - a, key_pos0=a, q_pos0=L - T,
                       scale=wl.scale, topk=topk, window=window)
        q = torch.zeros(1)   # the host ops read the queries' bits themselves
        o, lse, idx, ns = cp.cp_full_attn_select(q, None, s, ops)
        out.put((rank, o.numpy(), lse.numpy(), idx.numpy(), ns.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", sorted(CASES))
def test_two_ranks_match_the_whole_cache(case):
    import oracle
    from hs2_synth import WORKLOADS, make_attention_inputs

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, case, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        r, *vals = q.get(timeout=300)
        res[r] = vals
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    B, T, L, H, D, topk, window, _ = CASES[case]
    wl = WORKLOADS["decode_bf16_32k"].resized(B=B, T=T, L=L, H=H, D=D, topk=topk, window=window,
                                              n_needles=3, n_sparse=0)
    inp = make_attention_inputs(wl)
    orc = oracle.full_attn_select(inp.q, inp.k, inp.v, scale=wl.scale, topk=topk, window=window,
                                  want_score=True)
    for r in (0, 1):   # every rank ends with the same results
        o, lse, idx, ns = res[r]
        assert np.allclose(o.reshape(B * T, H, D), orc["o"], rtol=1e-9, atol=1e-12)
        assert np.allclose(lse.reshape(B * T, H), orc["lse"], rtol=1e-12, atol=1e-12)
        idx = idx.reshape(B * T, -1)
        ns = ns.reshape(-1)
        assert np.array_equal(ns, orc["n_sel"])
        for row in range(B * T):
            g, o_ = idx[row, : ns[row]], orc["idx"][row, : ns[row]]
            if np.array_equal(g, o_):
                continue
            i = L - T + row % T
            sc = orc["score"][row]
            kth = sc[o_[o_ <= i - window]].min()
            for j in np.setxor1d(g, o_):
                assert abs(sc[j] - kth) <= 1e-9 * kth
