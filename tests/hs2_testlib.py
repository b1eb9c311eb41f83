"""Helpers shared by the GPU parity tests: upload seeded inputs, run the CUDA
path through the C ABI, run the oracle on the same bytes, compare."""

import numpy as np
import torch

import long_context_hs2_b200 as hs2
import oracle

TOL_BF16 = 1e-2   # max-abs on O / O' with a bf16 cache
TOL_FP8 = 3e-2    # max-abs with an E4M3 cache
TIE_BAND = 1e-3   # index swaps allowed among scores within this relative band of the k-th


def dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


class DeviceInputs:
    """Inputs of one attention workload resident on the GPU."""

    def __init__(self, inp):
        self.inp = inp
        wl = inp.wl
        self.wl = wl
        self.fp8 = wl.kv_dtype == "fp8"
        self.dt = hs2.HS2_KV_FP8_E4M3 if self.fp8 else hs2.HS2_KV_BF16
        self.q = dev(inp.q.view(np.int16), None).view(torch.bfloat16)
        self.q_sparse = [dev(q.view(np.int16)).view(torch.bfloat16) for q in inp.q_sparse]
        if self.fp8:
            self.k = dev(inp.k)
            self.v = dev(inp.v)
            self.ks = dev(inp.k_scale)
            self.vs = dev(inp.v_scale)
        else:
            self.k = dev(inp.k.view(np.int16)).view(torch.bfloat16)
            self.v = dev(inp.v.view(np.int16)).view(torch.bfloat16)
            self.ks = self.vs = None
        self.kv = hs2.kv_cache(self.k, self.v, self.ks, self.vs)


def run_full(di: DeviceInputs, topk=None, window=None):
    wl = di.wl
    topk = wl.topk if topk is None else topk
    window = wl.window if window is None else window
    B, T, L, H, D = wl.B, wl.T, wl.L, wl.H, wl.D
    ws_bytes = hs2.hs2_full_attn_select_workspace(B, T, L, H, D, topk, window, di.dt)
    assert ws_bytes > 0
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    O = torch.empty(B, T, H, D, dtype=torch.float32, device="cuda")
    lse = torch.empty(B, T, H, dtype=torch.float32, device="cuda")
    idx = torch.empty(B, T, topk + window, dtype=torch.int32, device="cuda")
    nsel = torch.empty(B, T, dtype=torch.int32, device="cuda")
    hs2.hs2_full_attn_select(di.q, di.kv, B, T, L, H, D, wl.scale, topk, window, di.dt, O, lse,
                             idx, nsel, ws, ws_bytes)
    st = hs2.hs2_last_device_status()
    assert st == 0, hs2.hs2_status_string(st)
    return dict(o=O.cpu().numpy().reshape(B * T, H, D), lse=lse.cpu().numpy().reshape(B * T, H),
                idx=idx.cpu().numpy().reshape(B * T, -1), n_sel=nsel.cpu().numpy().reshape(-1),
                idx_dev=idx, nsel_dev=nsel)


def run_sparse(di: DeviceInputs, layer: int, idx, nsel, slots):
    wl = di.wl
    B, T, L, H, D = wl.B, wl.T, wl.L, wl.H, wl.D
    if not torch.is_tensor(idx):
        idx = dev(np.asarray(idx, dtype=np.int32))
        nsel = dev(np.asarray(nsel, dtype=np.int32))
    O = torch.empty(B, T, H, D, dtype=torch.float32, device="cuda")
    hs2.hs2_sparse_attn(di.q_sparse[layer], di.kv, B, T, L, H, D, wl.scale, idx, nsel, slots,
                        di.dt, O)
    st = hs2.hs2_last_device_status()
    assert st == 0, hs2.hs2_status_string(st)
    return O.cpu().numpy().reshape(B * T, H, D)


def oracle_full(inp, rows=None, topk=None, window=None):
    wl = inp.wl
    return oracle.full_attn_select(inp.q, inp.k, inp.v, inp.k_scale, inp.v_scale, scale=wl.scale,
                                   topk=wl.topk if topk is None else topk,
                                   window=wl.window if window is None else window, rows=rows,
                                   want_score=True)


def oracle_sparse(inp, layer, idx, nsel, rows=None):
    wl = inp.wl
    return oracle.sparse_attn(inp.q_sparse[layer], inp.k, inp.v, inp.k_scale, inp.v_scale, idx,
                              nsel, scale=wl.scale, rows=rows)


def check_selection(gpu_idx, gpu_nsel, orc, positions, topk, window, band=TIE_BAND):
    """GPU selected sets against the oracle's.

    Sets must be equal except for swaps among candidates whose oracle score is
    within `band` (relative) of the k-th candidate score.  Returns the number of
    rows whose sets differ (all such differences being inside the band).
    """
    differ = 0
    for r, i in enumerate(positions):
        ns = int(orc["n_sel"][r])
        assert int(gpu_nsel[r]) == ns, (r, int(gpu_nsel[r]), ns)
        g = gpu_idx[r, :ns]
        assert (np.diff(g) > 0).all(), "indices not strictly ascending"
        assert (gpu_idx[r, ns:] == -1).all()
        win = np.arange(max(0, i - window + 1), i + 1)
        assert np.isin(win, g).all(), "forced window missing"
        o = orc["idx"][r, :ns]
        if np.array_equal(g, o):
            continue
        differ += 1
        sc = orc["score"][r]
        cand_sel = o[o <= i - window]
        kth = sc[cand_sel].min()
        for j in np.setxor1d(g, o):
            assert j <= i - window, "non-candidate position differs"
            assert abs(sc[j] - kth) <= band * kth, (r, j, sc[j], kth)
    return differ


def max_abs(a, b) -> float:
    return float(np.max(np.abs(np.asarray(a, dtype=np.float64) - np.asarray(b, dtype=np.float64))))
