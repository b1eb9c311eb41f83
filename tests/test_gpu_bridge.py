"""GPU parity of hs2_bridge_kv (KV Bridging on tcgen05) against the oracle.

bf16 caches: the GPU accumulates in fp32 and rounds once to bf16; the oracle
accumulates in fp64.  The bound used is |gpu - y| <= 2^-8 |y| + 2^-8 * 2^-6:
half a bf16 ulp (2^-9 relative) of rounding, doubled for the fp32-vs-fp64
difference of the sum, plus an absolute term for values near zero (outputs
are ~N(0, 1/64^2)).  The max-abs 1e-2 acceptance bound is also checked.
E4M3 caches: a code is a rounding decision taken on Y/s.  The GPU takes it on
its fp32 accumulation of Y, the oracle on the exact (fp64) Y; the two differ
by at most eps = 2^-20 * sum_k |x_k w_k| (a few fp32 ulps of the sum of the
product magnitudes).  So a GPU code is valid when it is the round-to-nearest
E4M3 code of some value in [(Y - eps)/s, (Y + eps)/s].  Where eps is tiny next
to a code step (most values) this is the exact code; for values far below the
row maximum (E4M3 subnormals) it admits the neighbouring codes.  Scales must
agree to 1e-5 relative.
"""

import numpy as np
import pytest
import torch

import long_context_hs2_b200 as hs2
import oracle
from hs2_synth import WORKLOADS, make_bridge_inputs
import oracle_pins as P

pytestmark = pytest.mark.gpu


def _run(bi, fp8, row_offset=0, total_rows=None):
    wl = bi.wl
    T, hidden, nl, D = wl.T, wl.hidden, wl.n_layers, wl.D
    rows = T + row_offset if total_rows is None else total_rows
    x = torch.from_numpy(bi.x.view(np.int16)).cuda().view(torch.bfloat16)
    wt = torch.from_numpy(bi.wt.view(np.int16)).cuda().view(torch.bfloat16)
    caches, keep = [], []
    for _ in range(nl):
        if fp8:
            k = torch.full((rows, D), 0x55, dtype=torch.uint8, device="cuda")
            v = torch.full((rows, D), 0x55, dtype=torch.uint8, device="cuda")
            ks = torch.full((rows,), -1.0, device="cuda")
            vs = torch.full((rows,), -1.0, device="cuda")
        else:
            k = torch.full((rows, D), 7.0, dtype=torch.bfloat16, device="cuda")
            v = torch.full((rows, D), 7.0, dtype=torch.bfloat16, device="cuda")
            ks = vs = None
        keep.append((k, v, ks, vs))
        caches.append(hs2.kv_cache(k, v, ks, vs))
    hs2.hs2_bridge_kv(x, T, hidden, wt, nl, D,
                      hs2.HS2_KV_FP8_E4M3 if fp8 else hs2.HS2_KV_BF16, caches, row_offset)
    st = hs2.hs2_last_device_status()
    assert st == 0, hs2.hs2_status_string(st)
    out = []
    for k, v, ks, vs in keep:
        if fp8:
            out.append((k.cpu().numpy(), v.cpu().numpy(), ks.cpu().numpy(), vs.cpu().numpy()))
        else:
            out.append((k.view(torch.int16).cpu().numpy().view(np.uint16),
                        v.view(torch.int16).cpu().numpy().view(np.uint16), None, None))
    return out


def _check_bf16(gpu, orc, rows_gpu, l):
    for kv in (0, 1):
        y = orc["y"][:, l * 256 + kv * 128: l * 256 + (kv + 1) * 128]
        g = P.dec_bf16(gpu[l][kv][rows_gpu])
        err = np.abs(g - y)
        assert (err <= 2.0 ** -8 * np.abs(y) + 2.0 ** -14).all(), err.max()
        assert err.max() <= 1e-2


def _e4m3_rne(y):
    """RNE E4M3 code of float64 values (|y| <= 448) via torch's float32 cast."""
    y = np.clip(y, -448.0, 448.0)
    return torch.from_numpy(y.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _check_fp8(gpu, orc, rows_gpu, l, eps):
    vals = P.dec_e4m3(np.arange(256, dtype=np.uint8))
    for kv, name in ((0, "k"), (1, "v")):
        codes = gpu[l][kv][rows_gpu]
        scale = gpu[l][2 + kv][rows_gpu]
        oc = orc[name + "_fp8"][l]
        osc = orc[name + "_scale"][l]
        assert np.allclose(scale, osc, rtol=1e-5, atol=0)
        cols = slice(l * 256 + kv * 128, l * 256 + (kv + 1) * 128)
        y = orc["y"][:, cols]
        e = eps[:, cols]
        lo = vals[_e4m3_rne((y - e) / osc[:, None])]
        hi = vals[_e4m3_rne((y + e) / osc[:, None])]
        g = vals[codes]
        ok = (g >= np.minimum(lo, hi)) & (g <= np.maximum(lo, hi))
        assert ok.all(), (np.argwhere(~ok)[:5], g[~ok][:5], (y / osc[:, None])[~ok][:5])
        # every code is valid (above); codes off the oracle's own are the rare
        # rounding decisions within eps of a midpoint
        assert (codes != oc).sum() <= max(1, 1e-3 * codes.size)
        deq = P.dec_e4m3(codes, scale)
        assert np.abs(deq - y).max() <= 3e-2


def _eps(bi, rows):
    """2^-20 * sum_k |x_k w_k| for the given rows (bound on fp32-vs-exact Y)."""
    xa = np.abs(P.dec_bf16(bi.x[rows]))
    wa = np.abs(P.dec_bf16(bi.wt))
    return 2.0 ** -20 * (xa @ wa.T)


@pytest.mark.parametrize("fp8", [False, True])
def test_bridge_small_ragged(fp8):
    wl = WORKLOADS["bridge_131k"].resized(T=300, hidden=512, n_layers=3)
    bi = make_bridge_inputs(wl)
    gpu = _run(bi, fp8)
    orc = oracle.bridge(bi.x, bi.wt, wl.n_layers, wl.D)
    eps = _eps(bi, np.arange(wl.T)) if fp8 else None
    for l in range(wl.n_layers):
        if fp8:
            _check_fp8(gpu, orc, np.arange(wl.T), l, eps)
        else:
            _check_bf16(gpu, orc, np.arange(wl.T), l)


def test_bridge_row_offset_appends_in_place():
    wl = WORKLOADS["bridge_131k"].resized(T=130, hidden=256, n_layers=2)
    bi = make_bridge_inputs(wl)
    off, total = 37, 300
    gpu = _run(bi, False, row_offset=off, total_rows=total)
    orc = oracle.bridge(bi.x, bi.wt, wl.n_layers, wl.D)
    for l in range(wl.n_layers):
        _check_bf16(gpu, orc, np.arange(wl.T) + off, l)
        for kv in (0, 1):
            untouched = np.r_[0:off, off + wl.T:total]
            assert (gpu[l][kv][untouched] == 0x40E0).all()   # bf16 7.0 left as it was


@pytest.mark.parametrize("fp8", [False, True])
def test_bridge_full_size_sampled_rows(fp8):
    wl = WORKLOADS["bridge_131k"]
    bi = make_bridge_inputs(wl)
    gpu = _run(bi, fp8)
    rng = np.random.default_rng(5)
    rows = np.unique(np.r_[0, 127, 128, wl.T - 1, rng.integers(0, wl.T, 1020)])
    orc = oracle.bridge(bi.x, bi.wt, wl.n_layers, wl.D, rows=rows)
    eps = _eps(bi, rows) if fp8 else None
    for l in range(wl.n_layers):
        if fp8:
            _check_fp8(gpu, orc, rows, l, eps)
        else:
            _check_bf16(gpu, orc, rows, l)


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("T", [1, 7, 33, 64])
def test_bridge_decode_append_few_tokens(T, fp8):
    # the decode-time append: T new tokens bridged into all six target layers at
    # the full hidden size, written at a row offset of an existing cache (the
    # few-token path: clusters over the hidden dimension); rows outside the
    # append must be left as they were
    wl = WORKLOADS["bridge_131k"].resized(T=T, seed=WORKLOADS["bridge_131k"].seed + T)
    bi = make_bridge_inputs(wl)
    off, total = 4093, 4093 + T + 5
    gpu = _run(bi, fp8, row_offset=off, total_rows=total)
    orc = oracle.bridge(bi.x, bi.wt, wl.n_layers, wl.D)
    eps = _eps(bi, np.arange(wl.T)) if fp8 else None
    untouched = np.r_[0:off, off + T:total]
    for l in range(wl.n_layers):
        if fp8:
            _check_fp8(gpu, orc, np.arange(T) + off, l, eps)
            for kv in (0, 1):
                assert (gpu[l][kv][untouched] == 0x55).all()
                assert (gpu[l][2 + kv][untouched] == -1.0).all()
        else:
            _check_bf16(gpu, orc, np.arange(T) + off, l)
            for kv in (0, 1):
                assert (gpu[l][kv][untouched] == 0x40E0).all()


@pytest.mark.parametrize("fp8", [False, True])
def test_bridge_few_tokens_small_hidden(fp8):
    # hidden 256 is 4 slices of 64: half of each segment's cluster has no slice
    # of the hidden dimension and contributes zeros to the reduction
    wl = WORKLOADS["bridge_131k"].resized(T=5, hidden=256, n_layers=2)
    bi = make_bridge_inputs(wl)
    gpu = _run(bi, fp8, row_offset=3, total_rows=11)
    orc = oracle.bridge(bi.x, bi.wt, wl.n_layers, wl.D)
    eps = _eps(bi, np.arange(wl.T)) if fp8 else None
    for l in range(wl.n_layers):
        if fp8:
            _check_fp8(gpu, orc, np.arange(wl.T) + 3, l, eps)
        else:
            _check_bf16(gpu, orc, np.arange(wl.T) + 3, l)
