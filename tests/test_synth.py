"""The seeded input generator's storage-format packing (CPU).

The E4M3 packing with random-mantissa scales must give scales that are not
powers of two, codes that never saturate or encode NaN, and stored values
(decoded with torch's own float8 cast, independent of the packer) within half
an E4M3 step of the value they stand for.
"""

import numpy as np
import torch

from hs2_synth import WORKLOADS, make_attention_inputs


def _dec(codes, scale):
    x = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double().numpy()
    return x * scale.astype(np.float64)[..., None]


def test_mantissa_scales_pack_within_half_a_step():
    wl = WORKLOADS["decode_fp8_256k"].resized(B=2, L=3001, n_needles=5, fp8_scale="mantissa")
    inp = make_attention_inputs(wl)
    for codes, scale in ((inp.k, inp.k_scale), (inp.v, inp.v_scale)):
        assert scale.dtype == np.float32 and scale.shape == (wl.B, wl.L)
        mant, _ = np.frexp(scale)
        assert (mant != 0.5).mean() > 0.99           # not powers of two
        assert not np.isin(codes & 0x7F, [0x7F]).any()  # no NaN codes
        y = _dec(codes, scale) / scale.astype(np.float64)[..., None]
        assert np.abs(y).max() <= 448.0
    # K: re-derive the unpacked keys from the same stream and compare
    pow2 = make_attention_inputs(wl.resized(fp8_scale="pow2"))
    xk = _dec(pow2.k, pow2.k_scale)   # a second packing of the same normals
    got = _dec(inp.k, inp.k_scale)
    # both are within half a code step of the same float64 key, so within one
    # step of each other; a step is at most 2^-3 of the value (normal codes) or
    # 2^-9 * scale (subnormal codes)
    step = np.maximum(np.abs(got) * 2.0 ** -3,
                      2.0 ** -9 * inp.k_scale.astype(np.float64)[..., None])
    step = np.maximum(step, 2.0 ** -9 * pow2.k_scale.astype(np.float64)[..., None])
    assert (np.abs(got - xk) <= 2.0 * step + 1e-12).all()
