"""The synthetic workloads of the hybrid-block hot path, and their input recipes.

Shapes follow the pages' 80B-A3B long-context analysis as fixed for this
library: MQA with one KV head, head_dim 128 and 32 query heads ("a more compact
MQA configuration"), a top-1024 budget plus the 128 most recent tokens, one
full-attention layer followed by sparse layers that reuse its KV cache and
indices, and six bridged target layers fed from one source hidden state.

Values are iid N(0, 1) unless stated.  "Needles" are keys planted at 4 times
the expected key norm along the direction of a later query's head-sum, so that
a correct selection must keep them: for needle position j with target query
position i* >= j + window, k_j = 4 sqrt(D) u, u = sum_h q[i*, h] / |sum_h q[i*, h]|.
Needles are planted before FP8 packing.
"""

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

from .gen import (
    splitmix64_stream,
    normal_stream,
    uniform_stream,
    stream_seed,
    f32_to_bf16_bits,
    bf16_bits_to_f32,
    fp8_quantise_pow2,
    fp8_quantise_with_scales,
    random_mantissa_scales,
)


@dataclass(frozen=True)
class AttnWorkload:
    name: str
    B: int
    T: int
    L: int
    H: int
    D: int
    kv_dtype: str          # "bf16" or "fp8"
    n_sparse: int
    n_needles: int         # per sequence
    seed: int
    topk: int = 1024
    window: int = 128
    # E4M3 per-token scales: "pow2" (smallest power of two that fits the row)
    # or "mantissa" (random non-power-of-two scales, see random_mantissa_scales)
    fp8_scale: str = "pow2"

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.D))

    def resized(self, **kw) -> "AttnWorkload":
        d = dict(self.__dict__)
        d.update(kw)
        return AttnWorkload(**d)


@dataclass(frozen=True)
class BridgeWorkload:
    name: str
    T: int
    hidden: int
    n_layers: int
    D: int
    seed: int

    @property
    def n_cols(self) -> int:
        return self.n_layers * 2 * self.D

    def resized(self, **kw) -> "BridgeWorkload":
        d = dict(self.__dict__)
        d.update(kw)
        return BridgeWorkload(**d)


BASE_SEED = 2026

WORKLOADS = {
    # tiny hybrid block: causal chunk of 2048 queries over its own 2048 tokens
    "tiny": AttnWorkload("tiny", B=1, T=2048, L=2048, H=8, D=64, kv_dtype="bf16",
                         n_sparse=1, n_needles=16, seed=BASE_SEED + 1),
    # bf16 decode at 32K context, 8 sequences
    "decode_bf16_32k": AttnWorkload("decode_bf16_32k", B=8, T=1, L=32768, H=32, D=128,
                                    kv_dtype="bf16", n_sparse=3, n_needles=64,
                                    seed=BASE_SEED + 2),
    # KV bridging prefill of 131072 tokens into 6 target layers
    "bridge_131k": BridgeWorkload("bridge_131k", T=131072, hidden=4096, n_layers=6, D=128,
                                  seed=BASE_SEED + 3),
    # FP8 decode at 256K context, 4 sequences
    "decode_fp8_256k": AttnWorkload("decode_fp8_256k", B=4, T=1, L=262144, H=32, D=128,
                                    kv_dtype="fp8", n_sparse=3, n_needles=256,
                                    seed=BASE_SEED + 4),
    # 4096-token new-observation chunk over a 1M-token FP8 cache
    "chunk_fp8_1m": AttnWorkload("chunk_fp8_1m", B=1, T=4096, L=1048576, H=32, D=128,
                                 kv_dtype="fp8", n_sparse=3, n_needles=1024,
                                 seed=BASE_SEED + 5),
}


@dataclass
class AttnInputs:
    wl: AttnWorkload
    q: np.ndarray                 # uint16 bf16 bits [B, T, H, D], full-attention layer
    q_sparse: List[np.ndarray]    # per sparse layer, same shape
    k: np.ndarray                 # uint16 [B, L, D] (bf16) or uint8 [B, L, D] (E4M3)
    v: np.ndarray
    k_scale: Optional[np.ndarray]  # float32 [B, L] for E4M3, else None
    v_scale: Optional[np.ndarray]
    needles: np.ndarray           # int64 [n, 3]: (b, key position j, target query index t)
    extras: dict = field(default_factory=dict)


def _bf16(x: np.ndarray) -> np.ndarray:
    return f32_to_bf16_bits(x)


def _query(wl: AttnWorkload, layer: int) -> np.ndarray:
    n = wl.B * wl.T * wl.H * wl.D
    x = normal_stream(stream_seed(wl.seed, "q", layer), n)
    return _bf16(x).reshape(wl.B, wl.T, wl.H, wl.D)


def _needle_sites(wl: AttnWorkload, b: int) -> np.ndarray:
    """(j, t) pairs with distinct j and L - T + t >= j + window, drawn from a seeded stream."""
    first_t = max(0, wl.window - (wl.L - wl.T))
    if wl.n_needles == 0 or first_t >= wl.T:
        return np.zeros((0, 2), dtype=np.int64)
    seed = stream_seed(wl.seed, "needle", b)
    sites, used, ctr = [], set(), 0
    while len(sites) < wl.n_needles:
        u = uniform_stream(seed, 2, ctr)
        ctr += 2
        t = first_t + int(u[0] * (wl.T - first_t))
        i_star = wl.L - wl.T + t
        j = int(u[1] * (i_star - wl.window + 1))
        if j in used:
            continue
        used.add(j)
        sites.append((j, t))
        if ctr > 64 * wl.n_needles + 1024:
            break
    return np.asarray(sites, dtype=np.int64)


def make_attention_inputs(wl: AttnWorkload, needles: bool = True) -> AttnInputs:
    q = _query(wl, 0)
    q_sparse = [_query(wl, 1 + s) for s in range(wl.n_sparse)]
    kf = normal_stream(stream_seed(wl.seed, "k"), wl.B * wl.L * wl.D).reshape(wl.B, wl.L, wl.D)
    vf = normal_stream(stream_seed(wl.seed, "v"), wl.B * wl.L * wl.D).reshape(wl.B, wl.L, wl.D)
    planted = []
    if needles:
        qf = bf16_bits_to_f32(q).astype(np.float64)
        for b in range(wl.B):
            for j, t in _needle_sites(wl, b):
                s = qf[b, t].sum(axis=0)
                u = s / np.linalg.norm(s)
                kf[b, j] = 4.0 * np.sqrt(wl.D) * u
                planted.append((b, j, t))
    if wl.kv_dtype == "bf16":
        k, v = _bf16(kf), _bf16(vf)
        ks = vs = None
    elif wl.kv_dtype == "fp8" and wl.fp8_scale == "pow2":
        k, ks = fp8_quantise_pow2(kf)
        v, vs = fp8_quantise_pow2(vf)
    elif wl.kv_dtype == "fp8" and wl.fp8_scale == "mantissa":
        n = wl.B * wl.L
        ks = random_mantissa_scales(kf, uniform_stream(stream_seed(wl.seed, "k_scale"), n))
        vs = random_mantissa_scales(vf, uniform_stream(stream_seed(wl.seed, "v_scale"), n))
        ks, vs = ks.reshape(wl.B, wl.L), vs.reshape(wl.B, wl.L)
        k = fp8_quantise_with_scales(kf, ks)
        v = fp8_quantise_with_scales(vf, vs)
    else:
        raise ValueError(wl.kv_dtype)
    del kf, vf
    nd = np.asarray(planted, dtype=np.int64).reshape(-1, 3)
    return AttnInputs(wl, q, q_sparse, k, v, ks, vs, nd)


@dataclass
class BridgeInputs:
    wl: BridgeWorkload
    x: np.ndarray    # uint16 bf16 [T, hidden], iid N(0,1)/64
    wt: np.ndarray   # uint16 bf16 [n_layers*2*D, hidden]; row c is output column c, iid N(0, 1/hidden)


def make_bridge_inputs(wl: BridgeWorkload) -> BridgeInputs:
    x = np.empty((wl.T, wl.hidden), dtype=np.uint16)
    rows = max(1, (1 << 22) // wl.hidden)
    seed = stream_seed(wl.seed, "x")
    for r0 in range(0, wl.T, rows):
        r1 = min(wl.T, r0 + rows)
        x[r0:r1] = _bf16(_normal_block(seed, r0 * wl.hidden, (r1 - r0) * wl.hidden) / 64.0
                         ).reshape(r1 - r0, wl.hidden)
    w = normal_stream(stream_seed(wl.seed, "w"), wl.n_cols * wl.hidden) / np.sqrt(wl.hidden)
    return BridgeInputs(wl, x, _bf16(w).reshape(wl.n_cols, wl.hidden))


def _normal_block(seed: int, start: int, n: int) -> np.ndarray:
    """Normals start .. start+n-1 of a stream (start even), matching normal_stream."""
    assert start % 2 == 0
    m = (n + 1) // 2
    z = splitmix64_stream(seed, 2 * m, start)
    u1 = ((z[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * (1.0 / 9007199254740992.0)
    u2 = (z[1::2] >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)
    r = np.sqrt(-2.0 * np.log(u1))
    t = (2.0 * np.pi) * u2
    out = np.empty(2 * m, dtype=np.float64)
    out[0::2] = r * np.cos(t)
    out[1::2] = r * np.sin(t)
    return out[:n]
