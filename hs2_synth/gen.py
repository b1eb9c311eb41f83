"""Counter-based random streams and storage-format packing (numpy only).

SplitMix64 (Steele, Lea, Flood, OOPSLA 2014): with gamma = 0x9E3779B97F4A7C15,
the n-th output of a stream seeded with s is mix64(s + (n + 1) * gamma), where
mix64(z) = z1 ^ (z1 >> 31), z1 = (z0 ^ (z0 >> 27)) * 0x94D049BB133111EB,
z0 = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9, all modulo 2**64.

Uniforms take the top 53 bits.  Normals use Box-Muller on consecutive pairs:
r = sqrt(-2 ln u1), n0 = r cos(2 pi u2), n1 = r sin(2 pi u2), with u1 in (0, 1].
"""

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def _mix64(z):
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def splitmix64_stream(seed: int, n: int, start: int = 0) -> np.ndarray:
    """Outputs start .. start+n-1 of the SplitMix64 stream seeded with `seed`."""
    with np.errstate(over="ignore"):
        ctr = np.arange(start + 1, start + n + 1, dtype=np.uint64)
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + ctr * GAMMA
        return _mix64(z)


def stream_seed(base: int, tensor: str, layer: int = 0) -> int:
    """Seed of one named tensor stream: SplitMix64 of (base, FNV-1a(name), layer)."""
    h = 0xCBF29CE484222325
    for ch in tensor.encode():
        h = ((h ^ ch) * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    x = (base * 0x9E3779B97F4A7C15 + h + (layer + 1) * 0xD1B54A32D192ED03) & 0xFFFFFFFFFFFFFFFF
    return int(splitmix64_stream(x, 1)[0])


def uniform_stream(seed: int, n: int, start: int = 0) -> np.ndarray:
    """Uniforms in [0, 1) from the top 53 bits of each output."""
    z = splitmix64_stream(seed, n, start)
    return (z >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def normal_stream(seed: int, n: int) -> np.ndarray:
    """n standard normals (float64), generated in chunks to bound memory."""
    out = np.empty(n, dtype=np.float64)
    npairs = (n + 1) // 2
    done = 0
    while done < npairs:
        m = min(_CHUNK, npairs - done)
        z = splitmix64_stream(seed, 2 * m, 2 * done)
        u1 = ((z[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * (1.0 / 9007199254740992.0)
        u2 = (z[1::2] >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)
        r = np.sqrt(-2.0 * np.log(u1))
        t = (2.0 * np.pi) * u2
        lo = 2 * done
        pair = np.empty(2 * m, dtype=np.float64)
        pair[0::2] = r * np.cos(t)
        pair[1::2] = r * np.sin(t)
        take = min(2 * m, n - lo)
        out[lo:lo + take] = pair[:take]
        done += m
    return out


def f32_to_bf16_bits(x) -> np.ndarray:
    """Round float values to bf16 (round to nearest, ties to even); returns uint16 bits.

    The input is first rounded to float32.  Inputs here are finite.
    """
    b = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).view(np.uint32)
    with np.errstate(over="ignore"):
        bias = ((b >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
        return ((b + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def e4m3_value_table() -> np.ndarray:
    """Magnitudes of the 127 finite non-negative OCP E4M3 codes 0x00..0x7E (bias 7)."""
    codes = np.arange(127)
    e = codes >> 3
    m = codes & 7
    return np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))


_E4M3 = e4m3_value_table()


def _nearest_e4m3(y: np.ndarray) -> np.ndarray:
    """Nearest E4M3 code of |y| <= 448 (ties to the even code), sign in bit 7."""
    a = np.abs(y)
    hi = np.clip(np.searchsorted(_E4M3, a, side="left"), 1, 126)
    lo = hi - 1
    dlo = a - _E4M3[lo]
    dhi = _E4M3[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a >= _E4M3[126], 126, code)
    return (code | np.where(np.signbit(y), 0x80, 0)).astype(np.uint8)


def fp8_quantise_pow2(x: np.ndarray):
    """Store rows of x ([..., D]) as E4M3 codes with one fp32 power-of-two scale per row.

    The scale is the smallest power of two s with max|x_row| / s <= 448, so the
    division is exact and only the E4M3 rounding loses precision.  Rows of zeros
    get s = 1.  Returns (codes uint8 [..., D], scale float32 [...]).
    """
    x = np.asarray(x, dtype=np.float64)
    amax = np.max(np.abs(x), axis=-1)
    with np.errstate(divide="ignore"):
        ex = np.ceil(np.log2(np.where(amax > 0, amax, 448.0) / 448.0))
    scale = np.exp2(ex)
    scale = np.where(amax > 0, scale, 1.0)
    codes = _nearest_e4m3(x / scale[..., None])
    return codes, scale.astype(np.float32)


def fp8_quantise_with_scales(x: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """E4M3 codes of rows of x ([..., D]) for given fp32 per-row scales.

    Each element is stored as the nearest E4M3 code of x / scale (computed in
    float64 with the scale exactly as stored; ties to the even code; saturating
    at 448), so the stored value is code * scale.  Returns uint8 codes [..., D].
    """
    x = np.asarray(x, dtype=np.float64)
    s = np.asarray(scale, dtype=np.float32).astype(np.float64)
    return _nearest_e4m3(np.clip(x / s[..., None], -448.0, 448.0))


def random_mantissa_scales(x: np.ndarray, u: np.ndarray) -> np.ndarray:
    """Per-row fp32 scales with an arbitrary (non-power-of-two) mantissa.

    scale = max|x_row| / 448 * (1 + u_row / 2), rounded to fp32, with u_row a
    uniform in [0, 1): every row fits the E4M3 range, and the scale's mantissa
    bits are random, so a kernel that loses scale precision shows up in the
    results (a power-of-two scale would hide it: its products are exact at any
    precision).  Rows of zeros get 1.  Returns float32 [...].
    """
    amax = np.max(np.abs(np.asarray(x, dtype=np.float64)), axis=-1)
    s = amax / 448.0 * (1.0 + 0.5 * np.asarray(u, dtype=np.float64).reshape(amax.shape))
    return np.where(amax > 0, s, 1.0).astype(np.float32)


def fp8_dequantise(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """Value of E4M3 codes times their row scale (float64); used to plant and check inputs."""
    c = np.asarray(codes, dtype=np.uint8)
    mag = np.concatenate([_E4M3, [np.nan]])[c & 0x7F]
    val = np.where(c & 0x80, -mag, mag)
    return val * np.asarray(scale, dtype=np.float64)[..., None]
