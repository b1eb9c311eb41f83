"""Seeded synthetic inputs for the HySparse2 hybrid-block hot path.

This module is the only code shared by the CPU oracle (``oracle/``) and the
CUDA path (``long_context_hs2_b200``).  It draws random numbers and packs them
into the storage formats the kernels read (bf16 bit patterns, E4M3 bytes with a
per-token fp32 scale).  It holds none of the method's arithmetic: no attention,
no selection, no projection.

Random numbers come from SplitMix64 (Steele, Lea and Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014), used as a counter-based
generator: element n of a stream with seed s is mix(s + (n + 1) * gamma).
Normals come from the Box-Muller transform of pairs of uniforms.

Workloads follow the five shapes of the HySparse2 pages' 80B-A3B analysis as
sized for this library (tiny parity block, bf16 decode at 32K, bridge prefill
of 131072 tokens, FP8 decode at 256K, 4096-token chunk at 1M).  Planted
"needle" keys stand in for the long-context retrieval evaluations the pages
report (RULER-v2, MRCR-v2, GraphWalks), which are not available here.
"""

from .gen import (  # noqa: F401
    GAMMA,
    splitmix64_stream,
    uniform_stream,
    normal_stream,
    stream_seed,
    f32_to_bf16_bits,
    bf16_bits_to_f32,
    e4m3_value_table,
    fp8_quantise_pow2,
    fp8_quantise_with_scales,
    random_mantissa_scales,
    fp8_dequantise,
)
from .workloads import (  # noqa: F401
    WORKLOADS,
    AttnInputs,
    BridgeInputs,
    make_attention_inputs,
    make_bridge_inputs,
)
