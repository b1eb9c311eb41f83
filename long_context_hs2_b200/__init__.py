"""Python binding of libhs2, the sm_100a HySparse2 hybrid-block hot path.

Argument marshalling only: every function here forwards to the C ABI of
include/hs2.h with the same name, turning torch tensors into device pointers
and the current CUDA stream into a stream handle, and raises ``Hs2Error`` when
the library returns a non-OK status.  All computation runs in the library's
CUDA kernels; there is no fallback path.  Importing this package does not load
the library; the first call does, and fails loudly if ``libhs2.so`` has not
been built (``python -m long_context_hs2_b200.build``).
"""

import ctypes
import os
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhs2.so")

HS2_OK = 0
HS2_KV_BF16 = 0
HS2_KV_FP8_E4M3 = 1

_STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "CUDA error",
           4: "workspace", 5: "timeout", 6: "device index error"}

EXPORTED = ("hs2_bridge_kv", "hs2_full_attn_select_workspace", "hs2_full_attn_select",
            "hs2_full_attn_select_noalloc", "hs2_sparse_attn", "hs2_last_device_status",
            "hs2_status_string", "hs2_version", "hs2_set_stage_events",
            "hs2_set_fault_injection", "hs2_full_attn_select_blocks", "hs2_cp_workspace",
            "hs2_cp_attn_partial", "hs2_cp_lse_combine", "hs2_cp_rescale", "hs2_cp_select_local",
            "hs2_cp_merge_select", "hs2_set_phase_stamps")

# Global-timer stamps per CTA written by the fused full-attention kernel when enabled.
HS2_PHASES = 8

# Size of the scratch area built into the library for hs2_full_attn_select_noalloc.
HS2_NOALLOC_SCRATCH_BYTES = 16 << 20


class Hs2Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__("%s failed: %s (%d)" % (fn, _STATUS.get(status, "?"), status))
        self.status = status


class hs2_kv_cache(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("k_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Loads libhs2.so and declares its signatures.  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError("libhs2.so is not built at %s; run python -m long_context_hs2_b200.build"
                           % path)
    lib = ctypes.CDLL(path)
    P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    KV = ctypes.POINTER(hs2_kv_cache)
    lib.hs2_version.restype = i32
    lib.hs2_status_string.restype = ctypes.c_char_p
    lib.hs2_status_string.argtypes = [i32]
    lib.hs2_last_device_status.restype = i32
    lib.hs2_last_device_status.argtypes = [P]
    lib.hs2_bridge_kv.restype = i32
    lib.hs2_bridge_kv.argtypes = [P, i64, i32, P, i32, i32, i32, KV, i64, P]
    lib.hs2_full_attn_select_workspace.restype = sz
    lib.hs2_full_attn_select_workspace.argtypes = [i32, i32, i64, i32, i32, i32, i32, i32]
    lib.hs2_full_attn_select.restype = i32
    lib.hs2_full_attn_select.argtypes = [P, KV, i32, i32, i64, i32, i32, ctypes.c_float, i32, i32,
                                         i32, P, P, P, P, P, sz, P]
    lib.hs2_full_attn_select_blocks.restype = i32
    lib.hs2_full_attn_select_blocks.argtypes = [P, KV, i32, i32, i64, i32, i32, ctypes.c_float,
                                                i32, i32, i32, i32, P, P, P, P, P, sz, P]
    lib.hs2_cp_workspace.restype = sz
    lib.hs2_cp_workspace.argtypes = [i32, i32, i64, i32, i32, i32, i32, i32]
    lib.hs2_cp_attn_partial.restype = i32
    lib.hs2_cp_attn_partial.argtypes = [P, KV, i32, i32, i64, i64, i32, i32, ctypes.c_float, i32,
                                        P, P, P, sz, P]
    lib.hs2_cp_lse_combine.restype = i32
    lib.hs2_cp_lse_combine.argtypes = [P, i32, i64, P, P]
    lib.hs2_cp_rescale.restype = i32
    lib.hs2_cp_rescale.argtypes = [P, P, P, i64, i32, P]
    lib.hs2_cp_select_local.restype = i32
    lib.hs2_cp_select_local.argtypes = [P, KV, i32, i32, i64, i64, i64, i32, i32, ctypes.c_float,
                                        i32, i32, i32, P, P, P, P, sz, P]
    lib.hs2_cp_merge_select.restype = i32
    lib.hs2_cp_merge_select.argtypes = [P, P, i32, i32, i32, i64, i32, i32, P, P, P]
    lib.hs2_full_attn_select_noalloc.restype = i32
    lib.hs2_full_attn_select_noalloc.argtypes = [P, KV, i32, i32, i64, i32, i32, ctypes.c_float,
                                                 i32, i32, i32, P, P, P, P, P]
    lib.hs2_set_stage_events.restype = i32
    lib.hs2_set_fault_injection.restype = i32
    lib.hs2_set_fault_injection.argtypes = [ctypes.c_uint, ctypes.c_ulonglong]
    lib.hs2_set_phase_stamps.restype = i32
    lib.hs2_set_phase_stamps.argtypes = [ctypes.c_void_p, ctypes.c_int]
    lib.hs2_set_stage_events.argtypes = [P, P]
    lib.hs2_sparse_attn.restype = i32
    lib.hs2_sparse_attn.argtypes = [P, KV, i32, i32, i64, i32, i32, ctypes.c_float, P, P, i32, i32,
                                    P, P]
    _lib = lib
    return lib


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, st: int):
    if st != HS2_OK:
        raise Hs2Error(fn, st)


def kv_cache(k, v, k_scale=None, v_scale=None) -> hs2_kv_cache:
    """The C struct of one layer's cache from device tensors (or raw pointers).
    The struct holds references to the tensors it was made from, so that their
    memory stays allocated for as long as the struct (or a CUDA graph that
    captured calls with it, while the caller keeps the struct) is in use."""
    c = hs2_kv_cache(_ptr(k), _ptr(v), _ptr(k_scale), _ptr(v_scale))
    c._tensors = (k, v, k_scale, v_scale)
    return c


def hs2_version() -> int:
    return load_library().hs2_version()


def hs2_status_string(status: int) -> str:
    return load_library().hs2_status_string(int(status)).decode()


def hs2_last_device_status(stream=None) -> int:
    """Synchronises `stream`; returns (and clears) the device status code."""
    return load_library().hs2_last_device_status(_stream(stream))


def hs2_bridge_kv(X, T: int, hidden: int, Wt, n_layers: int, D: int, out_dtype: int,
                  caches: Sequence[hs2_kv_cache], cache_row_offset: int = 0, stream=None):
    arr = (hs2_kv_cache * n_layers)(*caches)
    _check("hs2_bridge_kv", load_library().hs2_bridge_kv(
        _ptr(X), int(T), int(hidden), _ptr(Wt), int(n_layers), int(D), int(out_dtype), arr,
        int(cache_row_offset), _stream(stream)))


def hs2_full_attn_select_workspace(B, T, L, H, D, topk, window, dt) -> int:
    return int(load_library().hs2_full_attn_select_workspace(int(B), int(T), int(L), int(H), int(D),
                                                             int(topk), int(window), int(dt)))


def hs2_full_attn_select(Q, kv: hs2_kv_cache, B, T, L, H, D, scale, topk, window, dt, O, lse,
                         idx, n_sel, workspace, workspace_bytes: int, stream=None):
    _check("hs2_full_attn_select", load_library().hs2_full_attn_select(
        _ptr(Q), ctypes.byref(kv), int(B), int(T), int(L), int(H), int(D), float(scale), int(topk),
        int(window), int(dt), _ptr(O), _ptr(lse), _ptr(idx), _ptr(n_sel), _ptr(workspace),
        int(workspace_bytes), _stream(stream)))


def hs2_full_attn_select_blocks(Q, kv: hs2_kv_cache, B, T, L, H, D, scale, topk, window, block,
                                dt, O, lse, idx, n_sel, workspace, workspace_bytes: int,
                                stream=None):
    """hs2_full_attn_select with the block-level selection (blocks of `block`
    positions, topk/block of them kept) instead of the token-level one."""
    _check("hs2_full_attn_select_blocks", load_library().hs2_full_attn_select_blocks(
        _ptr(Q), ctypes.byref(kv), int(B), int(T), int(L), int(H), int(D), float(scale),
        int(topk), int(window), int(block), int(dt), _ptr(O), _ptr(lse), _ptr(idx), _ptr(n_sel),
        _ptr(workspace), int(workspace_bytes), _stream(stream)))


def hs2_full_attn_select_noalloc(Q, kv: hs2_kv_cache, B, T, L, H, D, scale, topk, window, dt,
                                 O, lse, idx, n_sel, stream=None):
    """hs2_full_attn_select without a workspace argument, for callers that cannot
    allocate device memory; the library's built-in scratch area is used instead."""
    _check("hs2_full_attn_select_noalloc", load_library().hs2_full_attn_select_noalloc(
        _ptr(Q), ctypes.byref(kv), int(B), int(T), int(L), int(H), int(D), float(scale),
        int(topk), int(window), int(dt), _ptr(O), _ptr(lse), _ptr(idx), _ptr(n_sel),
        _stream(stream)))


def hs2_sparse_attn(Q, kv: hs2_kv_cache, B, T, L, H, D, scale, idx, n_sel, slots, dt, O,
                    stream=None):
    _check("hs2_sparse_attn", load_library().hs2_sparse_attn(
        _ptr(Q), ctypes.byref(kv), int(B), int(T), int(L), int(H), int(D), float(scale),
        _ptr(idx), _ptr(n_sel), int(slots), int(dt), _ptr(O), _stream(stream)))


def hs2_set_stage_events(begin=None, end=None):
    """Sets (or, with no arguments, clears) the events that this thread's
    full-attention calls record around their partial-attention kernel.
    `begin`/`end` are torch.cuda.Event objects (timing enabled) or raw handles."""
    def handle(e):
        if e is None or isinstance(e, int):
            return e
        return e.cuda_event
    _check("hs2_set_stage_events", load_library().hs2_set_stage_events(handle(begin), handle(end)))


def hs2_set_phase_stamps(stamps=None, max_ctas: int = 0):
    """Tracing: the fused full-attention kernel writes HS2_PHASES global-timer
    stamps per CTA into `stamps` (a device uint64/int64 buffer of max_ctas *
    HS2_PHASES values); None turns them off."""
    _check("hs2_set_phase_stamps",
           load_library().hs2_set_phase_stamps(_ptr(stamps), int(max_ctas) if stamps is not None else 0))


def hs2_set_fault_injection(extra_arrivals: int = 0, wait_limit_ns: int = 0):
    """Test hook: the fused kernel's group barriers wait for `extra_arrivals`
    arrivals that never come and give up after `wait_limit_ns` (0: one second).
    With no arguments, restores the defaults."""
    _check("hs2_set_fault_injection",
           load_library().hs2_set_fault_injection(int(extra_arrivals), int(wait_limit_ns)))


# ------------------------------------------------ context parallelism --
def hs2_cp_workspace(B, T, L_local, H, D, topk, window, dt) -> int:
    return int(load_library().hs2_cp_workspace(int(B), int(T), int(L_local), int(H), int(D),
                                                int(topk), int(window), int(dt)))


def hs2_cp_attn_partial(Q, kv: hs2_kv_cache, B, T, L_local, q_pos_local, H, D, scale, dt, O, lse,
                        workspace, workspace_bytes: int, stream=None):
    _check("hs2_cp_attn_partial", load_library().hs2_cp_attn_partial(
        _ptr(Q), ctypes.byref(kv), int(B), int(T), int(L_local), int(q_pos_local), int(H), int(D),
        float(scale), int(dt), _ptr(O), _ptr(lse), _ptr(workspace), int(workspace_bytes),
        _stream(stream)))


def hs2_cp_lse_combine(lse_parts, G, n, lse, stream=None):
    _check("hs2_cp_lse_combine", load_library().hs2_cp_lse_combine(
        _ptr(lse_parts), int(G), int(n), _ptr(lse), _stream(stream)))


def hs2_cp_rescale(O_part, lse_part, lse, n, D, stream=None):
    _check("hs2_cp_rescale", load_library().hs2_cp_rescale(
        _ptr(O_part), _ptr(lse_part), _ptr(lse), int(n), int(D), _stream(stream)))


def hs2_cp_select_local(Q, kv: hs2_kv_cache, B, T, L_local, q_pos_local, key_pos0, H, D, scale,
                        topk, window, dt, lse, cand_score, cand_idx, workspace,
                        workspace_bytes: int, stream=None):
    _check("hs2_cp_select_local", load_library().hs2_cp_select_local(
        _ptr(Q), ctypes.byref(kv), int(B), int(T), int(L_local), int(q_pos_local), int(key_pos0),
        int(H), int(D), float(scale), int(topk), int(window), int(dt), _ptr(lse),
        _ptr(cand_score), _ptr(cand_idx), _ptr(workspace), int(workspace_bytes),
        _stream(stream)))


def hs2_cp_merge_select(cand_score, cand_idx, G, B, T, q_pos0, topk, window, idx, n_sel,
                        stream=None):
    _check("hs2_cp_merge_select", load_library().hs2_cp_merge_select(
        _ptr(cand_score), _ptr(cand_idx), int(G), int(B), int(T), int(q_pos0), int(topk),
        int(window), _ptr(idx), _ptr(n_sel), _stream(stream)))
