"""CPU oracle of the HySparse2 hybrid-block hot path (plain C++ fp64, via ctypes).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The library under
``long_context_hs2_b200`` never imports this package, and this package never
imports the library.  Both read the same input bytes from ``hs2_synth``.

Each function cites the passage of the HySparse2 pages it restates; see the
header of ``hs2_oracle.cpp`` for the readings taken where the pages are silent.
"""

import contextlib
import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hs2_oracle.cpp")
_LIB = os.path.join(_HERE, "libhs2_oracle.so")
_lib = None


def compile_source(src: str, out: str) -> str:
    """g++ build of an oracle source file (plain IEEE fp64: no fast-math, no FMA contraction)."""
    tmp = out + ".tmp%d" % os.getpid()
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-pthread",
                           "-ffp-contract=off", "-fno-fast-math", src, "-o", tmp])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile oracle/libhs2_oracle.so if it is missing or older than its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        compile_source(_SRC, _LIB)
    return _LIB


def _configure(lib):
    """Declare argument and return types of the exported oracle functions."""
    P = ctypes.c_void_p
    i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
    lib.hs2o_bf16_to_f64.restype = dbl
    lib.hs2o_bf16_to_f64.argtypes = [ctypes.c_uint16]
    lib.hs2o_f64_to_bf16.restype = ctypes.c_uint16
    lib.hs2o_f64_to_bf16.argtypes = [dbl]
    lib.hs2o_e4m3_to_f64.restype = dbl
    lib.hs2o_e4m3_to_f64.argtypes = [ctypes.c_uint8]
    lib.hs2o_f64_to_e4m3.restype = ctypes.c_uint8
    lib.hs2o_f64_to_e4m3.argtypes = [dbl]
    lib.hs2o_threads.restype = i32
    lib.hs2o_set_threads.argtypes = [i32]
    lib.hs2o_bridge.restype = i32
    lib.hs2o_bridge.argtypes = [P, i64, i32, P, i32, i32, P, i64, P, P, P, P]
    lib.hs2o_full_attn_select.restype = i32
    lib.hs2o_full_attn_select.argtypes = [P, i32, P, P, P, P, i32, i32, i64, i32, i32, dbl,
                                          i32, i32, P, i64, P, P, P, P, P]
    lib.hs2o_select.restype = i32
    lib.hs2o_select.argtypes = [P, i64, i32, i32, P, P]
    lib.hs2o_attn_slice.restype = i32
    lib.hs2o_attn_slice.argtypes = [P, i32, P, P, P, P, i32, i32, i64, i64, i32, i32, dbl, i32, P,
                                    P, i64, P, P, P]
    lib.hs2o_select_blocks.restype = i32
    lib.hs2o_select_blocks.argtypes = [P, i64, i32, i32, i32, P, P]
    lib.hs2o_sparse_attn.restype = i32
    lib.hs2o_sparse_attn.argtypes = [P, i32, P, P, P, P, i32, i32, i64, i32, i32, dbl,
                                     P, P, i32, P, i64, P]
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _configure(ctypes.CDLL(_LIB))
    return _lib


@contextlib.contextmanager
def use_library(path: str):
    """Temporarily route every call to another build of hs2_oracle.cpp (used by the
    mutation test, which plants mistakes in copies of the source)."""
    global _lib
    saved = _load()
    _lib = _configure(ctypes.CDLL(os.path.abspath(path)))
    try:
        yield
    finally:
        _lib = saved


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def threads() -> int:
    return _load().hs2o_threads()


def set_threads(n: int) -> None:
    _load().hs2o_set_threads(int(n))


# ------------------------------------------------------------------ codecs --
def bf16_to_f64(bits) -> np.ndarray:
    lib = _load()
    b = np.asarray(bits, dtype=np.uint16).ravel()
    return np.array([lib.hs2o_bf16_to_f64(int(x)) for x in b]).reshape(np.shape(bits))


def f64_to_bf16(x) -> np.ndarray:
    lib = _load()
    a = np.asarray(x, dtype=np.float64).ravel()
    return np.array([lib.hs2o_f64_to_bf16(float(v)) for v in a], dtype=np.uint16).reshape(np.shape(x))


def e4m3_to_f64(codes) -> np.ndarray:
    lib = _load()
    c = np.asarray(codes, dtype=np.uint8).ravel()
    return np.array([lib.hs2o_e4m3_to_f64(int(v)) for v in c]).reshape(np.shape(codes))


def f64_to_e4m3(x) -> np.ndarray:
    lib = _load()
    a = np.asarray(x, dtype=np.float64).ravel()
    return np.array([lib.hs2o_f64_to_e4m3(float(v)) for v in a], dtype=np.uint8).reshape(np.shape(x))


# ------------------------------------------------------------ KV Bridging --
def bridge(x_bits: np.ndarray, wt_bits: np.ndarray, n_layers: int, D: int, rows=None):
    """KV Bridging of token rows of X (IT Home announcement, "KV Bridging" paragraph:
    every bridged full-attention layer builds its own K/V from the source layer's input
    hidden state with its own projection).

    Returns dict: y [n, n_cols] fp64, k_bf16/v_bf16 [n_layers, n, D] uint16,
    k_fp8/v_fp8 [n_layers, n, D] uint8, k_scale/v_scale [n_layers, n] fp64.
    """
    lib = _load()
    x = _c(x_bits, np.uint16)
    wt = _c(wt_bits, np.uint16)
    T, hidden = x.shape
    n_cols = wt.shape[0]
    assert n_cols == n_layers * 2 * D and wt.shape[1] == hidden
    rows = np.arange(T, dtype=np.int64) if rows is None else _c(rows, np.int64)
    n = len(rows)
    y = np.zeros((n, n_cols))
    ob = np.zeros((n_layers, 2, n, D), dtype=np.uint16)
    of = np.zeros((n_layers, 2, n, D), dtype=np.uint8)
    sc = np.zeros((n_layers, 2, n))
    rc = lib.hs2o_bridge(_p(x), T, hidden, _p(wt), n_layers, D, _p(rows), n, _p(y), _p(ob), _p(of),
                         _p(sc))
    if rc != 0:
        raise ValueError("hs2o_bridge: invalid arguments")
    return dict(y=y, k_bf16=ob[:, 0], v_bf16=ob[:, 1], k_fp8=of[:, 0], v_fp8=of[:, 1],
                k_scale=sc[:, 0], v_scale=sc[:, 1])


# ------------------------------------------- full attention and selection --
def full_attn_select(q, k, v, k_scale=None, v_scale=None, *, scale: float, topk: int = 1024,
                     window: int = 128, rows=None, want_score: bool = False):
    """Full-attention layer of a hybrid block plus token-level selection (IT Home
    announcement, "KV Reuse" paragraphs: the full layer picks important positions from its
    attention scores; "token-level selection" paragraph: 128 most recent tokens forced,
    1024 global tokens chosen from outside that window).

    q: uint16 [B, T, H, D]; k, v: uint16 [B, L, D] (bf16) or uint8 (E4M3) with float32
    scales [B, L].  Returns dict with o [n, H, D], lse [n, H], idx [n, topk+window],
    n_sel [n] and, if asked, score [n, L] (head-summed probability).
    """
    lib = _load()
    q = _c(q, np.uint16)
    fp8 = k.dtype == np.uint8
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    ks = _c(k_scale, np.float32)
    vs = _c(v_scale, np.float32)
    B, T, H, D = q.shape
    L = k.shape[1]
    rows_a = None if rows is None else _c(rows, np.int64)
    n = B * T if rows_a is None else len(rows_a)
    o = np.zeros((n, H, D))
    lse = np.zeros((n, H))
    sc = np.zeros((n, L)) if want_score else None
    idx = np.zeros((n, topk + window), dtype=np.int32)
    nsel = np.zeros(n, dtype=np.int32)
    rc = lib.hs2o_full_attn_select(_p(q), int(fp8), _p(k), _p(v), _p(ks), _p(vs), B, T, L, H, D,
                                   float(scale), topk, window, _p(rows_a), n, _p(o), _p(lse),
                                   _p(sc), _p(idx), _p(nsel))
    if rc != 0:
        raise ValueError("hs2o_full_attn_select: invalid arguments")
    out = dict(o=o, lse=lse, idx=idx, n_sel=nsel)
    if want_score:
        out["score"] = sc
    return out


def attn_slice(q, k, v, k_scale=None, v_scale=None, *, qpos: int, scale: float, window: int = 128,
               lse_in=None, rows=None, want_score: bool = False):
    """Attention of the queries over one slice of a context split across devices
    (dpshk.com explainer, section 05: million-token contexts): the slice's own
    normaliser lse and output O (normalised over the slice), and, if asked, the
    head-summed scores of the slice's candidates under lse_in (the normaliser
    over the whole context; the slice's own when None).

    q: uint16 [B, T, H, D]; k, v: the slice [B, L_slice, D]; query t sits at
    slice-relative position qpos + t.  lse_in: [B*T, H] float64 or None.
    Returns dict with o [n, H, D], lse [n, H] and optionally score [n, L_slice].
    """
    lib = _load()
    q = _c(q, np.uint16)
    fp8 = k.dtype == np.uint8
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    ks = _c(k_scale, np.float32)
    vs = _c(v_scale, np.float32)
    B, T, H, D = q.shape
    L = k.shape[1]
    rows_a = None if rows is None else _c(rows, np.int64)
    n = B * T if rows_a is None else len(rows_a)
    li = None if lse_in is None else _c(lse_in, np.float64)
    o = np.zeros((n, H, D))
    lse = np.zeros((n, H))
    sc = np.zeros((n, L)) if want_score else None
    rc = lib.hs2o_attn_slice(_p(q), int(fp8), _p(k), _p(v), _p(ks), _p(vs), B, T, L, int(qpos), H,
                             D, float(scale), int(window), _p(li), _p(rows_a), n, _p(o), _p(lse),
                             _p(sc))
    if rc != 0:
        raise ValueError("hs2o_attn_slice: invalid arguments")
    out = dict(o=o, lse=lse)
    if want_score:
        out["score"] = sc
    return out


def select(score_row: np.ndarray, i: int, topk: int, window: int):
    """Selection of query position i from a head-summed score row score[0..i]."""
    lib = _load()
    s = _c(score_row, np.float64)
    idx = np.zeros(topk + window, dtype=np.int32)
    ns = np.zeros(1, dtype=np.int32)
    if lib.hs2o_select(_p(s), int(i), topk, window, _p(idx), _p(ns)) != 0:
        raise ValueError("hs2o_select: invalid arguments")
    return idx, int(ns[0])


def select_blocks(score_row: np.ndarray, i: int, topk: int, window: int, block: int = 64):
    """Block-level selection of query position i from a head-summed score row
    score[0..i] (dpshk.com explainer, section 03: the earlier HySparse chose
    history in blocks of 64 tokens): the topk/block candidate blocks of largest
    summed score, ties to the lower block, plus the window."""
    lib = _load()
    s = _c(score_row, np.float64)
    idx = np.zeros(topk + window, dtype=np.int32)
    ns = np.zeros(1, dtype=np.int32)
    if lib.hs2o_select_blocks(_p(s), int(i), topk, window, block, _p(idx), _p(ns)) != 0:
        raise ValueError("hs2o_select_blocks: invalid arguments")
    return idx, int(ns[0])


# -------------------------------------------------------- sparse KV reuse --
def sparse_attn(q, k, v, k_scale, v_scale, idx, n_sel, *, scale: float, rows=None):
    """Sparse-attention layer reusing the block's KV cache and selection (IT Home
    announcement, "KV Reuse" paragraph).  idx [B*T, slots] int32, n_sel [B*T]."""
    lib = _load()
    q = _c(q, np.uint16)
    fp8 = k.dtype == np.uint8
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    ks = _c(k_scale, np.float32)
    vs = _c(v_scale, np.float32)
    idx = _c(idx, np.int32)
    nsel = _c(n_sel, np.int32)
    B, T, H, D = q.shape
    L = k.shape[1]
    slots = idx.shape[-1]
    rows_a = None if rows is None else _c(rows, np.int64)
    n = B * T if rows_a is None else len(rows_a)
    o = np.zeros((n, H, D))
    rc = lib.hs2o_sparse_attn(_p(q), int(fp8), _p(k), _p(v), _p(ks), _p(vs), B, T, L, H, D,
                              float(scale), _p(idx.reshape(B * T, slots)), _p(nsel.ravel()), slots,
                              _p(rows_a), n, _p(o))
    if rc != 0:
        raise ValueError("hs2o_sparse_attn: invalid arguments or indices")
    return o
