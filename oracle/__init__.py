"""fp64 CPU oracle for the paged KV-cache decode path.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg and reference arm import this package. The
product package ``paged_kv_cache_335_b200`` never imports it, and the C source
``pa_oracle.c`` shares no code with the CUDA sources.

What each function computes is documented in ``pa_oracle.c`` with the page and
section it follows. Arrays are numpy: element type ``float32`` for binary32
caches, ``uint16`` (raw bit patterns) for bfloat16 caches and ``uint8`` for
quantised caches (FP8 E4M3 or int8 codes, with per-kv-head binary32 scales).

Every function here is pinned by ``tests/test_oracle_pins.py`` against
something other than itself (a library attention routine, hand-written golden
layouts, invariants and closed forms); none is "parity unpinned".
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

F32 = 0
BF16 = 1
FP8_E4M3 = 2     # quantised cache codes (uint8 arrays)
INT8 = 3
QUANT_FORMATS = {"fp8": FP8_E4M3, "int8": INT8}


def build(force: bool = False) -> str:
    """Compile ``pa_oracle.c`` into ``liboracle.so`` next to it (gcc, OpenMP).

    No fast-math: the oracle keeps IEEE double semantics and source order.
    """
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    compile_source(_SRC, tmp)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(path: str):
    lib = ctypes.CDLL(path)
    p, i32 = ctypes.c_void_p, ctypes.c_int32
    lib.oracle_kv_append.argtypes = [p, p, p, i32, p, p, i32, i32, i32, i32, i32]
    lib.oracle_block_copy.argtypes = [p, i32, p, p, i32, i32, i32, i32, i32]
    lib.oracle_block_swap.argtypes = [p, i32, p, p, i32, p, p, i32, i32, i32, i32, i32]
    lib.oracle_decode_multi.argtypes = [p, p, p, p, p, i32, p, p, i32, i32, i32, i32, i32,
                                        i32, i32, ctypes.c_float, i32]
    lib.oracle_kv_append_quant.argtypes = [p, p, p, i32, p, p, p, p, i32, i32, i32, i32, i32]
    lib.oracle_quantize.argtypes = [p, ctypes.c_int64, ctypes.c_float, i32, p]
    lib.oracle_code_values.argtypes = [p, ctypes.c_int64, i32, p]
    lib.oracle_decode_quant.argtypes = [p, p, p, p, p, p, p, i32, p, i32, i32, i32, i32, i32,
                                        i32, i32, ctypes.c_float, i32]
    lib.oracle_decode.argtypes = [p, p, p, p, p, i32, p, i32, i32, i32, i32, i32,
                                  i32, i32, ctypes.c_float, i32]
    for f in (lib.oracle_kv_append, lib.oracle_block_copy, lib.oracle_block_swap,
              lib.oracle_decode, lib.oracle_decode_multi, lib.oracle_kv_append_quant,
              lib.oracle_quantize, lib.oracle_code_values, lib.oracle_decode_quant,
              lib.oracle_max_threads):
        f.restype = ctypes.c_int
    lib.oracle_max_threads.argtypes = []
    return lib


@contextlib.contextmanager
def use_library(path: str):
    """Temporarily route every call to another build of the oracle source (the
    mutation tests use it to check that planted slips fail the pins)."""
    global _lib
    with _lock:
        saved = _lib
        _lib = _bind(path)
    try:
        yield
    finally:
        with _lock:
            _lib = saved


def compile_source(src_path: str, out_path: str) -> str:
    """Compile an oracle C source with the same flags as ``build``."""
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-shared",
           "-fPIC", "-std=c11", src_path, "-o", out_path, "-lm"]
    subprocess.run(cmd, check=True)
    return out_path


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = _bind(_LIB_PATH)
    return _lib


class OracleError(RuntimeError):
    pass


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.uint8:
        return FP8_E4M3      # one-byte codes: moves do not look at their meaning
    raise TypeError(f"cache element type must be float32, uint16 (bf16 bits) or uint8 (codes), "
                    f"got {a.dtype}")


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _check(rc: int, what: str) -> None:
    if rc != 0:
        reason = {-1: "invalid argument", -2: "index outside the pool",
                  -3: "out of memory"}.get(rc, str(rc))
        raise OracleError(f"oracle {what}: {reason}")


def _contig(a: np.ndarray, dtype=None) -> np.ndarray:
    a = np.asarray(a)
    if dtype is not None and a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    if not a.flags.c_contiguous:
        raise ValueError("arrays passed to the oracle must be C-contiguous")
    return a


def kv_append(k: np.ndarray, v: np.ndarray, slot_mapping: np.ndarray,
              k_cache: np.ndarray, v_cache: np.ndarray) -> None:
    """In place: write k[i], v[i] ([T][Hkv][d]) into slot_mapping[i] (int64)."""
    k_cache = _contig(k_cache)
    v_cache = _contig(v_cache, k_cache.dtype)
    nb, hkv, bs, d = k_cache.shape
    k = _contig(k, k_cache.dtype)
    v = _contig(v, k_cache.dtype)
    slot = _contig(slot_mapping, np.int64)
    t = slot.shape[0]
    if k.shape != (t, hkv, d) or v.shape != (t, hkv, d):
        raise ValueError("k/v must be [num_tokens][num_kv_heads][head_dim]")
    rc = _load().oracle_kv_append(_ptr(k), _ptr(v), _ptr(slot), t, _ptr(k_cache),
                                  _ptr(v_cache), nb, hkv, bs, d, _dtype_code(k_cache))
    _check(rc, "kv_append")


def block_copy(pairs: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray) -> None:
    """In place: for every (src, dst) row of ``pairs`` (int64 [P][2]) copy block src to dst."""
    k_cache = _contig(k_cache)
    v_cache = _contig(v_cache, k_cache.dtype)
    nb, hkv, bs, d = k_cache.shape
    pairs = _contig(np.asarray(pairs, dtype=np.int64).reshape(-1, 2))
    rc = _load().oracle_block_copy(_ptr(pairs), pairs.shape[0], _ptr(k_cache), _ptr(v_cache),
                                   nb, hkv, bs, d, _dtype_code(k_cache))
    _check(rc, "block_copy")


def block_swap(pairs: np.ndarray, src_k: np.ndarray, src_v: np.ndarray, dst_k: np.ndarray,
               dst_v: np.ndarray) -> None:
    """In place on dst: for every (src, dst) row of ``pairs`` copy block src of the
    source pool to block dst of the destination pool (same block shape)."""
    src_k = _contig(src_k)
    src_v = _contig(src_v, src_k.dtype)
    dst_k = _contig(dst_k, src_k.dtype)
    dst_v = _contig(dst_v, src_k.dtype)
    if src_k.shape[1:] != dst_k.shape[1:] or src_v.shape != src_k.shape or \
            dst_v.shape != dst_k.shape:
        raise ValueError("the pools differ in block shape")
    pairs = _contig(np.asarray(pairs, dtype=np.int64).reshape(-1, 2))
    _, hkv, bs, d = src_k.shape
    rc = _load().oracle_block_swap(_ptr(pairs), pairs.shape[0], _ptr(src_k), _ptr(src_v),
                                   src_k.shape[0], _ptr(dst_k), _ptr(dst_v), dst_k.shape[0],
                                   hkv, bs, d, _dtype_code(src_k))
    _check(rc, "block_swap")


def decode(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
           block_tables: np.ndarray, context_lens: np.ndarray, scale: float,
           num_threads: int = 1) -> np.ndarray:
    """Return out (float64 [S][H][d]) = softmax(scale q K^T) V over the paged context."""
    k_cache = _contig(k_cache)
    v_cache = _contig(v_cache, k_cache.dtype)
    nb, hkv, bs, d = k_cache.shape
    q = _contig(q, k_cache.dtype)
    s, h, dq = q.shape
    if dq != d:
        raise ValueError("q head_dim differs from the cache's")
    tables = _contig(block_tables, np.int32)
    ctx = _contig(context_lens, np.int32)
    if tables.ndim != 2 or tables.shape[0] != s or ctx.shape != (s,):
        raise ValueError("block_tables must be [S][stride], context_lens [S]")
    out = np.zeros((s, h, d), dtype=np.float64)
    rc = _load().oracle_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                               _ptr(tables), tables.shape[1], _ptr(ctx), s, h, hkv, nb, bs, d,
                               _dtype_code(k_cache), float(np.float32(scale)), int(num_threads))
    _check(rc, "decode")
    return out


def decode_multi(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                 block_tables: np.ndarray, context_lens: np.ndarray, query_start: np.ndarray,
                 scale: float, num_threads: int = 1) -> np.ndarray:
    """Several query tokens per sequence: q [T][H][d], rows query_start[s] ..
    query_start[s+1]-1 of sequence s are its last n_s context positions, each
    attending causally. Returns out (float64 [T][H][d])."""
    k_cache = _contig(k_cache)
    v_cache = _contig(v_cache, k_cache.dtype)
    nb, hkv, bs, d = k_cache.shape
    q = _contig(q, k_cache.dtype)
    t, h, dq = q.shape
    if dq != d:
        raise ValueError("q head_dim differs from the cache's")
    tables = _contig(block_tables, np.int32)
    ctx = _contig(context_lens, np.int32)
    qs = _contig(query_start, np.int32)
    s = ctx.shape[0]
    if tables.ndim != 2 or tables.shape[0] != s or qs.shape != (s + 1,) or qs[-1] != t:
        raise ValueError("block_tables [S][stride], context_lens [S], query_start [S+1] ending at T")
    out = np.zeros((t, h, d), dtype=np.float64)
    rc = _load().oracle_decode_multi(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                     _ptr(tables), tables.shape[1], _ptr(ctx), _ptr(qs), s, h,
                                     hkv, nb, bs, d, _dtype_code(k_cache),
                                     float(np.float32(scale)), int(num_threads))
    _check(rc, "decode_multi")
    return out


def quantize(x: np.ndarray, scale: float, fmt: str) -> np.ndarray:
    """Codes (uint8) of binary32 values x under ``scale``: the code of x / scale
    (binary32 division) in FP8 E4M3 ("fp8", nearest-even, saturating to +-448,
    NaN -> 0x7F) or int8 ("int8", clamp to +-127 then nearest-even)."""
    x = _contig(np.asarray(x, dtype=np.float32))
    codes = np.zeros(x.shape, dtype=np.uint8)
    _check(_load().oracle_quantize(_ptr(x), x.size, float(np.float32(scale)),
                                   QUANT_FORMATS[fmt], _ptr(codes)), "quantize")
    return codes


def code_values(codes: np.ndarray, fmt: str) -> np.ndarray:
    """float64 values of stored codes (unscaled)."""
    codes = _contig(np.asarray(codes, dtype=np.uint8))
    out = np.zeros(codes.shape, dtype=np.float64)
    _check(_load().oracle_code_values(_ptr(codes), codes.size, QUANT_FORMATS[fmt], _ptr(out)),
           "code_values")
    return out


def kv_append_quant(k: np.ndarray, v: np.ndarray, slot_mapping: np.ndarray,
                    k_cache: np.ndarray, v_cache: np.ndarray, k_scale: np.ndarray,
                    v_scale: np.ndarray, fmt: str) -> None:
    """In place: bf16 (uint16 bits) k, v [T][Hkv][d] quantised into uint8 caches
    [NB][Hkv][B][d] with per-kv-head binary32 scales."""
    k = _contig(k, np.uint16)
    v = _contig(v, np.uint16)
    k_cache = _contig(k_cache, np.uint8)
    v_cache = _contig(v_cache, np.uint8)
    nb, hkv, bs, d = k_cache.shape
    ks = _contig(np.asarray(k_scale, np.float32))
    vs = _contig(np.asarray(v_scale, np.float32))
    slots = _contig(np.asarray(slot_mapping, np.int64))
    if ks.shape != (hkv,) or vs.shape != (hkv,) or k.shape != (slots.shape[0], hkv, d):
        raise ValueError("k, v [T][Hkv][d]; scales [Hkv]")
    _check(_load().oracle_kv_append_quant(_ptr(k), _ptr(v), _ptr(slots), slots.shape[0],
                                          _ptr(k_cache), _ptr(v_cache), _ptr(ks), _ptr(vs),
                                          nb, hkv, bs, d, QUANT_FORMATS[fmt]), "kv_append_quant")


def decode_quant(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                 k_scale: np.ndarray, v_scale: np.ndarray, block_tables: np.ndarray,
                 context_lens: np.ndarray, scale: float, fmt: str,
                 num_threads: int = 1) -> np.ndarray:
    """Decode over quantised caches (uint8 codes, per-kv-head scales); q bf16 bits."""
    k_cache = _contig(k_cache, np.uint8)
    v_cache = _contig(v_cache, np.uint8)
    nb, hkv, bs, d = k_cache.shape
    q = _contig(q, np.uint16)
    s, h, dq = q.shape
    ks = _contig(np.asarray(k_scale, np.float32))
    vs = _contig(np.asarray(v_scale, np.float32))
    tables = _contig(block_tables, np.int32)
    ctx = _contig(context_lens, np.int32)
    if dq != d or ks.shape != (hkv,) or vs.shape != (hkv,) or tables.shape[0] != s:
        raise ValueError("shapes: q [S][H][d], scales [Hkv], tables [S][stride]")
    out = np.zeros((s, h, d), dtype=np.float64)
    _check(_load().oracle_decode_quant(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                       _ptr(ks), _ptr(vs), _ptr(tables), tables.shape[1],
                                       _ptr(ctx), s, h, hkv, nb, bs, d, QUANT_FORMATS[fmt],
                                       float(np.float32(scale)), int(num_threads)),
           "decode_quant")
    return out


def max_threads() -> int:
    """Threads the oracle's OpenMP runtime would use by default."""
    return int(_load().oracle_max_threads())
