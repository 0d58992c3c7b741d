"""Paged KV-cache decode attention for one B200 (sm_100a).

Thin Python binding of the C ABI in ``include/pa.h`` (``libpa.so``). The
functions below keep the ABI's names and only marshal arguments: tensors to
device pointers, the current CUDA stream, status codes to exceptions. Every
step of the computation runs in the library's CUDA kernels; there is no CPU
or PyTorch fallback, and a call without the built library or on a tensor that
is not on a CUDA device raises.

    pa_kv_append(k, v, slot_mapping, k_cache, v_cache)
    pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, ...)
    pa_block_copy(src_dst_pairs, k_cache, v_cache)

Cache layout: ``k_cache``/``v_cache`` are ``[num_blocks][num_kv_heads]
[block_size][head_dim]`` tensors of float32 or bfloat16.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libpa.so")
INCLUDE_DIR = os.path.join(os.path.dirname(PKG_DIR), "include")
HEADER = os.path.join(INCLUDE_DIR, "pa.h")

PA_OK = 0
PA_ERR_INVALID_ARG = -1
PA_ERR_DTYPE = -2
PA_ERR_ALIGN = -3
PA_ERR_UNSUPPORTED = -4
PA_ERR_CUDA = -5
PA_ERR_BAD_INDEX = -6
PA_ERR_WORKSPACE = -7
PA_ERR_TIMEOUT = -8
PA_F32 = 0
PA_BF16 = 1
PA_FP8_E4M3 = 2             # quantised caches: torch.float8_e4m3fn / torch.int8 code tensors
PA_INT8 = 3
PA_NOALLOC_SCRATCH_BYTES = 32 << 20
PA_GROUPED_MMA_SYNC = 0     # pa_set_grouped_consumer() values
PA_GROUPED_TCGEN05 = 1
PA_KERNEL_SIMT = 0          # pa_test_last_decode_kernel() values
PA_KERNEL_MMA = 1
PA_KERNEL_GROUPED = 2
PA_KERNEL_GROUPED_TCGEN05 = 3

_lock = threading.Lock()
_lib = None


class PAError(RuntimeError):
    """A non-zero status from the library, with its code and message."""

    def __init__(self, code: int, message: str):
        super().__init__(f"{_status_name(code)} ({code}): {message}")
        self.code = code


class pa_cache_desc(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("dtype", ctypes.c_int32)]


def _status_name(code: int) -> str:
    try:
        return load_library().pa_status_string(code).decode()
    except Exception:  # library not loadable: fall back to the literal
        return str(code)


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load ``libpa.so`` (built by ``paged_kv_cache_335_b200.build``); raise if it is missing."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"{p} is not built: run `python -m paged_kv_cache_335_b200.build` "
                               "(or __graft_entry__.build()) first; there is no fallback path")
        lib = ctypes.CDLL(p)
        vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
        desc = ctypes.POINTER(pa_cache_desc)
        lib.pa_kv_append.argtypes = [vp, vp, vp, i32, vp, vp, desc, vp]
        lib.pa_decode.argtypes = [vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, f32, desc, i32,
                                  vp, sz, vp]
        lib.pa_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, f32, desc,
                                          i32, vp]
        lib.pa_decode_noalloc.restype = ctypes.c_int
        lib.pa_decode_workspace_size.argtypes = [i32, i32, i32, desc, i32]
        lib.pa_decode_workspace_size.restype = sz
        lib.pa_decode_num_partitions.argtypes = [i32, i32, i32, desc, i32]
        lib.pa_decode_grouped.argtypes = [vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, f32, desc,
                                          i32, i32, vp, sz, vp]
        lib.pa_decode_multi.argtypes = [vp, vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, i32,
                                        f32, desc, i32, vp, sz, vp]
        lib.pa_decode_multi_workspace_size.argtypes = [i32, i32, i32, i32, i32, desc, i32]
        lib.pa_decode_multi_workspace_size.restype = sz
        lib.pa_decode_multi_num_partitions.argtypes = [i32, i32, i32, i32, i32, desc, i32]
        lib.pa_decode_grouped_workspace_size.argtypes = [i32, i32, i32, desc, i32, i32]
        lib.pa_decode_grouped_workspace_size.restype = sz
        lib.pa_decode_grouped_num_partitions.argtypes = [i32, i32, i32, desc, i32, i32]
        lib.pa_block_copy.argtypes = [vp, i32, vp, vp, desc, vp]
        lib.pa_kv_append_quant.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, desc, vp]
        lib.pa_decode_quant.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, f32,
                                        desc, i32, vp, sz, vp]
        lib.pa_decode_grouped_quant.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, vp, i32, i32,
                                                i32, f32, desc, i32, i32, vp, sz, vp]
        lib.pa_decode_multi_quant.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, i32, i32,
                                              i32, i32, i32, f32, desc, i32, vp, sz, vp]
        lib.pa_block_swap.argtypes = [vp, i32, vp, vp, desc, vp, vp, desc, vp]
        lib.pa_sync_check.argtypes = [vp]
        lib.pa_stream_read.argtypes = [vp, sz, vp, i32, vp]
        lib.pa_test_skip_load.argtypes = [i32]
        lib.pa_test_skip_load.restype = None
        lib.pa_test_last_decode_kernel.argtypes = []
        lib.pa_set_grouped_consumer.argtypes = [ctypes.c_int]
        lib.pa_stream_read.restype = ctypes.c_int
        lib.pa_get_last_error.argtypes = []
        lib.pa_get_last_error.restype = ctypes.c_char_p
        lib.pa_status_string.argtypes = [ctypes.c_int]
        lib.pa_status_string.restype = ctypes.c_char_p
        for f in (lib.pa_kv_append, lib.pa_decode, lib.pa_decode_num_partitions,
                  lib.pa_block_copy, lib.pa_sync_check):
            f.restype = ctypes.c_int
        if path is None:
            _lib = lib
        return lib


def header_functions(header: str | None = None) -> list:
    """Names of the functions the headers under ``include/`` declare (or one header)."""
    paths = [header] if header else sorted(
        os.path.join(INCLUDE_DIR, f) for f in os.listdir(INCLUDE_DIR) if f.endswith(".h"))
    names = set()
    for path in paths:
        text = open(path, encoding="utf-8").read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names.update(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w]*\s*\*?\s*(pa_\w+)\s*\(",
                                text, flags=re.M))
    return sorted(names)


def _check(rc: int) -> None:
    if rc != PA_OK:
        msg = load_library().pa_get_last_error().decode(errors="replace")
        raise PAError(rc, msg)


# ---------------------------------------------------------------------------
# marshalling helpers (torch is imported lazily so the ABI can load without it)
# ---------------------------------------------------------------------------
def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return PA_F32
    if t.dtype == torch.bfloat16:
        return PA_BF16
    if t.dtype == torch.float8_e4m3fn:
        return PA_FP8_E4M3
    if t.dtype == torch.int8:
        return PA_INT8
    raise TypeError(f"unsupported element type {t.dtype}: float32, bfloat16, float8_e4m3fn "
                    "(FP8 E4M3 codes) or int8 (int8 codes)")


def _on_current_device(t, name: str):
    """The library launches on the current device and stream: a tensor of another
    GPU would hand its kernels a pointer they cannot use."""
    cur = _torch().cuda.current_device()
    if t.device.index != cur:
        raise ValueError(f"{name} is on {t.device}, but the current CUDA device is cuda:{cur}; "
                         "call under torch.cuda.device(...) of the tensors' device")


def _dev(t, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path exists)")
    _on_current_device(t, name)
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _addressable(t, name: str):
    """A CUDA tensor or a pinned host tensor (which the device addresses directly)."""
    if not (t.is_cuda or t.is_pinned()):
        raise ValueError(f"{name} must be a CUDA tensor or pinned host memory")
    if t.is_cuda:
        _on_current_device(t, name)
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def cache_desc(k_cache) -> pa_cache_desc:
    """Descriptor of a ``[num_blocks][num_kv_heads][block_size][head_dim]`` pool tensor."""
    if k_cache.dim() != 4:
        raise ValueError("cache must be [num_blocks][num_kv_heads][block_size][head_dim]")
    nb, hkv, bs, d = (int(x) for x in k_cache.shape)
    return pa_cache_desc(nb, hkv, bs, d, _dtype_code(k_cache))


def _same_pool(k_cache, v_cache):
    if k_cache.shape != v_cache.shape or k_cache.dtype != v_cache.dtype:
        raise ValueError("k_cache and v_cache must have the same shape and dtype")


# ---------------------------------------------------------------------------
# the three operations
# ---------------------------------------------------------------------------
def pa_kv_append(k, v, slot_mapping, k_cache, v_cache, stream=None) -> None:
    """Write k[i], v[i] ([T][num_kv_heads][head_dim]) into slot_mapping[i] (int64; <0 skips)."""
    torch = _torch()
    _same_pool(k_cache, v_cache)
    desc = cache_desc(k_cache)
    t = int(slot_mapping.shape[0])
    if tuple(k.shape) != (t, desc.num_kv_heads, desc.head_dim) or k.shape != v.shape:
        raise ValueError("k and v must be [num_tokens][num_kv_heads][head_dim]")
    if k.dtype != k_cache.dtype or v.dtype != k_cache.dtype:
        raise TypeError("k, v and the caches must share one dtype")
    _check(load_library().pa_kv_append(
        _dev(k, "k"), _dev(v, "v"), _dev(slot_mapping, "slot_mapping", torch.int64), t,
        _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"), ctypes.byref(desc), _stream(stream)))


def pa_block_copy(src_dst_pairs, k_cache, v_cache, stream=None) -> None:
    """Copy whole blocks: for each (src, dst) row of ``src_dst_pairs`` (int64 [P][2])."""
    torch = _torch()
    _same_pool(k_cache, v_cache)
    desc = cache_desc(k_cache)
    if src_dst_pairs.dim() != 2 or src_dst_pairs.shape[1] != 2:
        raise ValueError("src_dst_pairs must be [num_pairs][2]")
    _check(load_library().pa_block_copy(
        _dev(src_dst_pairs, "src_dst_pairs", torch.int64), int(src_dst_pairs.shape[0]),
        _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"), ctypes.byref(desc), _stream(stream)))


def pa_kv_append_quant(k, v, slot_mapping, k_cache, v_cache, k_scale, v_scale,
                       stream=None) -> None:
    """Quantising append: bf16 k, v [T][Hkv][D] into a float8_e4m3fn or int8 code
    pool, each element stored as the code of x / scale[kv head] (k_scale, v_scale:
    float32 [Hkv] on the device)."""
    torch = _torch()
    _same_pool(k_cache, v_cache)
    desc = cache_desc(k_cache)
    if k.shape != v.shape or k.dim() != 3 or k.shape[1:] != (desc.num_kv_heads, desc.head_dim):
        raise ValueError("k and v must be [num_tokens][num_kv_heads][head_dim]")
    if k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
        raise TypeError("k and v must be bfloat16")
    _check(load_library().pa_kv_append_quant(
        _dev(k, "k"), _dev(v, "v"), _dev(slot_mapping, "slot_mapping", torch.int64),
        int(k.shape[0]), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(k_scale, "k_scale", torch.float32), _dev(v_scale, "v_scale", torch.float32),
        ctypes.byref(desc), _stream(stream)))


def pa_decode_quant(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                    scale: float, max_context_len: int | None = None, partition_size: int = 0,
                    workspace=None, stream=None) -> None:
    """pa_decode over a quantised (float8_e4m3fn / int8 code) pool with per-kv-head
    float32 scales; q and out bfloat16."""
    torch = _torch()
    _same_pool(k_cache, v_cache)
    desc = cache_desc(k_cache)
    s, h, d = (int(x) for x in q.shape)
    if tuple(out.shape) != (s, h, d) or d != desc.head_dim:
        raise ValueError("q and out must be [num_seqs][num_heads][head_dim]")
    if q.dtype != torch.bfloat16 or out.dtype != torch.bfloat16:
        raise TypeError("q and out must be bfloat16")
    if max_context_len is None:
        max_context_len = int(context_lens.max().item()) if s else 0
    need = pa_decode_workspace_size(s, h, max_context_len, k_cache, partition_size)
    ws_ptr, ws_bytes = ctypes.c_void_p(0), 0
    if need:
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    _check(load_library().pa_decode_quant(
        _dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(k_scale, "k_scale", torch.float32), _dev(v_scale, "v_scale", torch.float32),
        _dev(block_tables, "block_tables", torch.int32), int(block_tables.shape[1]),
        _dev(context_lens, "context_lens", torch.int32), int(max_context_len), s, h,
        float(scale), ctypes.byref(desc), int(partition_size), ws_ptr, ws_bytes,
        _stream(stream)))


def _quant_ws(need, workspace, device):
    torch = _torch()
    if not need:
        return ctypes.c_void_p(0), 0
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    return _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()


def pa_decode_grouped_quant(out, q, k_cache, v_cache, k_scale, v_scale, block_tables,
                            context_lens, scale: float, group_size: int,
                            max_context_len: int | None = None, partition_size: int = 0,
                            workspace=None, stream=None) -> None:
    """pa_decode_grouped over a quantised pool (pa_decode_quant's arguments plus
    group_size): sequences [k group_size, (k + 1) group_size) decoded together."""
    torch = _torch()
    _same_pool(k_cache, v_cache)
    desc = cache_desc(k_cache)
    s, h, d = (int(x) for x in q.shape)
    if tuple(out.shape) != (s, h, d) or d != desc.head_dim:
        raise ValueError("q and out must be [num_seqs][num_heads][head_dim]")
    if q.dtype != torch.bfloat16 or out.dtype != torch.bfloat16:
        raise TypeError("q and out must be bfloat16")
    if max_context_len is None:
        max_context_len = int(context_lens.max().item()) if s else 0
    need = pa_decode_grouped_workspace_size(s, h, max_context_len, k_cache, int(group_size),
                                            partition_size)
    ws_ptr, ws_bytes = _quant_ws(need, workspace, q.device)
    _check(load_library().pa_decode_grouped_quant(
        _dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(k_scale, "k_scale", torch.float32), _dev(v_scale, "v_scale", torch.float32),
        _dev(block_tables, "block_tables", torch.int32), int(block_tables.shape[1]),
        _dev(context_lens, "context_lens", torch.int32), int(max_context_len), s, h,
        float(scale), ctypes.byref(desc), int(group_size), int(partition_size), ws_ptr,
        ws_bytes, _stream(stream)))


def pa_decode_multi_quant(out, q, k_cache, v_cache, k_scale, v_scale, block_tables,
                          context_lens, query_start, scale: float,
                          max_context_len: int | None = None, max_query_len: int | None = None,
                          partition_size: int = 0, workspace=None, stream=None) -> None:
    """pa_decode_multi over a quantised pool (q / out bfloat16 [T][H][D])."""
    torch = _torch()
    _same_pool(k_cache, v_cache)
    desc = cache_desc(k_cache)
    t, h, d = (int(x) for x in q.shape)
    s = int(context_lens.shape[0])
    if tuple(out.shape) != (t, h, d) or d != desc.head_dim:
        raise ValueError("q and out must be [num_query_tokens][num_heads][head_dim]")
    if q.dtype != torch.bfloat16 or out.dtype != torch.bfloat16:
        raise TypeError("q and out must be bfloat16")
    if block_tables.dim() != 2 or block_tables.shape[0] != s or query_start.shape != (s + 1,):
        raise ValueError("block_tables [S][stride], context_lens [S], query_start [S + 1]")
    if max_context_len is None:
        max_context_len = int(context_lens.max().item()) if s else 0
    if max_query_len is None:
        max_query_len = max(1, int((query_start[1:] - query_start[:-1]).max().item())) if s else 1
    need = pa_decode_multi_workspace_size(s, t, max_query_len, h, max_context_len, k_cache,
                                          partition_size)
    ws_ptr, ws_bytes = _quant_ws(need, workspace, q.device)
    _check(load_library().pa_decode_multi_quant(
        _dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(k_scale, "k_scale", torch.float32), _dev(v_scale, "v_scale", torch.float32),
        _dev(block_tables, "block_tables", torch.int32), int(block_tables.shape[1]),
        _dev(context_lens, "context_lens", torch.int32),
        _dev(query_start, "query_start", torch.int32), int(max_context_len), s, t,
        int(max_query_len), h, float(scale), ctypes.byref(desc), int(partition_size), ws_ptr,
        ws_bytes, _stream(stream)))


def pa_block_swap(src_dst_pairs, src_k, src_v, dst_k, dst_v, stream=None) -> None:
    """Copy whole blocks between two pools of the same block shape (swap-out to /
    swap-in from pinned host memory): for each (src, dst) row of ``src_dst_pairs``
    (int64 [P][2], on the device), block dst of (dst_k, dst_v) gets block src of
    (src_k, src_v). Either pool may be a CUDA tensor or a pinned host tensor."""
    torch = _torch()
    _same_pool(src_k, src_v)
    _same_pool(dst_k, dst_v)
    sd, dd = cache_desc(src_k), cache_desc(dst_k)
    if src_dst_pairs.dim() != 2 or src_dst_pairs.shape[1] != 2:
        raise ValueError("src_dst_pairs must be [num_pairs][2]")
    _check(load_library().pa_block_swap(
        _dev(src_dst_pairs, "src_dst_pairs", torch.int64), int(src_dst_pairs.shape[0]),
        _addressable(src_k, "src_k"), _addressable(src_v, "src_v"), ctypes.byref(sd),
        _addressable(dst_k, "dst_k"), _addressable(dst_v, "dst_v"), ctypes.byref(dd),
        _stream(stream)))


def pa_decode_workspace_size(num_seqs: int, num_heads: int, max_context_len: int, k_cache,
                             partition_size: int = 0) -> int:
    return pa_decode_grouped_workspace_size(num_seqs, num_heads, max_context_len, k_cache, 1,
                                            partition_size)


def pa_decode_num_partitions(num_seqs: int, num_heads: int, max_context_len: int, k_cache,
                             partition_size: int = 0) -> int:
    return pa_decode_grouped_num_partitions(num_seqs, num_heads, max_context_len, k_cache, 1,
                                            partition_size)


def pa_decode_grouped_workspace_size(num_seqs: int, num_heads: int, max_context_len: int,
                                     k_cache, group_size: int, partition_size: int = 0) -> int:
    lib = load_library()
    desc = cache_desc(k_cache)
    if group_size == 1:
        n = lib.pa_decode_workspace_size(num_seqs, num_heads, max_context_len,
                                         ctypes.byref(desc), partition_size)
    else:
        n = lib.pa_decode_grouped_workspace_size(num_seqs, num_heads, max_context_len,
                                                 ctypes.byref(desc), group_size, partition_size)
    if n == 0:
        msg = lib.pa_get_last_error().decode()
        rc = _num_partitions(num_seqs, num_heads, max_context_len, desc, group_size,
                             partition_size)
        if rc < 0:
            raise PAError(rc, msg)
    return int(n)


def _num_partitions(num_seqs, num_heads, max_context_len, desc, group_size, partition_size):
    lib = load_library()
    if group_size == 1:
        return lib.pa_decode_num_partitions(num_seqs, num_heads, max_context_len,
                                            ctypes.byref(desc), partition_size)
    return lib.pa_decode_grouped_num_partitions(num_seqs, num_heads, max_context_len,
                                                ctypes.byref(desc), group_size, partition_size)


def pa_decode_grouped_num_partitions(num_seqs: int, num_heads: int, max_context_len: int,
                                     k_cache, group_size: int, partition_size: int = 0) -> int:
    rc = _num_partitions(num_seqs, num_heads, max_context_len, cache_desc(k_cache), group_size,
                         partition_size)
    if rc < 0:
        _check(rc)
    return rc


def _decode_call(entry, extra, out, q, k_cache, v_cache, block_tables, context_lens, scale,
                 max_context_len, group_size, partition_size, workspace, stream):
    torch = _torch()
    _same_pool(k_cache, v_cache)
    desc = cache_desc(k_cache)
    s, h, d = (int(x) for x in q.shape)
    if tuple(out.shape) != (s, h, d) or d != desc.head_dim:
        raise ValueError("q and out must be [num_seqs][num_heads][head_dim]")
    if q.dtype != k_cache.dtype or out.dtype != k_cache.dtype:
        raise TypeError("q, out and the caches must share one dtype")
    if block_tables.dim() != 2 or block_tables.shape[0] != s or context_lens.shape != (s,):
        raise ValueError("block_tables must be [num_seqs][stride], context_lens [num_seqs]")
    if max_context_len is None:
        max_context_len = int(context_lens.max().item()) if s else 0
    need = pa_decode_grouped_workspace_size(s, h, max_context_len, k_cache, group_size,
                                            partition_size)
    ws_ptr, ws_bytes = ctypes.c_void_p(0), 0
    if need:
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    _check(entry(
        _dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32), int(block_tables.shape[1]),
        _dev(context_lens, "context_lens", torch.int32), int(max_context_len), s, h,
        float(scale), ctypes.byref(desc), *extra, int(partition_size), ws_ptr, ws_bytes,
        _stream(stream)))


def pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale: float,
              max_context_len: int | None = None, partition_size: int = 0, workspace=None,
              stream=None) -> None:
    """out[s][h] = softmax(scale q[s][h] . K) V over the context_lens[s] paged tokens.

    ``max_context_len`` is a host bound on context_lens (computed with a device
    sync if omitted). ``workspace``: a CUDA uint8 tensor of at least
    ``pa_decode_workspace_size`` bytes (allocated here if omitted and needed).
    """
    _decode_call(load_library().pa_decode, (), out, q, k_cache, v_cache, block_tables,
                 context_lens, scale, max_context_len, 1, partition_size, workspace, stream)


def pa_decode_grouped(out, q, k_cache, v_cache, block_tables, context_lens, scale: float,
                      group_size: int, max_context_len: int | None = None,
                      partition_size: int = 0, workspace=None, stream=None) -> None:
    """pa_decode with sequences [k group_size, (k + 1) group_size) decoded together,
    so blocks they share (beams, parallel samples of one prompt) are read once.

    Same result contract as ``pa_decode``; ``workspace`` is sized by
    ``pa_decode_grouped_workspace_size``.
    """
    _decode_call(load_library().pa_decode_grouped, (int(group_size),), out, q, k_cache, v_cache,
                 block_tables, context_lens, scale, max_context_len, int(group_size),
                 partition_size, workspace, stream)


def pa_decode_multi_workspace_size(num_seqs: int, num_query_tokens: int, max_query_len: int,
                                   num_heads: int, max_context_len: int, k_cache,
                                   partition_size: int = 0) -> int:
    lib = load_library()
    desc = cache_desc(k_cache)
    n = lib.pa_decode_multi_workspace_size(num_seqs, num_query_tokens, max_query_len, num_heads,
                                           max_context_len, ctypes.byref(desc), partition_size)
    if n == 0:
        msg = lib.pa_get_last_error().decode()
        rc = lib.pa_decode_multi_num_partitions(num_seqs, num_query_tokens, max_query_len,
                                                num_heads, max_context_len, ctypes.byref(desc),
                                                partition_size)
        if rc < 0:
            raise PAError(rc, msg)
    return int(n)


def pa_decode_multi_num_partitions(num_seqs: int, num_query_tokens: int, max_query_len: int,
                                   num_heads: int, max_context_len: int, k_cache,
                                   partition_size: int = 0) -> int:
    rc = load_library().pa_decode_multi_num_partitions(
        num_seqs, num_query_tokens, max_query_len, num_heads, max_context_len,
        ctypes.byref(cache_desc(k_cache)), partition_size)
    if rc < 0:
        _check(rc)
    return rc


def pa_decode_multi(out, q, k_cache, v_cache, block_tables, context_lens, query_start,
                    scale: float, max_context_len: int | None = None,
                    max_query_len: int | None = None, partition_size: int = 0, workspace=None,
                    stream=None) -> None:
    """Several query tokens per sequence (chunked prefill, draft verification):
    q / out [T][H][D] with rows query_start[s] .. query_start[s+1]-1 for sequence
    s, its last n_s context positions, each attending causally over the cache."""
    torch = _torch()
    _same_pool(k_cache, v_cache)
    desc = cache_desc(k_cache)
    t, h, d = (int(x) for x in q.shape)
    s = int(context_lens.shape[0])
    if tuple(out.shape) != (t, h, d) or d != desc.head_dim:
        raise ValueError("q and out must be [num_query_tokens][num_heads][head_dim]")
    if q.dtype != k_cache.dtype or out.dtype != k_cache.dtype:
        raise TypeError("q, out and the caches must share one dtype")
    if block_tables.dim() != 2 or block_tables.shape[0] != s or query_start.shape != (s + 1,):
        raise ValueError("block_tables [S][stride], context_lens [S], query_start [S + 1]")
    if max_context_len is None:
        max_context_len = int(context_lens.max().item()) if s else 0
    if max_query_len is None:
        max_query_len = max(1, int((query_start[1:] - query_start[:-1]).max().item())) if s else 1
    need = pa_decode_multi_workspace_size(s, t, max_query_len, h, max_context_len, k_cache,
                                          partition_size)
    ws_ptr, ws_bytes = ctypes.c_void_p(0), 0
    if need:
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    _check(load_library().pa_decode_multi(
        _dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32), int(block_tables.shape[1]),
        _dev(context_lens, "context_lens", torch.int32),
        _dev(query_start, "query_start", torch.int32), int(max_context_len), s, t,
        int(max_query_len), h, float(scale), ctypes.byref(desc), int(partition_size), ws_ptr,
        ws_bytes, _stream(stream)))


def pa_decode_noalloc(out, q, k_cache, v_cache, block_tables, context_lens, scale: float,
                      max_context_len: int | None = None, partition_size: int = 0,
                      stream=None) -> None:
    """pa_decode without a workspace argument, for callers that cannot allocate
    device memory: a split context uses the library's fixed scratch buffer of
    PA_NOALLOC_SCRATCH_BYTES per device. Calls that overlap on the GPU race on
    that buffer; make the first call on a device before any stream capture."""
    torch = _torch()
    _same_pool(k_cache, v_cache)
    desc = cache_desc(k_cache)
    s, h, d = (int(x) for x in q.shape)
    if tuple(out.shape) != (s, h, d) or d != desc.head_dim:
        raise ValueError("q and out must be [num_seqs][num_heads][head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != s or context_lens.shape != (s,):
        raise ValueError("block_tables must be [num_seqs][stride], context_lens [num_seqs]")
    if max_context_len is None:
        max_context_len = int(context_lens.max().item()) if s else 0
    _check(load_library().pa_decode_noalloc(
        _dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32), int(block_tables.shape[1]),
        _dev(context_lens, "context_lens", torch.int32), int(max_context_len), s, h,
        float(scale), ctypes.byref(desc), int(partition_size), _stream(stream)))


def pa_set_grouped_consumer(consumer: int) -> int:
    """Select the grouped / multi-token consumer (PA_GROUPED_MMA_SYNC or
    PA_GROUPED_TCGEN05); returns the previous one. Process-wide."""
    rc = load_library().pa_set_grouped_consumer(int(consumer))
    _check(min(rc, 0))
    return rc


def pa_sync_check(stream=None) -> None:
    """Wait for the stream; raise PAError if a kernel met an out-of-range index."""
    _check(load_library().pa_sync_check(_stream(stream)))


__all__ = ["pa_kv_append", "pa_decode", "pa_decode_noalloc", "pa_block_copy", "pa_decode_workspace_size",
           "pa_decode_num_partitions", "pa_decode_grouped", "pa_decode_grouped_workspace_size",
           "pa_decode_grouped_num_partitions", "pa_decode_multi", "pa_decode_multi_workspace_size",
           "pa_decode_multi_num_partitions", "pa_kv_append_quant", "pa_decode_quant", "pa_block_swap",
           "pa_set_grouped_consumer",
           "pa_sync_check", "pa_cache_desc", "cache_desc",
           "load_library", "header_functions", "PAError"]
