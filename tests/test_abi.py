"""The C-ABI library loads and exports what include/pa.h declares, and its
host-side argument checks answer without touching a GPU."""
import ctypes

import pytest

import paged_kv_cache_335_b200 as pa
from paged_kv_cache_335_b200 import build as pbuild


@pytest.fixture(scope="module")
def lib():
    pbuild.build()
    return pa.load_library()


def test_header_declares_the_hot_path():
    names = pa.header_functions()
    for f in ("pa_kv_append", "pa_decode", "pa_block_copy", "pa_decode_workspace_size",
              "pa_sync_check", "pa_get_last_error"):
        assert f in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in pa.header_functions() if not hasattr(lib, n)]
    assert not missing, f"libpa.so lacks {missing}"


def _desc(**kw):
    d = dict(num_blocks=64, num_kv_heads=4, block_size=16, head_dim=128, dtype=pa.PA_BF16)
    d.update(kw)
    return pa.pa_cache_desc(**d)


def _decode_rc(lib, desc, num_seqs=4, num_heads=4, max_ctx=100, stride=8, ptr=16, ps=0,
               scale=0.125):
    p = ctypes.c_void_p(ptr)
    return lib.pa_decode(p, p, p, p, p, stride, p, max_ctx, num_seqs, num_heads, scale,
                         ctypes.byref(desc), ps, None, 0, None)


@pytest.mark.parametrize("field,value,code", [
    ("head_dim", 96, pa.PA_ERR_UNSUPPORTED),
    ("block_size", 24, pa.PA_ERR_UNSUPPORTED),
    ("block_size", 8, pa.PA_ERR_UNSUPPORTED),
    ("dtype", 7, pa.PA_ERR_DTYPE),
    ("num_blocks", 0, pa.PA_ERR_INVALID_ARG),
])
def test_decode_rejects_bad_cache(lib, field, value, code):
    assert _decode_rc(lib, _desc(**{field: value})) == code
    assert lib.pa_get_last_error()


def test_decode_rejects_bad_arguments(lib):
    assert _decode_rc(lib, _desc(), num_heads=6) == pa.PA_ERR_INVALID_ARG   # 6 % 4 != 0
    assert _decode_rc(lib, _desc(), ptr=8) == pa.PA_ERR_ALIGN
    assert _decode_rc(lib, _desc(), max_ctx=200, stride=8) == pa.PA_ERR_INVALID_ARG
    assert _decode_rc(lib, _desc(), ps=24) == pa.PA_ERR_INVALID_ARG
    assert _decode_rc(lib, _desc(), scale=float("inf")) == pa.PA_ERR_INVALID_ARG
    assert _decode_rc(lib, _desc(), num_seqs=0) == pa.PA_OK                 # nothing to do


def test_decode_needs_workspace_when_split(lib):
    desc = _desc(num_kv_heads=1)
    n = lib.pa_decode_num_partitions(1, 8, 4096, ctypes.byref(desc), 512)
    assert n == 8
    need = lib.pa_decode_workspace_size(1, 8, 4096, ctypes.byref(desc), 512)
    assert need >= 8 * 8 * (128 + 2) * 4
    rc = _decode_rc(lib, desc, num_seqs=1, num_heads=8, max_ctx=4096, stride=256, ps=512)
    assert rc == pa.PA_ERR_WORKSPACE
    # unsplit: no partials, only the 256 bytes of the tensor-core kernel's dynamic
    # schedule, which a call may omit (it then runs the static schedule)
    assert lib.pa_decode_workspace_size(1, 8, 4096, ctypes.byref(desc), -1) == 256
    assert lib.pa_decode_workspace_size(1, 8, 4096, ctypes.byref(desc), 512) == \
        (8 * 8 * 128 * 4 + 255) // 256 * 256 + (8 * 8 * 2 * 4 + 255) // 256 * 256 + 256
    d13 = _desc(num_kv_heads=8)  # one query head per kv head: the CUDA-core kernel, no schedule
    assert lib.pa_decode_workspace_size(1, 8, 4096, ctypes.byref(d13), -1) == 0


def test_partition_policy(lib):
    # tensor-core GQA kernel (148 SMs x 4 CTA slots when no GPU is visible): equal
    # partitions, the count minimising waves x (sub-tiles per item + per-item overhead)
    d70 = _desc(num_kv_heads=8)
    assert lib.pa_decode_num_partitions(8, 64, 32768, ctypes.byref(d70), 0) == 9     # 576 items: 1 wave
    d70q = _desc(num_kv_heads=8, dtype=pa.PA_FP8_E4M3)
    assert lib.pa_decode_num_partitions(8, 64, 32768, ctypes.byref(d70q), 0) == 9
    assert lib.pa_decode_num_partitions(128, 64, 2303, ctypes.byref(d70), 0) == 1    # 1024 items already
    assert lib.pa_decode_num_partitions(1, 64, 4096, ctypes.byref(d70), 0) == 16     # >= 256 tokens each
    assert lib.pa_decode_num_partitions(1, 64, 300, ctypes.byref(d70), 0) == 2
    # CUDA-core kernel: split into 512-token partitions only when units cannot fill the GPU
    d13 = _desc(num_kv_heads=40)
    assert lib.pa_decode_num_partitions(256, 40, 4096, ctypes.byref(d13), 0) == 1
    assert lib.pa_decode_num_partitions(2, 40, 4096, ctypes.byref(d13), 0) == 8
    # explicit sizes and "never split"
    assert lib.pa_decode_num_partitions(8, 64, 32768, ctypes.byref(d70), 512) == 64
    assert lib.pa_decode_num_partitions(8, 64, 32768, ctypes.byref(d70), -1) == 1


def test_grouped_partition_policy(lib):
    d70 = _desc(num_kv_heads=8)
    f = lib.pa_decode_grouped_num_partitions
    # a group is the unit: 4-beam groups x 8 kv heads = 256 items fill 296 slots
    # (2 CTAs per SM for 32 query columns at head_dim 128) in one wave
    assert f(128, 64, 2303, ctypes.byref(d70), 4, 0) == 1
    # one group of 8 (64 columns, 1 CTA per SM): 8 items, so split into 18 partitions
    assert f(8, 64, 32768, ctypes.byref(d70), 8, 0) == 18
    assert f(8, 64, 32768, ctypes.byref(d70), 4, 512) == 64           # explicit size
    # group_size 1 and shapes without the grouped kernel follow pa_decode's policy
    assert f(8, 64, 32768, ctypes.byref(d70), 1, 0) == \
        lib.pa_decode_num_partitions(8, 64, 32768, ctypes.byref(d70), 0)
    f32 = _desc(num_kv_heads=8, dtype=pa.PA_F32)
    assert f(2, 64, 4096, ctypes.byref(f32), 4, 0) == \
        lib.pa_decode_num_partitions(2, 64, 4096, ctypes.byref(f32), 0)
    for bad in (0, 9, -1):
        assert f(128, 64, 2303, ctypes.byref(d70), bad, 0) == pa.PA_ERR_INVALID_ARG
    # the same partials as pa_decode's split (which adds its 256-byte schedule counter)
    assert lib.pa_decode_grouped_workspace_size(8, 64, 32768, ctypes.byref(d70), 4, 512) == \
        lib.pa_decode_workspace_size(8, 64, 32768, ctypes.byref(d70), 512) - 256


def test_grouped_decode_rejects_bad_group_size(lib):
    p = ctypes.c_void_p(256)
    desc = _desc()
    for bad in (0, 9):
        rc = lib.pa_decode_grouped(p, p, p, p, p, 8, p, 100, 4, 8, ctypes.c_float(0.1),
                                   ctypes.byref(desc), bad, 0, None, 0, None)
        assert rc == pa.PA_ERR_INVALID_ARG
        assert b"group_size" in lib.pa_get_last_error()


def test_multi_query_policy_and_arguments(lib):
    d70 = _desc(num_kv_heads=8)
    f = lib.pa_decode_multi_num_partitions
    # 8 sequences x 4 query tokens (one group of 4 per sequence and kv head):
    # 64 items for 296 slots, so the 32K context is split
    n = f(8, 32, 4, 64, 32768, ctypes.byref(d70), 0)
    assert 1 < n <= 32768 // 256
    assert f(8, 32, 4, 64, 32768, ctypes.byref(d70), 512) == 64
    assert lib.pa_decode_multi_workspace_size(8, 32, 4, 64, 32768, ctypes.byref(d70), 512) >= \
        32 * 64 * 64 * (128 + 2) * 4                                 # rows are query tokens
    assert f(8, 32, 0, 64, 32768, ctypes.byref(d70), 0) == pa.PA_ERR_INVALID_ARG   # max_query_len
    assert f(8, 32, 33, 64, 32768, ctypes.byref(d70), 0) == pa.PA_ERR_INVALID_ARG
    assert f(8, -1, 1, 64, 32768, ctypes.byref(d70), 0) == pa.PA_ERR_INVALID_ARG
    # fp32: one CUDA-core row per query token; 32 rows x 64 heads fill the GPU unsplit
    f32 = _desc(num_kv_heads=8, dtype=pa.PA_F32)
    assert f(8, 32, 4, 64, 32768, ctypes.byref(f32), 0) == 1
    assert f(8, 32, 4, 64, 32768, ctypes.byref(f32), 512) == 64
    assert f(8, 32, 4, 64, 32768, ctypes.byref(_desc(num_kv_heads=8, dtype=7)), 0) == pa.PA_ERR_DTYPE
    p = ctypes.c_void_p(256)
    rc = lib.pa_decode_multi(p, p, p, p, p, 8, p, None, 100, 2, 4, 2, 64, ctypes.c_float(0.1),
                             ctypes.byref(d70), -1, None, 0, None)
    assert rc == pa.PA_ERR_INVALID_ARG and b"query_start" in lib.pa_get_last_error()


def test_quantised_grouped_and_multi_arguments(lib):
    """pa_decode_grouped_quant / pa_decode_multi_quant: the scales are required,
    the pool must be quantised (and at head_dim 128), the group size and the
    multi-token arguments are checked as on the bf16 calls."""
    p = ctypes.c_void_p(256)
    fp8 = _desc(num_kv_heads=2, dtype=pa.PA_FP8_E4M3)
    bf16 = _desc(num_kv_heads=2)
    g = lib.pa_decode_grouped_quant

    def grouped(desc, ks=p, vs=p, gs=4):
        return g(p, p, p, p, ks, vs, p, 8, p, 100, 4, 16, ctypes.c_float(0.1), ctypes.byref(desc),
                 gs, -1, None, 0, None)
    assert grouped(fp8, ks=None) == pa.PA_ERR_INVALID_ARG
    assert grouped(bf16) == pa.PA_ERR_DTYPE
    assert grouped(_desc(num_kv_heads=2, dtype=pa.PA_INT8, head_dim=96)) == pa.PA_ERR_UNSUPPORTED
    # head_dim 64 over codes is accepted: its partition query answers without a GPU
    assert lib.pa_decode_grouped_num_partitions(8, 16, 100, ctypes.byref(
        _desc(num_kv_heads=2, dtype=pa.PA_INT8, head_dim=64)), 4, -1) == 1
    assert grouped(fp8, gs=9) == pa.PA_ERR_INVALID_ARG
    m = lib.pa_decode_multi_quant
    rc = m(p, p, p, p, p, p, p, 8, p, None, 100, 2, 4, 2, 16, ctypes.c_float(0.1),
           ctypes.byref(fp8), -1, None, 0, None)
    assert rc == pa.PA_ERR_INVALID_ARG and b"query_start" in lib.pa_get_last_error()
    rc = m(p, p, p, p, None, p, p, 8, p, p, 100, 2, 4, 2, 16, ctypes.c_float(0.1),
           ctypes.byref(fp8), -1, None, 0, None)
    assert rc == pa.PA_ERR_INVALID_ARG
    # the grouped and multi-token plans accept a quantised pool at head_dim 128
    d70 = _desc(num_kv_heads=8, dtype=pa.PA_FP8_E4M3)
    assert lib.pa_decode_grouped_num_partitions(128, 64, 2303, ctypes.byref(d70), 4, 0) == 1
    assert lib.pa_decode_multi_num_partitions(8, 32, 4, 64, 32768, ctypes.byref(d70), 512) == 64


def test_grouped_consumer_selector(lib):
    assert lib.pa_set_grouped_consumer(pa.PA_GROUPED_TCGEN05) == pa.PA_GROUPED_MMA_SYNC
    assert lib.pa_set_grouped_consumer(pa.PA_GROUPED_MMA_SYNC) == pa.PA_GROUPED_TCGEN05
    assert lib.pa_set_grouped_consumer(5) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_set_grouped_consumer(-1) == pa.PA_ERR_INVALID_ARG
    # the tcgen05 consumer's plan: 2 CTAs per SM, so the 4-beam CoW items (256) fit one wave
    d70 = _desc(num_kv_heads=8)
    lib.pa_set_grouped_consumer(pa.PA_GROUPED_TCGEN05)
    try:
        assert lib.pa_decode_grouped_num_partitions(128, 64, 2303, ctypes.byref(d70), 4, 0) == 1
    finally:
        lib.pa_set_grouped_consumer(pa.PA_GROUPED_MMA_SYNC)


def test_swap_rejects_bad_arguments(lib):
    p = ctypes.c_void_p(256)
    a, b = _desc(num_blocks=8), _desc(num_blocks=4)
    assert lib.pa_block_swap(p, 0, p, p, ctypes.byref(a), p, p, ctypes.byref(b), None) == pa.PA_OK
    assert lib.pa_block_swap(p, -1, p, p, ctypes.byref(a), p, p, ctypes.byref(b), None) \
        == pa.PA_ERR_INVALID_ARG
    c = _desc(num_blocks=4, head_dim=64)
    assert lib.pa_block_swap(p, 1, p, p, ctypes.byref(a), p, p, ctypes.byref(c), None) \
        == pa.PA_ERR_INVALID_ARG                                    # block shapes differ
    assert lib.pa_block_swap(None, 1, p, p, ctypes.byref(a), p, p, ctypes.byref(b), None) \
        == pa.PA_ERR_INVALID_ARG
    q = ctypes.c_void_p(1 << 20)
    assert lib.pa_block_swap(p, 1, p, p, ctypes.byref(a), q, q, ctypes.byref(b), None) \
        == pa.PA_ERR_INVALID_ARG                                    # dst_k == dst_v overlaps
    assert b"overlap" in lib.pa_get_last_error()
    assert lib.pa_block_swap(p, 1, p, ctypes.c_void_p(8 << 20), ctypes.byref(a),
                             ctypes.c_void_p(1 << 30), ctypes.c_void_p(3 << 20),
                             ctypes.byref(b), None) == pa.PA_ERR_INVALID_ARG   # src_k overlaps dst_v


def test_append_and_copy_reject_bad_arguments(lib):
    p = ctypes.c_void_p(16)
    assert lib.pa_kv_append(p, p, p, -1, p, p, ctypes.byref(_desc()), None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_kv_append(p, p, p, 0, p, p, ctypes.byref(_desc()), None) == pa.PA_OK
    assert lib.pa_kv_append(p, ctypes.c_void_p(4), p, 3, p, p, ctypes.byref(_desc()), None) \
        == pa.PA_ERR_ALIGN
    assert lib.pa_kv_append(None, p, p, 3, p, p, ctypes.byref(_desc()), None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_block_copy(p, 0, p, p, ctypes.byref(_desc()), None) == pa.PA_OK
    assert lib.pa_block_copy(None, 2, p, p, ctypes.byref(_desc()), None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_block_copy(ctypes.c_void_p(12), 2, p, p, ctypes.byref(_desc()), None) \
        == pa.PA_ERR_ALIGN


def test_status_strings(lib):
    assert lib.pa_status_string(pa.PA_ERR_BAD_INDEX) == b"PA_ERR_BAD_INDEX"
    assert lib.pa_status_string(0) == b"PA_OK"


def test_python_binding_refuses_cpu_tensors():
    import torch
    kc = torch.zeros((4, 1, 16, 64))
    with pytest.raises(ValueError, match="CUDA"):
        pa.pa_block_copy(torch.zeros((1, 2), dtype=torch.int64), kc, kc.clone())


def test_python_binding_quantised_calls_refuse_cpu_tensors():
    """The quantised grouped / multi-token bindings marshal device pointers only:
    host tensors are refused before anything reaches the library."""
    import torch
    kc = torch.zeros((8, 2, 16, 128), dtype=torch.float8_e4m3fn)
    q = torch.zeros((4, 16, 128), dtype=torch.bfloat16)
    scales = torch.ones(2)
    tables = torch.zeros((4, 2), dtype=torch.int32)
    ctx = torch.full((4,), 20, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        pa.pa_decode_grouped_quant(torch.empty_like(q), q, kc, kc.clone(), scales, scales, tables,
                                   ctx, 0.1, 2, max_context_len=20, partition_size=-1)
    qs = torch.tensor([0, 1, 2, 3, 4], dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        pa.pa_decode_multi_quant(torch.empty_like(q), q, kc, kc.clone(), scales, scales, tables,
                                 ctx, qs, 0.1, max_context_len=20, max_query_len=1,
                                 partition_size=-1)


def test_python_binding_refuses_a_tensor_of_another_device(monkeypatch):
    """The library launches on the current device: a tensor living on another
    GPU is refused in the binding instead of reaching a kernel as a foreign
    pointer (a stand-in tensor object plays the CUDA tensor; no GPU needed)."""
    import types

    import torch

    class OtherGpuTensor:
        is_cuda = True
        device = types.SimpleNamespace(index=1, type="cuda")

        def is_contiguous(self):
            return True

        def data_ptr(self):
            return 256

    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    with pytest.raises(ValueError, match="current CUDA device is cuda:0"):
        pa._dev(OtherGpuTensor(), "q")
    with pytest.raises(ValueError, match="current CUDA device"):
        pa._addressable(OtherGpuTensor(), "dst_k")
