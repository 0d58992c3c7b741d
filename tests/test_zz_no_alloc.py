"""pa_decode_noalloc: the decode entry point that allocates nothing.

Some callers cannot allocate device memory where they decode: code inside a
memory arena sized up front, plug-ins of an engine that owns every device
allocation, loops that must never enter an allocator. For them the library's
pa_decode_noalloc takes the split-context workspace from a fixed buffer inside
the library (PA_NOALLOC_SCRATCH_BYTES per GPU) instead of from the caller.

These tests call it through the C ABI and check that its output is bit for bit
the output of pa_decode with a caller-provided workspace (both run the same plan
and kernels, so any difference would be scratch contents leaking into a result),
on two calls in a row with different queries, and that the second call also
meets the bf16 bars against the fp64 oracle. This file sorts last so that a run
stopping at the first failure has run every other test before it.
"""
import ctypes

import pytest
import torch

import paged_kv_cache_335_b200 as pa
from paged_kv_cache_335_b200 import workloads as W
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def test_noalloc_matches_pa_decode_on_two_calls():
    wl = W.make("llama70b_gqa", num_seqs=4, context_len=8192)
    vals = W.make_values(wl, DEV)
    d = G.device_tensors(wl, vals)
    kc, vc = vals["k_cache"], vals["v_cache"]
    pa.pa_kv_append(vals["k_new"], vals["v_new"], d["slots"], kc, vc)
    parts = pa.pa_decode_num_partitions(wl.num_seqs, wl.num_heads, wl.max_context_len, kc, 512)
    need = pa.pa_decode_workspace_size(wl.num_seqs, wl.num_heads, wl.max_context_len, kc, 512)
    assert parts > 1 and 0 < need <= pa.PA_NOALLOC_SCRATCH_BYTES   # the scratch is really used
    g = torch.Generator(device=DEV).manual_seed(99)
    for call in range(2):
        q = torch.randn(vals["q"].shape, generator=g, device=DEV, dtype=torch.bfloat16)
        ref = torch.empty_like(q)
        ws = torch.empty(need, dtype=torch.uint8, device=DEV)
        pa.pa_decode(ref, q, kc, vc, d["tables"], d["ctx"], wl.scale,
                     max_context_len=wl.max_context_len, partition_size=512, workspace=ws)
        out = torch.full_like(q, float("nan"))
        pa.pa_decode_noalloc(out, q, kc, vc, d["tables"], d["ctx"], wl.scale,
                             max_context_len=wl.max_context_len, partition_size=512)
        torch.cuda.synchronize()
        pa.pa_sync_check()
        assert G.dev_bits_equal(out, ref), f"noalloc call {call} differs from pa_decode"
    # the last call against the oracle: the scratch path computes the right thing
    vals["q"] = q
    G.check_tolerance(G.to_f64(out), G.oracle_all(wl, vals), "bf16", "noalloc vs oracle")


def test_noalloc_without_split_needs_no_scratch():
    wl = W.decode_case(3, 8, 8, 128, 16, "bf16", [5, 300, 17], seed=4)
    vals = W.make_values(wl, DEV)
    d = G.device_tensors(wl, vals)
    kc, vc = vals["k_cache"], vals["v_cache"]
    ref, out = torch.empty_like(vals["q"]), torch.empty_like(vals["q"])
    pa.pa_decode(ref, vals["q"], kc, vc, d["tables"], d["ctx"], wl.scale,
                 max_context_len=wl.max_context_len, partition_size=-1)
    pa.pa_decode_noalloc(out, vals["q"], kc, vc, d["tables"], d["ctx"], wl.scale,
                         max_context_len=wl.max_context_len, partition_size=-1)
    torch.cuda.synchronize()
    assert G.dev_bits_equal(out, ref), "noalloc without split differs from pa_decode"


def test_noalloc_rejects_more_than_its_buffer():
    lib = pa.load_library()
    desc = pa.pa_cache_desc(1024, 64, 16, 128, pa.PA_BF16)
    need = lib.pa_decode_workspace_size(64, 64, 32768, ctypes.byref(desc), 512)
    assert need > pa.PA_NOALLOC_SCRATCH_BYTES
    p = ctypes.c_void_p(256)
    rc = lib.pa_decode_noalloc(p, p, p, p, p, 2048, p, 32768, 64, 64, 0.1, ctypes.byref(desc),
                               512, None)
    assert rc == pa.PA_ERR_WORKSPACE
    assert b"PA_NOALLOC_SCRATCH_BYTES" in lib.pa_get_last_error()
