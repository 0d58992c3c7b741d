"""Failure detection on the GPU without a fault or a hang: the decode kernels'
pipeline waits are bounded (about one second each). With one K/V load left out
on purpose (pa_test_skip_load), the waiting warps give up, the kernel still
terminates, pa_sync_check reports PA_ERR_TIMEOUT, and the context stays usable
for the next, normal call."""
import time

import pytest
import torch

import paged_kv_cache_335_b200 as pa
from paged_kv_cache_335_b200 import workloads as W
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _decode(wl, vals, d, out, gs, ps=0):
    kc, vc = vals["k_cache"], vals["v_cache"]
    if gs > 1:
        pa.pa_decode_grouped(out, vals["q"], kc, vc, d["tables"], d["ctx"], wl.scale, gs,
                             max_context_len=wl.max_context_len, partition_size=ps)
    else:
        pa.pa_decode(out, vals["q"], kc, vc, d["tables"], d["ctx"], wl.scale,
                     max_context_len=wl.max_context_len, partition_size=ps)


@pytest.mark.parametrize("name,kw,gs,ps", [
    ("llama70b_gqa", dict(num_seqs=1, context_len=1024), 1, 0),   # persistent tensor-core kernel
    # the same kernel under its dynamic item schedule (2048 items claimed from the
    # workspace's counter: the queue's waits give up too)
    ("llama70b_gqa", dict(num_seqs=8, context_len=8192), 1, 256),
    ("tiny", {}, 1, 0),                                             # CUDA-core kernel
    ("cow_beam4", dict(num_prompts=2, prompt_len=300, max_suffix=30), 4, 0),   # grouped kernel
])
def test_skipped_load_times_out_then_recovers(name, kw, gs, ps):
    wl = W.make(name, **kw)
    vals = W.make_values(wl, DEV)
    d = G.device_tensors(wl, vals)
    kc, vc = vals["k_cache"], vals["v_cache"]
    if wl.copy_pairs.shape[0]:
        pa.pa_block_copy(d["pairs"], kc, vc)
    pa.pa_kv_append(vals["k_new"], vals["v_new"], d["slots"], kc, vc)
    pa.pa_sync_check()
    lib = pa.load_library()
    out = torch.empty_like(vals["q"])
    lib.pa_test_skip_load(1)
    try:
        t0 = time.time()
        _decode(wl, vals, d, out, gs, ps)
        with pytest.raises(pa.PAError) as e:
            pa.pa_sync_check()
        assert e.value.code == pa.PA_ERR_TIMEOUT
        assert time.time() - t0 < 60
    finally:
        lib.pa_test_skip_load(-1)
    pa.pa_sync_check()                                  # status was cleared
    out2 = torch.empty_like(vals["q"])
    _decode(wl, vals, d, out2, gs, ps)
    pa.pa_sync_check()
    if gs > 1:
        assert G.last_kernel() in G.kernel_set(pa.PA_KERNEL_GROUPED)
    seqs = list(range(wl.num_seqs))
    ref = G.oracle_sampled(wl, vals, seqs)
    G.check_tolerance(G.to_f64(out2), ref, wl.dtype, f"{name} after a timed-out call")
