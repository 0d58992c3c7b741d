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


@pytest.mark.parametrize("name,kw", [
    ("llama70b_gqa", dict(num_seqs=1, context_len=1024)),   # persistent tensor-core kernel
    ("tiny", {}),                                             # CUDA-core kernel
])
def test_skipped_load_times_out_then_recovers(name, kw):
    wl = W.make(name, **kw)
    vals = W.make_values(wl, DEV)
    d = G.device_tensors(wl, vals)
    kc, vc = vals["k_cache"], vals["v_cache"]
    pa.pa_kv_append(vals["k_new"], vals["v_new"], d["slots"], kc, vc)
    pa.pa_sync_check()
    lib = pa.load_library()
    out = torch.empty_like(vals["q"])
    lib.pa_test_skip_load(1)
    try:
        t0 = time.time()
        pa.pa_decode(out, vals["q"], kc, vc, d["tables"], d["ctx"], wl.scale,
                     max_context_len=wl.max_context_len, partition_size=0)
        with pytest.raises(pa.PAError) as e:
            pa.pa_sync_check()
        assert e.value.code == pa.PA_ERR_TIMEOUT
        assert time.time() - t0 < 60
    finally:
        lib.pa_test_skip_load(-1)
    pa.pa_sync_check()                                  # status was cleared
    out2 = torch.empty_like(vals["q"])
    pa.pa_decode(out2, vals["q"], kc, vc, d["tables"], d["ctx"], wl.scale,
                 max_context_len=wl.max_context_len, partition_size=0)
    pa.pa_sync_check()
    seqs = list(range(wl.num_seqs))
    ref = G.oracle_sampled(wl, vals, seqs)
    G.check_tolerance(G.to_f64(out2), ref, wl.dtype, f"{name} after a timed-out call")
