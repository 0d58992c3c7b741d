"""A negative softmax scale (softmax(scale q . K) V with scale < 0) on every
decode kernel, against the fp64 oracle.

The grouped consumers take maxima of unscaled scores and scale them afterwards,
which is only right for a positive factor; they fold the scale's sign into q
(an exact negation) instead. The CUDA-core and tensor-core consumers scale
before the max. Each kernel is asserted to be the one the shape selects.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_335_b200 as pa
from paged_kv_cache_335_b200 import workloads as W
from tests import gpu_helpers as G
from tests.test_gpu_quant import _host, _oracle_step, _quant_step

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
CTX = [1, 16, 17, 64, 65, 300, 1000, 0]


@pytest.mark.parametrize("H,Hkv,gs,kernel", [
    (8, 8, 1, pa.PA_KERNEL_SIMT),       # CUDA cores
    (16, 2, 1, pa.PA_KERNEL_MMA),       # tensor cores, g = 8
    (16, 2, 4, pa.PA_KERNEL_GROUPED),   # grouped, 32 query columns
    (8, 8, 4, pa.PA_KERNEL_GROUPED),    # grouped, MHA
])
@pytest.mark.parametrize("consumer", [pa.PA_GROUPED_MMA_SYNC, pa.PA_GROUPED_TCGEN05])
def test_negative_scale_bf16(H, Hkv, gs, kernel, consumer):
    if gs == 1 and consumer == pa.PA_GROUPED_TCGEN05:
        pytest.skip("the grouped consumer applies to grouped calls only")
    wl = G.custom(len(CTX), H, Hkv, 128, 16, "bf16", CTX, seed=41)
    wl.scale = -abs(wl.scale)
    prev = pa.pa_set_grouped_consumer(consumer)
    try:
        vals = W.make_values(wl, DEV, poison=True)
        host = G.host_copy(vals)
        for ps in (-1, 64):
            v = {k: t.clone() for k, t in vals.items()}
            out = G.gpu_step(wl, v, partition_size=ps, group_size=gs)
            pa.pa_sync_check()
            assert G.last_kernel() in G.kernel_set(kernel)
            h = {k: a.copy() for k, a in host.items()}
            ref = G.oracle_step(wl, h)
            G.check_tolerance(G.to_f64(out), ref, "bf16", f"scale<0 H={H}/{Hkv} gs={gs} ps={ps}")
    finally:
        pa.pa_set_grouped_consumer(prev)


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
def test_negative_scale_codes(fmt):
    ctx = [1, 17, 300, 700]
    for H, Hkv in ((8, 8), (16, 2)):
        wl = W.quantized(G.custom(len(ctx), H, Hkv, 128, 16, "bf16", ctx, seed=43), fmt)
        wl.scale = -abs(wl.scale)
        vals = W.make_values(wl, DEV, poison=False)
        host = _host(vals)
        out = _quant_step(wl, vals, ps=-1)
        pa.pa_sync_check()
        ref = _oracle_step(wl, host)
        G.check_tolerance(G.to_f64(out), ref, "bf16", f"{fmt} scale<0 H={H}/{Hkv}")
        d = G.device_tensors(wl, vals)
        outg = torch.empty_like(vals["q"])
        pa.pa_decode_grouped_quant(outg, vals["q"], vals["k_cache"], vals["v_cache"],
                                   vals["k_scale"], vals["v_scale"], d["tables"], d["ctx"],
                                   wl.scale, 2, max_context_len=wl.max_context_len,
                                   partition_size=-1)
        pa.pa_sync_check()
        G.check_tolerance(G.to_f64(outg), ref, "bf16", f"{fmt} grouped scale<0 H={H}/{Hkv}")
