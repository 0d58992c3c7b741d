"""Work-item schedules of the persistent tensor-core (GQA) decode.

With the workspace size that pa_decode_workspace_size reports and more work
items (partition, kv head, sequence) than CTA slots, the kernel's CTAs claim
items from a counter in the workspace, so CTAs that stream faster take more
items; with a workspace that holds only the partial results (or none, unsplit),
or fewer than two items per slot, they take item u = CTA + k x grid. The cases below
with splits have thousands of items, so both schedules run. An item's arithmetic does not depend on the CTA that runs it, so the two
schedules must give the same output bit for bit, and both must meet the bf16
bar against the oracle: on ragged contexts (empty sequences and partitions past
a context included), with and without splits, over bf16 and over codes, with
more items than CTA slots.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_335_b200 as pa
from paged_kv_cache_335_b200 import workloads as W
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _workspaces(wl, kc, ps):
    """(dynamic, static) workspaces of one call: the reported size, and the
    partial results only (one byte when the call is not split)."""
    full = pa.pa_decode_workspace_size(wl.num_seqs, wl.num_heads, wl.max_context_len, kc, ps)
    assert full >= 256, "the tensor-core kernel reports its schedule counter"
    dyn = torch.empty(full, dtype=torch.uint8, device=DEV)
    static = torch.empty(max(full - 256, 1), dtype=torch.uint8, device=DEV)
    return dyn, static


def _decode(wl, vals, d, ps, ws):
    out = torch.full_like(vals["q"], float("nan"))
    if wl.kv_quant:
        pa.pa_decode_quant(out, vals["q"], vals["k_cache"], vals["v_cache"], vals["k_scale"],
                           vals["v_scale"], d["tables"], d["ctx"], wl.scale,
                           max_context_len=wl.max_context_len, partition_size=ps, workspace=ws)
    else:
        pa.pa_decode(out, vals["q"], vals["k_cache"], vals["v_cache"], d["tables"], d["ctx"],
                     wl.scale, max_context_len=wl.max_context_len, partition_size=ps,
                     workspace=ws)
    assert G.last_kernel() == pa.PA_KERNEL_MMA
    return out


def _append(wl, vals, d):
    if wl.kv_quant:
        pa.pa_kv_append_quant(vals["k_new"], vals["v_new"], d["slots"], vals["k_cache"],
                              vals["v_cache"], vals["k_scale"], vals["v_scale"])
    else:
        pa.pa_kv_append(vals["k_new"], vals["v_new"], d["slots"], vals["k_cache"], vals["v_cache"])


def _oracle(wl, host):
    kc, vc = host["k_cache"], host["v_cache"]
    if wl.kv_quant:
        oracle.kv_append_quant(host["k_new"], host["v_new"], wl.slot_mapping, kc, vc,
                               host["k_scale"], host["v_scale"], wl.kv_quant)
        return oracle.decode_quant(host["q"], kc, vc, host["k_scale"], host["v_scale"],
                                   wl.block_tables, wl.context_lens, wl.scale, wl.kv_quant,
                                   num_threads=G.THREADS)
    oracle.kv_append(host["k_new"], host["v_new"], wl.slot_mapping, kc, vc)
    return oracle.decode(host["q"], kc, vc, wl.block_tables, wl.context_lens, wl.scale,
                         num_threads=G.THREADS)


def _host(vals):
    return {k: (W.to_numpy(t).copy() if t.dtype != torch.float32 else t.cpu().numpy().copy())
            for k, t in vals.items()}


def _check(wl, partition_sizes):
    vals = W.make_values(wl, DEV, poison=True)
    host = _host(vals)
    d = G.device_tensors(wl, vals)
    _append(wl, vals, d)
    ref = _oracle(wl, host)
    for ps in partition_sizes:
        dyn_ws, static_ws = _workspaces(wl, vals["k_cache"], ps)
        a = _decode(wl, vals, d, ps, dyn_ws)
        b = _decode(wl, vals, d, ps, static_ws)
        c = _decode(wl, vals, d, ps, dyn_ws)  # the counter is reset for every call
        pa.pa_sync_check()
        assert G.dev_bits_equal(a, b), f"{wl.name} ps={ps}: dynamic and static schedules differ"
        assert G.dev_bits_equal(a, c), f"{wl.name} ps={ps}: a second dynamic call differs"
        G.check_tolerance(G.to_f64(a), ref, "bf16", f"{wl.name} ps={ps}")


@pytest.mark.parametrize("fmt", [None, "fp8", "int8"])
def test_ragged_contexts_both_schedules(fmt):
    """Empty sequences (zero output unsplit, no items split), contexts at block and
    partition edges, and one long context, at several partition sizes."""
    ctx = [0, 1, 15, 16, 17, 255, 256, 257, 1000, 0, 4097, 33, 2048, 511, 9000, 3]
    wl = G.custom(len(ctx), 64, 8, 128, 16, "bf16", ctx, seed=31)
    if fmt:
        wl = W.quantized(wl, fmt)
    _check(wl, (-1, 0, 256, 512))


def test_more_items_than_slots():
    """48 sequences x 8 kv heads at 256-token partitions: thousands of items of
    unequal length (contexts up to 8K, some empty) for the 592 CTA slots, so
    every CTA claims many."""
    rng = np.random.default_rng(7)
    ctx = [int(x) for x in rng.integers(0, 8192, size=48)]
    ctx[5] = 0
    ctx[17] = 8191
    wl = G.custom(len(ctx), 64, 8, 128, 16, "bf16", ctx, seed=32)
    _check(wl, (256, 0))


def test_head_dim_64_and_group_4():
    ctx = [700, 0, 1, 3000, 64, 65]
    wl = G.custom(len(ctx), 16, 4, 64, 32, "bf16", ctx, seed=33)
    _check(wl, (-1, 0, 128))


def test_full_size_70b_at_512_token_partitions():
    """The 70B-GQA configuration as benched (8 x 32K, 64 partitions): the two
    schedules bit for bit, and the dynamic one against the oracle on two
    sequences."""
    wl = W.make("llama70b_gqa")
    vals = W.make_values(wl, DEV, poison=True)
    d = G.device_tensors(wl, vals)
    _append(wl, vals, d)
    dyn_ws, static_ws = _workspaces(wl, vals["k_cache"], 512)
    a = _decode(wl, vals, d, 512, dyn_ws)
    b = _decode(wl, vals, d, 512, static_ws)
    pa.pa_sync_check()
    assert G.dev_bits_equal(a, b)
    ref = G.oracle_sampled(wl, vals, [0, 7])
    G.check_tolerance(G.to_f64(a[[0, 7]]), ref, "bf16", "llama70b_gqa sampled")
