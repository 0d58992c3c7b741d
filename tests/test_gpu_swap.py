"""Block swap between a device pool and a pinned host pool (pa_block_swap).

Moves must be bit-exact against the oracle over the whole destination pool
(untouched blocks included); a swap-out / swap-in round trip into other block
ids must leave decode results bit-identical; bad ids are reported, pageable
host memory is refused.
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


def _host_pool(like, blocks, fill=float("nan")):
    shape = (blocks,) + tuple(like.shape[1:])
    return (torch.full(shape, fill, dtype=like.dtype).pin_memory(),
            torch.full(shape, fill, dtype=like.dtype).pin_memory())


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_swap_out_and_in_bit_exact(dtype, d):
    wl = G.custom(5, 16, 4, d, 16, dtype, [700, 33, 1, 300, 129], seed=4)
    vals = W.make_values(wl, DEV, poison=True)
    kc, vc = vals["k_cache"], vals["v_cache"]
    hk, hv = _host_pool(kc, 40)
    rng = np.random.default_rng(1)
    out_pairs = np.stack([rng.choice(wl.num_blocks, 25, replace=False),
                          rng.choice(40, 25, replace=False)], 1).astype(np.int64)
    ref_k, ref_v = W.to_numpy(hk).copy(), W.to_numpy(hv).copy()
    oracle.block_swap(out_pairs, W.to_numpy(kc), W.to_numpy(vc), ref_k, ref_v)
    pa.pa_block_swap(torch.as_tensor(out_pairs, device=DEV), kc, vc, hk, hv)
    pa.pa_sync_check()
    assert G.bits_equal(hk, ref_k) and G.bits_equal(hv, ref_v)
    # swap in to other device blocks
    in_pairs = np.stack([out_pairs[:, 1], rng.choice(wl.num_blocks, 25, replace=False)],
                        1).astype(np.int64)
    dk, dv = W.to_numpy(kc).copy(), W.to_numpy(vc).copy()
    oracle.block_swap(in_pairs, W.to_numpy(hk), W.to_numpy(hv), dk, dv)
    pa.pa_block_swap(torch.as_tensor(in_pairs, device=DEV), hk, hv, kc, vc)
    pa.pa_sync_check()
    assert G.bits_equal(kc, dk) and G.bits_equal(vc, dv)


def test_device_to_device_pools():
    wl = G.custom(3, 8, 8, 128, 32, "bf16", [100, 64, 5], seed=2)
    vals = W.make_values(wl, DEV, poison=True)
    kc, vc = vals["k_cache"], vals["v_cache"]
    k2 = torch.zeros((7,) + tuple(kc.shape[1:]), dtype=kc.dtype, device=DEV)
    v2 = torch.zeros_like(k2)
    pairs = np.array([[0, 6], [wl.num_blocks - 1, 0], [3, 3]], np.int64)
    rk, rv = W.to_numpy(k2).copy(), W.to_numpy(v2).copy()
    oracle.block_swap(pairs, W.to_numpy(kc), W.to_numpy(vc), rk, rv)
    pa.pa_block_swap(torch.as_tensor(pairs, device=DEV), kc, vc, k2, v2)
    pa.pa_sync_check()
    assert G.bits_equal(k2, rk) and G.bits_equal(v2, rv)


def test_round_trip_preserves_decode_bitwise():
    """Preempt every sequence (swap all its blocks out), wipe the device pool,
    resume into a fresh permutation of block ids: decode is bit-identical."""
    wl = W.make("llama70b_gqa", num_seqs=3, context_len=1500)
    vals = W.make_values(wl, DEV, poison=True)
    before = G.gpu_step(wl, vals, partition_size=0)
    torch.cuda.synchronize()
    kc, vc = vals["k_cache"], vals["v_cache"]
    used = sorted({int(b) for s in range(wl.num_seqs)
                   for b in wl.block_tables[s, :-(-int(wl.context_lens[s]) // wl.block_size)]})
    hk, hv = _host_pool(kc, len(used))
    out = torch.as_tensor(np.stack([used, np.arange(len(used))], 1), dtype=torch.int64, device=DEV)
    pa.pa_block_swap(out, kc, vc, hk, hv)
    torch.cuda.synchronize()
    kc.fill_(float("nan"))
    vc.fill_(float("nan"))
    new_ids = np.random.default_rng(3).permutation(wl.num_blocks)[:len(used)]
    back = torch.as_tensor(np.stack([np.arange(len(used)), new_ids], 1), dtype=torch.int64,
                           device=DEV)
    pa.pa_block_swap(back, hk, hv, kc, vc)
    remap = dict(zip(used, new_ids.tolist()))
    tables = np.vectorize(lambda b: remap.get(int(b), int(b)))(wl.block_tables).astype(np.int32)
    after = torch.empty_like(before)
    pa.pa_decode(after, vals["q"], kc, vc, torch.as_tensor(tables, device=DEV),
                 torch.as_tensor(wl.context_lens, device=DEV), wl.scale,
                 max_context_len=wl.max_context_len, partition_size=0)
    pa.pa_sync_check()
    assert G.bits_equal(before, after)


def test_bad_ids_reported_and_pageable_memory_refused():
    wl = G.custom(2, 8, 8, 64, 16, "bf16", [20, 30], seed=2)
    vals = W.make_values(wl, DEV)
    kc, vc = vals["k_cache"], vals["v_cache"]
    hk, hv = _host_pool(kc, 4, 0.0)
    pa.pa_sync_check()
    pa.pa_block_swap(torch.tensor([[0, 4]], dtype=torch.int64, device=DEV), kc, vc, hk, hv)
    with pytest.raises(pa.PAError) as e:
        pa.pa_sync_check()
    assert e.value.code == pa.PA_ERR_BAD_INDEX
    assert torch.count_nonzero(hk.float()) == 0          # nothing written
    pageable = torch.zeros_like(hk, device="cpu")
    lib = pa.load_library()
    import ctypes
    sd, dd = pa.cache_desc(kc), pa.cache_desc(pageable)
    pairs = torch.tensor([[0, 0]], dtype=torch.int64, device=DEV)
    rc = lib.pa_block_swap(ctypes.c_void_p(pairs.data_ptr()), 1, ctypes.c_void_p(kc.data_ptr()),
                           ctypes.c_void_p(vc.data_ptr()), ctypes.byref(sd),
                           ctypes.c_void_p(pageable.data_ptr()),
                           ctypes.c_void_p(pageable.data_ptr() + pageable.numel() * 2 + 256),
                           ctypes.byref(dd), None)
    assert rc == pa.PA_ERR_INVALID_ARG
    assert b"pageable" in lib.pa_get_last_error()
