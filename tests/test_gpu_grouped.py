"""Parity of the grouped decode (pa_decode_grouped) with the fp64 oracle.

Sequences [k gs, (k + 1) gs) are decoded by one CTA, which reads each block
its members share once. The bar is pa_decode's: bf16 max abs error <= 1e-2
and mean abs error <= 1e-3 against the unrounded oracle (fp32 row-normwise
<= 1e-5 where a call falls back to the ungrouped kernels). Beyond parity:
a member's result must not depend on which blocks it shares (private copies,
other placements: bit-identical), shapes the grouped kernel cannot take must
run the ungrouped kernels, and bad block ids are reported, not faulted.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_335_b200 as pa
from paged_kv_cache_335_b200 import workloads as W
from tests import gpu_helpers as G
from tests.test_gpu_parity import EDGE_CTX, _permuted

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _check(wl, gs, ps, kernel=pa.PA_KERNEL_GROUPED):
    vals = W.make_values(wl, DEV, poison=True)
    host = G.host_copy(vals)
    out = G.gpu_step(wl, vals, partition_size=ps, group_size=gs)
    pa.pa_sync_check()
    assert G.last_kernel() in G.kernel_set(kernel)
    ref = G.oracle_step(wl, host)
    assert G.bits_equal(vals["k_cache"], host["k_cache"])
    assert G.bits_equal(vals["v_cache"], host["v_cache"])
    return G.check_tolerance(G.to_f64(out), ref, wl.dtype, f"{wl.name} gs={gs} ps={ps}")


def test_cow_beam4_full_size():
    """The measured copy-on-write step with its 4 beams decoded together, in the
    bench's launch configuration (library partition policy): every beam's output
    against the oracle, all outputs finite."""
    wl = W.make("cow_beam4")
    vals = W.make_values(wl, DEV, poison=True)
    out = G.gpu_step(wl, vals, partition_size=0, group_size=4)
    pa.pa_sync_check()
    assert G.last_kernel() in G.kernel_set(pa.PA_KERNEL_GROUPED)
    assert torch.isfinite(out.float()).all()
    ref = G.oracle_all(wl, vals)
    G.check_tolerance(G.to_f64(out), ref, "bf16", "cow_beam4")


@pytest.mark.parametrize("gs", [2, 3, 4, 8])
@pytest.mark.parametrize("ps", [0, -1, 32, 48])
def test_cow_small_full_pool(gs, ps):
    """Whole-pool CoW step (3 prompts x 4 beams, g = 8): groups that match the
    beams, split them (2), straddle prompts (3) or hold two prompts (8)."""
    wl = W.cow_beam4(num_prompts=3, prompt_len=200, max_suffix=40, num_heads=16, num_kv_heads=2,
                     head_dim=128)
    _check(wl, gs, ps)


def test_cow_small_head_dim_64_mha():
    """MHA (g = 1): the 4 beams of a prompt fill 4 columns of one n-tile."""
    wl = W.cow_beam4(num_prompts=3, prompt_len=150, max_suffix=30, num_heads=8, num_kv_heads=8,
                     head_dim=64)
    for ps in (0, 64):
        _check(wl, 4, ps)


def _private_copy(wl, vals):
    """Every sequence's logical blocks gathered into fresh private blocks."""
    B = wl.block_size
    rows, ids = [], []
    for s in range(wl.num_seqs):
        nb = -(-int(wl.context_lens[s]) // B)
        rows.append(list(range(len(ids), len(ids) + nb)))
        ids.extend(int(x) for x in wl.block_tables[s, :nb])
    idx = torch.as_tensor(ids, device=DEV)
    kc2 = vals["k_cache"].index_select(0, idx).contiguous()
    vc2 = vals["v_cache"].index_select(0, idx).contiguous()
    tables = np.zeros((wl.num_seqs, max(len(r) for r in rows)), np.int32)
    for s, r in enumerate(rows):
        tables[s, :len(r)] = r
    return kc2, vc2, torch.as_tensor(tables, device=DEV), len(set(ids)) < len(ids)


@pytest.mark.parametrize("ps", [0, 64])
def test_shared_equals_private_bitwise(ps):
    """A beam's output does not depend on whether its prompt blocks are shared
    with the other beams of its group or held as private copies."""
    wl = W.cow_beam4(num_prompts=2, prompt_len=300, max_suffix=30, num_heads=16, num_kv_heads=2,
                     head_dim=128)
    vals = W.make_values(wl, DEV, poison=False)
    shared = G.gpu_step(wl, vals, partition_size=ps, group_size=4)
    kc2, vc2, tables2, was_shared = _private_copy(wl, vals)
    out2 = torch.empty_like(vals["q"])
    pa.pa_decode_grouped(out2, vals["q"], kc2, vc2, tables2,
                         torch.as_tensor(wl.context_lens, device=DEV), wl.scale, 4,
                         max_context_len=wl.max_context_len, partition_size=ps)
    torch.cuda.synchronize()
    assert was_shared
    assert G.bits_equal(shared, out2)


@pytest.mark.parametrize("ps", [0, 48])
def test_members_sharing_blocks_with_different_lengths(ps):
    """Members that share every block but end at different tokens of one unit
    of the grouped kernel (a sequence and prefixes of it): each member takes
    its own units there, so results match the oracle and equal a private-copy
    layout bit for bit."""
    ctx = [150, 120, 97, 150, 64, 65, 0, 33]
    wl = G.custom(len(ctx), 16, 2, 128, 16, "bf16", ctx, seed=21)
    wl.block_tables[1:4, :] = wl.block_tables[0, :]   # 1..3 read 0's blocks
    wl.block_tables[5, :] = wl.block_tables[4, :]
    wl.slot_mapping[:] = -1                            # no appends into shared blocks
    vals = W.make_values(wl, DEV, poison=False)
    host = G.host_copy(vals)
    shared = G.gpu_step(wl, vals, partition_size=ps, group_size=4)
    pa.pa_sync_check()
    assert G.last_kernel() in G.kernel_set(pa.PA_KERNEL_GROUPED)
    ref = G.oracle_step(wl, host)
    G.check_tolerance(G.to_f64(shared), ref, "bf16", f"prefix members ps={ps}")
    kc2, vc2, tables2, was_shared = _private_copy(wl, vals)
    out2 = torch.empty_like(vals["q"])
    pa.pa_decode_grouped(out2, vals["q"], kc2, vc2, tables2,
                         torch.as_tensor(wl.context_lens, device=DEV), wl.scale, 4,
                         max_context_len=wl.max_context_len, partition_size=ps)
    torch.cuda.synchronize()
    assert was_shared
    assert G.bits_equal(shared, out2)


def test_placement_invariance_bitwise():
    wl = W.cow_beam4(num_prompts=2, prompt_len=250, max_suffix=40, num_heads=32, num_kv_heads=4,
                     head_dim=128)
    vals = W.make_values(wl, DEV, poison=True)
    outs = []
    for seed in (None, 5, 6):
        v = {k: t.clone() for k, t in vals.items()}
        w, v = (wl, v) if seed is None else _permuted(wl, v, seed)
        outs.append(G.gpu_step(w, v, partition_size=128, group_size=4))
    torch.cuda.synchronize()
    pa.pa_sync_check()
    for o in outs[1:]:
        assert G.bits_equal(outs[0], o)


def test_deterministic_repeat():
    wl = W.make("cow_beam4", num_prompts=4)
    vals = W.make_values(wl, DEV, poison=True)
    first = G.gpu_step(wl, vals, partition_size=0, group_size=4)
    d = G.device_tensors(wl, vals)
    for _ in range(2):
        out = torch.empty_like(vals["q"])
        pa.pa_decode_grouped(out, vals["q"], vals["k_cache"], vals["v_cache"], d["tables"],
                             d["ctx"], wl.scale, 4, max_context_len=wl.max_context_len)
        assert G.bits_equal(first, out)


@pytest.mark.parametrize("d,bs", [(64, 16), (128, 16), (128, 64)])
@pytest.mark.parametrize("H,Hkv", [(8, 8), (8, 4), (16, 4), (16, 2), (12, 3)])
@pytest.mark.parametrize("gs", [2, 3, 5, 8])
def test_unshared_shape_sweep_edges(d, bs, H, Hkv, gs):
    """Groups of unrelated sequences (nothing shared), contexts at every block
    and partition edge including 0, a ragged last group; n-tile layouts from
    one tile with idle columns (g = 1) to eight tiles (gs 8 x g 8)."""
    wl = G.custom(len(EDGE_CTX), H, Hkv, d, bs, "bf16", EDGE_CTX, seed=gs + bs + d + H)
    for ps in (-1, 64):
        _check(wl, gs, ps)


def test_members_with_empty_contexts():
    """A group whose members are all empty, and groups mixing empty and long ones."""
    ctx = [0, 0, 0, 0, 0, 700, 0, 33, 1, 0, 0, 0]
    wl = G.custom(len(ctx), 16, 2, 128, 16, "bf16", ctx, seed=11)
    for ps in (-1, 0, 128):
        _check(wl, 4, ps)


def test_shapes_without_the_grouped_kernel_fall_back():
    _check(W.tiny(), 2, 0, kernel=pa.PA_KERNEL_SIMT)                          # f32
    wl = G.custom(6, 32, 2, 128, 16, "bf16", [700, 5, 1200, 1, 0, 64], seed=9)   # 8 x 16 > 64
    _check(wl, 8, 0, kernel=pa.PA_KERNEL_SIMT)
    wl = G.custom(6, 16, 2, 128, 16, "bf16", [700, 5, 1200, 1, 0, 64], seed=9)
    _check(wl, 1, 0, kernel=pa.PA_KERNEL_MMA)                                 # group_size 1


def test_long_shared_context_many_partitions():
    """One group of 4 beams over a 20k-token shared prompt, split into many partitions."""
    wl = W.cow_beam4(num_prompts=1, prompt_len=20000, max_suffix=200, num_heads=64,
                     num_kv_heads=8, head_dim=128)
    for ps in (0, 512, 2048):
        vals = W.make_values(wl, DEV, poison=True)
        out = G.gpu_step(wl, vals, partition_size=ps, group_size=4)
        pa.pa_sync_check()
        ref = G.oracle_sampled(wl, vals, [0, 1, 2, 3])
        G.check_tolerance(G.to_f64(out), ref, "bf16", f"ps={ps}")


def test_bad_block_id_is_reported():
    wl = G.custom(4, 16, 2, 128, 16, "bf16", [40, 40, 50, 17], seed=1)
    vals = W.make_values(wl, DEV)
    d = G.device_tensors(wl, vals)
    d["tables"][1, 1] = wl.num_blocks + 5
    out = torch.empty_like(vals["q"])
    pa.pa_sync_check()
    pa.pa_decode_grouped(out, vals["q"], vals["k_cache"], vals["v_cache"], d["tables"], d["ctx"],
                         wl.scale, 4, max_context_len=50)
    with pytest.raises(pa.PAError) as e:
        pa.pa_sync_check()
    assert e.value.code == pa.PA_ERR_BAD_INDEX
    assert G.last_kernel() in G.kernel_set(pa.PA_KERNEL_GROUPED)
    pa.pa_sync_check()
