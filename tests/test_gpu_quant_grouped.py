"""Quantised caches on the grouped and multi-token calls (pa_decode_grouped_quant,
pa_decode_multi_quant) against the fp64 oracle.

The computation is pa_decode_quant's: every member of a group, and every query
token (with its causal end), gets the oracle's decode of value(code) x scale
within the bf16 bars. Beyond parity: a member's result does not depend on which
blocks it shares (bit-identical to a private-copy layout), and the full-size
configurations meet the bars on sampled sequences.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_335_b200 as pa
from paged_kv_cache_335_b200 import workloads as W
from tests import gpu_helpers as G
from tests.test_gpu_multi import CTX, NQ
from tests.test_gpu_quant import _codes, _host

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _append(wl, vals, d):
    kc, vc = vals["k_cache"], vals["v_cache"]
    if wl.copy_pairs.shape[0]:
        pa.pa_block_copy(d["pairs"], kc, vc)
    if wl.num_tokens:
        pa.pa_kv_append_quant(vals["k_new"], vals["v_new"], d["slots"], kc, vc, vals["k_scale"],
                              vals["v_scale"])


def _oracle_append(wl, host):
    kc, vc = host["k_cache"], host["v_cache"]
    if wl.copy_pairs.shape[0]:
        oracle.block_copy(wl.copy_pairs, kc, vc)
    if wl.num_tokens:
        oracle.kv_append_quant(host["k_new"], host["v_new"], wl.slot_mapping, kc, vc,
                               host["k_scale"], host["v_scale"], wl.kv_quant)


def _grouped(wl, vals, d, gs, ps, k_cache=None, v_cache=None, tables=None):
    out = torch.empty_like(vals["q"])
    pa.pa_decode_grouped_quant(out, vals["q"], vals["k_cache"] if k_cache is None else k_cache,
                               vals["v_cache"] if v_cache is None else v_cache, vals["k_scale"],
                               vals["v_scale"], d["tables"] if tables is None else tables,
                               d["ctx"], wl.scale, gs, max_context_len=wl.max_context_len,
                               partition_size=ps)
    return out


def _multi_rows(wl):
    """Query token t of sequence s as its own row: s's block table and the causal
    end ctx_s - n_s + j + 1 (j = t - query_start[s])."""
    qs = np.asarray(wl.query_start)
    tables, ctx = [], []
    for s in range(wl.num_seqs):
        n = int(qs[s + 1] - qs[s])
        for j in range(n):
            tables.append(wl.block_tables[s])
            ctx.append(int(wl.context_lens[s]) - n + j + 1)
    return (np.asarray(tables, dtype=np.int32).reshape(len(ctx), -1),
            np.asarray(ctx, dtype=np.int32))


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
@pytest.mark.parametrize("gs", [2, 4, 8])
@pytest.mark.parametrize("ps", [0, -1, 48])
def test_grouped_cow_parity(fmt, gs, ps):
    """Copy-on-write step over a quantised pool (3 prompts x 4 beams, g = 8): groups
    that match the beams, split them or hold two prompts; poisoned free slots."""
    wl = W.quantized(W.cow_beam4(num_prompts=3, prompt_len=200, max_suffix=40, num_heads=16,
                                 num_kv_heads=2, head_dim=128), fmt)
    vals = W.make_values(wl, DEV, poison=True)
    host = _host(vals)
    d = G.device_tensors(wl, vals)
    _append(wl, vals, d)
    out = _grouped(wl, vals, d, gs, ps)
    pa.pa_sync_check()
    assert G.last_kernel() in G.kernel_set(pa.PA_KERNEL_GROUPED)
    _oracle_append(wl, host)
    assert np.array_equal(_codes(vals["k_cache"]), host["k_cache"])
    assert np.array_equal(_codes(vals["v_cache"]), host["v_cache"])
    ref = oracle.decode_quant(host["q"], host["k_cache"], host["v_cache"], host["k_scale"],
                              host["v_scale"], wl.block_tables, wl.context_lens, wl.scale, fmt,
                              num_threads=G.THREADS)
    G.check_tolerance(G.to_f64(out), ref, "bf16", f"{wl.name} gs={gs} ps={ps}")


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
@pytest.mark.parametrize("H,Hkv", [(8, 8), (16, 4), (12, 3)])
@pytest.mark.parametrize("d", [64, 128])
def test_grouped_unshared_edges(fmt, H, Hkv, d):
    """Unrelated sequences grouped, contexts at block and unit edges including 0,
    head_dim 64 (zero-filled halves of 128-code rows) and 128."""
    ctx = [0, 1, 15, 16, 17, 63, 64, 65, 129, 300, 511, 513]
    wl = W.quantized(G.custom(len(ctx), H, Hkv, d, 16, "bf16", ctx, seed=H + 7 + d), fmt)
    for ps in (-1, 64):
        vals = W.make_values(wl, DEV, poison=True)
        host = _host(vals)
        d = G.device_tensors(wl, vals)
        _append(wl, vals, d)
        out = _grouped(wl, vals, d, 4, ps)
        pa.pa_sync_check()
        _oracle_append(wl, host)
        ref = oracle.decode_quant(host["q"], host["k_cache"], host["v_cache"], host["k_scale"],
                                  host["v_scale"], wl.block_tables, wl.context_lens, wl.scale,
                                  fmt, num_threads=G.THREADS)
        G.check_tolerance(G.to_f64(out), ref, "bf16", f"{wl.name} ps={ps}")


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
def test_grouped_shared_equals_private_bitwise(fmt):
    """A beam's output over codes does not depend on whether its prompt blocks are
    shared with the other beams of its group or held as private copies."""
    wl = W.quantized(W.cow_beam4(num_prompts=2, prompt_len=300, max_suffix=30, num_heads=16,
                                 num_kv_heads=2, head_dim=128), fmt)
    vals = W.make_values(wl, DEV, poison=False)
    d = G.device_tensors(wl, vals)
    _append(wl, vals, d)
    shared = _grouped(wl, vals, d, 4, 0)
    B = wl.block_size
    rows, ids = [], []
    for s in range(wl.num_seqs):
        nb = -(-int(wl.context_lens[s]) // B)
        rows.append(list(range(len(ids), len(ids) + nb)))
        ids.extend(int(x) for x in wl.block_tables[s, :nb])
    assert len(set(ids)) < len(ids)
    idx = torch.as_tensor(ids, device=DEV)
    kc, vc = vals["k_cache"], vals["v_cache"]
    kc2 = kc.view(torch.uint8).index_select(0, idx).contiguous().view(kc.dtype)
    vc2 = vc.view(torch.uint8).index_select(0, idx).contiguous().view(vc.dtype)
    tables = np.zeros((wl.num_seqs, max(len(r) for r in rows)), np.int32)
    for s, r in enumerate(rows):
        tables[s, :len(r)] = r
    private = _grouped(wl, vals, d, 4, 0, kc2, vc2, torch.as_tensor(tables, device=DEV))
    torch.cuda.synchronize()
    pa.pa_sync_check()
    assert G.bits_equal(shared, private)


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
@pytest.mark.parametrize("H,Hkv,d", [(8, 8, 128), (16, 2, 128), (64, 8, 128), (16, 2, 64)])
def test_multi_parity(fmt, H, Hkv, d):
    """Query counts from 0 to a 300-token chunk, contexts at block and partition
    edges; each query token against the oracle at its causal end."""
    wl = W.quantized(W.multi_query_case(len(CTX), H, Hkv, d, 16, "bf16", CTX, NQ, seed=H + 3 + d),
                     fmt)
    tables_r, ctx_r = _multi_rows(wl)
    for ps in (-1, 0, 64):
        vals = W.make_values(wl, DEV, poison=True)
        host = _host(vals)
        d = G.device_tensors(wl, vals)
        _append(wl, vals, d)
        out = torch.empty_like(vals["q"])
        pa.pa_decode_multi_quant(out, vals["q"], vals["k_cache"], vals["v_cache"], vals["k_scale"],
                                 vals["v_scale"], d["tables"], d["ctx"],
                                 torch.as_tensor(wl.query_start, device=DEV), wl.scale,
                                 max_context_len=wl.max_context_len,
                                 max_query_len=wl.max_query_len, partition_size=ps)
        pa.pa_sync_check()
        assert G.last_kernel() in G.kernel_set(pa.PA_KERNEL_GROUPED)
        _oracle_append(wl, host)
        ref = oracle.decode_quant(host["q"], host["k_cache"], host["v_cache"], host["k_scale"],
                                  host["v_scale"], tables_r, ctx_r, wl.scale, fmt,
                                  num_threads=G.THREADS)
        G.check_tolerance(G.to_f64(out), ref, "bf16", f"{wl.name} ps={ps}")


def test_full_size():
    """The 4-beam CoW step grouped and the 4-token 32K verification over FP8 pools,
    in the library's partition policy: every output row against the oracle."""
    wl = W.make("cow_beam4_fp8")
    vals = W.make_values(wl, DEV, poison=True)
    d = G.device_tensors(wl, vals)
    _append(wl, vals, d)
    out = _grouped(wl, vals, d, 4, 0)
    pa.pa_sync_check()
    assert torch.isfinite(out.float()).all()
    seqs = list(range(wl.num_seqs))
    sub = W.subproblem(wl, vals["k_cache"], vals["v_cache"], seqs, vals["q"])
    ref = oracle.decode_quant(sub["q"], sub["k_cache"], sub["v_cache"],
                              vals["k_scale"].cpu().numpy(), vals["v_scale"].cpu().numpy(),
                              sub["block_tables"], sub["context_lens"], wl.scale, "fp8",
                              num_threads=G.THREADS)
    G.check_tolerance(G.to_f64(out), ref, "bf16", wl.name)

    wl = W.make("llama70b_verify4_fp8")
    vals = W.make_values(wl, DEV, poison=False)
    d = G.device_tensors(wl, vals)
    _append(wl, vals, d)
    out = torch.empty_like(vals["q"])
    pa.pa_decode_multi_quant(out, vals["q"], vals["k_cache"], vals["v_cache"], vals["k_scale"],
                             vals["v_scale"], d["tables"], d["ctx"],
                             torch.as_tensor(wl.query_start, device=DEV), wl.scale,
                             max_context_len=wl.max_context_len, max_query_len=wl.max_query_len)
    pa.pa_sync_check()
    seq = list(range(wl.num_seqs))
    sub = W.subproblem(wl, vals["k_cache"], vals["v_cache"], seq)
    qs = np.asarray(wl.query_start)
    rows, tables_r, ctx_r = [], [], []
    for i, s in enumerate(seq):
        n = int(qs[s + 1] - qs[s])
        for j in range(n):
            rows.append(int(qs[s]) + j)
            tables_r.append(sub["block_tables"][i])
            ctx_r.append(int(sub["context_lens"][i]) - n + j + 1)
    rows_t = torch.as_tensor(rows, device=DEV)
    ref = oracle.decode_quant(W.to_numpy(vals["q"].index_select(0, rows_t)), sub["k_cache"],
                              sub["v_cache"], vals["k_scale"].cpu().numpy(),
                              vals["v_scale"].cpu().numpy(), np.asarray(tables_r, np.int32),
                              np.asarray(ctx_r, np.int32), wl.scale, "fp8", num_threads=G.THREADS)
    G.check_tolerance(G.to_f64(out.index_select(0, rows_t)), ref, "bf16", wl.name)


def test_refusals():
    """The quantised calls refuse a bf16 pool; the bf16 calls refuse a quantised one."""
    wl = G.custom(4, 16, 2, 128, 16, "bf16", [40, 17, 64, 5], seed=3)
    vals = W.make_values(wl, DEV)
    d = G.device_tensors(wl, vals)
    scales = torch.ones(wl.num_kv_heads, device=DEV)
    out = torch.empty_like(vals["q"])
    with pytest.raises(pa.PAError) as e:
        pa.pa_decode_grouped_quant(out, vals["q"], vals["k_cache"], vals["v_cache"], scales, scales,
                                   d["tables"], d["ctx"], wl.scale, 2, max_context_len=64)
    assert e.value.code == pa.PA_ERR_DTYPE
    wq = W.quantized(wl, "fp8")
    vq = W.make_values(wq, DEV)
    with pytest.raises((pa.PAError, TypeError)):   # the binding or the C ABI refuses
        pa.pa_decode_grouped(out, vals["q"], vq["k_cache"], vq["v_cache"], d["tables"], d["ctx"],
                             wl.scale, 2, max_context_len=64)
