"""Multi-token paged queries (pa_decode_multi) against the fp64 oracle.

Each sequence appends n_s tokens this step and every one of them attends
causally over the paged cache (chunked prefill, verification of draft tokens).
Bars: appended slots bit-exact; outputs within the bf16 tolerance of the
unrounded oracle; a query token's result bit-identical whether or not other
tokens share the call; bad inputs reported. fp32 caches meet the fp32 bar.
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


def _multi(wl, vals, ps=0, out=None):
    d = G.device_tensors(wl, vals)
    if out is None:
        out = torch.empty_like(vals["q"])
    pa.pa_decode_multi(out, vals["q"], vals["k_cache"], vals["v_cache"], d["tables"], d["ctx"],
                       torch.as_tensor(wl.query_start, device=DEV), wl.scale,
                       max_context_len=wl.max_context_len, max_query_len=wl.max_query_len,
                       partition_size=ps)
    return out


def _step_check(wl, ps):
    vals = W.make_values(wl, DEV, poison=True)
    host = G.host_copy(vals)
    d = G.device_tensors(wl, vals)
    pa.pa_kv_append(vals["k_new"], vals["v_new"], d["slots"], vals["k_cache"], vals["v_cache"])
    out = _multi(wl, vals, ps)
    pa.pa_sync_check()
    assert G.last_kernel() in G.kernel_set(pa.PA_KERNEL_GROUPED)
    oracle.kv_append(host["k_new"], host["v_new"], wl.slot_mapping, host["k_cache"], host["v_cache"])
    assert G.bits_equal(vals["k_cache"], host["k_cache"])
    assert G.bits_equal(vals["v_cache"], host["v_cache"])
    ref = oracle.decode_multi(host["q"], host["k_cache"], host["v_cache"], wl.block_tables,
                              wl.context_lens, wl.query_start, wl.scale, num_threads=G.THREADS)
    return G.check_tolerance(G.to_f64(out), ref, wl.dtype, f"{wl.name} ps={ps}"), out, vals


CTX = [1, 2, 15, 16, 17, 40, 64, 65, 129, 300, 511, 513]
NQ = [1, 2, 15, 3, 9, 8, 1, 17, 4, 300, 0, 33]


@pytest.mark.parametrize("d,bs", [(64, 16), (128, 16), (128, 64)])
@pytest.mark.parametrize("H,Hkv", [(8, 8), (8, 4), (16, 2), (12, 3), (64, 8)])
def test_parity_shape_sweep(d, bs, H, Hkv):
    """Query counts from 0 to a whole 300-token prompt (38 groups of 8), contexts
    at block and partition edges, every n-tile layout."""
    wl = W.multi_query_case(len(CTX), H, Hkv, d, bs, "bf16", CTX, NQ, seed=d + bs + H)
    for ps in (-1, 0, 64):
        _step_check(wl, ps)


def test_token_result_independent_of_the_other_tokens():
    """Row j of a 6-token verification equals, bit for bit, row j of a 2-token
    call holding only tokens j and j + 1 (j - 1 and j for the last token) with
    the context cut after them: same kernel (16 or more query columns), same
    partition size, other query tokens and context length changed."""
    wl = W.multi_query_case(2, 32, 4, 128, 16, "bf16", [900, 333], [6, 5], seed=3)
    vals = W.make_values(wl, DEV, poison=False)
    d = G.device_tensors(wl, vals)
    pa.pa_kv_append(vals["k_new"], vals["v_new"], d["slots"], vals["k_cache"], vals["v_cache"])
    for ps in (128, 912):
        full = _multi(wl, vals, ps)
        for s, j in ((0, 0), (0, 5), (1, 2), (1, 4)):
            r0 = int(wl.query_start[s])
            n = int(wl.query_start[s + 1] - wl.query_start[s])
            a = j if j + 1 < n else j - 1                  # the pair (a, a + 1) holds j
            cut = int(wl.context_lens[s]) - n + a + 2      # the pair are the last two positions
            two = torch.empty_like(vals["q"][r0 + a:r0 + a + 2])
            pa.pa_decode_multi(two, vals["q"][r0 + a:r0 + a + 2].contiguous(), vals["k_cache"],
                               vals["v_cache"], d["tables"][s:s + 1].contiguous(),
                               torch.tensor([cut], dtype=torch.int32, device=DEV),
                               torch.tensor([0, 2], dtype=torch.int32, device=DEV), wl.scale,
                               max_context_len=wl.max_context_len, max_query_len=2,
                               partition_size=ps)
            torch.cuda.synchronize()
            assert G.bits_equal(full[r0 + j:r0 + j + 1], two[j - a:j - a + 1]), (ps, s, j)


def test_verification_full_size():
    """8 x 32K-context sequences verifying 4 draft tokens (64/8 heads), library
    partition policy: every query row of every sequence against the oracle."""
    wl = W.make("llama70b_verify4")
    vals = W.make_values(wl, DEV, poison=True)
    d = G.device_tensors(wl, vals)
    pa.pa_kv_append(vals["k_new"], vals["v_new"], d["slots"], vals["k_cache"], vals["v_cache"])
    out = _multi(wl, vals, 0)
    pa.pa_sync_check()
    assert torch.isfinite(out.float()).all()
    sub = W.subproblem(wl, vals["k_cache"], vals["v_cache"], range(wl.num_seqs))
    ref = oracle.decode_multi(W.to_numpy(vals["q"]).copy(), sub["k_cache"], sub["v_cache"],
                              sub["block_tables"], sub["context_lens"],
                              np.asarray(wl.query_start, np.int32), wl.scale,
                              num_threads=G.THREADS)
    G.check_tolerance(G.to_f64(out), ref, "bf16", "verify4, every row")


def test_more_queries_than_context_reported():
    wl = W.multi_query_case(2, 16, 2, 128, 16, "bf16", [40, 30], [3, 2], seed=1)
    vals = W.make_values(wl, DEV)
    d = G.device_tensors(wl, vals)
    out = torch.empty_like(vals["q"])
    pa.pa_sync_check()
    qs = torch.tensor([0, 3, 5], dtype=torch.int32, device=DEV)
    d["ctx"][1] = 1                                          # 2 queries, 1 context position
    pa.pa_decode_multi(out, vals["q"], vals["k_cache"], vals["v_cache"], d["tables"], d["ctx"], qs,
                       wl.scale, max_context_len=40, max_query_len=3)
    with pytest.raises(pa.PAError) as e:
        pa.pa_sync_check()
    assert e.value.code == pa.PA_ERR_BAD_INDEX


@pytest.mark.parametrize("d,bs", [(64, 16), (128, 32)])
@pytest.mark.parametrize("H,Hkv", [(4, 4), (16, 2), (12, 3)])
def test_f32_cache_parity(d, bs, H, Hkv):
    """fp32 caches: each query token is a row of its own on the CUDA-core consumer
    (it reads its sequence's blocks up to its causal end); the fp32 bar of
    pa_decode (row-normwise relative error <= 1e-5) holds, split or not."""
    wl = W.multi_query_case(len(CTX), H, Hkv, d, bs, "f32", CTX, NQ, seed=d + bs + H + 1)
    for ps in (-1, 0, 64):
        vals = W.make_values(wl, DEV, poison=True)
        host = G.host_copy(vals)
        d_ = G.device_tensors(wl, vals)
        pa.pa_kv_append(vals["k_new"], vals["v_new"], d_["slots"], vals["k_cache"],
                        vals["v_cache"])
        out = _multi(wl, vals, ps)
        pa.pa_sync_check()
        assert G.last_kernel() == pa.PA_KERNEL_SIMT
        oracle.kv_append(host["k_new"], host["v_new"], wl.slot_mapping, host["k_cache"],
                         host["v_cache"])
        assert G.bits_equal(vals["k_cache"], host["k_cache"])
        ref = oracle.decode_multi(host["q"], host["k_cache"], host["v_cache"], wl.block_tables,
                                  wl.context_lens, wl.query_start, wl.scale,
                                  num_threads=G.THREADS)
        errs = G.check_tolerance(G.to_f64(out), ref, "f32", f"f32 multi ps={ps}")
        assert errs["row_rel"] <= G.F32_ROW_REL


def test_f32_more_queries_than_context_reported():
    """A sequence with more new tokens than context positions (not a valid step)
    on the fp32 path: reported, and the token without any position gets 0."""
    wl = W.multi_query_case(2, 4, 4, 64, 16, "f32", [40, 30], [3, 2], seed=1)
    vals = W.make_values(wl, DEV)
    d = G.device_tensors(wl, vals)
    out = torch.full_like(vals["q"], float("nan"))
    pa.pa_sync_check()
    qs = torch.tensor([0, 3, 5], dtype=torch.int32, device=DEV)
    d["ctx"][1] = 1                                          # 2 queries, 1 context position
    pa.pa_decode_multi(out, vals["q"], vals["k_cache"], vals["v_cache"], d["tables"], d["ctx"], qs,
                       wl.scale, max_context_len=40, max_query_len=3, partition_size=-1)
    with pytest.raises(pa.PAError) as e:
        pa.pa_sync_check()
    assert e.value.code == pa.PA_ERR_BAD_INDEX
    assert G.last_kernel() == pa.PA_KERNEL_SIMT
    assert torch.equal(out[3], torch.zeros_like(out[3]))      # causal end 0: nothing to attend
    assert torch.isfinite(out).all()


def test_bf16_query_groups_above_64_columns():
    """A query group of 128 heads per kv head: too many columns for the grouped
    kernel, so every query token takes a CUDA-core row of its own."""
    wl = W.multi_query_case(3, 128, 1, 128, 16, "bf16", [70, 33, 300], [3, 1, 5], seed=5)
    vals = W.make_values(wl, DEV, poison=True)
    host = G.host_copy(vals)
    d_ = G.device_tensors(wl, vals)
    pa.pa_kv_append(vals["k_new"], vals["v_new"], d_["slots"], vals["k_cache"], vals["v_cache"])
    out = _multi(wl, vals, 0)
    pa.pa_sync_check()
    assert G.last_kernel() == pa.PA_KERNEL_SIMT
    oracle.kv_append(host["k_new"], host["v_new"], wl.slot_mapping, host["k_cache"], host["v_cache"])
    ref = oracle.decode_multi(host["q"], host["k_cache"], host["v_cache"], wl.block_tables,
                              wl.context_lens, wl.query_start, wl.scale, num_threads=G.THREADS)
    G.check_tolerance(G.to_f64(out), ref, "bf16", "128 heads per kv head")


def test_large_outputs_of_short_causal_contexts():
    """Short causal contexts give outputs near single V values (|out| above 4
    here), where the bf16 output's own rounding exceeds 1e-2: the result must be
    within the bar of the exact value once that rounding is allowed (measured: a
    2-token context with exact value -4.20794 returns -4.21875, its correct
    rounding)."""
    ctx = [1, 2, 15, 16, 17, 40, 64, 65, 129, 300, 511, 513, 4000, 2500]
    nq = [1, 2, 15, 3, 9, 8, 1, 17, 4, 300, 0, 33, 4, 7]
    wl = W.multi_query_case(len(ctx), 64, 8, 128, 16, "bf16", ctx, nq, seed=41)
    for ps in (-1, 0, 256):
        errs, out, _ = _step_check(wl, ps)
        assert errs["max_abs_raw"] > G.BF16_MAX_ABS  # the case this test is for
