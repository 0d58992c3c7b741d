"""Quantised KV caches (FP8 E4M3 / int8 codes, per-kv-head scales) on the GPU.

The quantising append must match the oracle's codes bit for bit over the whole
pool (edge values included: ties, saturation, infinities, NaN, signed zero,
subnormals); decode over codes must meet the bf16 bars against the oracle's
fp64 decode of value(code) * scale; block copy / swap move code pools exactly;
the calls refuse descriptors of the wrong kind.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_335_b200 as pa
from paged_kv_cache_335_b200 import workloads as W
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _codes(t):
    return W.to_numpy(t)


def _quant_step(wl, vals, ps=0):
    d = G.device_tensors(wl, vals)
    kc, vc = vals["k_cache"], vals["v_cache"]
    if wl.copy_pairs.shape[0]:
        pa.pa_block_copy(d["pairs"], kc, vc)
    if wl.num_tokens:
        pa.pa_kv_append_quant(vals["k_new"], vals["v_new"], d["slots"], kc, vc, vals["k_scale"],
                              vals["v_scale"])
    out = torch.empty_like(vals["q"])
    pa.pa_decode_quant(out, vals["q"], kc, vc, vals["k_scale"], vals["v_scale"], d["tables"],
                       d["ctx"], wl.scale, max_context_len=wl.max_context_len, partition_size=ps)
    return out


def _oracle_step(wl, host):
    kc, vc = host["k_cache"], host["v_cache"]
    if wl.copy_pairs.shape[0]:
        oracle.block_copy(wl.copy_pairs, kc, vc)
    if wl.num_tokens:
        oracle.kv_append_quant(host["k_new"], host["v_new"], wl.slot_mapping, kc, vc,
                               host["k_scale"], host["v_scale"], wl.kv_quant)
    return oracle.decode_quant(host["q"], kc, vc, host["k_scale"], host["v_scale"],
                               wl.block_tables, wl.context_lens, wl.scale, wl.kv_quant,
                               num_threads=G.THREADS)


def _host(vals):
    return {k: (W.to_numpy(t).copy() if t.dtype != torch.float32 else t.cpu().numpy().copy())
            for k, t in vals.items()}


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
@pytest.mark.parametrize("H,Hkv", [(8, 8), (16, 2), (12, 3), (32, 2)])
@pytest.mark.parametrize("bs", [16, 64])
@pytest.mark.parametrize("d", [64, 128])
def test_step_parity_edges(fmt, H, Hkv, bs, d):
    """Contexts at block and partition edges (0 included) on the CUDA-core (MHA,
    group 16) and tensor-core (group 2..8) consumers over codes, head_dim 64
    (64-code rows read as 128-code rows whose upper half the TMA zero-fills) and
    128; appended codes bit-exact."""
    ctx = [0, 1, 2, 15, 16, 17, 33, 64, 129, 511, 513, 1000]
    wl = W.quantized(G.custom(len(ctx), H, Hkv, d, bs, "bf16", ctx, seed=bs + H + d), fmt)
    for ps in (-1, 64, 0):
        vals = W.make_values(wl, DEV, poison=True)
        host = _host(vals)
        out = _quant_step(wl, vals, ps)
        pa.pa_sync_check()
        ref = _oracle_step(wl, host)
        assert np.array_equal(_codes(vals["k_cache"]), host["k_cache"]), "k codes differ"
        assert np.array_equal(_codes(vals["v_cache"]), host["v_cache"]), "v codes differ"
        G.check_tolerance(G.to_f64(out), ref, "bf16", f"{wl.name} ps={ps}")


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
@pytest.mark.parametrize("d", [64, 128])
def test_append_codes_bit_exact_on_edge_values(fmt, d):
    """Ties, saturation, infinities, NaN, signed zero and subnormal quotients,
    through binary32 division by per-head scales."""
    wl = W.quantized(G.custom(4, 8, 4, d, 16, "bf16", [30, 1, 17, 64], seed=d), fmt)
    vals = W.make_values(wl, DEV, poison=False)
    special = torch.tensor([0.0, -0.0, float("inf"), -float("inf"), float("nan"), 1e30, -1e30,
                            2.5, 3.5, -2.5, 448.0, 449.0, 1e-30, -3e-38, 0.375, 7.0],
                           dtype=torch.float32)
    k_new = vals["k_new"].float()
    k_new.view(-1)[:special.numel()] = special.to(DEV)
    vals["k_new"] = k_new.to(torch.bfloat16)
    vals["k_scale"][0] = 0.5
    vals["k_scale"][1] = 1.0 / 3.0
    host = _host(vals)
    d_ = G.device_tensors(wl, vals)
    pa.pa_kv_append_quant(vals["k_new"], vals["v_new"], d_["slots"], vals["k_cache"],
                          vals["v_cache"], vals["k_scale"], vals["v_scale"])
    pa.pa_sync_check()
    oracle.kv_append_quant(host["k_new"], host["v_new"], wl.slot_mapping, host["k_cache"],
                           host["v_cache"], host["k_scale"], host["v_scale"], fmt)
    assert np.array_equal(_codes(vals["k_cache"]), host["k_cache"])
    assert np.array_equal(_codes(vals["v_cache"]), host["v_cache"])


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
def test_llama13b_full_size(fmt):
    """The headline 13B step over a quantised pool, in the bench's launch
    configuration: every output element against the oracle, codes of the
    appended slots bit-exact."""
    wl = W.make(f"llama13b_bs16_{fmt}")
    vals = W.make_values(wl, DEV, poison=(fmt == "fp8"))
    out = _quant_step(wl, vals)
    pa.pa_sync_check()
    assert torch.isfinite(out.float()).all()
    # appended codes against the oracle's quantiser on the same inputs
    slots = torch.as_tensor(wl.slot_mapping, device=DEV)
    b, o = slots // wl.block_size, slots % wl.block_size
    for cache, new, sc in ((vals["k_cache"], vals["k_new"], vals["k_scale"]),
                           (vals["v_cache"], vals["v_new"], vals["v_scale"])):
        got = _codes(cache.view(torch.uint8)[b, :, o, :])
        x = new.float().cpu().numpy()
        want = np.stack([np.stack([oracle.quantize(x[t, h], float(sc[h]), fmt)
                                   for h in range(wl.num_kv_heads)]) for t in range(x.shape[0])])
        assert np.array_equal(got, want)
    sub = W.subproblem(wl, vals["k_cache"], vals["v_cache"], range(wl.num_seqs), vals["q"])
    ref = oracle.decode_quant(sub["q"], sub["k_cache"], sub["v_cache"],
                              vals["k_scale"].cpu().numpy(), vals["v_scale"].cpu().numpy(),
                              sub["block_tables"], sub["context_lens"], wl.scale, fmt,
                              num_threads=G.THREADS)
    G.check_tolerance(G.to_f64(out), ref, "bf16", wl.name)


def test_copy_and_swap_move_code_pools():
    wl = W.quantized(W.cow_beam4(num_prompts=2, prompt_len=100, max_suffix=20, num_heads=16,
                                 num_kv_heads=2, head_dim=128), "fp8")
    vals = W.make_values(wl, DEV, poison=True)
    host = _host(vals)
    out = _quant_step(wl, vals)
    pa.pa_sync_check()
    ref = _oracle_step(wl, host)
    assert np.array_equal(_codes(vals["k_cache"]), host["k_cache"])
    G.check_tolerance(G.to_f64(out), ref, "bf16", "cow fp8")
    hk = torch.zeros((8,) + tuple(vals["k_cache"].shape[1:]), dtype=torch.uint8).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    pairs = np.array([[3, 0], [7, 5]], np.int64)
    pa.pa_block_swap(torch.as_tensor(pairs, device=DEV), vals["k_cache"], vals["v_cache"],
                     hk.view(torch.float8_e4m3fn), hv.view(torch.float8_e4m3fn))
    torch.cuda.synchronize()
    assert np.array_equal(hk.numpy()[0], host["k_cache"][3])
    assert np.array_equal(hv.numpy()[5], host["v_cache"][7])


def test_wrong_descriptor_kind_refused():
    wl = W.quantized(G.custom(2, 8, 8, 128, 16, "bf16", [20, 30], seed=2), "int8")
    vals = W.make_values(wl, DEV)
    d = G.device_tensors(wl, vals)
    out = torch.empty_like(vals["q"])
    lib = pa.load_library()
    desc = pa.cache_desc(vals["k_cache"])
    P = ctypes.c_void_p
    rc = lib.pa_decode(P(out.data_ptr()), P(vals["q"].data_ptr()), P(vals["k_cache"].data_ptr()),
                       P(vals["v_cache"].data_ptr()), P(d["tables"].data_ptr()), 2,
                       P(d["ctx"].data_ptr()), 30, 2, 8, ctypes.c_float(wl.scale),
                       ctypes.byref(desc), 0, None, 0, None)
    assert rc == pa.PA_ERR_DTYPE                       # codes need pa_decode_quant
    rc = lib.pa_kv_append(P(vals["k_new"].data_ptr()), P(vals["v_new"].data_ptr()),
                          P(d["slots"].data_ptr()), 2, P(vals["k_cache"].data_ptr()),
                          P(vals["v_cache"].data_ptr()), ctypes.byref(desc), None)
    assert rc == pa.PA_ERR_DTYPE                       # codes need pa_kv_append_quant
    wl3 = W.quantized(G.custom(2, 8, 8, 128, 16, "bf16", [20, 30], seed=2), "fp8")
    v3 = W.make_values(wl3, DEV)
    d3 = G.device_tensors(wl3, v3)
    with pytest.raises(TypeError):             # q must be bf16 over a quantised cache
        pa.pa_decode_quant(torch.empty_like(v3["q"]).float(), v3["q"].float(), v3["k_cache"],
                           v3["v_cache"], v3["k_scale"], v3["v_scale"], d3["tables"], d3["ctx"],
                           wl3.scale, max_context_len=30)


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
def test_llama70b_gqa_tensor_core_path(fmt):
    """The 70B GQA step (8 x 32K contexts, group 8) over codes runs the
    tensor-core consumer (f16 MMAs on exactly converted codes) with the library
    partition policy; every sequence against the oracle."""
    wl = W.make(f"llama70b_gqa_{fmt}")
    vals = W.make_values(wl, DEV, poison=(fmt == "fp8"))
    out = _quant_step(wl, vals, 0)
    pa.pa_sync_check()
    assert G.last_kernel() == pa.PA_KERNEL_MMA
    assert torch.isfinite(out.float()).all()
    sub = W.subproblem(wl, vals["k_cache"], vals["v_cache"], range(wl.num_seqs), vals["q"])
    ref = oracle.decode_quant(sub["q"], sub["k_cache"], sub["v_cache"],
                              vals["k_scale"].cpu().numpy(), vals["v_scale"].cpu().numpy(),
                              sub["block_tables"], sub["context_lens"], wl.scale, fmt,
                              num_threads=G.THREADS)
    G.check_tolerance(G.to_f64(out), ref, "bf16", wl.name)


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
def test_q_magnitudes_outside_f16_range(fmt):
    """Over codes q becomes an f16 MMA / fma operand, after a power-of-two shift
    that puts its largest magnitude in [2^14, 2^15), undone on the scores. So q
    of any magnitude is handled exactly: q x 2^20 (|q| ~ 1e6, far above f16's
    65504) with scale x 2^-20, and q x 2^-20 (|q| ~ 1e-6, below f16's normal
    range) with scale x 2^20, give bit for bit the output of (q, scale), which
    meets the bars against the oracle. Covers the CUDA-core consumer (MHA), the
    tensor-core consumer (GQA g = 8) and the grouped / multi-token consumer.
    (Comparing |q| ~ 1e6 with the fp64 oracle directly would test the
    conditioning of the softmax instead: scores ~1e6 carry fp32 rounding of the
    order of the gap between near-tied scores.)"""
    ctx = [1, 15, 16, 17, 130, 700]
    for H, Hkv in ((8, 8), (16, 2)):
        wl = W.quantized(G.custom(len(ctx), H, Hkv, 128, 16, "bf16", ctx, seed=31), fmt)
        vals = W.make_values(wl, DEV, poison=False)
        host = _host(vals)
        out = _quant_step(wl, vals, ps=-1)       # appends, then decodes (q, scale)
        pa.pa_sync_check()
        G.check_tolerance(G.to_f64(out), _oracle_step(wl, host), "bf16", f"{fmt} H={H}/{Hkv}")
        d = G.device_tensors(wl, vals)

        def decode(q, scale, grouped):
            o = torch.empty_like(q)
            args = (o, q, vals["k_cache"], vals["v_cache"], vals["k_scale"], vals["v_scale"],
                    d["tables"], d["ctx"], scale)
            if grouped:
                pa.pa_decode_grouped_quant(*args, 2, max_context_len=wl.max_context_len,
                                           partition_size=-1)
            else:
                pa.pa_decode_quant(*args, max_context_len=wl.max_context_len, partition_size=-1)
            pa.pa_sync_check()
            return o

        for grouped in (False, True):
            base = decode(vals["q"], wl.scale, grouped)
            for k in (20, -20):
                qk = (vals["q"].float() * 2.0 ** k).to(torch.bfloat16)   # exact: a power of two
                got = decode(qk, wl.scale * 2.0 ** -k, grouped)
                assert torch.isfinite(got.float()).all()
                assert G.dev_bits_equal(got, base), f"{fmt} H={H}/{Hkv} grouped={grouped} 2^{k}"


@pytest.mark.parametrize("fmt", ["int8", "fp8"])
def test_same_sign_q_long_context(fmt):
    """The worst case for the int8 offset the tensor-core consumers take out once
    per sum (scores minus 1152 x the sum of q): every q element of one sign, so
    the sum of q and the offset it carries are as large as they can be, over 4K-
    token contexts, on the GQA consumer (split and unsplit) and the grouped one.
    Must meet the bars against the oracle like any other q (fp8, which carries no
    offset, is the control)."""
    ctx = [4096, 3001, 17, 1]
    wl = W.quantized(G.custom(len(ctx), 16, 2, 128, 16, "bf16", ctx, seed=37), fmt)
    vals = W.make_values(wl, DEV, poison=False)
    vals["q"].copy_(vals["q"].abs())
    host = _host(vals)
    d = G.device_tensors(wl, vals)
    pa.pa_kv_append_quant(vals["k_new"], vals["v_new"], d["slots"], vals["k_cache"], vals["v_cache"],
                          vals["k_scale"], vals["v_scale"])
    ref = _oracle_step(wl, host)
    for grouped, ps in ((False, -1), (False, 512), (True, -1)):
        out = torch.empty_like(vals["q"])
        args = (out, vals["q"], vals["k_cache"], vals["v_cache"], vals["k_scale"], vals["v_scale"],
                d["tables"], d["ctx"], wl.scale)
        if grouped:
            pa.pa_decode_grouped_quant(*args, 2, max_context_len=wl.max_context_len, partition_size=ps)
        else:
            pa.pa_decode_quant(*args, max_context_len=wl.max_context_len, partition_size=ps)
        pa.pa_sync_check()
        assert G.last_kernel() in (pa.PA_KERNEL_MMA,) + G.kernel_set(pa.PA_KERNEL_GROUPED)
        G.check_tolerance(G.to_f64(out), ref, "bf16", f"{fmt} same-sign q grouped={grouped} ps={ps}")
