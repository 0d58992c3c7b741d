"""Shared helpers of the GPU parity tests: run one step on the CUDA path and on
the oracle from the same seeded inputs, and the acceptance tolerances."""
import os

import numpy as np
import torch

import oracle
import paged_kv_cache_335_b200 as pa
from paged_kv_cache_335_b200 import workloads as W

# Acceptance bars. fp32: row-normwise relative error max_d|g-r| / max_d|r| <= 1e-5
# per (sequence, head). bf16 caches with fp32 accumulation: max abs error <= 1e-2
# and mean abs error <= 1e-3 against the unrounded fp64 oracle. The output itself
# is bf16, whose rounding alone moves a value by up to half an ulp (1/64 for
# magnitudes in [4, 8)): the max bar bounds the arithmetic error, |got - ref|
# less half an ulp of the bf16 output (an output equal to the correctly rounded
# oracle value has none); the mean bar is taken on |got - ref| as it is.
F32_ROW_REL = 1e-5
BF16_MAX_ABS = 1e-2
BF16_MEAN_ABS = 1e-3


def bf16_half_ulp(x):
    """Half an ulp of bf16 values (8 significant bits) at their magnitude: the
    most that rounding to bf16 moves a value that lands on them."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126.0)
    return np.where(a > 0, np.exp2(e - 8.0), 2.0 ** -134)

THREADS = max(1, len(os.sched_getaffinity(0)))


def device_tensors(wl, vals):
    dev = vals["q"].device
    return {
        "tables": torch.as_tensor(wl.block_tables, device=dev),
        "ctx": torch.as_tensor(wl.context_lens, device=dev),
        "slots": torch.as_tensor(wl.slot_mapping, device=dev),
        "pairs": torch.as_tensor(wl.copy_pairs, device=dev),
    }


def gpu_step(wl, vals, partition_size=None, out=None, workspace=None, group_size=1):
    """One pass of the hot path on the GPU, in place on vals' caches:
    copy-on-write block copies, append of this step's tokens, decode (grouped
    by ``group_size`` sequences when > 1)."""
    d = device_tensors(wl, vals)
    kc, vc = vals["k_cache"], vals["v_cache"]
    if wl.copy_pairs.shape[0]:
        pa.pa_block_copy(d["pairs"], kc, vc)
    if wl.num_tokens:
        pa.pa_kv_append(vals["k_new"], vals["v_new"], d["slots"], kc, vc)
    if out is None:
        out = torch.empty_like(vals["q"])
    ps = wl.partition_size if partition_size is None else partition_size
    if group_size > 1:
        pa.pa_decode_grouped(out, vals["q"], kc, vc, d["tables"], d["ctx"], wl.scale, group_size,
                             max_context_len=wl.max_context_len, partition_size=ps,
                             workspace=workspace)
    else:
        pa.pa_decode(out, vals["q"], kc, vc, d["tables"], d["ctx"], wl.scale,
                     max_context_len=wl.max_context_len, partition_size=ps, workspace=workspace)
    return out


def last_kernel():
    return pa.load_library().pa_test_last_decode_kernel()


def kernel_set(kernel):
    """The decode kernels that count as `kernel`: the grouped kernel runs on either
    grouped consumer (pa_set_grouped_consumer)."""
    if kernel == pa.PA_KERNEL_GROUPED:
        return (pa.PA_KERNEL_GROUPED, pa.PA_KERNEL_GROUPED_TCGEN05)
    return (kernel,)


def oracle_step(wl, host):
    """The same step on the oracle. ``host``: numpy copies of the inputs taken
    before the GPU step (caches are modified in place)."""
    kc, vc = host["k_cache"], host["v_cache"]
    if wl.copy_pairs.shape[0]:
        oracle.block_copy(wl.copy_pairs, kc, vc)
    if wl.num_tokens:
        oracle.kv_append(host["k_new"], host["v_new"], wl.slot_mapping, kc, vc)
    return oracle.decode(host["q"], kc, vc, wl.block_tables, wl.context_lens, wl.scale,
                         num_threads=THREADS)


def host_copy(vals):
    return {k: W.to_numpy(v).copy() for k, v in vals.items()}


def to_f64(t):
    return t.detach().float().cpu().double().numpy()


def check_tolerance(got, ref, dtype, what=""):
    """Assert the acceptance bar; returns the error figures."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    if dtype == "f32":
        den = np.abs(ref).max(axis=-1)
        num = err.max(axis=-1)
        rel = np.where(den > 0, num / np.where(den > 0, den, 1), num)
        worst = float(rel.max()) if rel.size else 0.0
        assert worst <= F32_ROW_REL, f"{what}: row-normwise rel error {worst:.3e} > {F32_ROW_REL}"
        return {"row_rel": worst}
    arith = np.maximum(err - bf16_half_ulp(got), 0.0)  # less the output's own rounding
    mx = float(arith.max()) if err.size else 0.0
    mean = float(err.mean()) if err.size else 0.0
    assert mx <= BF16_MAX_ABS, f"{what}: max abs error {mx:.3e} beyond the output rounding > {BF16_MAX_ABS}"
    assert mean <= BF16_MEAN_ABS, f"{what}: mean abs error {mean:.3e} > {BF16_MEAN_ABS}"
    return {"max_abs": mx, "max_abs_raw": float(err.max()) if err.size else 0.0, "mean_abs": mean}


def bits_equal(a, b):
    """Bitwise equality of two tensors / arrays (NaN patterns included)."""
    if isinstance(a, torch.Tensor):
        a = W.to_numpy(a)
    if isinstance(b, torch.Tensor):
        b = W.to_numpy(b)
    a = np.ascontiguousarray(a)
    b = np.ascontiguousarray(b)
    if a.dtype == np.float32:
        a, b = a.view(np.uint32), b.view(np.uint32)
    return a.shape == b.shape and np.array_equal(a, b)


def dev_bits_equal(a: torch.Tensor, b: torch.Tensor) -> bool:
    """Bitwise equality of two device tensors, compared on the device."""
    if a.shape != b.shape or a.dtype != b.dtype:
        return False
    view = torch.int32 if a.element_size() == 4 else torch.int16
    return bool(torch.equal(a.contiguous().view(view), b.contiguous().view(view)))


def oracle_all(wl, vals_after):
    """Oracle decode of every sequence, read from the post-step device pool."""
    return oracle_sampled(wl, vals_after, range(wl.num_seqs))


def oracle_sampled(wl, vals_after, seq_ids):
    """Oracle decode of the sampled sequences read from the post-step device pool."""
    sub = W.subproblem(wl, vals_after["k_cache"], vals_after["v_cache"], seq_ids, vals_after["q"])
    return oracle.decode(sub["q"], sub["k_cache"], sub["v_cache"], sub["block_tables"],
                         sub["context_lens"], wl.scale, num_threads=THREADS)


def custom(S, H, Hkv, d, bs, dtype, ctx, seed=0, pool_factor=1.3, partition_size=0):
    """A decode workload with given context lengths (same construction as the configs)."""
    return W.decode_case(S, H, Hkv, d, bs, dtype, ctx, seed=seed, pool_factor=pool_factor,
                         partition_size=partition_size)
