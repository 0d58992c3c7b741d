"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Moves (append, block copy) must match bit for bit; decode must meet the
acceptance bars: fp32 row-normwise relative error <= 1e-5, bf16 max abs error
<= 1e-2 and mean abs error <= 1e-3 against the unrounded fp64 oracle.
Unfilled slots, unowned blocks and copy destinations are NaN-poisoned before
each step, so a read past a context or a missed write shows up as NaN.
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


def _full_step_check(wl, partition_size=None):
    """Whole-problem parity: pools bit-exact after the moves, decode within tolerance."""
    vals = W.make_values(wl, DEV, poison=True)
    host = G.host_copy(vals)
    out = G.gpu_step(wl, vals, partition_size=partition_size)
    pa.pa_sync_check()
    ref = G.oracle_step(wl, host)
    assert G.bits_equal(vals["k_cache"], host["k_cache"]), "k_cache differs from the oracle"
    assert G.bits_equal(vals["v_cache"], host["v_cache"]), "v_cache differs from the oracle"
    return G.check_tolerance(G.to_f64(out), ref, wl.dtype, wl.name), out, vals


# ---------------------------------------------------------------------------
# the five configurations
# ---------------------------------------------------------------------------
def test_tiny_fp32_full():
    errs, _, _ = _full_step_check(W.tiny())
    assert errs["row_rel"] <= G.F32_ROW_REL


def test_tiny_fp32_split_partitions():
    wl = W.tiny()
    for ps in (16, 32, 64, -1):
        _full_step_check(wl, partition_size=ps)


@pytest.mark.parametrize("name", ["llama7b", "llama13b_bs16", "llama13b_bs32", "llama70b_gqa",
                                  "cow_beam4"])
def test_config_full_size(name):
    """Full-size configuration in the bench's launch configuration: every
    element of the decode output against the oracle, the appended slots and
    copied blocks bit-exact, all outputs finite."""
    wl = W.make(name)
    vals = W.make_values(wl, DEV, poison=True)
    pre = {"k_cache": vals["k_cache"].clone(), "v_cache": vals["v_cache"].clone()}
    out = G.gpu_step(wl, vals)
    pa.pa_sync_check()
    assert torch.isfinite(out.float()).all(), "NaN/Inf in decode output (poisoned slot read?)"
    # appended slots hold exactly the new vectors
    if wl.num_tokens:
        slots = torch.as_tensor(wl.slot_mapping, device=DEV)
        b, o = slots // wl.block_size, slots % wl.block_size
        for cache, new in ((vals["k_cache"], vals["k_new"]), (vals["v_cache"], vals["v_new"])):
            assert G.dev_bits_equal(cache[b, :, o, :], new)
    # copy destinations hold the sources' pre-step bits, except slots appended after
    if wl.copy_pairs.shape[0]:
        src = torch.as_tensor(wl.copy_pairs[:, 0], device=DEV)
        dst = torch.as_tensor(wl.copy_pairs[:, 1], device=DEV)
        # every copied tail keeps at least this many prompt slots that no append overwrites
        fill = int((wl.extra["prompt_lens"] % wl.block_size).min())
        for cache, before in ((vals["k_cache"], pre["k_cache"]), (vals["v_cache"], pre["v_cache"])):
            assert G.dev_bits_equal(cache[dst, :, :fill], before[src, :, :fill])
    # blocks no step wrote to are untouched
    touched = set((wl.slot_mapping // wl.block_size).tolist()) | set(wl.copy_pairs[:, 1].tolist())
    keep = torch.as_tensor(sorted(set(range(wl.num_blocks)) - touched), device=DEV)
    for cache, before in ((vals["k_cache"], pre["k_cache"]), (vals["v_cache"], pre["v_cache"])):
        assert G.dev_bits_equal(cache.index_select(0, keep), before.index_select(0, keep))
    del pre
    ref = G.oracle_all(wl, vals)
    G.check_tolerance(G.to_f64(out), ref, wl.dtype, name)


def test_cow_small_full_pool_bit_exact():
    """Copy-on-write step on a pool small enough to compare whole: block copies,
    suffix appends, decode; the shared-prefix beams agree with the oracle."""
    wl = W.cow_beam4(num_prompts=3, prompt_len=200, max_suffix=40, num_heads=16, num_kv_heads=2,
                     head_dim=128)
    assert wl.copy_pairs.shape[0] == 9
    _full_step_check(wl)


def test_cow_aligned_prompt_no_copies():
    wl = W.cow_beam4(num_prompts=2, prompt_len=64, aligned=True, max_suffix=20, num_heads=16,
                     num_kv_heads=2, head_dim=64)
    assert wl.copy_pairs.shape[0] == 0
    _full_step_check(wl)


# ---------------------------------------------------------------------------
# invariants on the GPU
# ---------------------------------------------------------------------------
def _permuted(wl, vals, seed):
    """Same logical contents, different physical placement: block b -> perm[b]."""
    perm = np.random.default_rng(seed).permutation(wl.num_blocks)
    inv = torch.as_tensor(np.argsort(perm), device=DEV)
    wl2 = W.Workload(**{**wl.__dict__})
    wl2.block_tables = perm[wl.block_tables].astype(np.int32)
    wl2.slot_mapping = (perm[wl.slot_mapping // wl.block_size] * wl.block_size +
                        wl.slot_mapping % wl.block_size).astype(np.int64)
    wl2.copy_pairs = perm[wl.copy_pairs].astype(np.int64).reshape(-1, 2)
    vals2 = dict(vals)
    vals2["k_cache"] = vals["k_cache"].index_select(0, inv).contiguous()
    vals2["v_cache"] = vals["v_cache"].index_select(0, inv).contiguous()
    return wl2, vals2


@pytest.mark.parametrize("name,kw", [
    ("tiny", {}),
    ("custom_mha_bf16", dict(S=6, H=8, Hkv=8, d=128, bs=16, dtype="bf16")),
    ("custom_gqa_bf16", dict(S=5, H=32, Hkv=4, d=128, bs=32, dtype="bf16")),
])
def test_placement_invariance_bitwise(name, kw):
    if name == "tiny":
        wl = W.tiny()
    else:
        wl = G.custom(ctx=np.random.default_rng(3).integers(1, 700, size=kw["S"]), seed=3, **kw)
    vals = W.make_values(wl, DEV, poison=True)
    outs = []
    for seed in (None, 17, 18):
        w, v = (wl, {k: t.clone() for k, t in vals.items()}) if seed is None else \
            _permuted(wl, {k: t.clone() for k, t in vals.items()}, seed)
        outs.append(G.gpu_step(w, v, partition_size=128))
    torch.cuda.synchronize()
    pa.pa_sync_check()
    for o in outs[1:]:
        assert G.bits_equal(outs[0], o)


def test_deterministic_repeat():
    wl = W.make("llama70b_gqa", num_seqs=2, context_len=5000)
    vals = W.make_values(wl, DEV, poison=True)
    d = G.device_tensors(wl, vals)
    pa.pa_kv_append(vals["k_new"], vals["v_new"], d["slots"], vals["k_cache"], vals["v_cache"])
    outs = []
    for _ in range(3):
        out = torch.empty_like(vals["q"])
        pa.pa_decode(out, vals["q"], vals["k_cache"], vals["v_cache"], d["tables"], d["ctx"],
                     wl.scale, max_context_len=wl.max_context_len, partition_size=512)
        outs.append(out)
    for o in outs[1:]:
        assert G.bits_equal(outs[0], o)


def test_shared_prefix_equals_private_copy_bitwise():
    """Beams that share prompt blocks through reference counts decode exactly
    like sequences holding private copies of the same tokens."""
    wl = W.cow_beam4(num_prompts=2, prompt_len=300, max_suffix=30, num_heads=16, num_kv_heads=2,
                     head_dim=128)
    vals = W.make_values(wl, DEV, poison=False)
    shared_out = G.gpu_step(wl, vals)
    # rebuild every beam privately: gather its logical blocks into fresh blocks
    B = wl.block_size
    rows, ids = [], []
    for s in range(wl.num_seqs):
        nb = -(-int(wl.context_lens[s]) // B)
        rows.append(list(range(len(ids), len(ids) + nb)))
        ids.extend(int(x) for x in wl.block_tables[s, :nb])
    idx = torch.as_tensor(ids, device=DEV)
    kc2 = vals["k_cache"].index_select(0, idx).contiguous()
    vc2 = vals["v_cache"].index_select(0, idx).contiguous()
    width = max(len(r) for r in rows)
    tables = np.zeros((wl.num_seqs, width), np.int32)
    for s, r in enumerate(rows):
        tables[s, :len(r)] = r
    out2 = torch.empty_like(vals["q"])
    pa.pa_decode(out2, vals["q"], kc2, vc2, torch.as_tensor(tables, device=DEV),
                 torch.as_tensor(wl.context_lens, device=DEV), wl.scale,
                 max_context_len=wl.max_context_len)
    torch.cuda.synchronize()
    assert len(set(ids)) < len(ids)       # the shared layout really shared blocks
    assert G.bits_equal(shared_out, out2)


# ---------------------------------------------------------------------------
# edge cases and the shape sweep
# ---------------------------------------------------------------------------
EDGE_CTX = [0, 1, 2, 15, 16, 17, 31, 32, 33, 63, 64, 65, 127, 128, 129, 511, 512, 513, 1000]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bs", [16, 32, 64])
@pytest.mark.parametrize("H,Hkv", [(4, 4), (8, 4), (16, 4), (16, 2), (12, 3)])
def test_shape_sweep_edges(dtype, d, bs, H, Hkv):
    """Empty, 1-token, block-boundary and partition-boundary contexts, for every
    head dim, block size, group size (1, 2, 4, 8 and 4 with 3 kv heads) and dtype;
    one partition and 64-token partitions."""
    wl = G.custom(len(EDGE_CTX), H, Hkv, d, bs, dtype, EDGE_CTX, seed=bs + d + H)
    for ps in (-1, 64):
        _full_step_check(wl, partition_size=ps)


def test_ctx1_returns_v_exactly():
    wl = G.custom(8, 32, 4, 128, 16, "bf16", [1] * 8, seed=5)
    vals = W.make_values(wl, DEV, poison=True)
    out = G.gpu_step(wl, vals)
    torch.cuda.synchronize()
    # ctx 1: the only token is the one just appended, so out = its V exactly
    v_rows = vals["v_new"].repeat_interleave(8, dim=1)      # q head h reads kv head h // 8
    assert G.bits_equal(out, v_rows)


def test_group_above_eight_uses_cuda_cores():
    wl = G.custom(3, 32, 2, 128, 16, "bf16", [700, 5, 1200], seed=9)   # group 16
    _full_step_check(wl, partition_size=0)


def test_long_context_many_partitions():
    wl = W.make("llama70b_gqa", num_seqs=2, context_len=32768)
    for ps in (512, 2048, -1):
        vals = W.make_values(wl, DEV, poison=True)
        out = G.gpu_step(wl, vals, partition_size=ps)
        ref = G.oracle_all(wl, vals)
        G.check_tolerance(G.to_f64(out), ref, "bf16", f"ps={ps}")


# ---------------------------------------------------------------------------
# bounds checks: bad indices are skipped and reported, never faulted
# ---------------------------------------------------------------------------
def test_bad_block_id_is_reported():
    wl = G.custom(2, 8, 8, 128, 16, "bf16", [40, 40], seed=1)
    vals = W.make_values(wl, DEV)
    d = G.device_tensors(wl, vals)
    d["tables"][1, 1] = wl.num_blocks + 5          # outside the pool: checked before use
    out = torch.empty_like(vals["q"])
    pa.pa_sync_check()
    pa.pa_decode(out, vals["q"], vals["k_cache"], vals["v_cache"], d["tables"], d["ctx"],
                 wl.scale, max_context_len=40)
    with pytest.raises(pa.PAError) as e:
        pa.pa_sync_check()
    assert e.value.code == pa.PA_ERR_BAD_INDEX
    pa.pa_sync_check()                             # cleared


def test_bad_slot_and_pair_are_reported():
    wl = G.custom(2, 8, 8, 64, 16, "bf16", [20, 30], seed=2)
    vals = W.make_values(wl, DEV)
    kc0 = vals["k_cache"].clone()
    slots = torch.tensor([wl.num_blocks * 16 + 3, -1], dtype=torch.int64, device=DEV)
    pa.pa_kv_append(vals["k_new"], vals["v_new"], slots, vals["k_cache"], vals["v_cache"])
    with pytest.raises(pa.PAError):
        pa.pa_sync_check()
    assert torch.equal(vals["k_cache"], kc0)       # nothing written
    pairs = torch.tensor([[0, wl.num_blocks]], dtype=torch.int64, device=DEV)
    pa.pa_block_copy(pairs, vals["k_cache"], vals["v_cache"])
    with pytest.raises(pa.PAError):
        pa.pa_sync_check()
    assert torch.equal(vals["k_cache"], kc0)


def test_context_beyond_bound_is_reported():
    wl = G.custom(2, 8, 8, 64, 16, "bf16", [20, 30], seed=2)
    vals = W.make_values(wl, DEV)
    d = G.device_tensors(wl, vals)
    d["ctx"][0] = 10_000                            # > max_context_len: clipped, reported
    out = torch.empty_like(vals["q"])
    pa.pa_decode(out, vals["q"], vals["k_cache"], vals["v_cache"], d["tables"], d["ctx"],
                 wl.scale, max_context_len=32)
    with pytest.raises(pa.PAError):
        pa.pa_sync_check()


# ---------------------------------------------------------------------------
# canaries: nothing is written outside out / workspace
# ---------------------------------------------------------------------------
def test_no_writes_outside_outputs():
    wl = W.make("llama70b_gqa", num_seqs=2, context_len=3000)
    vals = W.make_values(wl, DEV, poison=True)
    G_ELEMS = 4096
    n = vals["q"].numel()
    buf = torch.full((n + 2 * G_ELEMS,), 7.0, dtype=torch.bfloat16, device=DEV)
    out = buf[G_ELEMS:G_ELEMS + n].view_as(vals["q"])
    need = pa.pa_decode_workspace_size(wl.num_seqs, wl.num_heads, wl.max_context_len,
                                       vals["k_cache"], 512)
    wbuf = torch.full((need + 2 * 4096,), 0xA5, dtype=torch.uint8, device=DEV)
    ws = wbuf[4096:4096 + need]
    G.gpu_step(wl, vals, partition_size=512, out=out, workspace=ws)
    torch.cuda.synchronize()
    assert (buf[:G_ELEMS] == 7.0).all() and (buf[G_ELEMS + n:] == 7.0).all()
    assert (wbuf[:4096] == 0xA5).all() and (wbuf[4096 + need:] == 0xA5).all()
    ref = G.oracle_sampled(wl, vals, [0, 1])
    G.check_tolerance(G.to_f64(out), ref, "bf16")
