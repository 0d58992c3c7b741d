"""Host-side allocator and workload construction (no GPU)."""
import numpy as np
import pytest

from paged_kv_cache_335_b200 import block_manager as bmod
from paged_kv_cache_335_b200 import workloads as W


def test_allocation_follows_permutation_and_exhausts():
    order = np.random.default_rng(0).permutation(10)
    bm = bmod.BlockManager(10, 4, order=order, reserved=(int(order[-1]),))
    got = [bm.allocate() for _ in range(9)]
    assert got == [int(x) for x in order[:9]]
    assert bm.num_free == 0
    with pytest.raises(bmod.PoolExhausted):
        bm.allocate()


def test_order_must_be_permutation():
    with pytest.raises(ValueError):
        bmod.BlockManager(4, 2, order=[0, 1, 1, 2])


def test_append_opens_block_when_full():
    """Flowchart: append into the current block; a full block asks for a new one."""
    bm = bmod.BlockManager(8, 4)
    seq = bm.new_sequence(0)
    slots = [bm.append_slot(seq) for _ in range(9)]
    assert len(seq.table) == 3
    for pos, slot in enumerate(slots):
        assert slot == seq.table[pos // 4] * 4 + pos % 4


def test_free_returns_blocks_and_refcounts_stay_non_negative():
    bm = bmod.BlockManager(8, 2)
    a = bm.new_sequence(5)
    b = bm.fork(a)
    assert all(bm.refcount[x] == 2 for x in a.table)
    bm.free(a)
    assert all(bm.refcount[x] == 1 for x in b.table)
    free_before = bm.num_free
    bm.free(b)
    assert bm.num_free == free_before + 3
    assert (bm.refcount >= 0).all() and bm.refcount.sum() == 0
    with pytest.raises(AssertionError):
        bm._release(0)


def test_copy_on_write_only_when_shared():
    bm = bmod.BlockManager(16, 4)
    p = bm.new_sequence(6)           # tail block half full
    kids = [bm.fork(p) for _ in range(3)]
    tail = p.table[1]
    bm.free(p)
    for k in kids:
        bm.append_slot(k)
    pairs = bm.take_copies()
    # first two writers copy the shared tail; the last one owns it and writes in place
    assert pairs.shape == (2, 2)
    assert (pairs[:, 0] == kids[2].table[1]).all()
    assert kids[2].table[1] == tail
    assert len({k.table[1] for k in kids}) == 3
    assert all(bm.refcount[k.table[1]] == 1 for k in kids)
    assert bm.refcount[kids[0].table[0]] == 3       # full prefix block still shared


def test_tiny_workload_structure():
    wl = W.tiny()
    assert wl.num_seqs == 4 and wl.num_blocks == 64
    assert ((wl.context_lens >= 1) & (wl.context_lens <= 200)).all()
    B = wl.block_size
    for s in range(wl.num_seqs):
        n = int(wl.context_lens[s])
        assert wl.slot_mapping[s] == wl.block_tables[s, (n - 1) // B] * B + (n - 1) % B
        nb = -(-n // B)
        assert (wl.block_tables[s, nb:] == wl.poison_block).all()
    live = [int(b) for s in range(4) for b in wl.block_tables[s, :-(-int(wl.context_lens[s]) // B)]]
    assert len(live) == len(set(live)) and wl.poison_block not in live


def test_workloads_deterministic():
    a, b = W.llama7b(), W.llama7b()
    assert np.array_equal(a.block_tables, b.block_tables)
    assert np.array_equal(a.context_lens, b.context_lens)
    assert ((a.context_lens >= 512) & (a.context_lens <= 2048)).all()


def test_llama13b_lengths():
    wl = W.llama13b(block_size=32)
    assert wl.num_seqs == 256 and wl.num_heads == 40
    assert wl.context_lens.min() >= 16 and wl.context_lens.max() <= 4096
    assert 900 < np.median(wl.context_lens) < 1400


def test_cow_workload_copies_tails():
    wl = W.cow_beam4()
    assert wl.num_seqs == 128
    assert wl.copy_pairs.shape == (96, 2)         # beams 0..2 of each of 32 prompts
    assert len(set(wl.copy_pairs[:, 1].tolist())) == 96
    assert not set(wl.copy_pairs[:, 1].tolist()) & set(wl.copy_pairs[:, 0].tolist())
    plen = wl.extra["prompt_lens"]
    assert ((plen >= 2033) & (plen <= 2047)).all()
    # every beam shares its prompt's full blocks with its 3 siblings
    for i in range(32):
        rows = wl.block_tables[4 * i:4 * i + 4]
        full = int(plen[i]) // wl.block_size
        assert (rows[:, :full] == rows[0, :full]).all()
    assert wl.unique_kv_bytes() < 0.4 * wl.kv_bytes()
    assert wl.num_tokens == int(wl.extra["suffix_lens"].sum())


def test_cow_aligned_prompt_copies_nothing():
    wl = W.cow_beam4(aligned=True)
    assert wl.copy_pairs.shape == (0, 2)


def test_poison_covers_unfilled_and_unowned():
    wl = W.tiny()
    blocks, offs, whole = W.poison_slots(wl)
    assert wl.poison_block in whole.tolist()
    # each sequence: the appended slot is poisoned before the step
    for s in range(wl.num_seqs):
        slot = int(wl.slot_mapping[s])
        b, o = divmod(slot, wl.block_size)
        assert any((blocks == b) & (offs == o))


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
def test_quantised_values_stay_below_four(fmt):
    """The quantised pools' values (code value x per-head scale) stay below 4 in
    magnitude, the range in which bf16 rounding of an output stays inside the
    1e-2 bar; poisoned slots are the NaN code (fp8) or -128 (int8)."""
    import numpy as np
    import oracle
    wl = W.quantized(W.cow_beam4(num_prompts=2, prompt_len=120, max_suffix=20, num_heads=8,
                                 num_kv_heads=2, head_dim=128), fmt)
    vals = W.make_values(wl, "cpu", poison=False)
    for cache, scale in (("k_cache", "k_scale"), ("v_cache", "v_scale")):
        codes = W.to_numpy(vals[cache])
        v = oracle.code_values(codes, fmt)
        s = vals[scale].numpy().astype(np.float64)
        assert np.all(np.isfinite(v))
        assert float((np.abs(v) * s[None, :, None, None]).max()) < 4.0
    poisoned = W.to_numpy(W.make_values(wl, "cpu", poison=True)["k_cache"])
    bad = 0x7F if fmt == "fp8" else 0x80
    assert (poisoned.view(np.uint8) == bad).any()
