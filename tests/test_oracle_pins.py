"""Pins of the fp64 oracle against things other than itself.

Each test names what fixes the expected value: a hand-written golden fixture,
a library attention routine (torch's scaled_dot_product_attention in float64
on the logically ordered, contiguous K/V), an invariant the pages state, or a
closed form. Together they are chosen so that a plausible slip in the oracle
(a dropped scale, a wrong kv-head grouping, a swapped block / offset, a
transposed layout, an off-by-one context, a missing max shift, a wrong bf16
widening) fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_335_b200 import block_manager as bmod
from paged_kv_cache_335_b200 import workloads as W
from tests.conftest import read_golden


def _bits_bf16(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _paged_from_stream(K, V, ctx, block_size, num_blocks, rng, dtype):
    """Build a permuted paged pool from logical token streams K, V [S][Tmax][Hkv][d]
    (float64 holding representable values) through the oracle's append and a block
    manager; returns (k_cache, v_cache, tables)."""
    S, Tmax, Hkv, d = K.shape
    order = rng.permutation(num_blocks)
    bm = bmod.BlockManager(num_blocks, block_size, order=order)
    seqs, slots, toks = [], [], []
    for s in range(S):
        seq = bm.new_sequence(0)
        for t in range(int(ctx[s])):
            slots.append(bm.append_slot(seq))
            toks.append((s, t))
        seqs.append(seq)
    width = max(1, max(len(q.table) for q in seqs))
    tables = bm.tables_array(seqs, width, 0)
    conv = (lambda a: a.astype(np.float32)) if dtype == "f32" else \
        (lambda a: _bits_bf16(torch.from_numpy(a)))
    kc = np.zeros((num_blocks, Hkv, block_size, d), dtype=np.float32 if dtype == "f32" else np.uint16)
    vc = np.zeros_like(kc)
    if toks:
        kt = np.stack([K[s, t] for s, t in toks])
        vt = np.stack([V[s, t] for s, t in toks])
        oracle.kv_append(np.ascontiguousarray(conv(kt)), np.ascontiguousarray(conv(vt)),
                         np.asarray(slots, dtype=np.int64), kc, vc)
    return kc, vc, tables


def _sdpa_reference(q, K, V, ctx, scale, num_kv_heads):
    """torch float64 scaled_dot_product_attention on the contiguous context."""
    S, H, d = q.shape
    out = np.zeros((S, H, d))
    for s in range(S):
        n = int(ctx[s])
        if n == 0:
            continue
        qs = torch.from_numpy(q[s]).view(1, H, 1, d)
        ks = torch.from_numpy(np.ascontiguousarray(K[s, :n].transpose(1, 0, 2))).view(1, num_kv_heads, n, d)
        vs = torch.from_numpy(np.ascontiguousarray(V[s, :n].transpose(1, 0, 2))).view(1, num_kv_heads, n, d)
        o = torch.nn.functional.scaled_dot_product_attention(
            qs, ks, vs, scale=scale, enable_gqa=(H != num_kv_heads))
        out[s] = o.view(H, d).numpy()
    return out


def _random_case(seed, S, H, Hkv, d, B, max_ctx, dtype, num_blocks=None, qmul=1.0):
    rng = np.random.default_rng(seed)
    ctx = rng.integers(1, max_ctx + 1, size=S)
    Tmax = int(ctx.max())
    g = torch.Generator().manual_seed(seed)
    qf = torch.randn((S, H, d), generator=g, dtype=torch.float64) * qmul
    Kf = torch.randn((S, Tmax, Hkv, d), generator=g, dtype=torch.float64)
    Vf = torch.randn((S, Tmax, Hkv, d), generator=g, dtype=torch.float64)
    if dtype == "f32":
        q_store = qf.to(torch.float32).numpy()
        q_val = q_store.astype(np.float64)
        K = Kf.to(torch.float32).double().numpy()
        V = Vf.to(torch.float32).double().numpy()
    else:
        q_store = _bits_bf16(qf)
        q_val = qf.to(torch.bfloat16).double().numpy()
        K = Kf.to(torch.bfloat16).double().numpy()
        V = Vf.to(torch.bfloat16).double().numpy()
    demand = int(sum(-(-int(n) // B) for n in ctx))
    nb = num_blocks or demand + 5
    kc, vc, tables = _paged_from_stream(K, V, ctx, B, nb, rng, dtype)
    return dict(ctx=ctx.astype(np.int32), q_store=q_store, q_val=q_val, K=K, V=V,
                kc=kc, vc=vc, tables=tables)


# ---------------------------------------------------------------------------
# golden fixtures
# ---------------------------------------------------------------------------
def test_golden_append_layout():
    g = read_golden("append_layout.txt")
    nb, hkv, bs, d = (int(x) for x in g["shape"][0])
    slots = np.asarray([int(x) for x in g["slots"][0]], dtype=np.int64)
    T = slots.shape[0]
    k = np.zeros((T, hkv, d), dtype=np.float32)
    for i in range(T):
        for h in range(hkv):
            for j in range(d):
                k[i, h, j] = 100 * i + 10 * h + j + 1
    v = -k
    kc = np.zeros((nb, hkv, bs, d), dtype=np.float32)
    vc = np.zeros_like(kc)
    oracle.kv_append(k, v, slots, kc, vc)
    expect = np.asarray([float(x) for x in g["k"][0]], dtype=np.float32)
    np.testing.assert_array_equal(kc.reshape(-1), expect)
    np.testing.assert_array_equal(vc.reshape(-1), -expect)


def test_golden_block_copy():
    g = read_golden("block_copy.txt")
    nb, hkv, bs, d = (int(x) for x in g["shape"][0])
    pairs = np.asarray([int(x) for x in g["pairs"][0]], dtype=np.int64).reshape(-1, 2)
    before = np.asarray([float(x) for x in g["before"][0]], dtype=np.float32)
    after = np.asarray([float(x) for x in g["after"][0]], dtype=np.float32)
    kc = before.reshape(nb, hkv, bs, d).copy()
    vc = -kc
    oracle.block_copy(pairs, kc, vc)
    np.testing.assert_array_equal(kc.reshape(-1), after)
    np.testing.assert_array_equal(vc.reshape(-1), -after)


@pytest.mark.parametrize("ctx_len", [48, 40, 33])
def test_block_table_worked_example(ctx_len):
    """Logical blocks 0,1,2 in physical 17,4,29: decode through that table equals
    attention over the contiguous K/V (torch SDPA, float64)."""
    table = [int(x) for x in read_golden("block_table_17_4_29.txt")["table"][0]]
    B, d, Hkv, H, nb = 16, 8, 2, 2, 32
    g = torch.Generator().manual_seed(7)
    K = torch.randn((1, ctx_len, Hkv, d), generator=g).float().double().numpy()
    V = torch.randn((1, ctx_len, Hkv, d), generator=g).float().double().numpy()
    q = torch.randn((1, H, d), generator=g).float().numpy()
    kc = np.full((nb, Hkv, B, d), np.nan, dtype=np.float32)
    vc = np.full_like(kc, np.nan)
    slots = np.asarray([table[t // B] * B + t % B for t in range(ctx_len)], dtype=np.int64)
    oracle.kv_append(np.ascontiguousarray(K[0].astype(np.float32)),
                     np.ascontiguousarray(V[0].astype(np.float32)), slots, kc, vc)
    out = oracle.decode(q, kc, vc, np.asarray([table], dtype=np.int32),
                        np.asarray([ctx_len], dtype=np.int32), 0.25)
    ref = _sdpa_reference(q.astype(np.float64), K, V, [ctx_len], float(np.float32(0.25)), Hkv)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-13)


def test_golden_closed_form():
    g = read_golden("decode_closed_form.txt")
    qv, k0, k1, v0, v1, expect, tol = (float(x) for x in g["case"][0])
    kc = np.asarray([k0, k1], dtype=np.float32).reshape(1, 1, 2, 1)
    vc = np.asarray([v0, v1], dtype=np.float32).reshape(1, 1, 2, 1)
    q = np.asarray([qv], dtype=np.float32).reshape(1, 1, 1)
    out = oracle.decode(q, kc, vc, np.zeros((1, 1), np.int32), np.asarray([2], np.int32), 1.0)
    assert abs(out[0, 0, 0] - expect) <= tol
    vals = [float(x) for x in g["case3"][0]]
    qv, k0, k1, k2, a, b, c, expect, tol = vals
    kc = np.asarray([k0, k1, k2, 0], dtype=np.float32).reshape(1, 1, 4, 1)
    vc = np.asarray([a, b, c, 0], dtype=np.float32).reshape(1, 1, 4, 1)
    q = np.asarray([qv], dtype=np.float32).reshape(1, 1, 1)
    out = oracle.decode(q, kc, vc, np.zeros((1, 1), np.int32), np.asarray([3], np.int32), 1.0)
    assert abs(out[0, 0, 0] - expect) <= tol


# ---------------------------------------------------------------------------
# library routine: contiguous attention
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B", [1, 2, 16])
@pytest.mark.parametrize("H,Hkv", [(4, 4), (4, 2), (8, 2)])
def test_decode_equals_contiguous_sdpa(dtype, B, H, Hkv):
    c = _random_case(seed=100 + B + 10 * H + Hkv, S=4, H=H, Hkv=Hkv, d=16, B=B,
                     max_ctx=40, dtype=dtype)
    scale = float(np.float32(1 / 4))
    out = oracle.decode(c["q_store"], c["kc"], c["vc"], c["tables"], c["ctx"], scale)
    ref = _sdpa_reference(c["q_val"], c["K"], c["V"], c["ctx"], scale, Hkv)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_large_logits_stable():
    """Scores of order 1e3: exp without the max shift overflows; SDPA does not."""
    c = _random_case(seed=5, S=2, H=2, Hkv=2, d=16, B=4, max_ctx=30, dtype="f32", qmul=300.0)
    out = oracle.decode(c["q_store"], c["kc"], c["vc"], c["tables"], c["ctx"], 1.0)
    ref = _sdpa_reference(c["q_val"], c["K"], c["V"], c["ctx"], 1.0, 2)
    assert np.all(np.isfinite(out))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-9)


# ---------------------------------------------------------------------------
# invariants and closed forms
# ---------------------------------------------------------------------------
def test_placement_invariance_bitwise():
    """Two different physical placements of the same logical K/V: identical bits."""
    outs = []
    for perm_seed in (11, 12):
        rng = np.random.default_rng(3)
        ctx = rng.integers(1, 60, size=3)
        g = torch.Generator().manual_seed(3)
        K = torch.randn((3, 60, 2, 16), generator=g).float().double().numpy()
        V = torch.randn((3, 60, 2, 16), generator=g).float().double().numpy()
        q = torch.randn((3, 4, 16), generator=g).float().numpy()
        kc, vc, tables = _paged_from_stream(K, V, ctx, 8, 40, np.random.default_rng(perm_seed), "f32")
        outs.append((oracle.decode(q, kc, vc, tables, ctx.astype(np.int32), 0.3), tables))
    assert not np.array_equal(outs[0][1], outs[1][1]), "placements should differ"
    assert np.array_equal(outs[0][0], outs[1][0])


def test_prefix_sharing_bitwise():
    """Sequences sharing prefix blocks through reference counts decode exactly like
    sequences holding private copies of the same tokens."""
    B, Hkv, d, H = 4, 2, 8, 4
    g = torch.Generator().manual_seed(9)
    prefix = torch.randn((10, Hkv, d), generator=g).float().numpy()
    suffix = [torch.randn((n, Hkv, d), generator=g).float().numpy() for n in (3, 6)]
    q = torch.randn((2, H, d), generator=g).float().numpy()
    vscale = np.float32(-0.5)

    # shared: one prefix, two forks, copy-on-write of the partly filled tail
    bm = bmod.BlockManager(32, B, order=np.random.default_rng(1).permutation(32))
    kc = np.full((32, Hkv, B, d), np.nan, np.float32)
    vc = np.full_like(kc, np.nan)
    parent = bm.new_sequence(0)
    pslots = np.asarray([bm.append_slot(parent) for _ in range(10)], np.int64)
    oracle.kv_append(prefix, prefix * vscale, pslots, kc, vc)
    kids = [bm.fork(parent) for _ in range(2)]
    bm.free(parent)
    slots, ks = [], []
    for kid, suf in zip(kids, suffix):
        for t in range(suf.shape[0]):
            slots.append(bm.append_slot(kid))
            ks.append(suf[t])
    pairs = bm.take_copies()
    assert pairs.shape[0] == 1          # first fork copies the shared tail, second writes in place
    oracle.block_copy(pairs, kc, vc)
    kt = np.stack(ks)
    oracle.kv_append(kt, kt * vscale, np.asarray(slots, np.int64), kc, vc)
    tables = bm.tables_array(kids, 4, 0)
    ctx = np.asarray([13, 16], np.int32)
    shared_out = oracle.decode(q, kc, vc, tables, ctx, 0.35)
    assert len(set(tables[0, :2]) & set(tables[1, :2])) == 2   # prefix blocks really shared

    # private: each sequence written separately into its own blocks
    bm2 = bmod.BlockManager(32, B, order=np.random.default_rng(2).permutation(32))
    kc2 = np.full((32, Hkv, B, d), np.nan, np.float32)
    vc2 = np.full_like(kc2, np.nan)
    seqs = []
    for suf in suffix:
        s = bm2.new_sequence(0)
        toks = np.concatenate([prefix, suf])
        sl = np.asarray([bm2.append_slot(s) for _ in range(toks.shape[0])], np.int64)
        oracle.kv_append(np.ascontiguousarray(toks), np.ascontiguousarray(toks * vscale), sl, kc2, vc2)
        seqs.append(s)
    private_out = oracle.decode(q, kc2, vc2, bm2.tables_array(seqs, 4, 0), ctx, 0.35)
    assert np.array_equal(shared_out, private_out)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_ctx1_returns_v_exactly(dtype):
    c = _random_case(seed=21, S=4, H=4, Hkv=2, d=16, B=2, max_ctx=1, dtype=dtype)
    out = oracle.decode(c["q_store"], c["kc"], c["vc"], c["tables"], c["ctx"], 0.5)
    for s in range(4):
        for h in range(4):
            assert np.array_equal(out[s, h], c["V"][s, 0, h // 2])


def test_bf16_widening_known_bits():
    """ctx = 1 returns V exactly, so known bf16 bit patterns must come back as their values."""
    bits = np.asarray([0x3F80, 0xC000, 0x4049, 0x0001, 0x7F7F, 0xBF00, 0x0000, 0x3E80], np.uint16)
    expect = np.asarray([1.0, -2.0, 3.140625, 2.0 ** -133, 3.3895313892515355e38, -0.5, 0.0, 0.25])
    kc = np.zeros((1, 1, 16, 8), np.uint16)
    vc = np.zeros_like(kc)
    vc[0, 0, 0, :] = bits
    q = np.zeros((1, 1, 8), np.uint16)
    out = oracle.decode(q, kc, vc, np.zeros((1, 1), np.int32), np.asarray([1], np.int32), 1.0)
    np.testing.assert_array_equal(out[0, 0], expect)


def test_zero_query_gives_mean_of_v():
    c = _random_case(seed=31, S=3, H=2, Hkv=2, d=16, B=4, max_ctx=37, dtype="f32")
    q0 = np.zeros_like(c["q_store"])
    out = oracle.decode(q0, c["kc"], c["vc"], c["tables"], c["ctx"], 0.7)
    for s in range(3):
        n = int(c["ctx"][s])
        mean = c["V"][s, :n].mean(axis=0)            # [Hkv][d]
        np.testing.assert_allclose(out[s], mean, rtol=0, atol=1e-14)


def test_linear_in_v():
    """V1, V2 small integers (exact in float32): out(V1 + V2) = out(V1) + out(V2)."""
    rng = np.random.default_rng(41)
    ctx = np.asarray([5, 17, 33], np.int32)
    nb, B, Hkv, d = 40, 4, 2, 8
    kc = rng.standard_normal((nb, Hkv, B, d)).astype(np.float32)
    v1 = rng.integers(-8, 9, size=(nb, Hkv, B, d)).astype(np.float32)
    v2 = rng.integers(-8, 9, size=(nb, Hkv, B, d)).astype(np.float32)
    tables = rng.permutation(nb)[:27].reshape(3, 9).astype(np.int32)
    q = rng.standard_normal((3, 2, d)).astype(np.float32)
    o1 = oracle.decode(q, kc, v1, tables, ctx, 0.4)
    o2 = oracle.decode(q, kc, v2, tables, ctx, 0.4)
    o12 = oracle.decode(q, kc, v1 + v2, tables, ctx, 0.4)
    np.testing.assert_allclose(o12, o1 + o2, rtol=0, atol=1e-12)
    o3 = oracle.decode(q, kc, 2 * v1, tables, ctx, 0.4)
    assert np.array_equal(o3, 2 * o1)


def test_ctx0_gives_zeros():
    kc = np.full((2, 1, 16, 8), np.nan, np.float32)
    out = oracle.decode(np.ones((2, 1, 8), np.float32), kc, kc.copy(),
                        np.zeros((2, 1), np.int32), np.asarray([0, 0], np.int32), 1.0)
    assert np.array_equal(out, np.zeros_like(out))


def test_scale_is_applied():
    """scale 0 makes every weight equal: out = mean(V), unlike scale 1."""
    c = _random_case(seed=51, S=2, H=2, Hkv=2, d=16, B=4, max_ctx=20, dtype="f32")
    out0 = oracle.decode(c["q_store"], c["kc"], c["vc"], c["tables"], c["ctx"], 0.0)
    for s in range(2):
        n = int(c["ctx"][s])
        np.testing.assert_allclose(out0[s], c["V"][s, :n].mean(axis=0), rtol=0, atol=1e-14)


def test_threads_do_not_change_bits():
    c = _random_case(seed=61, S=4, H=8, Hkv=2, d=16, B=16, max_ctx=40, dtype="bf16")
    o1 = oracle.decode(c["q_store"], c["kc"], c["vc"], c["tables"], c["ctx"], 0.25, num_threads=1)
    o8 = oracle.decode(c["q_store"], c["kc"], c["vc"], c["tables"], c["ctx"], 0.25, num_threads=8)
    assert np.array_equal(o1, o8)


def test_rejects_block_outside_pool():
    kc = np.zeros((4, 1, 2, 4), np.float32)
    with pytest.raises(oracle.OracleError):
        oracle.decode(np.zeros((1, 1, 4), np.float32), kc, kc.copy(),
                      np.asarray([[0, 9]], np.int32), np.asarray([3], np.int32), 1.0)
    with pytest.raises(oracle.OracleError):
        oracle.kv_append(np.zeros((1, 1, 4), np.float32), np.zeros((1, 1, 4), np.float32),
                         np.asarray([8], np.int64), kc, kc.copy())


# ---------------------------------------------------------------------------
# the seeded workloads feed the oracle consistently
# ---------------------------------------------------------------------------
def test_tiny_workload_step_matches_sdpa():
    """The tiny configuration end to end on the oracle (append, then decode) equals
    SDPA on the logical token streams rebuilt from the pool."""
    wl = W.tiny()
    vals = W.make_values(wl, "cpu", poison=True)
    kc = W.to_numpy(vals["k_cache"]).copy()
    vc = W.to_numpy(vals["v_cache"]).copy()
    oracle.kv_append(W.to_numpy(vals["k_new"]), W.to_numpy(vals["v_new"]), wl.slot_mapping, kc, vc)
    out = oracle.decode(W.to_numpy(vals["q"]), kc, vc, wl.block_tables, wl.context_lens, wl.scale)
    assert np.all(np.isfinite(out))
    # rebuild logical streams by walking tables in the test (independent of the oracle)
    S, B = wl.num_seqs, wl.block_size
    Tmax = wl.max_context_len
    K = np.zeros((S, Tmax, wl.num_kv_heads, wl.head_dim))
    V = np.zeros_like(K)
    for s in range(S):
        for t in range(int(wl.context_lens[s])):
            b = wl.block_tables[s, t // B]
            K[s, t] = kc[b, :, t % B, :]
            V[s, t] = vc[b, :, t % B, :]
    ref = _sdpa_reference(W.to_numpy(vals["q"]).astype(np.float64), K, V, wl.context_lens,
                          wl.scale, wl.num_kv_heads)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# swap between pools
# ---------------------------------------------------------------------------
def test_block_swap_equals_indexed_assignment():
    """Swap out / in against numpy's own indexed assignment (a library routine)."""
    rng = np.random.default_rng(7)
    dev_k = rng.standard_normal((11, 3, 16, 8)).astype(np.float32)
    dev_v = rng.standard_normal((11, 3, 16, 8)).astype(np.float32)
    host_k = np.full((6, 3, 16, 8), np.nan, np.float32)
    host_v = np.full((6, 3, 16, 8), np.nan, np.float32)
    pairs = np.array([[9, 0], [2, 5], [4, 3]], np.int64)
    want_k, want_v = host_k.copy(), host_v.copy()
    want_k[pairs[:, 1]] = dev_k[pairs[:, 0]]
    want_v[pairs[:, 1]] = dev_v[pairs[:, 0]]
    oracle.block_swap(pairs, dev_k, dev_v, host_k, host_v)
    assert want_k.view(np.uint32).tobytes() == host_k.view(np.uint32).tobytes()
    assert want_v.view(np.uint32).tobytes() == host_v.view(np.uint32).tobytes()
    # round trip into fresh device blocks restores every bit
    back = np.array([[0, 1], [5, 6], [3, 10]], np.int64)
    k2, v2 = dev_k.copy(), dev_v.copy()
    oracle.block_swap(back, host_k, host_v, k2, v2)
    for (s, _), (_, d) in zip(pairs, back):
        assert k2[d].tobytes() == dev_k[s].tobytes() and v2[d].tobytes() == dev_v[s].tobytes()


def test_block_swap_rejects_bad_ids_and_shapes():
    a = np.zeros((4, 2, 16, 8), np.float32)
    b = np.zeros((2, 2, 16, 8), np.float32)
    with pytest.raises(oracle.OracleError):
        oracle.block_swap(np.array([[3, 2]]), a, a.copy(), b, b.copy())     # dst 2 of 2
    with pytest.raises(ValueError):
        oracle.block_swap(np.array([[0, 0]]), a, a.copy(), np.zeros((2, 2, 16, 4), np.float32),
                          np.zeros((2, 2, 16, 4), np.float32))


# ---------------------------------------------------------------------------
# multi-token queries (chunked prefill / draft verification)
# ---------------------------------------------------------------------------
def _sdpa_multi_reference(q_rows, K, V, ctx, nq, scale, num_kv_heads):
    """torch float64 SDPA per sequence with an explicit bottom-right causal mask:
    query j of n sees keys 0 .. ctx - n + j (a library routine on the contiguous
    context, independent of the oracle's own code)."""
    out = np.zeros_like(q_rows)
    row = 0
    H, d = q_rows.shape[1], q_rows.shape[2]
    for s in range(len(ctx)):
        n, c = int(nq[s]), int(ctx[s])
        if n == 0:
            continue
        qs = torch.from_numpy(np.ascontiguousarray(q_rows[row:row + n].transpose(1, 0, 2))).view(1, H, n, d)
        ks = torch.from_numpy(np.ascontiguousarray(K[s, :c].transpose(1, 0, 2))).view(1, num_kv_heads, c, d)
        vs = torch.from_numpy(np.ascontiguousarray(V[s, :c].transpose(1, 0, 2))).view(1, num_kv_heads, c, d)
        mask = torch.arange(c).view(1, c) <= (c - n + torch.arange(n)).view(n, 1)
        o = torch.nn.functional.scaled_dot_product_attention(
            qs, ks, vs, attn_mask=mask, scale=scale, enable_gqa=(H != num_kv_heads))
        out[row:row + n] = o.view(H, n, d).permute(1, 0, 2).numpy()
        row += n
    return out


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,H,Hkv", [(1, 4, 4), (16, 8, 2), (2, 4, 1)])
def test_decode_multi_equals_masked_sdpa(dtype, B, H, Hkv):
    c = _random_case(seed=300 + B + H, S=4, H=H, Hkv=Hkv, d=16, B=B, max_ctx=40, dtype=dtype)
    nq = np.minimum(np.array([1, 5, 0, 12]), c["ctx"])
    nq[3] = c["ctx"][3]                       # a whole prompt as one chunk (full causal prefill)
    qs = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    g = torch.Generator().manual_seed(9)
    qf = torch.randn((int(qs[-1]), H, 16), generator=g, dtype=torch.float64)
    if dtype == "f32":
        q_store = qf.to(torch.float32).numpy()
        q_val = q_store.astype(np.float64)
    else:
        q_store = _bits_bf16(qf)
        q_val = qf.to(torch.bfloat16).double().numpy()
    scale = float(np.float32(1 / 4))
    out = oracle.decode_multi(q_store, c["kc"], c["vc"], c["tables"], c["ctx"], qs, scale)
    ref = _sdpa_multi_reference(q_val, c["K"], c["V"], c["ctx"], nq, scale, Hkv)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_decode_multi_rejects_more_queries_than_context():
    kc = np.zeros((2, 1, 4, 4), np.float32)
    with pytest.raises(oracle.OracleError):
        oracle.decode_multi(np.zeros((3, 1, 4), np.float32), kc, kc.copy(),
                            np.zeros((1, 1), np.int32), np.array([2], np.int32),
                            np.array([0, 3], np.int32), 1.0)


# ---------------------------------------------------------------------------
# quantised KV cache: FP8 E4M3 / int8 codes with per-kv-head scales
# ---------------------------------------------------------------------------
def test_e4m3_values_match_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    mine = oracle.code_values(codes, "fp8")
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(mine), np.isnan(lib))
    assert np.array_equal(mine[~np.isnan(mine)], lib[~np.isnan(lib)])
    assert mine[0x7E] == 448.0 and mine[0x01] == 2.0 ** -9 and mine[0x38] == 1.0 and mine[0xB8] == -1.0


def test_e4m3_encoding_matches_torch_round_to_nearest_even():
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(20000) * 40, rng.standard_normal(5000) * 0.01,
        oracle.code_values(np.arange(0x7F, dtype=np.uint8), "fp8"),            # exact codes
        (oracle.code_values(np.arange(0x7E, dtype=np.uint8), "fp8") +
         oracle.code_values(np.arange(1, 0x7F, dtype=np.uint8), "fp8")) / 2,   # exact ties
    ]).astype(np.float32)
    vals = np.concatenate([vals, -vals])
    vals = vals[np.abs(vals) < 448]
    mine = oracle.quantize(vals, 1.0, "fp8")
    lib = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(mine, lib)


def test_e4m3_saturation_nan_and_scale():
    x = np.array([448, 449, 1e30, np.inf, -np.inf, np.nan, -0.0, 2.0 ** -10, 3 * 2.0 ** -10],
                 np.float32)
    assert [int(c) for c in oracle.quantize(x, 1.0, "fp8")] == \
        [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x7F, 0x80, 0x00, 0x02]
    # the code is that of x / scale, divided in binary32
    assert int(oracle.quantize(np.array([3.0], np.float32), 2.0, "fp8")[0]) == 0x3C   # 1.5


def test_int8_codes():
    x = np.array([2.5, 3.5, -2.5, -3.5, 126.6, 127.4, 200, -1e9, np.inf, -np.inf, np.nan, -0.4],
                 np.float32)
    assert oracle.quantize(x, 1.0, "int8").view(np.int8).tolist() == \
        [2, 4, -2, -4, 127, 127, 127, -127, 127, -127, -127, 0]
    rng = np.random.default_rng(2)
    y = (rng.standard_normal(50000) * 60).astype(np.float32)
    s = np.float32(0.37)
    lib = np.clip(np.rint(y / s), -127, 127).astype(np.int8)         # numpy: IEEE binary32 divide
    assert np.array_equal(oracle.quantize(y, float(s), "int8").view(np.int8), lib)


def test_quantisation_error_bounds():
    rng = np.random.default_rng(3)
    s = 0.05
    x = (rng.uniform(-1, 1, 40000) * 127 * s).astype(np.float32)
    deq = oracle.code_values(oracle.quantize(x, s, "int8"), "int8") * np.float32(s)
    assert np.max(np.abs(deq - x)) <= s / 2 * (1 + 1e-6)
    xf = (rng.uniform(2.0 ** -6, 440, 40000) * rng.choice([-1, 1], 40000)).astype(np.float32)
    deqf = oracle.code_values(oracle.quantize(xf, 1.0, "fp8"), "fp8")
    assert np.max(np.abs(deqf - xf) / np.abs(xf)) <= 2.0 ** -4


def test_quant_append_places_codes():
    """Codes land in (slot / B, head, slot % B): numpy placement of torch / numpy
    quantised values."""
    rng = np.random.default_rng(4)
    T, Hkv, B, d, NB = 6, 3, 4, 8, 5
    k = torch.randn((T, Hkv, d), generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    v = torch.randn((T, Hkv, d), generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    ks = np.array([0.01, 0.02, 0.5], np.float32)
    vs = np.array([0.03, 0.04, 0.25], np.float32)
    slots = np.array([19, 0, -1, 7, 12, 3], np.int64)
    for fmt in ("fp8", "int8"):
        kc = np.zeros((NB, Hkv, B, d), np.uint8)
        vc = np.zeros_like(kc)
        oracle.kv_append_quant(_bits_bf16(k), _bits_bf16(v), slots, kc, vc, ks, vs, fmt)
        want_k, want_v = np.zeros_like(kc), np.zeros_like(vc)
        for t, sl in enumerate(slots):
            if sl < 0:
                continue
            for h in range(Hkv):
                for src, sc, dst in ((k, ks, want_k), (v, vs, want_v)):
                    y = src[t, h].float().numpy() / sc[h]
                    if fmt == "int8":
                        code = np.clip(np.rint(y), -127, 127).astype(np.int8).view(np.uint8)
                    else:
                        code = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
                    dst[sl // B, h, sl % B] = code
        assert np.array_equal(kc, want_k) and np.array_equal(vc, want_v), fmt


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
@pytest.mark.parametrize("B,H,Hkv", [(16, 8, 2), (2, 4, 4)])
def test_decode_quant_equals_sdpa_on_dequantised_values(fmt, B, H, Hkv):
    """Decode over codes = contiguous SDPA over value(code) * scale, the values
    taken through torch's float8 type (fp8) or plain integers (int8)."""
    rng = np.random.default_rng(5 + B + H)
    S, d, NB = 3, 16, 40
    ctx = np.array([1, 37, 20], np.int32)
    ks = rng.uniform(0.005, 0.05, Hkv).astype(np.float32)
    vs = rng.uniform(0.005, 0.05, Hkv).astype(np.float32)
    kc = rng.integers(0, 256, (NB, Hkv, B, d), dtype=np.uint8)
    vc = rng.integers(0, 256, (NB, Hkv, B, d), dtype=np.uint8)
    if fmt == "fp8":                                # no NaN codes
        kc[(kc & 0x7F) == 0x7F] = 0x7E
        vc[(vc & 0x7F) == 0x7F] = 0x7E
    perm = rng.permutation(NB)
    tables = np.zeros((S, -(-int(ctx.max()) // B)), np.int32)
    used = 0
    for s in range(S):
        nb = -(-int(ctx[s]) // B)
        tables[s, :nb] = perm[used:used + nb]
        used += nb
    qf = torch.randn((S, H, d), generator=torch.Generator().manual_seed(7))
    q_bits = _bits_bf16(qf)
    q_val = qf.to(torch.bfloat16).double().numpy()
    if fmt == "fp8":
        kval = torch.from_numpy(kc).view(torch.float8_e4m3fn).double().numpy()
        vval = torch.from_numpy(vc).view(torch.float8_e4m3fn).double().numpy()
    else:
        kval = kc.view(np.int8).astype(np.float64)
        vval = vc.view(np.int8).astype(np.float64)
    kval = kval * ks.astype(np.float64)[None, :, None, None]
    vval = vval * vs.astype(np.float64)[None, :, None, None]
    Tm = int(ctx.max())
    K = np.zeros((S, Tm, Hkv, d))
    V = np.zeros((S, Tm, Hkv, d))
    for s in range(S):
        for t in range(int(ctx[s])):
            K[s, t] = kval[tables[s, t // B], :, t % B]
            V[s, t] = vval[tables[s, t // B], :, t % B]
    scale = float(np.float32(0.25))
    out = oracle.decode_quant(q_bits, kc, vc, ks, vs, tables, ctx, scale, fmt)
    ref = _sdpa_reference(q_val, K, V, ctx, scale, Hkv)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
