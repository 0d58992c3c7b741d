"""Seeded synthetic decode workloads shared by the tests, the smoke check and
the bench. Input construction only: it holds no attention arithmetic, and both
the CUDA path and the CPU oracle consume exactly the bits it produces.

Shapes follow the pages' workloads (LLaMA-shaped head counts, prompts around
1024 tokens, contexts up to 32K, beam width 4 sharing a prompt):

* "PagedAttention：大模型推理性能优化的核心技术解析", § 实际性能对比与量化数据:
  LLaMA-2-13B, prompt 1024, 256 generated tokens.
* "PagedAttention原理详解：GPU显存优化与模型路由技术", § 显存消耗的三大来源
  (70B-shaped heads) and § PagedAttention的三大核心优势 (beam_width = 4 sharing).
* "vLLM的Paged Attention技术：高效注意力机制解析", § 3.1 (HEAD_SIZE 128,
  BLOCK_SIZE 16/32).

Structure (context lengths, the shuffled pool, block tables, slots, copy
pairs) is drawn on the host with ``numpy.random.default_rng(seed)``. Values
(q, new k/v, both pools) are N(0, 1) drawn with a seeded ``torch.Generator`` on
the device that will hold them; a test that needs them on the host copies them.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

from .block_manager import BlockManager

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass
class Workload:
    name: str
    dtype: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    scale: float
    seed: int
    context_lens: np.ndarray          # int32 [S], includes this step's appended tokens
    history_lens: np.ndarray          # int32 [S], tokens already in the cache before the step
    block_tables: np.ndarray          # int32 [S][MB]; padding entries = poison_block
    slot_mapping: np.ndarray          # int64 [T], this step's appended tokens
    token_seq: np.ndarray             # int32 [T], sequence of each appended token
    copy_pairs: np.ndarray            # int64 [P][2], this step's copy-on-write pairs
    poison_block: int
    partition_size: int = 0           # 0 = library policy
    description: str = ""
    extra: dict = field(default_factory=dict)
    # multi-token queries: int32 [S + 1]; sequence s owns q rows query_start[s] ..
    # query_start[s+1]-1, its last n_s context positions (None: one query per sequence)
    query_start: np.ndarray | None = None
    # quantised caches: "fp8" (E4M3 codes) or "int8" codes with per-kv-head scales;
    # q, new k / v and out stay in `dtype` (bf16)
    kv_quant: str | None = None

    @property
    def torch_dtype(self):
        return DTYPES[self.dtype]

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def kv_elem_bytes(self) -> int:
        """Bytes per cached element: 1 for a quantised cache."""
        return 1 if self.kv_quant else self.elem_bytes

    @property
    def num_tokens(self) -> int:
        return int(self.slot_mapping.shape[0])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    def kv_bytes(self) -> int:
        """Logical K+V bytes one decode call reads: every context token, K and V."""
        return int(self.context_lens.astype(np.int64).sum()) * self.num_kv_heads * \
            self.head_dim * 2 * self.kv_elem_bytes

    @property
    def num_query_rows(self) -> int:
        """Rows of q / out: one per sequence, or every query token."""
        return self.num_seqs if self.query_start is None else int(self.query_start[-1])

    @property
    def max_query_len(self) -> int:
        return 1 if self.query_start is None else int(np.diff(self.query_start).max(initial=1))

    def decode_bytes(self) -> int:
        """Algorithmic bytes of one decode call: K/V of every context token (once
        per sequence, whatever its query count) + q + out."""
        qo = 2 * self.num_query_rows * self.num_heads * self.head_dim * self.elem_bytes
        return self.kv_bytes() + qo

    def append_bytes(self) -> int:
        """Bytes one append call moves: new k, v read and written once each."""
        return 2 * self.num_tokens * self.num_kv_heads * self.head_dim * \
            (self.elem_bytes + self.kv_elem_bytes)

    def copy_bytes(self) -> int:
        """Bytes one block-copy call moves: K and V block read + written per pair."""
        blk = self.num_kv_heads * self.block_size * self.head_dim * self.kv_elem_bytes
        return 2 * 2 * int(self.copy_pairs.shape[0]) * blk

    def unique_kv_bytes(self) -> int:
        """K+V bytes of distinct (block, filled slot) pairs the decode reads."""
        seen = {}
        for s in range(self.num_seqs):
            n = int(self.context_lens[s])
            nb = -(-n // self.block_size)
            for j in range(nb):
                b = int(self.block_tables[s, j])
                fill = min(self.block_size, n - j * self.block_size)
                seen[b] = max(seen.get(b, 0), fill)
        toks = sum(seen.values())
        return toks * self.num_kv_heads * self.head_dim * 2 * self.kv_elem_bytes


# ---------------------------------------------------------------------------
# structure
# ---------------------------------------------------------------------------
def _decode_structure(name, dtype, ctx, num_heads, num_kv_heads, head_dim, block_size,
                      num_blocks, scale, seed, rng, partition_size=0, description="",
                      new_tokens=None):
    """Sequences of the given final context lengths, each holding ctx - n tokens
    before the step and appending n in it (positions ctx-n .. ctx-1); n = 1
    unless ``new_tokens`` gives one count per sequence (multi-token queries)."""
    ctx = np.asarray(ctx, dtype=np.int64)
    s_count = ctx.shape[0]
    news = np.ones(s_count, np.int64) if new_tokens is None else np.asarray(new_tokens, np.int64)
    news = np.minimum(news, ctx)
    order = rng.permutation(num_blocks)
    poison = int(order[-1])                      # a valid id that no sequence owns
    bm = BlockManager(num_blocks, block_size, order=order, reserved=(poison,))
    seqs, slots, token_seq = [], [], []
    for s in range(s_count):
        n = int(ctx[s])
        seq = bm.new_sequence(n - int(news[s]))
        for _ in range(int(news[s])):
            slots.append(bm.append_slot(seq))
            token_seq.append(s)
        seqs.append(seq)
    width = max(1, max(len(q.table) for q in seqs) if seqs else 1)
    tables = bm.tables_array(seqs, width, poison)
    return Workload(
        name=name, dtype=dtype, num_seqs=s_count, num_heads=num_heads,
        num_kv_heads=num_kv_heads, head_dim=head_dim, block_size=block_size,
        num_blocks=num_blocks, scale=float(np.float32(scale)), seed=seed,
        context_lens=ctx.astype(np.int32), history_lens=(ctx - news).astype(np.int32),
        block_tables=tables, slot_mapping=np.asarray(slots, dtype=np.int64),
        token_seq=np.asarray(token_seq, dtype=np.int32),
        copy_pairs=np.zeros((0, 2), dtype=np.int64), poison_block=poison,
        partition_size=partition_size, description=description,
        query_start=None if new_tokens is None else
        np.concatenate([[0], np.cumsum(news)]).astype(np.int32))


def _pool_size(ctx, block_size, factor=1.2):
    demand = int(sum(-(-int(n) // block_size) for n in ctx))
    return int(math.ceil(factor * demand)) + 1


def tiny(seed: int = 0) -> Workload:
    """4 seqs, 4 heads = 4 kv heads, d 64, bs 16, fp32, ctx U[1,200], 64-block
    permuted pool, scale 1/8."""
    rng = np.random.default_rng(seed)
    ctx = rng.integers(1, 201, size=4)
    return _decode_structure("tiny", "f32", ctx, 4, 4, 64, 16, 64, 0.125, seed, rng,
                             description="4 seqs, 4/4 heads, d64, bs16, fp32, ctx U[1,200]")


def llama7b(seed: int = 1, block_size: int = 16) -> Workload:
    """LLaMA-7B-shaped layer: 64 seqs, 32 heads = 32 kv heads, d 128, bf16,
    ctx U[512,2048] (including the token appended this step), pool 1.2x demand."""
    rng = np.random.default_rng(seed)
    ctx = rng.integers(512, 2049, size=64)
    nb = _pool_size(ctx, block_size)
    return _decode_structure("llama7b", "bf16", ctx, 32, 32, 128, block_size, nb,
                             1.0 / math.sqrt(128), seed, rng,
                             description="64 seqs, 32/32 heads, d128, bs16, bf16, ctx U[512,2048]")


def llama13b(seed: int = 2, block_size: int = 16, sigma: float = 0.5) -> Workload:
    """LLaMA-13B-shaped layer: 256 seqs, 40 heads = 40 kv heads, d 128, bf16,
    ctx = clip(round(LogNormal(ln 1152, sigma)), 16, 4096): median = prompt 1024
    + 128 generated. sigma is not given by the pages; 0.5 is this build's reading."""
    rng = np.random.default_rng(seed)
    ctx = np.clip(np.rint(rng.lognormal(math.log(1152.0), sigma, size=256)), 16, 4096)
    ctx = ctx.astype(np.int64)
    nb = _pool_size(ctx, block_size)
    return _decode_structure(f"llama13b_bs{block_size}", "bf16", ctx, 40, 40, 128, block_size,
                             nb, 1.0 / math.sqrt(128), seed, rng,
                             description=f"256 seqs, 40/40 heads, d128, bs{block_size}, bf16, "
                                         "ctx lognormal(median 1152, sigma 0.5) in [16,4096]")


def llama70b_gqa(seed: int = 3, num_seqs: int = 8, context_len: int = 32768) -> Workload:
    """70B-GQA long context: 8 seqs, 64 q heads / 8 kv heads, d 128, bs 16, bf16,
    ctx 32768 each, split into partitions of 512 tokens."""
    rng = np.random.default_rng(seed)
    ctx = np.full(num_seqs, context_len, dtype=np.int64)
    nb = _pool_size(ctx, 16)
    return _decode_structure("llama70b_gqa", "bf16", ctx, 64, 8, 128, 16, nb,
                             1.0 / math.sqrt(128), seed, rng, partition_size=512,
                             description=f"{num_seqs} seqs, 64/8 heads, d128, bs16, bf16, "
                                         f"ctx {context_len}, partitions of 512")


def cow_beam4(seed: int = 4, num_prompts: int = 32, beam_width: int = 4,
              prompt_len: int = 2048, aligned: bool = False, max_suffix: int = 256,
              num_heads: int = 64, num_kv_heads: int = 8, head_dim: int = 128,
              block_size: int = 16, dtype: str = "bf16") -> Workload:
    """Copy-on-write parallel sampling: each prompt is prefilled once and shared
    by ``beam_width`` beams through reference counts; in this step every beam
    appends its own suffix of U[1, max_suffix] tokens. The first suffix token of
    a beam falls into the prompt's partly filled tail block, which is still
    shared, so beams 0..W-2 get a private copy (a ``pa_block_copy`` pair) and the
    last beam, then the tail's only owner, writes in place.

    A 2048-token prompt fills its last block exactly at block_size 16, leaving
    nothing to copy; the reading used here shortens each prompt by U{1..15}
    tokens (``aligned=False``). ``aligned=True`` keeps prompt_len exactly and
    must give zero copies."""
    rng = np.random.default_rng(seed)
    if aligned:
        plen = np.full(num_prompts, prompt_len, dtype=np.int64)
    else:
        plen = prompt_len - rng.integers(1, block_size, size=num_prompts)
    suffix = rng.integers(1, max_suffix + 1, size=num_prompts * beam_width)
    demand = sum(-(-int(p) // block_size) for p in plen)
    for i in range(num_prompts):
        for b in range(beam_width):
            total = int(plen[i] + suffix[i * beam_width + b])
            demand += -(-total // block_size) - int(plen[i]) // block_size
    nb = int(math.ceil(1.2 * demand)) + 1
    order = rng.permutation(nb)
    poison = int(order[-1])
    bm = BlockManager(nb, block_size, order=order, reserved=(poison,))
    seqs, hist, ctx, slots, token_seq = [], [], [], [], []
    for i in range(num_prompts):
        prompt = bm.new_sequence(int(plen[i]))
        beams = [bm.fork(prompt) for _ in range(beam_width)]
        bm.free(prompt)                       # the prompt itself is no longer a sequence
        for b, beam in enumerate(beams):
            s = len(seqs)
            n_new = int(suffix[i * beam_width + b])
            hist.append(beam.length)
            for _ in range(n_new):
                slots.append(bm.append_slot(beam))
                token_seq.append(s)
            ctx.append(beam.length)
            seqs.append(beam)
    pairs = bm.take_copies()
    width = max(len(s.table) for s in seqs)
    tables = bm.tables_array(seqs, width, poison)
    name = "cow_beam4_aligned" if aligned else "cow_beam4"
    return Workload(
        name=name, dtype=dtype, num_seqs=len(seqs), num_heads=num_heads,
        num_kv_heads=num_kv_heads, head_dim=head_dim, block_size=block_size, num_blocks=nb,
        scale=float(np.float32(1.0 / math.sqrt(head_dim))), seed=seed,
        context_lens=np.asarray(ctx, dtype=np.int32), history_lens=np.asarray(hist, np.int32),
        block_tables=tables, slot_mapping=np.asarray(slots, dtype=np.int64),
        token_seq=np.asarray(token_seq, dtype=np.int32), copy_pairs=pairs, poison_block=poison,
        description=f"{num_prompts} prompts x beam {beam_width}, prompt ~{prompt_len} shared, "
                    f"suffix U[1,{max_suffix}], {num_heads}/{num_kv_heads} heads, d{head_dim}, "
                    f"bs{block_size}, {dtype}",
        extra={"prompt_lens": plen.astype(np.int32), "suffix_lens": suffix.astype(np.int32),
               "beam_width": beam_width, "refcount": bm.refcount.copy()})


def decode_case(num_seqs, num_heads, num_kv_heads, head_dim, block_size, dtype, context_lens,
                seed=0, pool_factor=1.3, partition_size=0, name=None) -> Workload:
    """A decode workload with the given final context lengths, built like the
    named configurations (shuffled pool, one appended token per sequence)."""
    rng = np.random.default_rng(seed)
    ctx = np.asarray(context_lens, dtype=np.int64)
    assert ctx.shape == (num_seqs,)
    demand = int(sum(-(-int(n) // block_size) for n in ctx))
    nb = int(math.ceil(pool_factor * max(demand, 1))) + 2
    name = name or f"case_{num_seqs}x{num_heads}/{num_kv_heads}_d{head_dim}_bs{block_size}_{dtype}"
    return _decode_structure(name, dtype, ctx, num_heads, num_kv_heads, head_dim, block_size, nb,
                             1.0 / math.sqrt(head_dim), seed, rng, partition_size=partition_size)


def multi_query_case(num_seqs, num_heads, num_kv_heads, head_dim, block_size, dtype,
                     context_lens, query_lens, seed=0, pool_factor=1.3, partition_size=0,
                     name=None) -> Workload:
    """Multi-token queries: sequence s appends query_lens[s] tokens this step
    (its last positions) and each of them attends causally over the cache, as
    in chunked prefill or the verification of draft tokens."""
    rng = np.random.default_rng(seed)
    ctx = np.asarray(context_lens, dtype=np.int64)
    demand = int(sum(-(-int(n) // block_size) for n in ctx))
    nb = int(math.ceil(pool_factor * max(demand, 1))) + 2
    name = name or (f"multi_{num_seqs}x{num_heads}/{num_kv_heads}_d{head_dim}_bs{block_size}_"
                    f"{dtype}")
    return _decode_structure(name, dtype, ctx, num_heads, num_kv_heads, head_dim, block_size, nb,
                             1.0 / math.sqrt(head_dim), seed, rng, partition_size=partition_size,
                             new_tokens=query_lens)


def llama70b_verify(seed: int = 6, num_seqs: int = 8, context_len: int = 32768,
                    draft: int = 4) -> Workload:
    """Speculative verification on the 70B-shaped layer: 8 sequences of 32K
    context each check ``draft`` new tokens in one pass (64/8 heads, d128, bf16)."""
    wl = multi_query_case(num_seqs, 64, 8, 128, 16, "bf16", [context_len] * num_seqs,
                          [draft] * num_seqs, seed=seed, pool_factor=1.05,
                          name=f"llama70b_verify{draft}")
    wl.description = (f"{num_seqs} seqs x {context_len} ctx, {draft} query tokens each "
                      "(verification), 64/8 heads, d128, bs16, bf16")
    return wl


CONFIGS = {
    "tiny": tiny,
    "llama7b": llama7b,
    "llama13b_bs16": lambda seed=2: llama13b(seed, 16),
    "llama13b_bs32": lambda seed=2: llama13b(seed, 32),
    "llama70b_gqa": llama70b_gqa,
    "cow_beam4": cow_beam4,
    "llama70b_verify4": llama70b_verify,
}


def restrict(wl: Workload, seq_ids) -> Workload:
    """The same step for a subset of sequences on a compact pool: their blocks
    (and the sources of their copy pairs) renumbered 0..n-1 in first-use order,
    plus one fresh poison block. Used to size bounded CPU samples."""
    seq_ids = sorted({int(s) for s in seq_ids})
    B = wl.block_size
    remap = {}

    def new_id(b):
        b = int(b)
        if b not in remap:
            remap[b] = len(remap)
        return remap[b]

    nbs = [-(-int(wl.context_lens[s]) // B) for s in seq_ids]
    for s, nb in zip(seq_ids, nbs):
        for j in range(nb):
            new_id(wl.block_tables[s, j])
    dsts = set(remap)
    pairs = [(new_id(a), remap[int(b)]) for a, b in wl.copy_pairs.tolist() if int(b) in dsts]
    poison = len(remap)
    width = max([1] + nbs)
    tables = np.full((len(seq_ids), width), poison, dtype=np.int32)
    for i, (s, nb) in enumerate(zip(seq_ids, nbs)):
        tables[i, :nb] = [remap[int(b)] for b in wl.block_tables[s, :nb]]
    pos = {s: i for i, s in enumerate(seq_ids)}
    keep = [t for t, s in enumerate(wl.token_seq.tolist()) if s in pos]
    slots = [remap[int(wl.slot_mapping[t]) // B] * B + int(wl.slot_mapping[t]) % B for t in keep]
    sub = Workload(**{**wl.__dict__})
    sub.name = f"{wl.name}[{len(seq_ids)} of {wl.num_seqs} seqs]"
    sub.num_seqs = len(seq_ids)
    sub.num_blocks = poison + 1
    sub.context_lens = wl.context_lens[seq_ids].copy()
    sub.history_lens = wl.history_lens[seq_ids].copy()
    sub.block_tables = tables
    sub.slot_mapping = np.asarray(slots, dtype=np.int64)
    sub.token_seq = np.asarray([pos[int(wl.token_seq[t])] for t in keep], dtype=np.int32)
    sub.copy_pairs = np.asarray(pairs, dtype=np.int64).reshape(-1, 2)
    sub.poison_block = poison
    sub.extra = dict(wl.extra)
    if wl.query_start is not None:
        counts = np.diff(wl.query_start)[seq_ids]
        sub.query_start = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return sub


def quantized(wl: Workload, fmt: str) -> Workload:
    """The same step over a quantised cache ("fp8" E4M3 or "int8" codes); q, the
    new k / v and the output stay bf16."""
    if fmt not in ("fp8", "int8") or wl.dtype != "bf16":
        raise ValueError("quantised caches: fmt fp8 / int8 over a bf16 workload")
    sub = Workload(**{**wl.__dict__})
    sub.name = f"{wl.name}_{fmt}"
    sub.kv_quant = fmt
    sub.description = f"{wl.description}; {fmt} KV codes with per-kv-head scales"
    return sub


def make(name: str, **kw) -> Workload:
    for fmt in ("fp8", "int8"):
        if name.endswith("_" + fmt) and name[:-len(fmt) - 1] in CONFIGS:
            return quantized(CONFIGS[name[:-len(fmt) - 1]](**kw), fmt)
    if name not in CONFIGS:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(CONFIGS)}")
    return CONFIGS[name](**kw)


# ---------------------------------------------------------------------------
# values
# ---------------------------------------------------------------------------
def make_values(wl: Workload, device="cpu", poison: bool = False, seed_offset: int = 0):
    """q, new k/v and both pools, N(0,1) in the workload's dtype on ``device``.

    With ``poison``, every cache slot that no sequence may read before this
    step's writes is set to NaN: blocks no table references, the slots of each
    sequence from its history length to the end of its last block (including
    the slots this step's append must fill), and every copy destination. A
    read of any of them, or a missed append or copy, turns outputs into NaN.
    """
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(wl.seed * 1000003 + seed_offset)
    dt = wl.torch_dtype
    S, H, Hkv, d = wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim
    q = torch.randn((wl.num_query_rows, H, d), generator=g, device=device, dtype=dt)
    k_new = torch.randn((wl.num_tokens, Hkv, d), generator=g, device=device, dtype=dt)
    v_new = torch.randn((wl.num_tokens, Hkv, d), generator=g, device=device, dtype=dt)
    shape = (wl.num_blocks, Hkv, wl.block_size, d)
    if wl.kv_quant:
        return _quant_values(wl, device, g, q, k_new, v_new, shape, poison)
    k_cache = torch.randn(shape, generator=g, device=device, dtype=dt)
    v_cache = torch.randn(shape, generator=g, device=device, dtype=dt)
    if poison:
        blocks, offs, whole = poison_slots(wl)
        if blocks.size:
            bi = torch.as_tensor(blocks, device=device)
            oi = torch.as_tensor(offs, device=device)
            k_cache[bi, :, oi, :] = float("nan")
            v_cache[bi, :, oi, :] = float("nan")
        if whole.size:
            wi = torch.as_tensor(whole, device=device)
            k_cache[wi] = float("nan")
            v_cache[wi] = float("nan")
    return {"q": q, "k_new": k_new, "v_new": v_new, "k_cache": k_cache, "v_cache": v_cache}


def _quant_values(wl, device, g, q, k_new, v_new, shape, poison):
    """Quantised pools drawn as codes (no quantiser runs here): FP8 E4M3 codes
    with a random sign, exponent field 4..10 and mantissa (values 2^-3 .. 15),
    or int8 codes uniform in [-127, 127]; per-kv-head scales U(0.15, 0.25) (fp8)
    or U(0.02, 0.03) (int8), so every cached value stays below 4 in magnitude
    (3.75, 3.81), the range in which bf16 rounding of an output stays inside the
    1e-2 bar. Poisoned slots hold the NaN code (fp8) or -128."""
    Hkv = wl.num_kv_heads

    def codes():
        if wl.kv_quant == "fp8":
            sign = torch.randint(0, 2, shape, generator=g, device=device, dtype=torch.int32) << 7
            exp = torch.randint(4, 11, shape, generator=g, device=device, dtype=torch.int32) << 3
            man = torch.randint(0, 8, shape, generator=g, device=device, dtype=torch.int32)
            return (sign | exp | man).to(torch.uint8)
        return (torch.randint(-127, 128, shape, generator=g, device=device,
                              dtype=torch.int32) & 0xFF).to(torch.uint8)

    k_cache, v_cache = codes(), codes()
    lo, hi = (0.15, 0.25) if wl.kv_quant == "fp8" else (0.02, 0.03)
    k_scale = lo + (hi - lo) * torch.rand((Hkv,), generator=g, device=device, dtype=torch.float32)
    v_scale = lo + (hi - lo) * torch.rand((Hkv,), generator=g, device=device, dtype=torch.float32)
    if poison:
        bad = 0x7F if wl.kv_quant == "fp8" else 0x80
        blocks, offs, whole = poison_slots(wl)
        if blocks.size:
            bi = torch.as_tensor(blocks, device=device)
            oi = torch.as_tensor(offs, device=device)
            k_cache[bi, :, oi, :] = bad
            v_cache[bi, :, oi, :] = bad
        if whole.size:
            wi = torch.as_tensor(whole, device=device)
            k_cache[wi] = bad
            v_cache[wi] = bad
    view = torch.float8_e4m3fn if wl.kv_quant == "fp8" else torch.int8
    return {"q": q, "k_new": k_new, "v_new": v_new, "k_cache": k_cache.view(view),
            "v_cache": v_cache.view(view), "k_scale": k_scale, "v_scale": v_scale}


def poison_slots(wl: Workload):
    """(block ids, slot offsets) of per-sequence unfilled slots, and ids of
    whole blocks to poison (unreferenced blocks and copy destinations)."""
    B = wl.block_size
    blocks, offs = [], []
    referenced = np.zeros(wl.num_blocks, dtype=bool)
    for s in range(wl.num_seqs):
        n = int(wl.context_lens[s])
        h = int(wl.history_lens[s])
        nb = -(-n // B)
        referenced[wl.block_tables[s, :nb]] = True
        for pos in range(h, nb * B):
            blocks.append(int(wl.block_tables[s, pos // B]))
            offs.append(pos % B)
    whole = set(np.nonzero(~referenced)[0].tolist())
    whole.update(int(x) for x in wl.copy_pairs[:, 1].tolist())
    whole.add(wl.poison_block)
    return (np.asarray(blocks, dtype=np.int64), np.asarray(offs, dtype=np.int64),
            np.asarray(sorted(whole), dtype=np.int64))


def to_numpy(t: torch.Tensor) -> np.ndarray:
    """Host numpy view of a tensor: float32 stays float32; bfloat16 becomes its
    uint16 bit patterns (the oracle's bf16 representation)."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    if t.dtype in (torch.float8_e4m3fn, torch.int8, torch.uint8):
        return t.view(torch.uint8).numpy()           # quantised codes, raw bytes
    raise TypeError(f"unsupported dtype {t.dtype}")


def subproblem(wl: Workload, k_cache: torch.Tensor, v_cache: torch.Tensor,
               seq_ids, q: torch.Tensor | None = None):
    """Host copy of the part of a (possibly device-resident) pool that the
    sequences ``seq_ids`` read, with their block tables renumbered onto the
    compact copy. Renumbering is a change of physical placement only.

    Returns dict(q, k_cache, v_cache, block_tables, context_lens) as numpy.
    """
    seq_ids = [int(s) for s in seq_ids]
    B = wl.block_size
    used = []
    index = {}
    rows = []
    for s in seq_ids:
        n = int(wl.context_lens[s])
        nb = -(-n // B)
        row = []
        for j in range(nb):
            b = int(wl.block_tables[s, j])
            if b not in index:
                index[b] = len(used)
                used.append(b)
            row.append(index[b])
        rows.append(row)
    width = max([1] + [len(r) for r in rows])
    tables = np.zeros((len(seq_ids), width), dtype=np.int32)
    for i, r in enumerate(rows):
        tables[i, :len(r)] = r
    ids = torch.as_tensor(used if used else [0], dtype=torch.long, device=k_cache.device)
    if k_cache.dtype in (torch.float8_e4m3fn, torch.int8):     # code pools: gather raw bytes
        k_cache, v_cache = k_cache.view(torch.uint8), v_cache.view(torch.uint8)
    out = {
        "k_cache": to_numpy(k_cache.index_select(0, ids)),
        "v_cache": to_numpy(v_cache.index_select(0, ids)),
        "block_tables": tables,
        "context_lens": wl.context_lens[seq_ids].astype(np.int32),
    }
    if q is not None:
        qi = torch.as_tensor(seq_ids, dtype=torch.long, device=q.device)
        out["q"] = to_numpy(q.index_select(0, qi))
    return out
