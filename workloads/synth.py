"""Seeded synthetic batches for PagedAttention over a block-paged KV pool.

The shapes follow the workloads named for this library: a tiny correctness case,
Llama-2-7B/13B/70B-shaped attention layers and a Qwen-32B-like continuous-batching
step.  The structure follows the pages' description of the KV cache manager
("vLLM 基本原理", sections "PagedAttention" / "内存共享"; "当大模型推理遇上内存瓶颈"
section 2.2-2.3):

* a sequence's KV is split into logical blocks of ``block_size`` tokens;
* each logical block maps to any free physical block of one pool (here drawn by a
  seeded shuffle, so the blocks are scattered);
* only the last block of a sequence may be partly filled;
* parallel samples of one prompt point at the same physical prompt blocks
  (ref-counted), and a sharer that must own a block gets a copied one
  (copy-on-write pairs).

Everything here is index bookkeeping and random-number filling.  None of the
attention arithmetic lives in this module, and it imports neither the oracle nor
the CUDA library.  Integer arrays are NumPy; bf16 tensors are NumPy ``uint16`` bit
patterns (``fill_host``) or torch tensors on a device (``fill_device``).

Poisoning, so that a kernel that reads what it must not read is caught:

* table entries past ``ceil(L / block_size)`` hold ``INT32_MAX``;
* slots at positions ``>= L`` of a sequence's last block hold bf16 NaN;
* physical blocks no table references hold NaN;
* slots that this step's new tokens will be written to hold NaN until the
  cache-write call fills them;
* copy-on-write destination blocks hold NaN until the block copy fills them.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

INT32_MAX = 2**31 - 1
BF16_NAN = 0x7FC0
BLOCK_SIZE = 16

__all__ = [
    "INT32_MAX", "BF16_NAN", "BLOCK_SIZE", "Layout", "f32_to_bf16_bits",
    "normal_bf16", "build_layout", "tiny", "llama7b_decode", "llama13b_sampling",
    "gqa70b_long", "mixed_qwen32b", "CONFIGS", "fill_host", "fill_device",
    "chunk_schedule", "decode_kv_bytes", "kv_cache_bytes_per_layer",
    "prefill_flops", "unique_kv_bytes", "subset", "token_rows",
]


# ----------------------------------------------------------------------------
# bf16 bit patterns
# ----------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even).

    Returns the 16-bit patterns as ``uint16``.  Inputs are finite here.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = ((u >> np.uint64(16)) & np.uint64(1)) + np.uint64(0x7FFF)
    return ((u + bias) >> np.uint64(16)).astype(np.uint16)


def normal_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    """N(0, 1) float32 samples rounded to bf16 bit patterns."""
    return f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))


# ----------------------------------------------------------------------------
# Layout: the integer side of one batch step
# ----------------------------------------------------------------------------
@dataclass
class Layout:
    """One batch step over one paged KV pool.

    ``context_lens[s]`` counts every token of sequence ``s`` after this step's
    new tokens are written (so a decode sequence's own new token is included).
    ``q_lens[s]`` is the number of new tokens of ``s`` this step: 1 for a decode
    sequence, the chunk length for a chunked-prefill sequence.
    """

    name: str
    seed: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    context_lens: np.ndarray  # int32 [S]
    block_tables: np.ndarray  # int32 [S, max_blocks], padding INT32_MAX
    q_lens: np.ndarray  # int32 [S]
    is_prefill: np.ndarray  # bool [S]
    copy_pairs: np.ndarray = field(default_factory=lambda: np.zeros((0, 2), np.int64))
    ref_counts: np.ndarray | None = None  # int32 [num_blocks]
    notes: str = ""

    # -- sizes --------------------------------------------------------------
    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def max_blocks(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def group_size(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def pool_shape(self) -> tuple:
        return (self.num_blocks, self.num_kv_heads, self.block_size, self.head_dim)

    def blocks_used(self, s: int) -> int:
        return -(-int(self.context_lens[s]) // self.block_size)

    # -- sub-batches --------------------------------------------------------
    def decode_rows(self) -> np.ndarray:
        return np.nonzero(~self.is_prefill)[0]

    def prefill_rows(self) -> np.ndarray:
        return np.nonzero(self.is_prefill)[0]

    # -- new tokens ---------------------------------------------------------
    def new_positions(self, rows=None) -> tuple[np.ndarray, np.ndarray]:
        """(seq index, absolute position) of every new token, seq-major order."""
        rows = np.arange(self.num_seqs) if rows is None else np.asarray(rows)
        seqs, poss = [], []
        for s in rows:
            L, n = int(self.context_lens[s]), int(self.q_lens[s])
            seqs.append(np.full(n, s, np.int64))
            poss.append(np.arange(L - n, L, dtype=np.int64))
        if not seqs:
            return np.zeros(0, np.int64), np.zeros(0, np.int64)
        return np.concatenate(seqs), np.concatenate(poss)

    def slot_mapping(self, rows=None) -> np.ndarray:
        """Flat slot (physical_block * block_size + offset) of every new token."""
        seqs, poss = self.new_positions(rows)
        bs = self.block_size
        phys = self.block_tables[seqs, poss // bs].astype(np.int64)
        return phys * bs + poss % bs

    def cu_q_lens(self, rows) -> np.ndarray:
        ql = self.q_lens[np.asarray(rows)]
        return np.concatenate([[0], np.cumsum(ql)]).astype(np.int32)


def _alloc_order(rng: np.random.Generator, num_blocks: int, shuffle: bool) -> list:
    order = rng.permutation(num_blocks) if shuffle else np.arange(num_blocks)
    return [int(b) for b in order]


def build_layout(name, seed, context_lens, *, num_q_heads, num_kv_heads, head_dim,
                 block_size=BLOCK_SIZE, q_lens=None, is_prefill=None, pool_factor=1.25,
                 num_blocks=None, shuffle=True, extra_table_cols=0, rng=None,
                 notes="") -> Layout:
    """Private (unshared) blocks for every sequence, drawn from a shuffled pool.

    ``num_blocks`` defaults to ``ceil(pool_factor * blocks needed)``.  Block
    ``k`` of the draw order goes to the ``k``-th logical block, sequence-major.
    """
    rng = np.random.default_rng(seed) if rng is None else rng
    context_lens = np.asarray(context_lens, dtype=np.int32)
    S = context_lens.shape[0]
    need = [-(-int(L) // block_size) for L in context_lens]
    total = int(sum(need))
    if num_blocks is None:
        num_blocks = max(1, int(math.ceil(pool_factor * total)))
    if num_blocks < total:
        raise ValueError("pool too small")
    order = _alloc_order(rng, num_blocks, shuffle)
    max_blocks = max([1] + need) + extra_table_cols
    tables = np.full((S, max_blocks), INT32_MAX, dtype=np.int32)
    ref = np.zeros(num_blocks, np.int32)
    k = 0
    for s in range(S):
        for b in range(need[s]):
            tables[s, b] = order[k]
            ref[order[k]] += 1
            k += 1
    if q_lens is None:
        q_lens = np.ones(S, np.int32)
    if is_prefill is None:
        is_prefill = np.zeros(S, bool)
    return Layout(name, seed, num_q_heads, num_kv_heads, head_dim, block_size,
                  num_blocks, context_lens, tables, np.asarray(q_lens, np.int32),
                  np.asarray(is_prefill, bool), ref_counts=ref, notes=notes)


# ----------------------------------------------------------------------------
# The five named workloads
# ----------------------------------------------------------------------------
def tiny(seed: int = 0) -> Layout:
    """4 sequences, contexts {1, 17, 33, 64}, 4 q heads = 4 KV heads, head_dim 64,
    32 physical blocks assigned by a seeded permutation, one decode query each."""
    return build_layout("tiny", seed, [1, 17, 33, 64], num_q_heads=4, num_kv_heads=4,
                        head_dim=64, num_blocks=32)


def llama7b_decode(seed: int = 1, batch: int = 64) -> Layout:
    """Llama-2-7B-shaped layer decode: MHA 32/32, head_dim 128, contexts
    uniform in [128, 2048], pool 1.25x the blocks needed, shuffled."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(128, 2048 + 1, size=batch)
    return build_layout("llama7b_decode", seed, lens, num_q_heads=32, num_kv_heads=32,
                        head_dim=128, rng=rng)


def llama13b_sampling(seed: int = 2, groups: int = 64, samples: int = 4,
                      prefix: int = 512, max_suffix: int = 512, batch: int | None = None) -> Layout:
    """Llama-2-13B-shaped parallel sampling: ``groups`` prompts x ``samples``
    samples, MHA 40/40, head_dim 128.  Every sample of a group points at the
    same physical prompt blocks (ref count = samples).  Samples 1.. take a
    copy-on-write copy of the last prompt block (``copy_pairs``); every sample
    then owns a private suffix of uniform [1, max_suffix] tokens.  ``batch``,
    when given, is the number of sequences (groups = batch // samples)."""
    if batch is not None:
        groups = max(1, batch // samples)
    rng = np.random.default_rng(seed)
    bs = BLOCK_SIZE
    pre_blocks = -(-prefix // bs)
    suffix = rng.integers(1, max_suffix + 1, size=groups * samples)
    lens = prefix + suffix
    suf_blocks = [-(-(int(L)) // bs) - pre_blocks for L in lens]
    need = groups * pre_blocks + groups * (samples - 1) + int(sum(suf_blocks))
    num_blocks = int(math.ceil(1.25 * need))
    order = _alloc_order(rng, num_blocks, True)
    max_blocks = max(-(-int(L) // bs) for L in lens)
    S = groups * samples
    tables = np.full((S, max_blocks), INT32_MAX, dtype=np.int32)
    ref = np.zeros(num_blocks, np.int32)
    pairs = []
    k = 0
    for g in range(groups):
        shared = order[k:k + pre_blocks]
        k += pre_blocks
        for j in range(samples):
            s = g * samples + j
            tables[s, :pre_blocks] = shared
            if j > 0:  # copy-on-write of the last prompt block
                dst = order[k]
                k += 1
                pairs.append((shared[-1], dst))
                tables[s, pre_blocks - 1] = dst
            for b in range(suf_blocks[s]):
                tables[s, pre_blocks + b] = order[k]
                k += 1
    for s in range(S):
        for b in range(-(-int(lens[s]) // bs)):
            ref[tables[s, b]] += 1
    return Layout("llama13b_sampling", seed, 40, 40, 128, bs, num_blocks,
                  lens.astype(np.int32), tables, np.ones(S, np.int32), np.zeros(S, bool),
                  copy_pairs=np.asarray(pairs, np.int64).reshape(-1, 2), ref_counts=ref,
                  notes=f"{groups} groups x {samples} samples; {prefix}-token shared prefix")


def prefix_runs(name: str, seed: int, run_sizes, prefix, max_suffix: int, *, num_q_heads: int,
                num_kv_heads: int, head_dim: int = 128, min_suffix: int = 1,
                cow: bool = True) -> Layout:
    """Runs of sequences sharing a prompt: run ``r`` has ``run_sizes[r]``
    sequences that all point at the same physical blocks for the first
    ``prefix[r]`` tokens (``prefix`` may be one number for every run).  With
    ``cow`` the sequences after the first take a copy-on-write copy of the last
    prompt block (``copy_pairs``); each then owns a private suffix of uniform
    [min_suffix, max_suffix] tokens.  A run of size 1 is an unshared sequence;
    a prefix of 0 gives an empty context when the suffix is empty too.  Pool
    1.25x the blocks needed, shuffled."""
    rng = np.random.default_rng(seed)
    bs = BLOCK_SIZE
    run_sizes = [int(n) for n in run_sizes]
    prefix = [int(prefix)] * len(run_sizes) if np.isscalar(prefix) else [int(x) for x in prefix]
    S = int(sum(run_sizes))
    suffix = rng.integers(min_suffix, max_suffix + 1, size=S)
    lens = np.zeros(S, np.int64)
    need = 0
    s = 0
    for n, pre in zip(run_sizes, prefix):
        pb = -(-pre // bs)
        need += pb + (n - 1 if cow and pb else 0)
        for j in range(n):
            lens[s] = pre + suffix[s]
            need += -(-int(lens[s]) // bs) - pb
            s += 1
    num_blocks = max(1, int(math.ceil(1.25 * need)))
    order = _alloc_order(rng, num_blocks, True)
    max_blocks = max(1, max(-(-int(L) // bs) for L in lens))
    tables = np.full((S, max_blocks), INT32_MAX, dtype=np.int32)
    pairs = []
    k = 0
    s = 0
    for n, pre in zip(run_sizes, prefix):
        pb = -(-pre // bs)
        shared = order[k:k + pb]
        k += pb
        for j in range(n):
            tables[s, :pb] = shared
            if j > 0 and cow and pb:
                tables[s, pb - 1] = order[k]
                pairs.append((shared[-1], order[k]))
                k += 1
            for b in range(pb, -(-int(lens[s]) // bs)):
                tables[s, b] = order[k]
                k += 1
            s += 1
    ref = np.zeros(num_blocks, np.int32)
    for s in range(S):
        for b in range(-(-int(lens[s]) // bs)):
            ref[tables[s, b]] += 1
    return Layout(name, seed, num_q_heads, num_kv_heads, head_dim, bs, num_blocks,
                  lens.astype(np.int32), tables, np.ones(S, np.int32), np.zeros(S, bool),
                  copy_pairs=np.asarray(pairs, np.int64).reshape(-1, 2), ref_counts=ref,
                  notes=f"runs {run_sizes} sharing prompt prefixes")


def gqa70b_long(seed: int = 3, batch: int = 128) -> Layout:
    """70B-like GQA long context: 64 q heads / 8 KV heads, head_dim 128,
    contexts log-uniform in [1024, 32768] (floor of exp(U(ln 1024, ln 32768))),
    pool 1.25x the blocks needed, shuffled."""
    rng = np.random.default_rng(seed)
    lens = np.floor(np.exp(rng.uniform(math.log(1024), math.log(32768), size=batch)))
    lens = np.clip(lens, 1024, 32768).astype(np.int64)
    return build_layout("gqa70b_long", seed, lens, num_q_heads=64, num_kv_heads=8,
                        head_dim=128, rng=rng)


def mixed_qwen32b(seed: int = 4, n_prefill: int = 8, chunk: int = 512,
                  n_decode: int = 192, batch: int | None = None) -> Layout:
    """Continuous-batching mixed step, Qwen-32B-like: 40 q heads / 8 KV heads,
    head_dim 128.  ``n_prefill`` sequences each add a ``chunk``-token causal
    chunk onto an existing context uniform in [0, 4096]; ``n_decode`` decode
    sequences have contexts uniform in [256, 8192].  ``batch``, when given,
    replaces ``n_decode`` (a smaller step of the same shape)."""
    if batch is not None:
        n_decode = batch
    rng = np.random.default_rng(seed)
    cached = rng.integers(0, 4096 + 1, size=n_prefill)
    dec = rng.integers(256, 8192 + 1, size=n_decode)
    lens = np.concatenate([cached + chunk, dec])
    q_lens = np.concatenate([np.full(n_prefill, chunk), np.ones(n_decode)]).astype(np.int32)
    is_pf = np.concatenate([np.ones(n_prefill, bool), np.zeros(n_decode, bool)])
    return build_layout("mixed_qwen32b", seed, lens, num_q_heads=40, num_kv_heads=8,
                        head_dim=128, q_lens=q_lens, is_prefill=is_pf, rng=rng)


CONFIGS = {
    "tiny": tiny,
    "llama7b_decode": llama7b_decode,
    "llama13b_sampling": llama13b_sampling,
    "gqa70b_long": gqa70b_long,
    "mixed_qwen32b": mixed_qwen32b,
}


# ----------------------------------------------------------------------------
# Poison lists (index bookkeeping only)
# ----------------------------------------------------------------------------
def _poison_slots(layout: Layout):
    """Return (unused_blocks, slot_blocks, slot_offsets) to be filled with NaN:
    tails past each context, new-token slots, and copy-on-write destinations."""
    bs = layout.block_size
    referenced = np.zeros(layout.num_blocks, bool)
    for s in range(layout.num_seqs):
        nb = layout.blocks_used(s)
        referenced[layout.block_tables[s, :nb]] = True
    if layout.copy_pairs.size:
        referenced[layout.copy_pairs[:, 0]] = True
    unused = np.nonzero(~referenced)[0]
    # A copy-on-write source is copied whole to its destinations, whose
    # sequences may read past the source owner's context: its slots stay finite.
    src = set(layout.copy_pairs[:, 0].tolist()) if layout.copy_pairs.size else set()
    blocks, offs = [], []
    for s in range(layout.num_seqs):
        L = int(layout.context_lens[s])
        if L % bs:
            last = int(layout.block_tables[s, L // bs])
            if last in src:
                continue
            for o in range(L % bs, bs):
                blocks.append(last)
                offs.append(o)
    sm = layout.slot_mapping()
    keep = np.array([int(b) not in src for b in (sm // bs).tolist()], bool)
    blocks.extend((sm[keep] // bs).tolist())
    offs.extend((sm[keep] % bs).tolist())
    if layout.copy_pairs.size:
        for dst in layout.copy_pairs[:, 1]:
            for o in range(bs):
                blocks.append(int(dst))
                offs.append(o)
    return unused, np.asarray(blocks, np.int64), np.asarray(offs, np.int64)


# ----------------------------------------------------------------------------
# Fillers
# ----------------------------------------------------------------------------
def fill_host(layout: Layout, seed: int | None = None, poison: bool = True) -> dict:
    """bf16 bit-pattern tensors (NumPy uint16) for a layout, drawn from N(0, 1).

    Keys: ``q`` [T_new, Hq, D], ``key`` / ``value`` [T_new, Hkv, D] (this step's
    new tokens, seq-major, matching ``layout.slot_mapping()``), ``k_pool`` /
    ``v_pool`` [num_blocks, Hkv, block_size, D].
    """
    rng = np.random.default_rng(layout.seed + 1000 if seed is None else seed)
    T = int(layout.q_lens.sum())
    Hq, Hkv, D = layout.num_q_heads, layout.num_kv_heads, layout.head_dim
    out = {
        "q": normal_bf16(rng, (T, Hq, D)),
        "key": normal_bf16(rng, (T, Hkv, D)),
        "value": normal_bf16(rng, (T, Hkv, D)),
        "k_pool": normal_bf16(rng, layout.pool_shape),
        "v_pool": normal_bf16(rng, layout.pool_shape),
    }
    if poison:
        unused, pb, po = _poison_slots(layout)
        for name in ("k_pool", "v_pool"):
            pool = out[name]
            pool[unused] = BF16_NAN
            pool[pb, :, po, :] = BF16_NAN
    return out


def fill_device(layout: Layout, device, seed: int | None = None, poison: bool = True,
                chunk_blocks: int = 4096) -> dict:
    """Same tensors as :func:`fill_host`, drawn on ``device`` with torch's seeded
    generator (for pools too large to draw on the host).  Values differ from
    ``fill_host`` (a different generator); callers that check results take host
    copies of exactly these tensors."""
    import torch

    seed = layout.seed + 2000 if seed is None else seed
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    T = int(layout.q_lens.sum())
    Hq, Hkv, D = layout.num_q_heads, layout.num_kv_heads, layout.head_dim

    def randn_bf16(shape):
        return torch.randn(shape, generator=gen, device=device,
                           dtype=torch.float32).to(torch.bfloat16)

    out = {
        "q": randn_bf16((T, Hq, D)),
        "key": randn_bf16((T, Hkv, D)),
        "value": randn_bf16((T, Hkv, D)),
    }
    for name in ("k_pool", "v_pool"):
        pool = torch.empty(layout.pool_shape, dtype=torch.bfloat16, device=device)
        for b0 in range(0, layout.num_blocks, chunk_blocks):
            b1 = min(layout.num_blocks, b0 + chunk_blocks)
            pool[b0:b1] = randn_bf16((b1 - b0,) + layout.pool_shape[1:])
        out[name] = pool
    if poison:
        unused, pb, po = _poison_slots(layout)
        nan = float("nan")
        for name in ("k_pool", "v_pool"):
            pool = out[name]
            if unused.size:
                pool[torch.as_tensor(unused, device=device)] = nan
            if pb.size:
                pool[torch.as_tensor(pb, device=device), :,
                     torch.as_tensor(po, device=device), :] = nan
    return out


# ----------------------------------------------------------------------------
# Chunk schedule of the pages' chunked-prefill example
# ----------------------------------------------------------------------------
def chunk_schedule(prompt_len: int, chunk: int, budget: int) -> list:
    """Rounds of a chunked prefill: each round takes the next ``chunk`` prompt
    tokens (the last round takes what is left) and gives the rest of the
    ``budget`` to decode tokens.  Returns ``[(start, end, decode_tokens), ...]``.

    The pages' example ("vLLM 定位与核心机制详解", section 六.4): a budget of 6
    tokens per round and a 12-token prompt read 4 at a time take 3 rounds,
    with the decoding requests still served in every round.
    """
    if chunk <= 0 or chunk > budget:
        raise ValueError("chunk must be in [1, budget]")
    rounds = []
    start = 0
    while start < prompt_len:
        end = min(prompt_len, start + chunk)
        rounds.append((start, end, budget - (end - start)))
        start = end
    return rounds


# ----------------------------------------------------------------------------
# Byte / flop accounting used by the measurement
# ----------------------------------------------------------------------------
def kv_cache_bytes_per_layer(num_heads: int, seq_len: int, head_dim: int,
                             elem_bytes: int) -> int:
    """K plus V bytes of one layer for one sequence: 2 * heads * len * dim * size
    ("当大模型推理遇上内存瓶颈", section 2.1, worked for Llama 2-7B)."""
    return 2 * num_heads * seq_len * head_dim * elem_bytes


def decode_kv_bytes(layout: Layout, rows=None) -> dict:
    """Algorithmic bytes of one paged decode over ``rows`` (default: all decode
    rows): K/V of every context token of every KV head, q in, out, the used
    table entries and the lengths.  ``logical`` counts shared blocks once per
    sequence that reads them; ``unique`` counts each physical block once."""
    rows = layout.decode_rows() if rows is None else np.asarray(rows)
    Hq, Hkv, D, bs = layout.num_q_heads, layout.num_kv_heads, layout.head_dim, layout.block_size
    lens = layout.context_lens[rows].astype(np.int64)
    kv = int(sum(kv_cache_bytes_per_layer(Hkv, int(L), D, 2) for L in lens))
    qo = int(len(rows) * 2 * Hq * D * 2)
    meta = int(sum(4 * (-(-int(L) // bs)) for L in lens) + 4 * len(rows))
    uniq = unique_kv_bytes(layout, rows)
    return {"kv": kv, "q_out": qo, "meta": meta, "logical": kv + qo + meta,
            "unique_kv": uniq, "unique": uniq + qo + meta}


def unique_kv_bytes(layout: Layout, rows) -> int:
    """K/V bytes of the distinct (physical block, token offset) slots read."""
    bs = layout.block_size
    seen = {}
    for s in rows:
        L = int(layout.context_lens[s])
        for b in range(-(-L // bs)):
            p = int(layout.block_tables[s, b])
            n = min(bs, L - b * bs)
            seen[p] = max(seen.get(p, 0), n)
    toks = sum(seen.values())
    return int(2 * layout.num_kv_heads * toks * layout.head_dim * 2)


def prefill_flops(layout: Layout, rows=None) -> int:
    """Multiply-add flops (2 per MAC) of causal chunked-prefill attention: for
    query i of a chunk on cached length c, QK and PV over c + i + 1 keys."""
    rows = layout.prefill_rows() if rows is None else np.asarray(rows)
    D, Hq = layout.head_dim, layout.num_q_heads
    total = 0
    for s in rows:
        L, n = int(layout.context_lens[s]), int(layout.q_lens[s])
        c = L - n
        keys = n * c + n * (n + 1) // 2
        total += 4 * D * Hq * keys
    return int(total)


# ----------------------------------------------------------------------------
# Restriction of a batch to some sequences (for checking sampled outputs)
# ----------------------------------------------------------------------------
def subset(layout: Layout, rows) -> tuple[Layout, np.ndarray]:
    """The batch restricted to ``rows``, over a compact pool holding only the
    blocks those rows read or write (plus the sources of the copy-on-write
    pairs whose destinations they use).

    Returns ``(sub_layout, blocks)`` where ``blocks[i]`` is the original
    physical id of the sub-layout's block ``i``; the caller gathers
    ``pool[blocks]`` to build the compact pools.  Token order of the new tokens
    follows ``rows``.
    """
    rows = [int(r) for r in rows]
    need = []
    for s in rows:
        need.extend(int(b) for b in layout.block_tables[s, : layout.blocks_used(s)])
    used = set(need)
    pairs = [(int(a), int(b)) for a, b in layout.copy_pairs if int(b) in used]
    need.extend(a for a, _ in pairs)
    blocks = np.asarray(sorted(set(need)), dtype=np.int64)
    remap = {int(b): i for i, b in enumerate(blocks)}
    mb = max([1] + [layout.blocks_used(s) for s in rows])
    tables = np.full((len(rows), mb), INT32_MAX, dtype=np.int32)
    for i, s in enumerate(rows):
        for j in range(layout.blocks_used(s)):
            tables[i, j] = remap[int(layout.block_tables[s, j])]
    ref = np.zeros(len(blocks), np.int32)
    for i in range(len(rows)):
        for j in range(-(-int(layout.context_lens[rows[i]]) // layout.block_size)):
            ref[tables[i, j]] += 1
    cp = np.asarray([(remap[a], remap[b]) for a, b in pairs], np.int64).reshape(-1, 2)
    sub = Layout(layout.name + "-subset", layout.seed, layout.num_q_heads, layout.num_kv_heads,
                 layout.head_dim, layout.block_size, len(blocks),
                 layout.context_lens[rows].copy(), tables, layout.q_lens[rows].copy(),
                 layout.is_prefill[rows].copy(), copy_pairs=cp, ref_counts=ref)
    return sub, blocks


def token_rows(layout: Layout, rows) -> np.ndarray:
    """Indices, into the step's packed new-token arrays (q, key, value), of the
    new tokens of ``rows`` in ``rows`` order."""
    starts = np.concatenate([[0], np.cumsum(layout.q_lens)]).astype(np.int64)
    return np.concatenate([np.arange(starts[s], starts[s + 1]) for s in rows]).astype(np.int64)
