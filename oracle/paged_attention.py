"""Plain NumPy float64 definition of paged attention (TEST INFRASTRUCTURE ONLY).

Sources, by page title and section:

* "vLLM 基本原理", section "PagedAttention" (logical blocks, physical blocks,
  block table; "the CUDA kernel fetches data from every corner of physical
  memory according to the table") and section "Transformer 和 Attention"
  (attention as a weighted lookup: each query scores every context token and
  mixes their values by those weights).
* "当大模型推理遇上内存瓶颈", section 3.1 (paged layout
  ``[num_blocks, num_heads, block_size, head_dim]`` and indexing
  ``block_tables[seq_idx][logic_block]`` -> ``physical_block``) and section 3.3
  (copying one shared block into a sharer's own block).
* "vLLM 定位与核心机制详解", section 六.4 (chunked prefill: a long prompt is read
  a chunk per round; each chunk's tokens attend causally).

Readings taken where the pages are silent:

* GQA: q head ``h`` reads KV head ``h // (Hq / Hkv)`` (contiguous groups).
* A decode step's own new token is part of its context (``context_lens``
  includes it; the cache write happens first).
* Chunked prefill: the query at absolute position ``p`` sees keys ``0..p``
  inclusive; the chunk's own K/V are in the pool before attention runs.
* ``context_len == 0``: output zeros and log-sum-exp ``-inf``.
* Cache write: a negative slot is padding and is skipped.
* Block copy: destinations must be distinct and none may also be a source,
  so the result does not depend on the order the copies run in.

Every function works on bf16 *bit patterns* (``uint16``) for its tensor inputs
and widens them exactly to float64; arithmetic is float64 with no blocking,
splitting or reordering beyond the definition.  The max subtraction inside the
softmax is the identity ``exp(x)/sum(exp(x)) == exp(x-m)/sum(exp(x-m))``.
"""
from __future__ import annotations

import numpy as np


class CopyBlocksError(ValueError):
    """A block-copy list breaks the rules above (range, duplicate or chained)."""


# ----------------------------------------------------------------------------
# bf16 <-> float64
# ----------------------------------------------------------------------------
def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact value of bf16 bit patterns: a bf16 number is the float32 whose upper
    16 bits are the pattern and whose lower 16 bits are zero."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x) -> np.ndarray:
    """Round float64 to bf16, to nearest with ties to even, through the exact
    float32 value nearest to ``x`` (used to compare kernel outputs that are
    exact copies of bf16 inputs)."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    bias = ((u >> np.uint64(16)) & np.uint64(1)) + np.uint64(0x7FFF)
    return ((u + bias) >> np.uint64(16)).astype(np.uint16)


# ----------------------------------------------------------------------------
# Addressing ("vLLM 基本原理" / PagedAttention; "当大模型推理遇上内存瓶颈" 3.1)
# ----------------------------------------------------------------------------
def slot_of(block_table_row, position: int, block_size: int) -> int:
    """Flat slot of the token at ``position`` of one sequence.

    The token lies in logical block ``position // block_size`` at offset
    ``position % block_size``; the block table maps the logical block to its
    physical block, and the slot is ``physical * block_size + offset``.
    """
    logical, offset = divmod(int(position), int(block_size))
    return int(block_table_row[logical]) * int(block_size) + offset


def gather_kv(k_pool, v_pool, block_table_row, context_len: int):
    """Contiguous ``[Hkv, L, D]`` K and V (bit patterns) of one sequence.

    Walks the sequence's logical blocks in order; logical block ``b`` holds
    tokens ``b*bs .. b*bs+bs-1`` and lives in physical block
    ``block_table_row[b]`` of the pool ``[num_blocks, Hkv, bs, D]``.  Only the
    first ``L - b*bs`` tokens of the last block belong to the sequence.
    """
    num_blocks, hkv, bs, d = k_pool.shape
    L = int(context_len)
    K = np.empty((hkv, L, d), dtype=k_pool.dtype)
    V = np.empty((hkv, L, d), dtype=v_pool.dtype)
    for b in range(-(-L // bs)):
        p = int(block_table_row[b])
        if not 0 <= p < num_blocks:
            raise IndexError(f"block table entry {p} outside pool of {num_blocks}")
        n = min(bs, L - b * bs)
        K[:, b * bs:b * bs + n, :] = k_pool[p, :, :n, :]
        V[:, b * bs:b * bs + n, :] = v_pool[p, :, :n, :]
    return K, V


# ----------------------------------------------------------------------------
# Attention ("vLLM 基本原理" / Transformer 和 Attention)
# ----------------------------------------------------------------------------
def attend(q, K, V, scale: float):
    """Softmax attention of one query over ``L`` keys, float64.

    ``x_t = scale * (q . k_t)``;  ``w = softmax(x)``;  ``out = sum_t w_t v_t``;
    ``lse = log(sum_t exp(x_t))``.  With no keys: zeros and ``-inf``.
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    if K.shape[0] == 0:
        return np.zeros(V.shape[-1]), -np.inf
    x = scale * (K @ q)
    m = x.max()
    w = np.exp(x - m)
    z = w.sum()
    return (w @ V) / z, m + np.log(z)


def _kv_head_of(h: int, num_q_heads: int, num_kv_heads: int) -> int:
    """KV head read by q head ``h``: contiguous groups of ``Hq / Hkv`` q heads."""
    return h // (num_q_heads // num_kv_heads)


def decode(q, k_pool, v_pool, block_tables, context_lens, scale: float):
    """Single-query paged attention for every sequence and q head.

    ``q``: bf16 bits ``[S, Hq, D]``; pools: bf16 bits ``[num_blocks, Hkv, bs, D]``;
    ``block_tables``: ``[S, max_blocks]``; ``context_lens``: ``[S]``.
    Returns ``out`` float64 ``[S, Hq, D]`` and ``lse`` float64 ``[S, Hq]``.
    """
    S, hq, d = q.shape
    hkv = k_pool.shape[1]
    if hq % hkv:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    qf = bf16_bits_to_f64(q)
    out = np.zeros((S, hq, d))
    lse = np.full((S, hq), -np.inf)
    for s in range(S):
        Kb, Vb = gather_kv(k_pool, v_pool, block_tables[s], int(context_lens[s]))
        K, V = bf16_bits_to_f64(Kb), bf16_bits_to_f64(Vb)
        for h in range(hq):
            g = _kv_head_of(h, hq, hkv)
            out[s, h], lse[s, h] = attend(qf[s, h], K[g], V[g], scale)
    return out, lse


def chunked_prefill(q, cu_q_lens, k_pool, v_pool, block_tables, context_lens, scale: float):
    """Causal attention of each sequence's new chunk over its cached context
    plus the chunk itself.

    Sequence ``s`` owns query rows ``cu_q_lens[s] .. cu_q_lens[s+1]-1`` of ``q``
    (bf16 bits ``[Nq, Hq, D]``), i.e. ``n`` new tokens on top of
    ``c = context_lens[s] - n`` cached ones.  Query ``i`` is at absolute
    position ``c + i`` and attends to keys ``0 .. c + i``.
    Returns ``out`` float64 ``[Nq, Hq, D]`` and ``lse`` ``[Nq, Hq]``.
    """
    nq, hq, d = q.shape
    hkv = k_pool.shape[1]
    qf = bf16_bits_to_f64(q)
    out = np.zeros((nq, hq, d))
    lse = np.full((nq, hq), -np.inf)
    for s in range(len(context_lens)):
        r0, r1 = int(cu_q_lens[s]), int(cu_q_lens[s + 1])
        n, L = r1 - r0, int(context_lens[s])
        c = L - n
        if c < 0:
            raise ValueError("context_lens must include the chunk")
        Kb, Vb = gather_kv(k_pool, v_pool, block_tables[s], L)
        K, V = bf16_bits_to_f64(Kb), bf16_bits_to_f64(Vb)
        for i in range(n):
            limit = c + i + 1
            for h in range(hq):
                g = _kv_head_of(h, hq, hkv)
                out[r0 + i, h], lse[r0 + i, h] = attend(qf[r0 + i, h], K[g, :limit],
                                                        V[g, :limit], scale)
    return out, lse


# ----------------------------------------------------------------------------
# Cache writes and block copies
# ----------------------------------------------------------------------------
def reshape_and_cache(k_pool, v_pool, key, value, slot_mapping):
    """Write each new token's K and V into its slot; returns new pools.

    Token ``t`` goes to physical block ``slot // bs`` at offset ``slot % bs``
    for every KV head ("vLLM 基本原理", 按需分配: tokens fill the current block
    and a new block is taken only when it is full).  A negative slot is skipped.
    """
    num_blocks, hkv, bs, d = k_pool.shape
    k, v = k_pool.copy(), v_pool.copy()
    slots = [int(x) for x in slot_mapping]
    live = [x for x in slots if x >= 0]
    if len(set(live)) != len(live):
        raise ValueError("two tokens map to one slot")
    for t, slot in enumerate(slots):
        if slot < 0:
            continue
        b, o = divmod(slot, bs)
        if b >= num_blocks:
            raise IndexError(f"slot {slot} outside pool")
        k[b, :, o, :] = key[t]
        v[b, :, o, :] = value[t]
    return k, v


def copy_blocks(k_pool, v_pool, pairs):
    """Copy whole K and V blocks (all heads, all slots) ``src -> dst``; returns
    new pools ("当大模型推理遇上内存瓶颈" 3.3: a sharer that must write gets its own
    copy of the shared block).  Raises :class:`CopyBlocksError` for a pair out of
    range, a repeated destination or a destination that is also a source."""
    num_blocks = k_pool.shape[0]
    pairs = np.asarray(pairs, dtype=np.int64).reshape(-1, 2)
    srcs = [int(x) for x in pairs[:, 0]]
    dsts = [int(x) for x in pairs[:, 1]]
    for x in srcs + dsts:
        if not 0 <= x < num_blocks:
            raise CopyBlocksError(f"block {x} outside pool of {num_blocks}")
    if len(set(dsts)) != len(dsts):
        raise CopyBlocksError("repeated destination block")
    if set(dsts) & set(srcs):
        raise CopyBlocksError("a destination block is also a source")
    k, v = k_pool.copy(), v_pool.copy()
    for s, d in zip(srcs, dsts):
        k[d] = k_pool[s]
        v[d] = v_pool[s]
    return k, v


def swap_blocks(src_k, src_v, dst_k, dst_v, pairs):
    """Copy whole K and V blocks from the source pools to the destination pools
    (``src -> dst`` per pair; "当大模型推理遇上内存瓶颈" 5.1 and 7.3: KV blocks moved
    to a CPU swap space and read back).  The two sides are different pools, so
    only the destinations must be distinct.  Returns the new destination pools."""
    pairs = np.asarray(pairs, dtype=np.int64).reshape(-1, 2)
    ns, nd = src_k.shape[0], dst_k.shape[0]
    for s_, d_ in pairs:
        if not (0 <= s_ < ns and 0 <= d_ < nd):
            raise CopyBlocksError(f"pair ({s_}, {d_}) outside the pools ({ns}, {nd})")
    if len(set(int(d_) for d_ in pairs[:, 1])) != len(pairs):
        raise CopyBlocksError("repeated destination block")
    k, v = dst_k.copy(), dst_v.copy()
    for s_, d_ in pairs:
        k[d_] = src_k[s_]
        v[d_] = src_v[s_]
    return k, v
