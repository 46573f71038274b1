"""PagedAttention over a block-paged KV pool, for NVIDIA B200 (sm_100a).

The work runs in ``libpa.so`` (hand-written CUDA, C ABI in ``include/pa.h``).
This module only marshals torch tensors (device memory, streams) into that ABI;
the function names are the C names.  There is no fallback: if the library is
missing or a tensor is not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import _abi
from ._abi import (PA_DEV_ERR_BLOCK_ID, PA_DEV_ERR_CONTEXT, PA_DEV_ERR_SLOT,  # noqa: F401
                   PA_DEV_ERR_TIMEOUT, PA_KERNEL_AUTO, PA_KERNEL_SIMT, PA_KERNEL_TCGEN05,
                   PA_PREFILL_EXACT_WEIGHTS, PaError, PoolDesc)

__all__ = [
    "pa_reshape_and_cache", "pa_copy_blocks", "pa_decode", "pa_decode_workspace_size",
    "pa_decode_noalloc",
    "pa_chunked_prefill", "pa_gather_kv", "pa_get_device_error", "pa_sample", "pa_swap_blocks",
    "pa_read_probe",
    "pool_desc", "lib",
    "PaError", "PA_KERNEL_AUTO", "PA_KERNEL_SIMT", "PA_KERNEL_TCGEN05",
    "PA_PREFILL_EXACT_WEIGHTS",
]


def lib():
    return _abi.load()


def _torch():
    import torch
    return torch


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _need_cuda(name, t, dtype=None, contiguous=True):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def pool_desc(k_pool) -> PoolDesc:
    """Descriptor of a ``[num_blocks, num_kv_heads, block_size, head_dim]`` pool."""
    nb, hkv, bs, d = k_pool.shape
    return PoolDesc(nb, hkv, bs, d)


def _check_pools(k_pool, v_pool):
    torch = _torch()
    _need_cuda("k_pool", k_pool, torch.bfloat16)
    _need_cuda("v_pool", v_pool, torch.bfloat16)
    if k_pool.dim() != 4 or k_pool.shape != v_pool.shape:
        raise ValueError("k_pool and v_pool must be [num_blocks, Hkv, block_size, D] alike")


def _row_stride(name, t):
    """Token stride (elements) of a [T, H, D] tensor whose heads are packed."""
    if t.dim() != 3 or t.stride(2) != 1 or t.stride(1) != t.shape[2]:
        raise ValueError(f"{name} must be [T, H, D] with packed heads")
    return t.stride(0)


def pa_reshape_and_cache(key, value, k_pool, v_pool, slot_mapping, stream=None) -> None:
    """Write new tokens' K/V (bf16 [T, Hkv, D]) into the pools at ``slot_mapping``
    (int64 [T]; negative = skip)."""
    torch = _torch()
    _check_pools(k_pool, v_pool)
    _need_cuda("key", key, torch.bfloat16, contiguous=False)
    _need_cuda("value", value, torch.bfloat16, contiguous=False)
    _need_cuda("slot_mapping", slot_mapping, torch.int64)
    ks, vs = _row_stride("key", key), _row_stride("value", value)
    if ks != vs:
        raise ValueError("key and value must share a token stride")
    _abi.check("pa_reshape_and_cache", lib().pa_reshape_and_cache(
        _ptr(key), _ptr(value), ks, _ptr(k_pool), _ptr(v_pool), pool_desc(k_pool),
        _ptr(slot_mapping), key.shape[0], _stream(stream)))


def pa_copy_blocks(k_pool, v_pool, pairs, stream=None) -> None:
    """Copy whole blocks src -> dst in both pools.  ``pairs``: host int64 [P, 2]."""
    _check_pools(k_pool, v_pool)
    arr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int64).reshape(-1, 2))
    _abi.check("pa_copy_blocks", lib().pa_copy_blocks(
        _ptr(k_pool), _ptr(v_pool), pool_desc(k_pool),
        arr.ctypes.data_as(ctypes.c_void_p), arr.shape[0], _stream(stream)))


def pa_decode_workspace_size(num_seqs, num_q_heads, k_pool, max_blocks_per_seq,
                             partition_tokens=0) -> int:
    return int(lib().pa_decode_workspace_size_ex(num_seqs, num_q_heads, pool_desc(k_pool),
                                                 max_blocks_per_seq, partition_tokens))


def pa_decode(q, k_pool, v_pool, block_tables, context_lens, scale, out=None, lse=None,
              workspace=None, partition_tokens=0, kernel=PA_KERNEL_AUTO, stream=None,
              want_lse=False):
    """Single-query paged attention.  ``q`` bf16 [S, Hq, D]; ``block_tables`` int32
    [S, max_blocks]; ``context_lens`` int32 [S].  Returns ``(out, lse)``; ``lse``
    is None unless given or ``want_lse``."""
    torch = _torch()
    _check_pools(k_pool, v_pool)
    _need_cuda("q", q, torch.bfloat16, contiguous=False)
    _need_cuda("block_tables", block_tables, torch.int32)
    _need_cuda("context_lens", context_lens, torch.int32)
    S, hq, d = q.shape
    qs = _row_stride("q", q)
    if out is None:
        out = torch.empty((S, hq, d), dtype=torch.bfloat16, device=q.device)
    _need_cuda("out", out, torch.bfloat16)
    if lse is None and want_lse:
        lse = torch.empty((S, hq), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need_cuda("lse", lse, torch.float32)
    mb = block_tables.shape[1]
    if workspace is None:
        n = pa_decode_workspace_size(S, hq, k_pool, mb, partition_tokens)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
    _need_cuda("workspace", workspace, torch.uint8)
    _abi.check("pa_decode_ex", lib().pa_decode_ex(
        _ptr(q), qs, _ptr(k_pool), _ptr(v_pool), pool_desc(k_pool), _ptr(block_tables), mb,
        _ptr(context_lens), S, hq, float(scale), _ptr(out), _ptr(lse), _ptr(workspace),
        workspace.numel(), int(partition_tokens), int(kernel), _stream(stream)))
    return out, lse


def pa_decode_noalloc(q, k_pool, v_pool, block_tables, context_lens, scale, out=None, lse=None,
                      stream=None, want_lse=False):
    """``pa_decode`` for callers that cannot allocate device memory: the split
    scratch comes from a fixed array inside the library (``_abi.PA_NOALLOC_SCRATCH_BYTES``
    per device, shared by all calls on the device, so calls must not overlap on
    the GPU).  This wrapper itself allocates ``out``/``lse`` only when they are
    not given."""
    torch = _torch()
    _check_pools(k_pool, v_pool)
    _need_cuda("q", q, torch.bfloat16, contiguous=False)
    _need_cuda("block_tables", block_tables, torch.int32)
    _need_cuda("context_lens", context_lens, torch.int32)
    S, hq, d = q.shape
    qs = _row_stride("q", q)
    if out is None:
        out = torch.empty((S, hq, d), dtype=torch.bfloat16, device=q.device)
    _need_cuda("out", out, torch.bfloat16)
    if lse is None and want_lse:
        lse = torch.empty((S, hq), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need_cuda("lse", lse, torch.float32)
    _abi.check("pa_decode_noalloc", lib().pa_decode_noalloc(
        _ptr(q), qs, _ptr(k_pool), _ptr(v_pool), pool_desc(k_pool), _ptr(block_tables),
        block_tables.shape[1], _ptr(context_lens), S, hq, float(scale), _ptr(out), _ptr(lse),
        _stream(stream)))
    return out, lse


def pa_chunked_prefill(q, cu_q_lens, max_q_len, k_pool, v_pool, block_tables, context_lens,
                       scale, out=None, lse=None, stream=None, want_lse=False,
                       exact_weights=False):
    """Causal attention of each sequence's new chunk over its cached context plus
    itself.  ``q`` bf16 [total_q, Hq, D]; ``cu_q_lens`` int32 [S+1] (device).
    ``exact_weights`` asks for the weights' bf16 remainder on every key tile
    (``pa_chunked_prefill_ex`` with ``PA_PREFILL_EXACT_WEIGHTS``)."""
    torch = _torch()
    _check_pools(k_pool, v_pool)
    _need_cuda("q", q, torch.bfloat16, contiguous=False)
    _need_cuda("cu_q_lens", cu_q_lens, torch.int32)
    _need_cuda("block_tables", block_tables, torch.int32)
    _need_cuda("context_lens", context_lens, torch.int32)
    total_q, hq, d = q.shape
    qs = _row_stride("q", q)
    if out is None:
        out = torch.empty((total_q, hq, d), dtype=torch.bfloat16, device=q.device)
    _need_cuda("out", out, torch.bfloat16)
    if lse is None and want_lse:
        lse = torch.empty((total_q, hq), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need_cuda("lse", lse, torch.float32)
    S = context_lens.shape[0]
    if exact_weights:
        _abi.check("pa_chunked_prefill_ex", lib().pa_chunked_prefill_ex(
            _ptr(q), qs, _ptr(cu_q_lens), total_q, int(max_q_len), _ptr(k_pool), _ptr(v_pool),
            pool_desc(k_pool), _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), S,
            hq, float(scale), _ptr(out), _ptr(lse), PA_PREFILL_EXACT_WEIGHTS, _stream(stream)))
    else:
        _abi.check("pa_chunked_prefill", lib().pa_chunked_prefill(
            _ptr(q), qs, _ptr(cu_q_lens), total_q, int(max_q_len), _ptr(k_pool), _ptr(v_pool),
            pool_desc(k_pool), _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), S,
            hq, float(scale), _ptr(out), _ptr(lse), _stream(stream)))
    return out, lse


def pa_gather_kv(k_pool, v_pool, block_tables, context_lens, cu_kv_lens, max_context,
                 total_tokens, stream=None):
    """Contiguous copies ``[total_tokens, Hkv, D]`` of every sequence's K and V."""
    torch = _torch()
    _check_pools(k_pool, v_pool)
    _need_cuda("block_tables", block_tables, torch.int32)
    _need_cuda("context_lens", context_lens, torch.int32)
    _need_cuda("cu_kv_lens", cu_kv_lens, torch.int32)
    _, hkv, _, d = k_pool.shape
    k_out = torch.empty((total_tokens, hkv, d), dtype=torch.bfloat16, device=k_pool.device)
    v_out = torch.empty_like(k_out)
    _abi.check("pa_gather_kv", lib().pa_gather_kv(
        _ptr(k_pool), _ptr(v_pool), pool_desc(k_pool), _ptr(block_tables), block_tables.shape[1],
        _ptr(context_lens), _ptr(cu_kv_lens), context_lens.shape[0], int(max_context),
        _ptr(k_out), _ptr(v_out), _stream(stream)))
    return k_out, v_out


def pa_get_device_error(stream=None) -> int:
    """Wait for ``stream`` and return-and-clear the device error word."""
    v = ctypes.c_uint32(0)
    _abi.check("pa_get_device_error", lib().pa_get_device_error(ctypes.byref(v), _stream(stream)))
    return int(v.value)


def pa_sample(logits, temperature, top_k, top_p, uniform, out=None, stream=None):
    """Fused temperature / Top-K / Top-P sampling, one token per row of ``logits``
    (fp32 [rows, vocab], rows contiguous).  ``temperature``, ``top_p``, ``uniform``:
    fp32 [rows]; ``top_k``: int32 [rows]; all CUDA tensors.  Returns int32 [rows]."""
    torch = _torch()
    _need_cuda("logits", logits, torch.float32, contiguous=False)
    if logits.dim() != 2 or logits.stride(1) != 1:
        raise ValueError("logits must be [rows, vocab] with unit stride along the vocabulary")
    rows, vocab = logits.shape
    for name, t, dt in (("temperature", temperature, torch.float32), ("top_k", top_k, torch.int32),
                        ("top_p", top_p, torch.float32), ("uniform", uniform, torch.float32)):
        _need_cuda(name, t, dt)
        if t.shape != (rows,):
            raise ValueError(f"{name} must have shape ({rows},)")
    if out is None:
        out = torch.empty(rows, dtype=torch.int32, device=logits.device)
    _need_cuda("out", out, torch.int32)
    _abi.check("pa_sample", lib().pa_sample(
        _ptr(logits), logits.stride(0), rows, vocab, _ptr(temperature), _ptr(top_k),
        _ptr(top_p), _ptr(uniform), _ptr(out), _stream(stream)))
    return out


def pa_swap_blocks(k_pool, v_pool, k_host, v_host, pairs, direction, stream=None) -> None:
    """Copy whole blocks between the device pools and page-locked host pools of
    the same block shape (``k_host``/``v_host``: pinned CPU tensors).
    ``direction``: ``_abi.PA_SWAP_OUT`` (device src -> host dst) or
    ``_abi.PA_SWAP_IN`` (host src -> device dst); ``pairs``: int64 [P, 2]."""
    torch = _torch()
    _check_pools(k_pool, v_pool)
    for name, t in (("k_host", k_host), ("v_host", v_host)):
        if not isinstance(t, torch.Tensor) or t.is_cuda or not t.is_pinned():
            raise TypeError(f"{name} must be a pinned CPU tensor")
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.shape[1:] != k_pool.shape[1:]:
            raise ValueError(f"{name} must be bf16 [num_host_blocks, {tuple(k_pool.shape[1:])}]")
    arr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int64).reshape(-1, 2))
    _abi.check("pa_swap_blocks", lib().pa_swap_blocks(
        _ptr(k_pool), _ptr(v_pool), pool_desc(k_pool), _ptr(k_host), _ptr(v_host),
        k_host.shape[0], arr.ctypes.data_as(ctypes.c_void_p), arr.shape[0], int(direction),
        _stream(stream)))


def pa_read_probe(k_pool, v_pool, block_tables, context_lens, num_ctas=None, out=None,
                  stream=None):
    """Read every K/V page a decode over ``block_tables`` / ``context_lens``
    reads, and nothing else (a read-bandwidth measurement).  Returns the
    per-CTA sums (int64 [num_ctas], the bits of uint64 sums modulo 2^64) of the
    pages' 32-bit words; ``num_ctas`` defaults to the SM count."""
    torch = _torch()
    _check_pools(k_pool, v_pool)
    _need_cuda("block_tables", block_tables, torch.int32)
    _need_cuda("context_lens", context_lens, torch.int32)
    if block_tables.dim() != 2 or block_tables.shape[0] != context_lens.shape[0]:
        raise ValueError("block_tables must be [S, max_blocks] with S = len(context_lens)")
    if num_ctas is None:
        num_ctas = torch.cuda.get_device_properties(k_pool.device).multi_processor_count
    if out is None:
        out = torch.empty(num_ctas, dtype=torch.int64, device=k_pool.device)
    _need_cuda("out", out, torch.int64)
    if out.numel() < num_ctas:
        raise ValueError("out holds fewer than num_ctas sums")
    _abi.check("pa_read_probe", lib().pa_read_probe(
        _ptr(k_pool), _ptr(v_pool), pool_desc(k_pool), _ptr(block_tables), block_tables.shape[1],
        _ptr(context_lens), context_lens.shape[0], _ptr(out), int(num_ctas), _stream(stream)))
    return out
