"""Python handle on the library's host KV-cache block manager (``pa_kvm_*``,
declared in ``include/pa_kv_manager.h``).

Argument marshalling only: every decision (allocation, reference counts,
copy-on-write pairs, prefix-cache lookups) is made by the C++ manager in
``libpa.so``.  Method names follow the C calls without the prefix.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import _abi


class KvManagerError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = _abi.load().pa_status_string(status)
        super().__init__(f"{fn} failed: {msg.decode() if msg else status}")


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _p(a: np.ndarray) -> int:
    # the address as a plain int (the argument types are c_void_p): half the
    # cost of building a c_void_p object per argument
    return a.ctypes.data


class KvManager:
    """One pool of ``num_blocks`` blocks of ``block_size`` token slots."""

    def __init__(self, num_blocks: int, block_size: int = 16, prefix_caching: bool = False,
                 num_host_blocks: int = 0):
        self._lib = _abi.load()
        self._h = self._lib.pa_kvm_create(num_blocks, block_size, 1 if prefix_caching else 0,
                                          num_host_blocks)
        if not self._h:
            raise ValueError("pa_kvm_create failed (bad sizes or out of memory)")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.prefix_caching = prefix_caching
        # scratch the per-step call reuses: copy pairs and their count
        self._pairs = np.empty((0, 2), np.int64)
        self._pairs_addr = self._pairs.ctypes.data
        self._npairs = ctypes.c_int32(0)
        self._npairs_ref = ctypes.byref(self._npairs)

    def close(self):
        if self._h:
            self._lib.pa_kvm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # noqa: BLE001 -- interpreter shutdown
            pass

    def _check(self, fn, st):
        if st != _abi.PA_OK:
            raise KvManagerError(fn, st)

    # ------------------------------------------------------------------ calls
    def num_free_blocks(self) -> int:
        return self._lib.pa_kvm_num_free_blocks(self._h)

    def add_sequence(self, seq_id: int, tokens):
        """Returns (slots int64[n], cached_tokens)."""
        t = _i32(tokens)
        slots = np.empty(len(t), np.int64)
        cached = ctypes.c_int32(0)
        self._check("pa_kvm_add_sequence",
                    self._lib.pa_kvm_add_sequence(self._h, seq_id, _p(t), len(t), _p(slots),
                                                  ctypes.byref(cached)))
        return slots, cached.value

    def append_tokens(self, seq_id: int, tokens):
        """Returns (slots int64[n], copy pairs as a list of (src, dst))."""
        t = _i32(tokens)
        slots = np.empty(len(t), np.int64)
        pair = np.empty(2, np.int64)
        npairs = ctypes.c_int32(0)
        self._check("pa_kvm_append_tokens",
                    self._lib.pa_kvm_append_tokens(self._h, seq_id, _p(t), len(t), _p(slots),
                                                   _p(pair), ctypes.byref(npairs)))
        return slots, [(int(pair[0]), int(pair[1]))] if npairs.value else []

    def decode_step(self, seq_ids, tokens, slots=None):
        """One new token per sequence, all or nothing.  Returns (slots int64[S],
        copy pairs as a list of (src, dst)); ``slots`` may be given to fill."""
        ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int64))
        t = _i32(tokens)
        if slots is None:
            slots = np.empty(len(ids), np.int64)
        elif slots.shape != (len(ids),) or slots.dtype != np.int64:
            raise ValueError("slots does not match the batch")
        if self._pairs.shape[0] < max(len(ids), 1):
            self._pairs = np.empty((max(len(ids), 1), 2), np.int64)
            self._pairs_addr = self._pairs.ctypes.data
        self._check("pa_kvm_decode_step",
                    self._lib.pa_kvm_decode_step(self._h, _p(ids), len(ids), _p(t), _p(slots),
                                                 self._pairs_addr, self._npairs_ref))
        n = self._npairs.value
        return slots, [(int(a), int(b)) for a, b in self._pairs[:n]] if n else []

    def fork(self, parent: int, child: int):
        self._check("pa_kvm_fork", self._lib.pa_kvm_fork(self._h, parent, child))

    def share_prefix(self, src: int, dst: int, n_blocks: int):
        self._check("pa_kvm_share_prefix", self._lib.pa_kvm_share_prefix(self._h, src, dst, n_blocks))

    def share_blocks(self, src: int, dst: int, idx):
        i = _i32(idx)
        self._check("pa_kvm_share_blocks",
                    self._lib.pa_kvm_share_blocks(self._h, src, dst, _p(i), len(i)))

    def free_sequence(self, seq_id: int):
        self._check("pa_kvm_free_sequence", self._lib.pa_kvm_free_sequence(self._h, seq_id))

    def sequence_info(self, seq_id: int):
        """Returns (context_len, num_blocks)."""
        L, nb = ctypes.c_int32(0), ctypes.c_int32(0)
        self._check("pa_kvm_sequence_info",
                    self._lib.pa_kvm_sequence_info(self._h, seq_id, ctypes.byref(L),
                                                   ctypes.byref(nb)))
        return L.value, nb.value

    def context_len(self, seq_id: int) -> int:
        return self.sequence_info(seq_id)[0]

    def block_table(self, seq_id: int) -> list:
        _, nb = self.sequence_info(seq_id)
        t = np.empty(max(nb, 1), np.int32)
        self._check("pa_kvm_block_table", self._lib.pa_kvm_block_table(self._h, seq_id, _p(t), nb))
        return [int(x) for x in t[:nb]]

    def batch(self, seq_ids, max_blocks: int, out=None):
        """Decode inputs of a batch: (block_tables int32[S, max_blocks], context_lens int32[S]).
        ``out``: optional (tables, lens) arrays of those shapes to fill instead."""
        ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int64))
        if out is None:
            tables = np.empty((len(ids), max_blocks), np.int32)
            lens = np.empty(len(ids), np.int32)
        else:
            tables, lens = out
            if (tables.shape != (len(ids), max_blocks) or tables.dtype != np.int32
                    or not tables.flags.c_contiguous or lens.shape != (len(ids),)
                    or lens.dtype != np.int32):
                raise ValueError("out arrays do not match the batch")
        self._check("pa_kvm_batch",
                    self._lib.pa_kvm_batch(self._h, _p(ids), len(ids), max_blocks, _p(tables),
                                           _p(lens)))
        return tables, lens

    def batch_update(self, seq_ids, out):
        """Bring ``out`` = (tables, lens) from ``batch`` up to date after a
        ``decode_step`` of the same sequences in the same order (writes only
        each sequence's last table entry and its length)."""
        ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int64))
        tables, lens = out
        if (tables.ndim != 2 or tables.shape[0] != len(ids) or tables.dtype != np.int32
                or not tables.flags.c_contiguous or lens.shape != (len(ids),)
                or lens.dtype != np.int32):
            raise ValueError("out arrays do not match the batch")
        self._check("pa_kvm_batch_update",
                    self._lib.pa_kvm_batch_update(self._h, _p(ids), len(ids), tables.shape[1],
                                                  _p(tables), _p(lens)))
        return tables, lens

    def _swap(self, fn, seq_id):
        _, nb = self.sequence_info(seq_id)
        pairs = np.empty((max(nb, 1), 2), np.int64)
        n = ctypes.c_int32(0)
        self._check(fn, getattr(self._lib, fn)(self._h, seq_id, _p(pairs), nb, ctypes.byref(n)))
        return [(int(a), int(b)) for a, b in pairs[:n.value]]

    def swap_out(self, seq_id: int):
        """Move the sequence to host swap space; returns the (device, host) pairs."""
        return self._swap("pa_kvm_swap_out", seq_id)

    def swap_in(self, seq_id: int):
        """Bring it back to fresh device blocks; returns the (host, device) pairs."""
        return self._swap("pa_kvm_swap_in", seq_id)

    def num_free_host_blocks(self) -> int:
        return self._lib.pa_kvm_num_free_host_blocks(self._h)

    def ref_count(self, block: int) -> int:
        return self._lib.pa_kvm_ref_count(self._h, block)
