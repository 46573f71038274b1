"""The library's C++ block manager (``pa_kvm_*``) against the oracle
(``oracle.KvManager``), operation by operation: every returned slot, copy
pair, cached-token count and error, and after every operation every block's
reference count, the free count and each live sequence's table and length.
All integer work, so the comparison is exact.  Runs on the host; no GPU."""
from __future__ import annotations

import ctypes

import numpy as np
import pytest

import oracle
from paged_kv_cache_454_b200 import _abi
from paged_kv_cache_454_b200.kv_manager import KvManager, KvManagerError
from test_kv_manager_oracle import random_ops


def run(target, op):
    kind = op[0]
    try:
        if kind == "add":
            slots, cached = target.add_sequence(op[1], op[2])
            return ("ok", [int(s) for s in slots], cached)
        if kind == "append":
            slots, pairs = target.append_tokens(op[1], op[2])
            return ("ok", [int(s) for s in slots], [tuple(map(int, p)) for p in pairs])
        if kind == "step":
            slots, pairs = target.decode_step(op[1], op[2])
            return ("ok", [int(s) for s in slots], [tuple(map(int, p)) for p in pairs])
        if kind == "fork":
            target.fork(op[1], op[2])
        elif kind == "share_prefix":
            target.share_prefix(op[1], op[2], op[3])
        elif kind == "share_blocks":
            target.share_blocks(op[1], op[2], op[3])
        elif kind == "swap_out":
            return ("ok", [tuple(map(int, p)) for p in target.swap_out(op[1])])
        elif kind == "swap_in":
            return ("ok", [tuple(map(int, p)) for p in target.swap_in(op[1])])
        else:
            target.free_sequence(op[1])
        return ("ok",)
    except oracle.NoBlocks:
        return ("no_blocks",)
    except oracle.KvManagerError:
        return ("arg",)
    except KvManagerError as e:
        return {_abi.PA_ERR_NO_BLOCKS: ("no_blocks",), _abi.PA_ERR_ARG: ("arg",)}.get(
            e.status, ("status", e.status))


def compare_state(ref, lib, live):
    assert lib.num_free_blocks() == ref.num_free_blocks()
    assert lib.num_free_host_blocks() == ref.num_free_host_blocks()
    assert [lib.ref_count(b) for b in range(ref.num_blocks)] == ref.ref
    for sid in live:
        assert lib.block_table(sid) == ref.block_table(sid), sid
        assert lib.context_len(sid) == ref.context_len(sid), sid


@pytest.mark.parametrize("prefix_caching", [False, True])
@pytest.mark.parametrize("seed", range(8))
def test_cpp_manager_matches_oracle_op_by_op(seed, prefix_caching):
    nb, bs = 24, 4
    ref = oracle.KvManager(nb, bs, prefix_caching, 10)
    lib = KvManager(nb, bs, prefix_caching, 10)
    for op in random_ops(seed, 500, nb, bs, prefix_caching):
        a, b = run(ref, op), run(lib, op)
        assert a == b, (op, a, b)
        compare_state(ref, lib, list(ref.seqs))


@pytest.mark.parametrize("prefix_caching", [False, True])
def test_cpp_manager_matches_oracle_on_a_larger_pool(prefix_caching):
    nb, bs = 300, 16
    ref = oracle.KvManager(nb, bs, prefix_caching, 60)
    lib = KvManager(nb, bs, prefix_caching, 60)
    for i, op in enumerate(random_ops(100 + int(prefix_caching), 1500, nb, bs, prefix_caching)):
        assert run(ref, op) == run(lib, op), op
        if i % 50 == 0:
            compare_state(ref, lib, list(ref.seqs))
    compare_state(ref, lib, list(ref.seqs))


def test_batch_builds_decode_inputs():
    m = KvManager(64, 16)
    m.add_sequence(7, np.arange(40))
    m.add_sequence(3, np.arange(5))
    m.fork(7, 8)
    m.append_tokens(8, [1])
    tables, lens = m.batch([7, 3, 8], 4)
    assert lens.tolist() == [40, 5, 41]
    assert tables[0, :3].tolist() == m.block_table(7) and tables[0, 3] == -1
    assert tables[1, 0] == m.block_table(3)[0] and (tables[1, 1:] == -1).all()
    assert tables[2, :3].tolist() == m.block_table(8)
    with pytest.raises(KvManagerError) as e:
        m.batch([7], 2)
    assert e.value.status == _abi.PA_ERR_SHAPE
    with pytest.raises(KvManagerError) as e:
        m.batch([99], 4)
    assert e.value.status == _abi.PA_ERR_ARG


def test_host_argument_checks():
    lib = _abi.load()
    assert not lib.pa_kvm_create(0, 16, 0, 0)
    assert not lib.pa_kvm_create(4, 0, 0, 0)
    h = lib.pa_kvm_create(8, 4, 1, 0)
    try:
        slots = (ctypes.c_int64 * 4)()
        toks = (ctypes.c_int32 * 4)(1, 2, 3, 4)
        # prefix caching needs token ids
        assert lib.pa_kvm_add_sequence(h, 1, None, 4, slots, None) == _abi.PA_ERR_ARG
        assert lib.pa_kvm_add_sequence(h, 1, toks, -1, slots, None) == _abi.PA_ERR_ARG
        assert lib.pa_kvm_add_sequence(h, 1, toks, 4, None, None) == _abi.PA_ERR_ARG
        assert lib.pa_kvm_add_sequence(h, 1, toks, 4, slots, None) == _abi.PA_OK
        assert lib.pa_kvm_add_sequence(h, 1, toks, 4, slots, None) == _abi.PA_ERR_ARG  # duplicate
        npairs = ctypes.c_int32(0)
        assert lib.pa_kvm_append_tokens(h, 2, toks, 1, slots, None, ctypes.byref(npairs)) == \
            _abi.PA_ERR_ARG  # unknown sequence
        assert lib.pa_kvm_ref_count(h, -1) == -1 and lib.pa_kvm_ref_count(h, 8) == -1
        assert lib.pa_kvm_num_free_blocks(h) == 7
    finally:
        lib.pa_kvm_destroy(h)
    lib.pa_kvm_destroy(None)


def test_without_prefix_caching_tokens_may_be_omitted():
    lib = _abi.load()
    h = lib.pa_kvm_create(8, 4, 0, 0)
    try:
        slots = (ctypes.c_int64 * 6)()
        assert lib.pa_kvm_add_sequence(h, 1, None, 6, slots, None) == _abi.PA_OK
        assert list(slots) == [0, 1, 2, 3, 4, 5]
        npairs = ctypes.c_int32(0)
        pair = (ctypes.c_int64 * 2)()
        assert lib.pa_kvm_append_tokens(h, 1, None, 3, slots, pair, ctypes.byref(npairs)) == _abi.PA_OK
        assert list(slots)[:3] == [6, 7, 8] and npairs.value == 0
    finally:
        lib.pa_kvm_destroy(h)


def test_batch_update_tracks_decode_steps():
    m = KvManager(400, 16, prefix_caching=False)
    rng = np.random.default_rng(3)
    ids = list(range(12))
    for i in ids:
        m.add_sequence(i, np.zeros(int(rng.integers(1, 60)), np.int32))
    for i in (1, 2, 3):
        m.fork(0, 100 + i)          # shared partial blocks: steps copy them
    ids += [101, 102, 103]
    out = m.batch(ids, 12)
    for step in range(40):
        _, pairs = m.decode_step(ids, np.zeros(len(ids), np.int32))
        m.batch_update(ids, out)
        full = m.batch(ids, 12)
        assert np.array_equal(out[0], full[0]) and np.array_equal(out[1], full[1]), step
