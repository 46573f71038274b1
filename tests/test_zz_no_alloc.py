"""pa_decode_noalloc: the decode entry point for callers that cannot allocate
device memory (a process that gave all free HBM to its KV pool, or a framework
op interface with no workspace argument).  It takes its split-context scratch
from a fixed array inside the library instead of a caller workspace.

Checked through the C ABI against pa_decode (which takes a caller workspace)
on calls in a row over different batches: the shared array keeps the previous
call's contents, and no call may depend on them.  This file is collected last
so that a run stopping at the first failure has run every other test first.
"""
import ctypes

import numpy as np
import pytest

from workloads import synth

import gpu_helpers as H

pytestmark = pytest.mark.gpu


def _layouts():
    # several 128-token tiles, split partitions and ragged tails; a GQA batch
    # (group 8), a group-5 batch and an MHA batch
    return [
        synth.build_layout("na_gqa8", 201, [1, 130, 1025, 3000, 4100], num_q_heads=16,
                           num_kv_heads=2, head_dim=128),
        synth.build_layout("na_gqa5", 202, [700, 2222, 9], num_q_heads=10, num_kv_heads=2,
                           head_dim=128),
        synth.build_layout("na_mha", 203, [17, 1500, 2049, 64], num_q_heads=4, num_kv_heads=4,
                           head_dim=128),
    ]


def _prepared(lay):
    import paged_kv_cache_454_b200 as pa
    st = H.Step.from_host(lay)
    pa.pa_reshape_and_cache(st.key, st.value, st.k_pool, st.v_pool, st.slot_mapping)
    return st


def _noalloc_via_abi(st):
    """Call pa_decode_noalloc through the C ABI; returns (out, lse) tensors."""
    import torch
    from paged_kv_cache_454_b200 import _abi
    lay = st.layout
    lib = _abi.load()
    out = torch.full(st.q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full(st.q.shape[:2], float("nan"), dtype=torch.float32, device="cuda")
    status = lib.pa_decode_noalloc(
        st.q.data_ptr(), st.q.stride(0), st.k_pool.data_ptr(), st.v_pool.data_ptr(),
        _abi.PoolDesc(*st.k_pool.shape), st.tables.data_ptr(), lay.max_blocks,
        st.lens.data_ptr(), lay.num_seqs, lay.num_q_heads, ctypes.c_float(lay.scale),
        out.data_ptr(), lse.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert status == _abi.PA_OK, lib.pa_status_string(status)
    torch.cuda.synchronize()
    return out, lse


def test_noalloc_matches_pa_decode_on_calls_in_a_row():
    import paged_kv_cache_454_b200 as pa
    steps = [_prepared(lay) for lay in _layouts()]
    refs = []
    for st in steps:
        out, lse = pa.pa_decode(st.q, st.k_pool, st.v_pool, st.tables, st.lens, st.layout.scale,
                                want_lse=True)
        refs.append((H.host_f64(out), lse.cpu().numpy()))
    # A, B, C, then A again: each call follows one on a different batch
    for i in [0, 1, 2, 0]:
        out, lse = _noalloc_via_abi(steps[i])
        H.assert_close(H.host_f64(out), refs[i][0], what=f"noalloc {steps[i].layout.name}")
        H.assert_lse_close(lse.cpu().numpy(), refs[i][1], what=f"noalloc {steps[i].layout.name}")
    assert pa.pa_get_device_error() == 0


def test_noalloc_rejects_batches_beyond_its_scratch():
    import torch
    from paged_kv_cache_454_b200 import _abi
    lib = _abi.load()
    lay = _layouts()[0]
    st = _prepared(lay)
    # 64 sequences with tables of 16384 blocks (4 MiB of int32) need about
    # 135 MB of split-context scratch, twice what the array holds: rejected on
    # the host, nothing launched.  Every buffer is sized for the declared
    # shapes (q rows, lengths, table width), so a launch, were the check ever
    # to regress, would read nothing out of bounds and the assert below fails
    # cleanly instead.
    S, hq, mb = 64, lay.num_q_heads, 16384
    pool = _abi.PoolDesc(*st.k_pool.shape)
    need = lib.pa_decode_workspace_size(S, hq, pool, mb)
    assert need > _abi.PA_NOALLOC_SCRATCH_BYTES
    q = torch.zeros((S, hq, lay.head_dim), dtype=torch.bfloat16, device="cuda")
    lens = torch.zeros(S, dtype=torch.int32, device="cuda")
    tables = torch.zeros((S, mb), dtype=torch.int32, device="cuda")
    out = torch.zeros((S, hq, lay.head_dim), dtype=torch.bfloat16, device="cuda")
    status = lib.pa_decode_noalloc(
        q.data_ptr(), q.stride(0), st.k_pool.data_ptr(), st.v_pool.data_ptr(), pool,
        tables.data_ptr(), mb, lens.data_ptr(), S, hq, ctypes.c_float(lay.scale),
        out.data_ptr(), None, torch.cuda.current_stream().cuda_stream)
    assert status == _abi.PA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0  # nothing ran
