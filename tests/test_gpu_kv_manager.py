"""The C++ block manager driving the device path, end to end on a GPU.

A prompt is prefilled, forked into samples that decode step by step (the
first writers of the shared partial block get copy-on-write pairs), and a
later request reuses the prompt's full blocks through the prefix cache.  At
every step the manager's slots, copy pairs and batch tables feed
``pa_copy_blocks``, ``pa_reshape_and_cache`` and ``pa_decode``; the test keeps
each sequence's own K/V rows on the host, unshared.  Checks:

* ``pa_gather_kv`` through the manager's tables returns exactly each
  sequence's rows (bit-exact: sharing, copies and cached blocks are right);
* decode equals the oracle run on an unshared, contiguous copy of every
  sequence ("vLLM 基本原理", memory sharing: shared physical blocks give the
  same attention as private copies).
"""
from __future__ import annotations

import numpy as np
import pytest

import gpu_helpers as H
import oracle
from workloads import synth

pytestmark = pytest.mark.gpu

HKV, HQ, D, BS, NB = 2, 8, 128, 16, 64


def pa():
    import paged_kv_cache_454_b200 as m
    return m


def unshared_pools(rows):
    """Each sequence's (K, V) rows [L, Hkv, D] copied into private blocks of a
    fresh pool: tables, lengths, k_pool, v_pool (bf16 bits)."""
    nblk = [-(-len(k) // BS) for k, _ in rows]
    total = max(1, sum(nblk))
    kp = np.zeros((total, HKV, BS, D), np.uint16)
    vp = np.zeros_like(kp)
    tables = np.zeros((len(rows), max(nblk + [1])), np.int32)
    b = 0
    for s, (k, v) in enumerate(rows):
        for j in range(nblk[s]):
            tables[s, j] = b
            seg = slice(j * BS, min((j + 1) * BS, len(k)))
            n = seg.stop - seg.start
            kp[b, :, :n] = k[seg].transpose(1, 0, 2)
            vp[b, :, :n] = v[seg].transpose(1, 0, 2)
            b += 1
    return tables, np.array([len(k) for k, _ in rows], np.int32), kp, vp


def test_manager_drives_cache_writes_copies_and_decode():
    torch = H.torch()
    from paged_kv_cache_454_b200.kv_manager import KvManager
    rng = np.random.default_rng(7)
    m = KvManager(NB, BS, prefix_caching=True)
    k_pool = H.dev_bf16(synth.normal_bf16(rng, (NB, HKV, BS, D)))
    v_pool = H.dev_bf16(synth.normal_bf16(rng, (NB, HKV, BS, D)))
    rows = {}  # seq -> [K rows, V rows] (bf16 bits [L, Hkv, D])

    def write(slots, k, v):
        pa().pa_reshape_and_cache(H.dev_bf16(k), H.dev_bf16(v), k_pool, v_pool, H.dev_i64(slots))

    # prompt of 40 tokens: two full blocks and a partial one
    prompt = list(rng.integers(0, 1000, 40))
    k0, v0 = synth.normal_bf16(rng, (40, HKV, D)), synth.normal_bf16(rng, (40, HKV, D))
    slots, cached = m.add_sequence(0, prompt)
    assert cached == 0
    write(slots, k0, v0)
    rows[0] = [k0, v0]
    for c in (1, 2):
        m.fork(0, c)
        rows[c] = [k0.copy(), v0.copy()]
    # a later request whose first 32 tokens match: those rows come from the cache
    p3 = prompt[:32] + list(rng.integers(0, 1000, 9))
    slots3, cached3 = m.add_sequence(3, p3)
    assert cached3 == 32 and (slots3[:32] == -1).all()
    k3 = np.concatenate([k0[:32], synth.normal_bf16(rng, (9, HKV, D))])
    v3 = np.concatenate([v0[:32], synth.normal_bf16(rng, (9, HKV, D))])
    write(slots3, k3, v3)  # the cached rows are skipped (slot -1)
    rows[3] = [k3, v3]

    seqs = [0, 1, 2, 3]
    pairs_seen = 0
    for step in range(20):
        # one new token per sequence: slots and copy-on-write pairs from the manager
        new_slots, pairs = m.decode_step(seqs, rng.integers(0, 1000, len(seqs)))
        if pairs:
            pa().pa_copy_blocks(k_pool, v_pool, np.array(pairs, np.int64))
            pairs_seen += len(pairs)
        new_k = synth.normal_bf16(rng, (len(seqs), HKV, D))
        new_v = synth.normal_bf16(rng, (len(seqs), HKV, D))
        for i, s in enumerate(seqs):
            rows[s][0] = np.concatenate([rows[s][0], new_k[i:i + 1]])
            rows[s][1] = np.concatenate([rows[s][1], new_v[i:i + 1]])
        write(new_slots, new_k, new_v)
        tables, lens = m.batch(seqs, 8)
        q = synth.normal_bf16(rng, (len(seqs), HQ, D))
        scale = 1.0 / np.sqrt(D)
        out, lse = pa().pa_decode(H.dev_bf16(q), k_pool, v_pool, H.dev_i32(tables),
                                  H.dev_i32(lens), scale, want_lse=True)
        ut, ul, ukp, uvp = unshared_pools([rows[s] for s in seqs])
        ref_o, ref_l = oracle.decode(q, ukp, uvp, ut, ul, scale)
        H.assert_close(H.host_f64(out), ref_o, what=f"step {step}")
        H.assert_lse_close(lse.cpu().numpy(), ref_l, what=f"step {step}")
    # the two forks and the parent shared a partial block: the first two writers copied it
    assert pairs_seen == 2

    # every sequence read back through the manager's tables, bit for bit
    tables, lens = m.batch(seqs, 8)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    k, v = pa().pa_gather_kv(k_pool, v_pool, H.dev_i32(tables), H.dev_i32(lens), H.dev_i32(cu),
                             int(lens.max()), int(cu[-1]))
    kb, vb = H.host_bits(k), H.host_bits(v)
    for i, s in enumerate(seqs):
        assert np.array_equal(kb[cu[i]:cu[i + 1]], rows[s][0])
        assert np.array_equal(vb[cu[i]:cu[i + 1]], rows[s][1])
    assert pa().pa_get_device_error() == 0
    torch.cuda.synchronize()


def test_swap_blocks_bit_exact():
    torch = H.torch()
    rng = np.random.default_rng(9)
    nb, nh = 40, 12
    kd = synth.normal_bf16(rng, (nb, HKV, BS, D))
    vd = synth.normal_bf16(rng, (nb, HKV, BS, D))
    kh = synth.normal_bf16(rng, (nh, HKV, BS, D))
    vh = synth.normal_bf16(rng, (nh, HKV, BS, D))
    k_pool, v_pool = H.dev_bf16(kd), H.dev_bf16(vd)
    k_host = torch.from_numpy(kh.view(np.int16)).view(torch.bfloat16).pin_memory()
    v_host = torch.from_numpy(vh.view(np.int16)).view(torch.bfloat16).pin_memory()
    out_pairs = np.array([[3, 0], [7, 5], [39, 11], [7, 2]], np.int64)   # a source twice
    pa().pa_swap_blocks(k_pool, v_pool, k_host, v_host, out_pairs, 0)
    torch.cuda.synchronize()
    rk, rv = oracle.swap_blocks(kd, vd, kh, vh, out_pairs)
    assert np.array_equal(k_host.view(torch.int16).numpy().view(np.uint16), rk)
    assert np.array_equal(v_host.view(torch.int16).numpy().view(np.uint16), rv)
    in_pairs = np.array([[0, 1], [11, 2], [4, 30]], np.int64)
    pa().pa_swap_blocks(k_pool, v_pool, k_host, v_host, in_pairs, 1)
    rk2, rv2 = oracle.swap_blocks(rk, rv, kd, vd, in_pairs)
    assert np.array_equal(H.host_bits(k_pool), rk2) and np.array_equal(H.host_bits(v_pool), rv2)
    from paged_kv_cache_454_b200 import _abi
    with pytest.raises(pa().PaError):
        pa().pa_swap_blocks(k_pool, v_pool, k_host, v_host, np.array([[0, 12]]), 0)  # host id out
    with pytest.raises(pa().PaError):
        pa().pa_swap_blocks(k_pool, v_pool, k_host, v_host, np.array([[0, 1], [2, 1]]), 0)
    assert _abi.PA_SWAP_IN == 1


def test_manager_swaps_a_sequence_out_and_back():
    torch = H.torch()
    from paged_kv_cache_454_b200.kv_manager import KvManager
    rng = np.random.default_rng(13)
    nb, nh = 8, 8
    m = KvManager(nb, BS, num_host_blocks=nh)
    k_pool = H.dev_bf16(synth.normal_bf16(rng, (nb, HKV, BS, D)))
    v_pool = H.dev_bf16(synth.normal_bf16(rng, (nb, HKV, BS, D)))
    k_host = torch.empty((nh, HKV, BS, D), dtype=torch.bfloat16).pin_memory()
    v_host = torch.empty((nh, HKV, BS, D), dtype=torch.bfloat16).pin_memory()
    rows = {}
    for s, n in ((0, 70), (1, 20)):
        slots, _ = m.add_sequence(s, np.zeros(n, np.int32))
        k, v = synth.normal_bf16(rng, (n, HKV, D)), synth.normal_bf16(rng, (n, HKV, D))
        pa().pa_reshape_and_cache(H.dev_bf16(k), H.dev_bf16(v), k_pool, v_pool, H.dev_i64(slots))
        rows[s] = [k, v]
    # sequence 0 (5 blocks) moves out; sequence 2 takes its device blocks
    pa().pa_swap_blocks(k_pool, v_pool, k_host, v_host, m.swap_out(0), 0)
    slots2, _ = m.add_sequence(2, np.zeros(80, np.int32))
    k2, v2 = synth.normal_bf16(rng, (80, HKV, D)), synth.normal_bf16(rng, (80, HKV, D))
    pa().pa_reshape_and_cache(H.dev_bf16(k2), H.dev_bf16(v2), k_pool, v_pool, H.dev_i64(slots2))
    rows[2] = [k2, v2]
    m.free_sequence(2)
    del rows[2]
    pa().pa_swap_blocks(k_pool, v_pool, k_host, v_host, m.swap_in(0), 1)
    seqs = [0, 1]
    tables, lens = m.batch(seqs, 8)
    q = synth.normal_bf16(rng, (2, HQ, D))
    out, lse = pa().pa_decode(H.dev_bf16(q), k_pool, v_pool, H.dev_i32(tables), H.dev_i32(lens),
                              0.125, want_lse=True)
    ut, ul, ukp, uvp = unshared_pools([rows[s] for s in seqs])
    ref_o, ref_l = oracle.decode(q, ukp, uvp, ut, ul, 0.125)
    H.assert_close(H.host_f64(out), ref_o, what="after swap in")
    H.assert_lse_close(lse.cpu().numpy(), ref_l, what="after swap in")
    assert pa().pa_get_device_error() == 0
