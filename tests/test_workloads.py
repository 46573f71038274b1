"""Host-side checks of the seeded batch builder (integer bookkeeping only)."""
import math

import numpy as np
import pytest

from workloads import synth


def _check_layout(lay):
    bs = lay.block_size
    S = lay.num_seqs
    # on-demand allocation: a sequence holds exactly ceil(L / bs) blocks, and
    # only its last block may be partly filled
    for s in range(S):
        nb = lay.blocks_used(s)
        assert nb == math.ceil(int(lay.context_lens[s]) / bs)
        row = lay.block_tables[s]
        assert np.all((row[:nb] >= 0) & (row[:nb] < lay.num_blocks))
        assert np.all(row[nb:] == synth.INT32_MAX)
    # ref counts match the tables
    ref = np.zeros(lay.num_blocks, np.int64)
    for s in range(S):
        for p in lay.block_tables[s, : lay.blocks_used(s)]:
            ref[p] += 1
    assert np.array_equal(ref, lay.ref_counts)
    # new-token slots are distinct and inside the pool
    sm = lay.slot_mapping()
    assert len(np.unique(sm)) == len(sm) == int(lay.q_lens.sum())
    assert np.all((sm >= 0) & (sm < lay.num_blocks * bs))
    # a new token's slot is never in a block another sequence reads
    for slot in sm:
        assert ref[slot // bs] == 1


@pytest.mark.parametrize("name", list(synth.CONFIGS))
def test_named_layouts(name):
    lay = synth.CONFIGS[name]()
    _check_layout(lay)
    assert lay.block_size == 16


def test_tiny_matches_its_description():
    lay = synth.tiny()
    assert list(lay.context_lens) == [1, 17, 33, 64]
    assert (lay.num_q_heads, lay.num_kv_heads, lay.head_dim, lay.num_blocks) == (4, 4, 64, 32)
    assert sum(lay.blocks_used(s) for s in range(4)) == 10
    assert lay.scale == 1 / 8


def test_llama7b_shape():
    lay = synth.llama7b_decode()
    assert lay.num_seqs == 64 and lay.num_q_heads == lay.num_kv_heads == 32
    assert lay.context_lens.min() >= 128 and lay.context_lens.max() <= 2048
    need = sum(lay.blocks_used(s) for s in range(64))
    assert lay.num_blocks == math.ceil(1.25 * need)


def test_llama13b_sharing_and_cow():
    lay = synth.llama13b_sampling()
    assert lay.num_seqs == 256 and lay.copy_pairs.shape == (192, 2)
    for g in range(64):
        rows = lay.block_tables[4 * g: 4 * g + 4]
        # 31 prompt blocks shared by all four samples (ref count 4)
        assert np.all(rows[:, :31] == rows[0, :31])
        assert np.all(lay.ref_counts[rows[0, :31]] == 4)
        # logical block 31: sample 0 keeps the original, samples 1-3 own copies
        assert len(set(rows[:, 31].tolist())) == 4
        assert np.all(lay.ref_counts[rows[:, 31]] == 1)
    src, dst = lay.copy_pairs[:, 0], lay.copy_pairs[:, 1]
    assert len(set(dst.tolist())) == 192 and not set(dst.tolist()) & set(src.tolist())
    assert np.all(lay.context_lens >= 513) and np.all(lay.context_lens <= 1024)


def test_gqa70b_lengths():
    lay = synth.gqa70b_long()
    assert lay.group_size == 8
    assert lay.context_lens.min() >= 1024 and lay.context_lens.max() <= 32768
    b = synth.decode_kv_bytes(lay)
    assert 4.0e9 < b["kv"] < 6.0e9


def test_mixed_step():
    lay = synth.mixed_qwen32b()
    pf, dc = lay.prefill_rows(), lay.decode_rows()
    assert len(pf) == 8 and len(dc) == 192
    assert int(lay.q_lens.sum()) == 8 * 512 + 192
    assert np.all(lay.context_lens[pf] >= 512) and np.all(lay.context_lens[pf] <= 4096 + 512)
    cu = lay.cu_q_lens(pf)
    assert cu[-1] == 4096


def test_fill_host_poison():
    lay = synth.tiny()
    t = synth.fill_host(lay)
    bs = lay.block_size
    # slot past the end of the 17-token sequence holds NaN
    last = lay.block_tables[1, 1]
    assert np.all(t["k_pool"][last, :, 1:, :] == synth.BF16_NAN)
    # new-token slot of sequence 3 (position 63) holds NaN before the write
    p = lay.block_tables[3, 3]
    assert np.all(t["v_pool"][p, :, 15, :] == synth.BF16_NAN)
    # a referenced, non-new slot holds finite data
    assert np.all(t["k_pool"][lay.block_tables[3, 0], :, 0, :] != synth.BF16_NAN)
    assert t["q"].shape == (4, 4, 64) and t["key"].shape == (4, 4, 64)


def test_chunk_schedule_rules():
    assert synth.chunk_schedule(10, 4, 6) == [(0, 4, 2), (4, 8, 2), (8, 10, 4)]
    with pytest.raises(ValueError):
        synth.chunk_schedule(10, 7, 6)


def test_prefill_flops_closed_form():
    lay = synth.build_layout("f", 0, [5 + 3], num_q_heads=2, num_kv_heads=1, head_dim=4,
                             q_lens=[3], is_prefill=[True], num_blocks=2)
    # queries see 6, 7, 8 keys: 21 keys x 2 heads x 4 dims x 2 MACs x 2 flops
    assert synth.prefill_flops(lay) == 21 * 2 * 4 * 4


def test_decode_bytes_formula():
    lay = synth.build_layout("b", 0, [20, 16], num_q_heads=4, num_kv_heads=2, head_dim=8,
                             num_blocks=4)
    b = synth.decode_kv_bytes(lay)
    assert b["kv"] == 2 * 2 * 36 * 8 * 2
    assert b["q_out"] == 2 * 2 * 4 * 8 * 2
    assert b["meta"] == 4 * (2 + 1) + 4 * 2
    assert b["unique_kv"] == b["kv"]
