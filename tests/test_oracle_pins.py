"""Pins for the CPU oracle: closed forms, the pages' invariants, a brute-force
scalar implementation and the pages' worked numbers.

Each check is a plain function that raises ``AssertionError`` on a mismatch, so
``test_oracle_mutations.py`` can plant a plausible mistake in the oracle and show
that some check here catches it.
"""
import functools
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import paged_attention as pa
from workloads import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BS = 16


def bits(x):
    return synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def f64(b):
    return oracle.bf16_bits_to_f64(b)


def contiguous_to_pool(K, V, bs=BS, table=None, num_blocks=None, fill=None):
    """Lay contiguous [Hkv, L, D] bit arrays into a pool with the given table
    (default: identity).  Unused slots get ``fill`` (default: NaN)."""
    hkv, L, d = K.shape
    nb = -(-L // bs)
    table = np.arange(nb) if table is None else np.asarray(table)
    num_blocks = int(table.max()) + 1 if num_blocks is None else num_blocks
    fillv = synth.BF16_NAN if fill is None else fill
    kp = np.full((num_blocks, hkv, bs, d), fillv, np.uint16)
    vp = np.full((num_blocks, hkv, bs, d), fillv, np.uint16)
    for t in range(L):
        b, o = divmod(t, bs)
        kp[table[b], :, o, :] = K[:, t, :]
        vp[table[b], :, o, :] = V[:, t, :]
    return kp, vp, table


# ----------------------------------------------------------------------------
# bf16 widening / rounding
# ----------------------------------------------------------------------------
def check_bf16_widening():
    pats = np.array([0x3F80, 0xC000, 0x3F81, 0x0000, 0x8000, 0x4049], np.uint16)
    want = [1.0, -2.0, 1.0 + 2.0**-7, 0.0, -0.0, 3.140625]
    got = f64(pats)
    assert list(got) == want
    assert np.isnan(f64(np.array([synth.BF16_NAN], np.uint16)))[0]


def test_bf16_widening():
    check_bf16_widening()


def test_bf16_rounding_ties_to_even():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties go to the even pattern 0x3F80.
    assert synth.f32_to_bf16_bits(np.float32(1 + 2.0**-8)) == 0x3F80
    # 1 + 3*2^-8 is halfway between 1+2^-7 (odd) and 1+2^-6 (even): rounds up.
    assert synth.f32_to_bf16_bits(np.float32(1 + 3 * 2.0**-8)) == 0x3F82
    assert synth.f32_to_bf16_bits(np.float32(1 + 2.0**-8 + 2.0**-20)) == 0x3F81
    assert oracle.f64_to_bf16_bits(1 + 2.0**-8) == 0x3F80


# ----------------------------------------------------------------------------
# Addressing (pages' worked numbers)
# ----------------------------------------------------------------------------
def check_addressing_golden():
    g = json.load(open(os.path.join(GOLDEN, "block_table_addressing.json")))
    bs, H, D = g["block_size"], g["num_heads"], g["head_dim"]
    table = g["block_table"]
    # a pool whose every element holds its own flat index (as int64) lets the
    # gather report which element it read
    nb = max(table) + 1
    flat = np.arange(nb * H * bs * D, dtype=np.int64).reshape(nb, H, bs, D)
    for c in g["cases"]:
        assert oracle.slot_of(table, c["position"], bs) == c["slot"]
        L = c["position"] + 1
        K, _ = oracle.gather_kv(flat, flat, table, L)
        assert K[c["head"], c["position"], 0] == c["k_element_offset"]


def test_addressing_golden():
    check_addressing_golden()


def test_kv_bytes_golden():
    g = json.load(open(os.path.join(GOLDEN, "kv_cache_bytes_llama2_7b.json")))
    per_layer = synth.kv_cache_bytes_per_layer(g["num_heads"], g["seq_len"], g["head_dim"],
                                               g["elem_bytes"])
    assert per_layer == g["per_layer_mib"] * 2**20
    assert per_layer * g["num_layers"] == g["all_layers_gib"] * 2**30


def test_chunk_schedule_golden():
    g = json.load(open(os.path.join(GOLDEN, "chunked_prefill_schedule.json")))
    rounds = synth.chunk_schedule(g["prompt_tokens"], g["chunk_tokens"], g["budget_tokens_per_round"])
    assert len(rounds) == g["rounds"]
    assert [e - s for s, e, _ in rounds] == g["prefill_tokens_per_round"]
    assert [d for _, _, d in rounds] == g["decode_tokens_per_round"]
    # the unchunked column: one round reads the whole prompt
    assert len(synth.chunk_schedule(12, 12, 12)) == 1


# ----------------------------------------------------------------------------
# Gather: identity table, permutation of physical blocks
# ----------------------------------------------------------------------------
def check_identity_table():
    rng = np.random.default_rng(11)
    K = synth.normal_bf16(rng, (3, 45, 8))
    V = synth.normal_bf16(rng, (3, 45, 8))
    kp, vp, table = contiguous_to_pool(K, V)
    Kg, Vg = oracle.gather_kv(kp, vp, table, 45)
    assert np.array_equal(Kg, K) and np.array_equal(Vg, V)


def test_identity_table():
    check_identity_table()


def check_permutation_invariance():
    rng = np.random.default_rng(12)
    lay = synth.build_layout("p", 12, [5, 40, 16, 33], num_q_heads=4, num_kv_heads=2,
                             head_dim=16, num_blocks=20)
    t = synth.fill_host(lay)
    k0, v0 = oracle.reshape_and_cache(t["k_pool"], t["v_pool"], t["key"], t["value"],
                                      lay.slot_mapping())
    out0, lse0 = oracle.decode(t["q"], k0, v0, lay.block_tables, lay.context_lens, lay.scale)
    perm = rng.permutation(lay.num_blocks)  # physical block b moves to perm[b]
    kp = np.empty_like(k0)
    vp = np.empty_like(v0)
    kp[perm] = k0
    vp[perm] = v0
    tab = lay.block_tables.copy()
    m = tab != synth.INT32_MAX
    tab[m] = perm[tab[m]]
    out1, lse1 = oracle.decode(t["q"], kp, vp, tab, lay.context_lens, lay.scale)
    assert np.array_equal(out0, out1) and np.array_equal(lse0, lse1)
    assert np.all(np.isfinite(out0))


def test_permutation_invariance():
    check_permutation_invariance()


# ----------------------------------------------------------------------------
# Attention: hand example, closed forms
# ----------------------------------------------------------------------------
def check_hand_example():
    # q = (1, 0), k0 = (1, 0), k1 = (0, 1): scores (1, 0) at scale 1, so the
    # weights are (e, 1)/(1 + e).  V rows (2, 0) and (0, -3) differ from K.
    e = math.e
    q = np.array([1.0, 0.0])
    K = np.array([[1.0, 0.0], [0.0, 1.0]])
    V = np.array([[2.0, 0.0], [0.0, -3.0]])
    o, lse = oracle.attend(q, K, V, 1.0)
    assert np.allclose(o, [2 * e / (1 + e), -3 / (1 + e)], rtol=0, atol=1e-15)
    assert abs(lse - math.log(1 + e)) < 1e-15
    # scale 1/2: scores (1/2, 0)
    r = math.exp(0.5)
    o, lse = oracle.attend(q, K, V, 0.5)
    assert np.allclose(o, [2 * r / (1 + r), -3 / (1 + r)], rtol=0, atol=1e-15)
    assert abs(lse - math.log(1 + r)) < 1e-15
    # the same numbers through a scattered pool and decode()
    Kb = bits(K.reshape(1, 2, 2))
    Vb = bits(V.reshape(1, 2, 2))
    kp, vp, table = contiguous_to_pool(Kb, Vb, table=[5], num_blocks=8)
    qb = bits(q.reshape(1, 1, 2))
    out, lse = oracle.decode(qb, kp, vp, np.array([[5, synth.INT32_MAX]]), [2], 0.5)
    assert np.allclose(out[0, 0], [2 * r / (1 + r), -3 / (1 + r)], rtol=0, atol=1e-15)


def test_hand_example():
    check_hand_example()


def check_single_token_is_v0():
    rng = np.random.default_rng(3)
    D = 32
    q = synth.normal_bf16(rng, (1, 2, D))
    K = synth.normal_bf16(rng, (1, 1, D))
    V = synth.normal_bf16(rng, (1, 1, D))
    kp, vp, _ = contiguous_to_pool(K, V, table=[3], num_blocks=4)
    out, lse = oracle.decode(q, kp, vp, np.array([[3]]), [1], 0.25)
    for h in range(2):
        assert np.array_equal(out[0, h], f64(V[0, 0]))
        assert abs(lse[0, h] - 0.25 * float(f64(q[0, h]) @ f64(K[0, 0]))) < 1e-12


def test_single_token_is_v0():
    check_single_token_is_v0()


def check_equal_keys_mean_of_values():
    rng = np.random.default_rng(4)
    L, D = 37, 16
    k = synth.normal_bf16(rng, (D,))
    K = np.broadcast_to(k, (1, L, D)).copy()
    V = synth.normal_bf16(rng, (1, L, D))
    q = synth.normal_bf16(rng, (1, 1, D))
    kp, vp, table = contiguous_to_pool(K, V, table=[2, 0, 1], num_blocks=3)
    out, lse = oracle.decode(q, kp, vp, table[None, :], [L], 0.3)
    assert np.allclose(out[0, 0], f64(V[0]).mean(axis=0), rtol=0, atol=1e-13)
    s = 0.3 * float(f64(q[0, 0]) @ f64(k))
    assert abs(lse[0, 0] - (s + math.log(L))) < 1e-12
    # q = 0: uniform weights whatever the keys
    K2 = synth.normal_bf16(rng, (1, L, D))
    kp2, vp2, _ = contiguous_to_pool(K2, V, table=[2, 0, 1], num_blocks=3)
    out, lse = oracle.decode(np.zeros((1, 1, D), np.uint16), kp2, vp2, table[None, :], [L], 0.3)
    assert np.allclose(out[0, 0], f64(V[0]).mean(axis=0), rtol=0, atol=1e-13)
    assert abs(lse[0, 0] - math.log(L)) < 1e-12


def test_equal_keys_mean_of_values():
    check_equal_keys_mean_of_values()


def check_gqa_mapping():
    # Hq = 8, Hkv = 2: q heads 0-3 read KV head 0, heads 4-7 read KV head 1.
    # V of KV head g is the constant c_g, so every output of a q head is the
    # constant of the KV head it reads.
    rng = np.random.default_rng(5)
    L, D = 29, 8
    K = synth.normal_bf16(rng, (2, L, D))
    V = np.empty((2, L, D), np.uint16)
    V[0] = bits(1.5)
    V[1] = bits(-0.75)
    kp, vp, table = contiguous_to_pool(K, V, table=[1, 0], num_blocks=2)
    q = synth.normal_bf16(rng, (1, 8, D))
    out, _ = oracle.decode(q, kp, vp, table[None, :], [L], 0.4)
    for h in range(8):
        assert np.allclose(out[0, h], 1.5 if h < 4 else -0.75, rtol=0, atol=1e-14), h


def test_gqa_mapping():
    check_gqa_mapping()


def check_last_token_counts_and_tail_is_ignored():
    # The key at position L-1 is 16*q, so its score dominates by ~e^40 and the
    # output is v_{L-1}.  The slot at position L holds NaN and must not be read.
    rng = np.random.default_rng(6)
    L, D = 21, 8
    q = np.ones(D, np.float32) * 0.5
    K = synth.normal_bf16(rng, (1, L + 1, D))
    K[0, L - 1] = bits(q * 16)
    V = synth.normal_bf16(rng, (1, L + 1, D))
    K[0, L] = synth.BF16_NAN
    V[0, L] = synth.BF16_NAN
    kp, vp, table = contiguous_to_pool(K, V, table=[4, 1], num_blocks=6)
    out, _ = oracle.decode(bits(q.reshape(1, 1, D)), kp, vp, table[None, :], [L], 1.0)
    assert np.all(np.isfinite(out))
    assert np.allclose(out[0, 0], f64(V[0, L - 1]), rtol=0, atol=1e-9)


def test_last_token_counts_and_tail_is_ignored():
    check_last_token_counts_and_tail_is_ignored()


def check_lse_single_and_uniform():
    rng = np.random.default_rng(7)
    D = 8
    K = synth.normal_bf16(rng, (1, 1, D))
    V = synth.normal_bf16(rng, (1, 1, D))
    q = synth.normal_bf16(rng, (1, 1, D))
    kp, vp, table = contiguous_to_pool(K, V)
    _, lse = oracle.decode(q, kp, vp, table[None, :], [1], 0.7)
    assert abs(lse[0, 0] - 0.7 * float(f64(q[0, 0]) @ f64(K[0, 0]))) < 1e-12


def test_lse_single_and_uniform():
    check_lse_single_and_uniform()


def test_empty_context_convention():
    kp = np.zeros((2, 1, BS, 4), np.uint16)
    out, lse = oracle.decode(np.zeros((1, 1, 4), np.uint16), kp, kp, np.array([[0]]), [0], 1.0)
    assert np.all(out == 0) and lse[0, 0] == -np.inf


# ----------------------------------------------------------------------------
# Brute force: scalar Python loops addressing the pool directly
# ----------------------------------------------------------------------------
@functools.lru_cache(maxsize=None)
def _bf(x):
    """bf16 bit pattern -> float by its fields (sign, 8-bit exponent, 7-bit
    mantissa), independently of the oracle's widening."""
    x = int(x)
    sign = -1.0 if x & 0x8000 else 1.0
    e, m = (x >> 7) & 0xFF, x & 0x7F
    if e == 0xFF:
        return math.nan if m else sign * math.inf
    if e == 0:
        return sign * m * 2.0**-133
    return sign * (1 + m / 128) * 2.0 ** (e - 127)


def brute_force_query(qrow, k_pool, v_pool, table_row, limit, g, scale):
    """softmax over keys 0..limit-1 by explicit loops; no max shift."""
    bs, D = k_pool.shape[2], k_pool.shape[3]
    weights, rows = [], []
    for t in range(limit):
        p = int(table_row[t // bs])
        o = t % bs
        s = 0.0
        for d in range(D):
            s += _bf(qrow[d]) * _bf(k_pool[p, g, o, d])
        weights.append(math.exp(scale * s))
        rows.append([_bf(v_pool[p, g, o, d]) for d in range(D)])
    z = sum(weights)
    out = [sum(w * r[d] for w, r in zip(weights, rows)) / z for d in range(D)]
    return out, math.log(z)


def check_brute_force_decode():
    for lay in (synth.tiny(),
                synth.build_layout("gqa", 9, [3, 18, 40], num_q_heads=8, num_kv_heads=2,
                                   head_dim=8, num_blocks=12)):
        t = synth.fill_host(lay)
        # decode reads the pool after the cache write of this step's tokens
        kp, vp = oracle.reshape_and_cache(t["k_pool"], t["v_pool"], t["key"], t["value"],
                                          lay.slot_mapping())
        out, lse = oracle.decode(t["q"], kp, vp, lay.block_tables, lay.context_lens, lay.scale)
        G = lay.group_size
        for s in range(lay.num_seqs):
            for h in range(lay.num_q_heads):
                o, l = brute_force_query(t["q"][s, h], kp, vp, lay.block_tables[s],
                                         int(lay.context_lens[s]), h // G, lay.scale)
                assert np.allclose(out[s, h], o, rtol=0, atol=1e-12), (lay.name, s, h)
                assert abs(lse[s, h] - l) < 1e-12


def test_brute_force_decode():
    check_brute_force_decode()


def check_brute_force_prefill():
    # two sequences: a fresh prompt (c = 0) and a chunk on 21 cached tokens
    lay = synth.build_layout("pf", 13, [7, 26], num_q_heads=4, num_kv_heads=2, head_dim=8,
                             q_lens=[7, 5], is_prefill=[True, True], num_blocks=6)
    t = synth.fill_host(lay)
    kp, vp = oracle.reshape_and_cache(t["k_pool"], t["v_pool"], t["key"], t["value"],
                                      lay.slot_mapping())
    cu = lay.cu_q_lens([0, 1])
    out, lse = oracle.chunked_prefill(t["q"], cu, kp, vp, lay.block_tables, lay.context_lens,
                                      lay.scale)
    for s in range(2):
        n = int(lay.q_lens[s])
        c = int(lay.context_lens[s]) - n
        for i in range(n):
            for h in range(4):
                o, l = brute_force_query(t["q"][cu[s] + i, h], kp, vp, lay.block_tables[s],
                                         c + i + 1, h // 2, lay.scale)
                assert np.allclose(out[cu[s] + i, h], o, rtol=0, atol=1e-12)
                assert abs(lse[cu[s] + i, h] - l) < 1e-12


def test_brute_force_prefill():
    check_brute_force_prefill()


# ----------------------------------------------------------------------------
# Chunked prefill invariants
# ----------------------------------------------------------------------------
def check_prefill_one_token_is_decode():
    lay = synth.build_layout("d", 21, [19, 50], num_q_heads=6, num_kv_heads=3, head_dim=8,
                             num_blocks=9)
    t = synth.fill_host(lay, poison=False)
    out_d, lse_d = oracle.decode(t["q"], t["k_pool"], t["v_pool"], lay.block_tables,
                                 lay.context_lens, lay.scale)
    out_p, lse_p = oracle.chunked_prefill(t["q"], np.array([0, 1, 2]), t["k_pool"], t["v_pool"],
                                          lay.block_tables, lay.context_lens, lay.scale)
    assert np.array_equal(out_d, out_p) and np.array_equal(lse_d, lse_p)


def test_prefill_one_token_is_decode():
    check_prefill_one_token_is_decode()


def check_chunk_split_equivalence():
    # the pages' example: a 12-token prompt read 4 tokens a round equals one
    # 12-token prefill
    rng = np.random.default_rng(22)
    D, hkv, hq = 8, 1, 2
    K = synth.normal_bf16(rng, (hkv, 12, D))
    V = synth.normal_bf16(rng, (hkv, 12, D))
    q = synth.normal_bf16(rng, (12, hq, D))
    kp, vp, table = contiguous_to_pool(K, V, table=[2], num_blocks=3)
    tab = table[None, :]
    whole, lse_w = oracle.chunked_prefill(q, np.array([0, 12]), kp, vp, tab, [12], 0.35)
    parts = []
    for s, e, _ in synth.chunk_schedule(12, 4, 6):
        o, _ = oracle.chunked_prefill(q[s:e], np.array([0, e - s]), kp, vp, tab, [e], 0.35)
        parts.append(o)
    assert np.array_equal(np.concatenate(parts), whole)


def test_chunk_split_equivalence():
    check_chunk_split_equivalence()


def check_prefill_causal_boundary():
    # Query i of a chunk on c cached tokens sees key c+i but not key c+i+1.
    rng = np.random.default_rng(23)
    D, c, n = 8, 5, 4
    L = c + n
    q = np.full((n, 1, D), 0.5, np.float32)
    K = synth.normal_bf16(rng, (1, L, D))
    V = synth.normal_bf16(rng, (1, L, D))
    i = 1
    K[0, c + i] = bits(np.full(D, 8.0))        # dominates query i
    K[0, c + i + 1] = bits(np.full(D, 16.0))   # would dominate if visible
    kp, vp, table = contiguous_to_pool(K, V, table=[1], num_blocks=2)
    out, _ = oracle.chunked_prefill(bits(q), np.array([0, n]), kp, vp, table[None, :], [L], 1.0)
    assert np.allclose(out[i, 0], f64(V[0, c + i]), rtol=0, atol=1e-9)
    assert np.allclose(out[i + 1, 0], f64(V[0, c + i + 1]), rtol=0, atol=1e-9)


def test_prefill_causal_boundary():
    check_prefill_causal_boundary()


# ----------------------------------------------------------------------------
# Cache write, block copy, sharing
# ----------------------------------------------------------------------------
def check_reshape_and_cache():
    lay = synth.tiny()
    t = synth.fill_host(lay)
    sm = lay.slot_mapping()
    kp, vp = oracle.reshape_and_cache(t["k_pool"], t["v_pool"], t["key"], t["value"], sm)
    seqs, pos = lay.new_positions()
    for j, (s, p) in enumerate(zip(seqs, pos)):
        Kg, Vg = oracle.gather_kv(kp, vp, lay.block_tables[s], int(p) + 1)
        assert np.array_equal(Kg[:, p], t["key"][j]) and np.array_equal(Vg[:, p], t["value"][j])
    touched = np.zeros(kp.shape[:1] + kp.shape[2:3], bool)
    touched[sm // BS, sm % BS] = True
    assert np.array_equal(kp.transpose(0, 2, 1, 3)[~touched],
                          t["k_pool"].transpose(0, 2, 1, 3)[~touched])
    # a negative slot is padding
    sm2 = sm.copy()
    sm2[1] = -1
    kp2, vp2 = oracle.reshape_and_cache(t["k_pool"], t["v_pool"], t["key"], t["value"], sm2)
    keep = np.arange(len(sm)) != 1
    kp3, vp3 = oracle.reshape_and_cache(t["k_pool"], t["v_pool"], t["key"][keep],
                                        t["value"][keep], sm[keep])
    assert np.array_equal(kp2, kp3) and np.array_equal(vp2, vp3)
    with pytest.raises(ValueError):
        oracle.reshape_and_cache(t["k_pool"], t["v_pool"], t["key"], t["value"], [3, 3, 4, 5])


def test_reshape_and_cache():
    check_reshape_and_cache()


def check_copy_blocks():
    rng = np.random.default_rng(31)
    kp = synth.normal_bf16(rng, (10, 2, BS, 8))
    vp = synth.normal_bf16(rng, (10, 2, BS, 8))
    pairs = np.array([[1, 4], [1, 7], [2, 9]])
    k2, v2 = oracle.copy_blocks(kp, vp, pairs)
    for s, d in pairs:
        assert np.array_equal(k2[d], kp[s]) and np.array_equal(v2[d], vp[s])
    for b in set(range(10)) - {4, 7, 9}:
        assert np.array_equal(k2[b], kp[b]) and np.array_equal(v2[b], vp[b])
    for bad in ([[1, 4], [2, 4]], [[1, 4], [4, 5]], [[1, 10]], [[-1, 3]]):
        with pytest.raises(oracle.CopyBlocksError):
            oracle.copy_blocks(kp, vp, bad)


def test_copy_blocks():
    check_copy_blocks()


def unshare(layout, k_pool, v_pool):
    """Give every sequence its own physical copy of every block it reads."""
    bs = layout.block_size
    nb = sum(layout.blocks_used(s) for s in range(layout.num_seqs))
    kp = np.empty((nb,) + k_pool.shape[1:], k_pool.dtype)
    vp = np.empty_like(kp)
    tab = np.full_like(layout.block_tables, synth.INT32_MAX)
    k = 0
    for s in range(layout.num_seqs):
        for b in range(layout.blocks_used(s)):
            p = layout.block_tables[s, b]
            kp[k], vp[k] = k_pool[p], v_pool[p]
            tab[s, b] = k
            k += 1
    return kp, vp, tab


def check_shared_prefix_equals_unshared():
    lay = synth.llama13b_sampling(seed=2, groups=3, samples=4, prefix=48, max_suffix=20)
    lay.num_q_heads = lay.num_kv_heads = 2
    lay.head_dim = 8
    t = synth.fill_host(lay)
    # prompt blocks are shared: sample 0's prefix block 0 is every sample's
    assert len({int(lay.block_tables[j, 0]) for j in range(4)}) == 1
    assert lay.ref_counts[lay.block_tables[0, 0]] == 4
    kp, vp = oracle.copy_blocks(t["k_pool"], t["v_pool"], lay.copy_pairs)
    kp, vp = oracle.reshape_and_cache(kp, vp, t["key"], t["value"], lay.slot_mapping())
    out_s, lse_s = oracle.decode(t["q"], kp, vp, lay.block_tables, lay.context_lens, lay.scale)
    ku, vu, tab = unshare(lay, kp, vp)
    out_u, lse_u = oracle.decode(t["q"], ku, vu, tab, lay.context_lens, lay.scale)
    assert np.all(np.isfinite(out_s))
    assert np.array_equal(out_s, out_u) and np.array_equal(lse_s, lse_u)


def test_shared_prefix_equals_unshared():
    check_shared_prefix_equals_unshared()


def check_poison_is_never_read():
    lay = synth.tiny()
    t = synth.fill_host(lay, poison=True)
    kp, vp = oracle.reshape_and_cache(t["k_pool"], t["v_pool"], t["key"], t["value"],
                                      lay.slot_mapping())
    out, lse = oracle.decode(t["q"], kp, vp, lay.block_tables, lay.context_lens, lay.scale)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    # replacing every poisoned slot with other finite values changes nothing
    t2 = synth.fill_host(lay, poison=False)
    k2, v2 = t2["k_pool"].copy(), t2["v_pool"].copy()
    live = ~(np.isnan(f64(t["k_pool"])))
    k2[live], v2[live] = t["k_pool"][live], t["v_pool"][live]
    k2, v2 = oracle.reshape_and_cache(k2, v2, t["key"], t["value"], lay.slot_mapping())
    out2, lse2 = oracle.decode(t["q"], k2, v2, lay.block_tables, lay.context_lens, lay.scale)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_poison_is_never_read():
    check_poison_is_never_read()


# ----------------------------------------------------------------------------
# Library softmax on contiguous tensors
# ----------------------------------------------------------------------------
def check_matches_library_softmax():
    """Decode and causal prefill through an identity table equal
    ``scipy.special.softmax(scale * Q K^T) V`` on the contiguous tensors, and the
    log-sum-exp equals ``scipy.special.logsumexp`` of the scaled scores."""
    from scipy.special import logsumexp, softmax
    rng = np.random.default_rng(31)
    hq, hkv, d, L, n = 4, 2, 32, 45, 7
    K = bits(rng.normal(size=(hkv, L, d)))
    V = bits(rng.normal(size=(hkv, L, d)))
    kp, vp, table = contiguous_to_pool(K, V)
    Kf, Vf = f64(K), f64(V)
    scale = 0.37
    # decode: one query per head over all L keys
    q = bits(rng.normal(size=(1, hq, d)))
    out, lse = oracle.decode(q, kp, vp, table[None, :], np.array([L]), scale)
    for h in range(hq):
        g = h // (hq // hkv)
        s = scale * (Kf[g] @ f64(q[0, h]))
        assert np.allclose(out[0, h], softmax(s) @ Vf[g], rtol=0, atol=1e-12)
        assert abs(lse[0, h] - logsumexp(s)) < 1e-12
    # prefill: the last n positions as the chunk (and, with n = L, no cached
    # context: plain causal self-attention), causal mask as -inf
    for nn in (n, L):
        qp = bits(rng.normal(size=(nn, hq, d)))
        outp, lsep = oracle.chunked_prefill(qp, np.array([0, nn]), kp, vp, table[None, :],
                                            np.array([L]), scale)
        for i in range(nn):
            for h in range(hq):
                g = h // (hq // hkv)
                s = scale * (Kf[g] @ f64(qp[i, h]))
                s[L - nn + i + 1:] = -np.inf
                assert np.allclose(outp[i, h], softmax(s) @ Vf[g], rtol=0, atol=1e-12)
                assert abs(lsep[i, h] - logsumexp(s)) < 1e-12


def test_matches_library_softmax():
    check_matches_library_softmax()


ALL_CHECKS = [
    check_bf16_widening, check_addressing_golden, check_identity_table,
    check_permutation_invariance, check_hand_example, check_single_token_is_v0,
    check_equal_keys_mean_of_values, check_gqa_mapping,
    check_last_token_counts_and_tail_is_ignored, check_lse_single_and_uniform,
    check_brute_force_decode, check_brute_force_prefill, check_prefill_one_token_is_decode,
    check_chunk_split_equivalence, check_prefill_causal_boundary, check_reshape_and_cache,
    check_copy_blocks, check_shared_prefix_equals_unshared, check_poison_is_never_read,
    check_matches_library_softmax,
]

