"""Parity of the CUDA path (through the C ABI) with the CPU oracle, on seeded
inputs at sizes the oracle finishes in seconds: several 128-token tiles, several
split-context partitions, ragged tails, every poison of the batch builder.

Bit-exact: cache writes, block copies, gathers.  Attention outputs: each element
within 2e-3 absolute or 1e-2 relative of the fp64 oracle (bf16 inputs, fp32
accumulation, bf16 output); log-sum-exp within 1e-3.
"""
import numpy as np
import pytest

import oracle
from workloads import synth

import gpu_helpers as H

pytestmark = pytest.mark.gpu


def pa():
    import paged_kv_cache_454_b200 as m
    return m


# ----------------------------------------------------------------------------
# Layouts (small enough for the oracle; big enough for tiles, splits, tails)
# ----------------------------------------------------------------------------
def lay_mha128():
    return synth.build_layout("mha128", 101, [1, 15, 16, 17, 700, 2049], num_q_heads=4,
                              num_kv_heads=4, head_dim=128)


def lay_gqa8():
    return synth.build_layout("gqa8", 102, [1, 130, 1025, 3000, 4100], num_q_heads=16,
                              num_kv_heads=2, head_dim=128)


def lay_gqa5():
    return synth.build_layout("gqa5", 103, [33, 600, 1500, 2222], num_q_heads=10, num_kv_heads=2,
                              head_dim=128)


def lay_gqa4_d64():
    return synth.build_layout("gqa4d64", 104, [5, 300, 999], num_q_heads=8, num_kv_heads=2,
                              head_dim=64)


def lay_g16():
    return synth.build_layout("g16", 105, [64, 777], num_q_heads=32, num_kv_heads=2,
                              head_dim=128)


def lay_shared():
    lay = synth.llama13b_sampling(seed=106, groups=3, samples=4, prefix=512, max_suffix=300)
    lay.num_q_heads = lay.num_kv_heads = 4
    return lay


def lay_shared_many():
    # 160 short sequences x 32 KV heads sharing first blocks: the plan finds the
    # sharing, but the batch is too small for prefix order (an item would be
    # more than 1/16 of an SM's share), so it runs longest first.  Prefix order
    # needs about a GB of context at 148 SMs; the full-size sampling batch
    # (tests/test_gpu_fullsize.py) runs it.
    lay = synth.llama13b_sampling(seed=112, groups=40, samples=4, prefix=64, max_suffix=60)
    lay.num_q_heads = lay.num_kv_heads = 32
    return lay


def lay_gqa4():
    # group 4: two KV heads share a tile (4 KiB copies)
    return synth.build_layout("gqa4", 113, [1, 40, 700, 1500, 3000], num_q_heads=16,
                              num_kv_heads=4, head_dim=128)


def lay_gqa2_h6():
    # group 2 over 6 KV heads: tiles of 2 heads (4 does not divide 6)
    return synth.build_layout("gqa2_h6", 114, [3, 129, 900, 2100], num_q_heads=12,
                              num_kv_heads=6, head_dim=128)


def lay_gqa8_h3():
    # group 8 over 3 KV heads: no pairs, one KV head per tile
    return synth.build_layout("gqa8_h3", 117, [5, 200, 1800], num_q_heads=24, num_kv_heads=3,
                              head_dim=128)


def lay_mha_h5():
    # one q head per KV head, 5 KV heads: one head per tile
    return synth.build_layout("mha_h5", 115, [2, 17, 300, 1300], num_q_heads=5,
                              num_kv_heads=5, head_dim=128)


def lay_mha_h16():
    # 16 KV heads: two tiles of 8 heads per page
    return synth.build_layout("mha_h16", 116, [1, 16, 33, 1000, 2500], num_q_heads=16,
                              num_kv_heads=16, head_dim=128)


def lay_mixed(hq=10, hkv=2, d=128):
    # prefill chunks: fresh prompt, short cache, long cache with a ragged chunk;
    # plus two decode sequences
    cached = [0, 100, 1000]
    chunk = [37, 128, 300]
    lens = [c + n for c, n in zip(cached, chunk)] + [513, 70]
    return synth.build_layout("mixed", 107, lens, num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                              q_lens=chunk + [1, 1], is_prefill=[True] * 3 + [False] * 2)


def lay_short_gqa():
    # contexts of a few keys, where rounding of the softmax weights matters most
    return synth.build_layout("short_gqa", 109, [2, 3, 4, 5, 6, 7, 8, 9, 12, 16, 2, 3] * 3,
                              num_q_heads=16, num_kv_heads=2, head_dim=128)


def lay_short_mha():
    return synth.build_layout("short_mha", 110, [2, 3, 5, 8, 13, 16, 17, 2] * 4, num_q_heads=8,
                              num_kv_heads=8, head_dim=128)


# Groups 9-16 take the 16-column tensor-core tile (remainder of p in columns
# 16..31).  Contexts of 2-16 keys are where bf16 weights alone miss the
# tolerance, so these pin that the remainder is carried at this width too.
def lay_short_g16():
    return synth.build_layout("short_g16", 118, [2, 3, 4, 5, 8, 12, 16] * 3, num_q_heads=32,
                              num_kv_heads=2, head_dim=128)


def lay_short_g12():
    return synth.build_layout("short_g12", 119, [2, 3, 4, 5, 8, 12, 16] * 3, num_q_heads=24,
                              num_kv_heads=2, head_dim=128)


def lay_gqa3():
    # group 3 (3 of 8 columns live) over 4 KV heads: tiles of 2 heads
    return synth.build_layout("gqa3", 130, [1, 15, 16, 17, 300, 2049], num_q_heads=12,
                              num_kv_heads=4, head_dim=128)


def lay_gqa7():
    # group 7 (7 of 8 columns live) over 2 KV heads, short and long contexts
    return synth.build_layout("gqa7", 131, [2, 9, 33, 640, 3000], num_q_heads=14,
                              num_kv_heads=2, head_dim=128)


def lay_g12():
    # group 12 (12 of 16 columns live) over several tiles, splits and tails
    return synth.build_layout("g12", 120, [1, 40, 300, 1100, 2600], num_q_heads=36,
                              num_kv_heads=3, head_dim=128)


# Shared-prefix cascade: runs of sequences over common prompt blocks.  The plan
# takes the longest run for the sharers per item (at most 16 / group) and packs
# KV heads into the rest of the item's 16 q columns.
def lay_casc_mha4():
    # runs of 4: four sharers x four KV heads per item; a run of 3 and one of 2
    # under-fill their items; an unshared sequence; two prompt lengths
    return synth.prefix_runs("casc_mha4", 121, [4, 4, 4, 4, 2, 3, 1], [300, 600, 300, 600, 300, 600, 300],
                             400, num_q_heads=8, num_kv_heads=8)


def lay_casc_mha17():
    # a run of 17: sixteen sharers x one KV head per item, the 17th on its own
    return synth.prefix_runs("casc_mha17", 122, [17, 4, 2], 200, 150, num_q_heads=4,
                             num_kv_heads=4)


def lay_casc_gqa8():
    # group 8: two sharers per item; long prompts over several partitions; a run
    # of 5 cut into 2 + 2 + 1
    return synth.prefix_runs("casc_gqa8", 123, [2, 2, 3, 1, 5], [1000, 2000, 700, 0, 1500], 1500,
                             num_q_heads=16, num_kv_heads=2)


def lay_casc_gqa5():
    # group 5: three sharers (15 of 16 columns); a run of 4 cut into 3 + 1
    return synth.prefix_runs("casc_gqa5", 124, [3, 3, 2, 4], 500, 300, num_q_heads=10,
                             num_kv_heads=2)


def lay_casc_gqa4():
    # group 4, runs of 2: two sharers x two KV heads per item
    return synth.prefix_runs("casc_gqa4", 125, [2, 2, 2], 900, 700, num_q_heads=16,
                             num_kv_heads=4)


def lay_casc_edges():
    # empty contexts (no prompt, empty suffix), a prompt of 128 tokens whose
    # shared span (7 whole blocks after the copy-on-write) is too short to
    # cascade, suffixes of zero tokens after a shared prompt
    return synth.prefix_runs("casc_edges", 126, [4, 1, 1, 2, 3], [256, 0, 0, 128, 400], 20,
                             num_q_heads=8, num_kv_heads=8, min_suffix=0)


def lay_casc_g2_many():
    # group 2: 70 runs of two sharers -- more sub-runs than one round of the
    # plan's span search takes (64) -- and four unshared sequences; prompts of
    # 160 tokens (9 shared blocks after the copy-on-write)
    return synth.prefix_runs("casc_g2_many", 127, [2] * 70 + [1] * 4, 160, 40, num_q_heads=8,
                             num_kv_heads=4)


def lay_casc_g3():
    # group 3: two sharers per item; the run of 3 cut into 2 + 1
    return synth.prefix_runs("casc_g3", 128, [2, 2, 3, 1], 400, 200, num_q_heads=12,
                             num_kv_heads=4)


CASCADE_LAYOUTS = ["casc_mha4", "casc_mha17", "casc_gqa8", "casc_gqa5", "casc_gqa4", "casc_edges",
                   "casc_g2_many", "casc_g3"]


DECODE_LAYOUTS = {
    "tiny": synth.tiny,
    "mha128": lay_mha128,
    "gqa8": lay_gqa8,
    "gqa5": lay_gqa5,
    "gqa4_d64": lay_gqa4_d64,
    "g16": lay_g16,
    "shared_prefix": lay_shared,
    "shared_many": lay_shared_many,
    "gqa4": lay_gqa4,
    "gqa2_h6": lay_gqa2_h6,
    "mha_h5": lay_mha_h5,
    "mha_h16": lay_mha_h16,
    "gqa8_h3": lay_gqa8_h3,
    "short_gqa": lay_short_gqa,
    "short_mha": lay_short_mha,
    "short_g16": lay_short_g16,
    "short_g12": lay_short_g12,
    "g12": lay_g12,
    "gqa3": lay_gqa3,
    "gqa7": lay_gqa7,
    "casc_mha4": lay_casc_mha4,
    "casc_mha17": lay_casc_mha17,
    "casc_gqa8": lay_casc_gqa8,
    "casc_gqa5": lay_casc_gqa5,
    "casc_gqa4": lay_casc_gqa4,
    "casc_edges": lay_casc_edges,
    "casc_g2_many": lay_casc_g2_many,
    "casc_g3": lay_casc_g3,
}


# ----------------------------------------------------------------------------
# Bit-exact data movement
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("make", [synth.tiny, lay_mha128, lay_shared, lambda: lay_mixed()],
                         ids=["tiny", "mha128", "shared", "mixed"])
def test_reshape_and_cache_and_copy_blocks_bit_exact(make):
    lay = make()
    st = H.Step.from_host(lay)
    if lay.copy_pairs.size:
        pa().pa_copy_blocks(st.k_pool, st.v_pool, lay.copy_pairs)
    pa().pa_reshape_and_cache(st.key, st.value, st.k_pool, st.v_pool, st.slot_mapping)
    ref = st.run_oracle()["pools"]
    assert np.array_equal(H.host_bits(st.k_pool), ref[0])
    assert np.array_equal(H.host_bits(st.v_pool), ref[1])
    assert pa().pa_get_device_error() == 0


def test_copy_blocks_many_pairs_bit_exact():
    # more pairs than one launch carries (480), on D = 64 pools
    rng = np.random.default_rng(7)
    nb = 1200
    kp = synth.normal_bf16(rng, (nb, 2, 16, 64))
    vp = synth.normal_bf16(rng, (nb, 2, 16, 64))
    perm = rng.permutation(nb)
    pairs = np.stack([perm[:500], perm[500:1000]], axis=1)
    k, v = H.dev_bf16(kp), H.dev_bf16(vp)
    pa().pa_copy_blocks(k, v, pairs)
    rk, rv = oracle.copy_blocks(kp, vp, pairs)
    assert np.array_equal(H.host_bits(k), rk) and np.array_equal(H.host_bits(v), rv)


def test_reshape_and_cache_strided_and_padding():
    lay = lay_mha128()
    h = synth.fill_host(lay)
    T, hkv, d = h["key"].shape
    # key/value as views into a wider [T, 3*Hkv, D] buffer (a fused projection)
    wide = np.zeros((T, 3 * hkv, d), np.uint16)
    wide[:, :hkv] = h["key"]
    wide[:, hkv:2 * hkv] = h["value"]
    wd = H.dev_bf16(wide)
    sm = lay.slot_mapping().copy()
    sm[2] = -1  # padding token
    kp, vp = H.dev_bf16(h["k_pool"]), H.dev_bf16(h["v_pool"])
    pa().pa_reshape_and_cache(wd[:, :hkv], wd[:, hkv:2 * hkv], kp, vp, H.dev_i64(sm))
    rk, rv = oracle.reshape_and_cache(h["k_pool"], h["v_pool"], h["key"], h["value"], sm)
    assert np.array_equal(H.host_bits(kp), rk) and np.array_equal(H.host_bits(vp), rv)


@pytest.mark.parametrize("make", [synth.tiny, lay_gqa8, lay_shared], ids=["tiny", "gqa8", "shared"])
def test_gather_kv_bit_exact(make):
    lay = make()
    st = H.Step.from_host(lay)
    ref_pools = st.run_oracle()["pools"]
    if lay.copy_pairs.size:
        pa().pa_copy_blocks(st.k_pool, st.v_pool, lay.copy_pairs)
    pa().pa_reshape_and_cache(st.key, st.value, st.k_pool, st.v_pool, st.slot_mapping)
    cu = np.concatenate([[0], np.cumsum(lay.context_lens)]).astype(np.int32)
    k, v = pa().pa_gather_kv(st.k_pool, st.v_pool, st.tables, st.lens, H.dev_i32(cu),
                             int(lay.context_lens.max()), int(cu[-1]))
    kb, vb = H.host_bits(k), H.host_bits(v)
    for s in range(lay.num_seqs):
        K, V = oracle.gather_kv(ref_pools[0], ref_pools[1], lay.block_tables[s],
                                int(lay.context_lens[s]))
        assert np.array_equal(kb[cu[s]:cu[s + 1]], K.transpose(1, 0, 2))
        assert np.array_equal(vb[cu[s]:cu[s + 1]], V.transpose(1, 0, 2))


# ----------------------------------------------------------------------------
# Decode
# ----------------------------------------------------------------------------
_oracle_cache = {}


def _step_and_ref(name):
    if name not in _oracle_cache:
        lay = DECODE_LAYOUTS[name]()
        st = H.Step.from_host(lay)
        _oracle_cache[name] = (lay, st.host, st.run_oracle())
    lay, host, ref = _oracle_cache[name]
    return H.Step(lay, host), ref


@pytest.mark.parametrize("name", list(DECODE_LAYOUTS))
@pytest.mark.parametrize("partition", [0, 128, 512, 1 << 20])
def test_decode_simt(name, partition):
    st, ref = _step_and_ref(name)
    got = st.run_gpu(kernel=pa().PA_KERNEL_SIMT, partition=partition)
    H.compare_step(got, ref, what=f"{name} simt p={partition}")
    assert pa().pa_get_device_error() == 0


@pytest.mark.parametrize("name", ["gqa8", "gqa5", "g16", "shared_prefix", "shared_many", "mha128",
                                  "short_gqa", "short_mha", "gqa4", "gqa2_h6", "mha_h5",
                                  "mha_h16", "gqa8_h3", "short_g16", "short_g12", "g12", "gqa3",
                                  "gqa7"]
                         + CASCADE_LAYOUTS)
@pytest.mark.parametrize("partition", [0, 128, 1024, 1 << 20])
def test_decode_tcgen05(name, partition):
    st, ref = _step_and_ref(name)
    lay = st.layout
    from paged_kv_cache_454_b200 import _abi
    try:
        got = st.run_gpu(kernel=pa().PA_KERNEL_TCGEN05, partition=partition)
    except pa().PaError as e:
        if e.status == _abi.PA_ERR_UNSUPPORTED:
            pytest.skip(f"tcgen05 decode not built for D={lay.head_dim}, G={lay.group_size}")
        raise
    H.compare_step(got, ref, what=f"{name} tcgen05 p={partition}")
    assert pa().pa_get_device_error() == 0


@pytest.mark.parametrize("tail", [0, 5], ids=["whole_blocks", "ragged"])
@pytest.mark.parametrize("partition", [0, 128])
def test_decode_cascade_identical_tables(tail, partition):
    # sequences whose tables are identical over their whole context: the shared
    # span is every whole block, so a sequence with no tokens after it has no
    # items of its own and the shared-prefix items alone produce its output
    # (written directly when it has a single partition).  Decode only, on the
    # pool as drawn: no new tokens are written into the shared blocks.
    import torch
    rng = np.random.default_rng(127)
    lens, tables, nb = [], [], 0
    for n, blocks in [(4, 20), (3, 8), (2, 40), (5, 9)]:
        row = list(range(nb, nb + blocks))
        nb += blocks
        for j in range(n):
            lens.append(16 * blocks - (tail if j % 2 else 0))
            tables.append(row)
    S = len(lens)
    mb = max(len(r) for r in tables)
    tab = np.full((S, mb), synth.INT32_MAX, np.int32)
    for s, r in enumerate(tables):
        tab[s, :len(r)] = r
    perm = rng.permutation(nb).astype(np.int32)
    tab = np.where(tab == synth.INT32_MAX, tab, perm[np.minimum(tab, nb - 1)])
    hq, hkv, d = 8, 8, 128
    kp = synth.normal_bf16(rng, (nb, hkv, 16, d))
    vp = synth.normal_bf16(rng, (nb, hkv, 16, d))
    q = synth.normal_bf16(rng, (S, hq, d))
    lens = np.asarray(lens, np.int32)
    want, want_lse = oracle.decode(q, kp, vp, tab, lens, 1 / np.sqrt(d))
    out, lse = pa().pa_decode(H.dev_bf16(q), H.dev_bf16(kp), H.dev_bf16(vp), H.dev_i32(tab),
                              H.dev_i32(lens), float(1 / np.sqrt(d)),
                              kernel=pa().PA_KERNEL_TCGEN05, partition_tokens=partition,
                              want_lse=True)
    torch.cuda.synchronize()
    H.assert_close(H.host_f64(out), want, what=f"identical tables tail={tail}")
    H.assert_lse_close(H.host_f64(lse), want_lse, what=f"identical tables tail={tail}")
    assert pa().pa_get_device_error() == 0


def _expected_cascade(lay):
    """Sharers per item and log2 of the KV heads per item the plan should pick
    (items of 8 q columns, groups up to 4), and whether any sub-run's shared
    span reaches 128 tokens (never for larger groups: no shared-prefix items)."""
    G, hkv = lay.group_size, lay.num_kv_heads
    cols = 8
    lens, tab = lay.context_lens, lay.block_tables
    runs = {}
    for s in range(lay.num_seqs):
        if lens[s] > 0:
            runs.setdefault(int(tab[s, 0]), []).append(s)
    rmax = max(len(v) for v in runs.values())
    if G > 4:
        return 1, 0, False
    M = min(rmax, cols // G)
    hts = 0
    while hts < 3 and G * (2 << hts) * M <= cols and hkv % (2 << hts) == 0:
        hts += 1
    any_span = False
    for members in runs.values():
        members = sorted(members)
        for i in range(0, len(members), M):
            sub = members[i:i + M]
            if len(sub) < 2:
                continue
            full = min(int(lens[s]) // 16 for s in sub)
            lcp = 0
            while lcp < full and all(tab[s, lcp] == tab[sub[0], lcp] for s in sub):
                lcp += 1
            any_span |= lcp * 16 >= 128
    return M, hts, any_span


@pytest.mark.parametrize("name", CASCADE_LAYOUTS + ["shared_prefix", "mha128"])
def test_decode_cascade_plan(name):
    # white box: the plan's header in the caller's workspace (int32 [8]: own
    # items, partitions, their counter, partition length, shared-prefix items,
    # their counter, log2 KV heads | sharers << 8 per shared-prefix item,
    # their partition length) shows the cascade ran where the layout has shared prompts, with
    # the expected sharers and heads per item, and that every item was taken
    import torch
    st, ref = _step_and_ref(name)
    lay = st.layout
    S, hq = lay.num_seqs, lay.num_q_heads
    n = pa().pa_decode_workspace_size(S, hq, st.k_pool, lay.max_blocks)
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    got = {}
    if lay.copy_pairs.size:
        pa().pa_copy_blocks(st.k_pool, st.v_pool, lay.copy_pairs)
    pa().pa_reshape_and_cache(st.key, st.value, st.k_pool, st.v_pool, st.slot_mapping)
    out, lse = pa().pa_decode(st.q, st.k_pool, st.v_pool, st.tables, st.lens, lay.scale,
                              workspace=ws, kernel=pa().PA_KERNEL_TCGEN05, want_lse=True)
    torch.cuda.synchronize()
    hdr = ws[:32].view(torch.int32).cpu().numpy()
    H.compare_step({"decode": (out, lse)}, {"decode": ref["decode"]}, what=f"{name} cascade")
    # every item was taken (each CTA's last, empty grab also counts)
    assert hdr[2] >= hdr[0] and hdr[5] >= hdr[4], hdr
    shared = len(set(int(lay.block_tables[s, 0]) for s in range(S) if lay.context_lens[s] > 0)) < \
        int((lay.context_lens > 0).sum())
    if not shared:
        assert hdr[4] == 0, hdr
        return
    M, hts, any_span = _expected_cascade(lay)
    assert (hdr[4] > 0) == any_span, hdr
    if not any_span:
        return
    assert hdr[6] & 0xff == hts and hdr[6] >> 8 == M, (hdr, M, hts)
    if any_span:
        assert hdr[7] % 128 == 0 and hdr[7] >= 128, hdr


def test_decode_default_kernel_choice():
    st, ref = _step_and_ref("gqa8")
    H.compare_step(st.run_gpu(), ref, what="gqa8 auto")


# ----------------------------------------------------------------------------
# Chunked prefill
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("hq,hkv,d", [(10, 2, 128), (16, 2, 128), (4, 4, 128), (8, 2, 64),
                                     (32, 2, 128), (24, 2, 128), (8, 4, 128), (12, 4, 128),
                                     (14, 2, 128)],
                         ids=["g5", "g8", "mha", "g4_d64", "g16", "g12", "g2", "g3", "g7"])
def test_chunked_prefill(hq, hkv, d):
    lay = lay_mixed(hq, hkv, d)
    st = H.Step.from_host(lay)
    ref = st.run_oracle()
    got = st.run_gpu()
    H.compare_step(got, ref, what=f"mixed {hq}/{hkv}/{d}")
    assert pa().pa_get_device_error() == 0


@pytest.mark.parametrize("hq,hkv", [(16, 2), (10, 2), (4, 4), (32, 2), (24, 2)],
                         ids=["g8", "g5", "mha", "g16", "g12"])
def test_chunked_prefill_short_prompts(hq, hkv):
    # fresh prompts of a few tokens (c = 0) and short chunks on short caches
    chunks = [2, 3, 5, 8, 16, 1, 4, 7]
    cached = [0, 0, 0, 0, 0, 3, 2, 9]
    lens = [c + n for c, n in zip(cached, chunks)]
    lay = synth.build_layout("pf_short", 111, lens, num_q_heads=hq, num_kv_heads=hkv,
                             head_dim=128, q_lens=chunks, is_prefill=[True] * len(chunks))
    st = H.Step.from_host(lay)
    H.compare_step(st.run_gpu(), st.run_oracle(), what=f"short prefill {hq}/{hkv}")


@pytest.mark.parametrize("hq,hkv,short", [(10, 2, False), (32, 2, True), (4, 4, True)],
                         ids=["g5_mixed", "g16_short", "mha_short"])
def test_chunked_prefill_exact_weights(hq, hkv, short):
    # With every key tile's P.V carrying the weights' bf16 remainder, each
    # weight reaches the product to within 2^-15 of itself, so the output is
    # the exact attention up to its own bf16 rounding (half an ulp: at most
    # 2^-8 of the value) and fp32 accumulation.
    if short:
        chunks, cached = [2, 3, 5, 8, 16, 1, 4, 7], [0, 0, 0, 0, 0, 3, 2, 9]
        lay = synth.build_layout("pf_exact", 112, [c + n for c, n in zip(cached, chunks)],
                                 num_q_heads=hq, num_kv_heads=hkv, head_dim=128, q_lens=chunks,
                                 is_prefill=[True] * len(chunks))
    else:
        lay = lay_mixed(hq, hkv, 128)
    st = H.Step.from_host(lay)
    ref = st.run_oracle()
    got = st.run_gpu(exact_weights=True)
    out = H.host_f64(got["prefill"][0])
    want = ref["prefill"][0]
    bound = 2.0 ** -8 * np.abs(want) * 1.001 + 1e-4
    diff = np.abs(out - want)
    assert np.all(diff <= bound), (
        f"{int((diff > bound).sum())} of {diff.size} over; worst excess "
        f"{float((diff - bound).max()):.3e}")
    # the default (weights' remainder where a tile's share calls for it) stays
    # inside the stated tolerance on the same inputs
    H.compare_step(st.run_gpu(), ref, what=f"adaptive {hq}/{hkv}")
    assert pa().pa_get_device_error() == 0


def test_chunked_prefill_rejects_unknown_flags():
    import ctypes
    lib = pa().lib()
    st = H.Step.from_host(lay_mixed(10, 2, 128))
    assert lib.pa_chunked_prefill_ex(None, 0, None, 0, 0, None, None, pa().pool_desc(st.k_pool),
                                     None, 1, None, 0, 10, ctypes.c_float(1.0), None, None,
                                     ctypes.c_uint32(0x2), None) == 1  # PA_ERR_ARG


def test_prefill_of_twelve_tokens_in_chunks_of_four_equals_one_chunk():
    # the pages' example (budget 6, 12-token prompt, 4 tokens a round), run as
    # three chunked-prefill calls against one 12-token call
    lay = synth.build_layout("p12", 108, [12], num_q_heads=8, num_kv_heads=2, head_dim=128,
                             q_lens=[12], is_prefill=[True])
    st = H.Step.from_host(lay)
    ref = st.run_oracle()
    pa().pa_reshape_and_cache(st.key, st.value, st.k_pool, st.v_pool, st.slot_mapping)
    whole, _ = pa().pa_chunked_prefill(st.q, H.dev_i32([0, 12]), 12, st.k_pool, st.v_pool,
                                       st.tables, st.lens, lay.scale)
    parts = []
    for s, e, _ in synth.chunk_schedule(12, 4, 6):
        o, _ = pa().pa_chunked_prefill(st.q[s:e].contiguous(), H.dev_i32([0, e - s]), e - s,
                                       st.k_pool, st.v_pool, st.tables, H.dev_i32([e]), lay.scale)
        parts.append(H.host_f64(o))
    H.assert_close(np.concatenate(parts), ref["prefill"][0], what="chunks of 4")
    H.assert_close(H.host_f64(whole), ref["prefill"][0], what="one chunk")


# ----------------------------------------------------------------------------
# Edge cases and device-side checks
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("kernel", [1, 2])
def test_empty_and_single_token_contexts(kernel):
    lay = synth.build_layout("edge", 109, [0, 1, 2], num_q_heads=8, num_kv_heads=1, head_dim=128,
                             num_blocks=4)
    lay.q_lens = np.array([0, 1, 1], np.int32)
    st = H.Step.from_host(lay)
    pa().pa_reshape_and_cache(st.key, st.value, st.k_pool, st.v_pool, st.slot_mapping)
    try:
        out, lse = pa().pa_decode(st.q[[0, 0, 1]].contiguous(), st.k_pool, st.v_pool, st.tables,
                                  st.lens, lay.scale, kernel=kernel, want_lse=True)
    except pa().PaError:
        pytest.skip("kernel not built for this shape")
    o = H.host_f64(out)
    assert np.all(o[0] == 0) and np.all(np.isneginf(lse[0].cpu().numpy()))
    # one token: the output is that token's value, exactly
    v0 = oracle.bf16_bits_to_f64(st.host["value"][0])
    assert np.array_equal(o[1], np.broadcast_to(v0, o[1].shape))


@pytest.mark.parametrize("kernel", [1, 2])
def test_bad_block_id_is_flagged_not_read(kernel):
    lay = lay_gqa8()
    st = H.Step.from_host(lay)
    pa().pa_reshape_and_cache(st.key, st.value, st.k_pool, st.v_pool, st.slot_mapping)
    assert pa().pa_get_device_error() == 0
    tab = lay.block_tables.copy()
    tab[3, 5] = lay.num_blocks + 7  # needed by sequence 3 (3000 tokens)
    try:
        out, _ = pa().pa_decode(st.q, st.k_pool, st.v_pool, H.dev_i32(tab), st.lens, lay.scale,
                                kernel=kernel)
    except pa().PaError:
        pytest.skip("kernel not built for this shape")
    flags = pa().pa_get_device_error()
    assert flags & pa().PA_DEV_ERR_BLOCK_ID
    assert np.all(np.isfinite(H.host_f64(out)))
    assert pa().pa_get_device_error() == 0  # cleared by the read


def test_bad_slot_and_context_are_flagged():
    lay = synth.tiny()
    st = H.Step.from_host(lay)
    sm = lay.slot_mapping().copy()
    sm[0] = lay.num_blocks * 16 + 3
    pa().pa_reshape_and_cache(st.key, st.value, st.k_pool, st.v_pool, H.dev_i64(sm))
    assert pa().pa_get_device_error() & pa().PA_DEV_ERR_SLOT
    lens = lay.context_lens.copy()
    lens[1] = lay.max_blocks * 16 + 1
    pa().pa_decode(st.q, st.k_pool, st.v_pool, st.tables, H.dev_i32(lens), lay.scale)
    assert pa().pa_get_device_error() & pa().PA_DEV_ERR_CONTEXT
