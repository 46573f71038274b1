"""The paged read-bandwidth probe (``pa_read_probe``) reads exactly the pages a
decode over the same tables reads.

Its per-CTA sums, added modulo 2^64, must equal the sum of the 32-bit words of
every (block, KV head) page of K and of V under ceil(L / block_size) table
entries of each sequence -- computed here with NumPy from host copies of the
pools -- whatever the number of CTAs.  Pages a sequence names twice count
twice; a table entry outside the pool is skipped and flagged."""
from __future__ import annotations

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

MASK64 = (1 << 64) - 1


def pa():
    import paged_kv_cache_454_b200 as m
    return m


def page_sums(pool_np):
    """uint64 [num_blocks, Hkv]: sum of each page's 32-bit words."""
    nb, hkv = pool_np.shape[:2]
    words = pool_np.reshape(nb, hkv, -1).view(np.uint32).astype(np.uint64)
    return words.sum(axis=2)


def expected(kp, vp, tables, lens, bs=16):
    ks, vs = page_sums(kp), page_sums(vp)
    nb = kp.shape[0]
    tot = 0
    for s, L in enumerate(lens):
        L = max(0, min(int(L), tables.shape[1] * bs))
        for b in range(-(-L // bs)):
            p = int(tables[s, b])
            if 0 <= p < nb:
                tot += int(ks[p].sum()) + int(vs[p].sum())
    return tot & MASK64


def make(seed, nb, hkv, d, lens, max_blocks):
    import torch
    rng = np.random.default_rng(seed)
    bits = rng.integers(0, 1 << 16, size=(2, nb, hkv, 16, d), dtype=np.uint16)
    tables = rng.integers(0, nb, size=(len(lens), max_blocks), dtype=np.int32)
    dev = torch.device("cuda")
    kp = torch.from_numpy(bits[0].view(np.int16)).to(dev).view(torch.bfloat16)
    vp = torch.from_numpy(bits[1].view(np.int16)).to(dev).view(torch.bfloat16)
    t = torch.from_numpy(tables).to(dev)
    l = torch.from_numpy(np.asarray(lens, np.int32)).to(dev)
    return bits[0], bits[1], tables, kp, vp, t, l


def total(out):
    return int(sum(int(x) & MASK64 for x in out.cpu().numpy().astype(np.int64))) & MASK64


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("ctas", [1, 3, 148, 300])
def test_sums_match_every_page(d, ctas):
    lens = [0, 1, 15, 16, 17, 127, 128, 129, 300, 1000, 5]
    kb, vb, tables, kp, vp, t, l = make(d + ctas, 97, 3, d, lens, 64)
    out = pa().pa_read_probe(kp, vp, t, l, num_ctas=ctas)
    assert pa().pa_get_device_error() == 0
    assert total(out) == expected(kb, vb, tables, lens)


def test_empty_batch_writes_zero_sums():
    import torch
    kb, vb, tables, kp, vp, t, l = make(1, 8, 2, 128, [0, 0, 0], 4)
    out = pa().pa_read_probe(kp, vp, t, l, num_ctas=5)
    assert out.cpu().tolist() == [0] * 5
    kp2, vp2 = kp, vp
    t0 = torch.empty((0, 4), dtype=torch.int32, device="cuda")
    l0 = torch.empty((0,), dtype=torch.int32, device="cuda")
    out = pa().pa_read_probe(kp2, vp2, t0, l0, num_ctas=2)
    assert out.cpu().tolist() == [0, 0]


def test_bad_block_id_is_skipped_and_flagged():
    lens = [40, 70]
    kb, vb, tables, kp, vp, t, l = make(5, 31, 4, 128, lens, 8)
    tables[1, 2] = 31          # one past the pool
    tables[0, 1] = -3
    import torch
    t.copy_(torch.from_numpy(tables))
    out = pa().pa_read_probe(kp, vp, t, l, num_ctas=7)
    err = pa().pa_get_device_error()
    assert err & pa().PA_DEV_ERR_BLOCK_ID
    assert total(out) == expected(kb, vb, tables, lens)


def test_context_beyond_the_table_is_clamped_and_flagged():
    lens = [16 * 6 + 3, 10]    # 6 table entries hold 96 tokens
    kb, vb, tables, kp, vp, t, l = make(6, 40, 2, 64, lens, 6)
    out = pa().pa_read_probe(kp, vp, t, l, num_ctas=4)
    assert pa().pa_get_device_error() & pa().PA_DEV_ERR_CONTEXT
    assert total(out) == expected(kb, vb, tables, lens)


def test_larger_batch_many_units_per_cta():
    rng = np.random.default_rng(9)
    lens = rng.integers(0, 4096, size=200).tolist()
    kb, vb, tables, kp, vp, t, l = make(9, 1024, 8, 128, lens, 256)
    out = pa().pa_read_probe(kp, vp, t, l)
    assert pa().pa_get_device_error() == 0
    assert total(out) == expected(kb, vb, tables, lens)


def test_host_argument_checks():
    import torch
    kb, vb, tables, kp, vp, t, l = make(2, 8, 2, 128, [5], 2)
    with pytest.raises(pa().PaError):
        pa().pa_read_probe(kp, vp, t, l, num_ctas=0)
    with pytest.raises(pa().PaError):
        pa().pa_read_probe(kp, vp, t, l, num_ctas=70000)
    big = torch.zeros((5000, 1), dtype=torch.int32, device="cuda")
    lens = torch.zeros((5000,), dtype=torch.int32, device="cuda")
    with pytest.raises(pa().PaError):
        pa().pa_read_probe(kp, vp, big, lens, num_ctas=2)
