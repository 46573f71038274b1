"""Pins of the block-swap oracle (``oracle.swap_blocks``), CPU only.

"当大模型推理遇上内存瓶颈", 5.1 and 7.3: KV blocks move to a CPU swap space and
come back when needed.  What fixes the result without retyping the copy:
a hand-worked three-block example, the round trip (out and back restores the
device pool bit for bit), untouched blocks staying untouched, agreement with
``copy_blocks`` when both sides are one pool, and the range / repeated
destination rules."""
from __future__ import annotations

import numpy as np
import pytest

from oracle import CopyBlocksError, copy_blocks, swap_blocks


def filled(nb, value0, shape=(2, 16, 8)):
    """Pools whose block b holds the constant value0 + b (K) and 1000 + value0 + b (V)."""
    k = np.empty((nb,) + shape, np.uint16)
    v = np.empty_like(k)
    for b in range(nb):
        k[b] = value0 + b
        v[b] = 1000 + value0 + b
    return k, v


def test_hand_worked_example():
    dk, dv = filled(3, 10)       # device blocks hold 10, 11, 12
    hk, hv = filled(4, 50)       # host blocks hold 50, 51, 52, 53
    # out: device 0 -> host 3, device 2 -> host 0
    k, v = swap_blocks(dk, dv, hk, hv, [[0, 3], [2, 0]])
    assert [int(k[b].flat[0]) for b in range(4)] == [12, 51, 52, 10]
    assert [int(v[b].flat[0]) for b in range(4)] == [1012, 1051, 1052, 1010]
    # every element of a moved block moved, not only its first
    assert np.all(k[3] == 10) and np.all(v[0] == 1012)
    # the inputs are not modified
    assert int(hk[3].flat[0]) == 53 and int(dk[0].flat[0]) == 10


def test_round_trip_restores_the_device_pool():
    rng = np.random.default_rng(3)
    dk = rng.integers(0, 1 << 16, size=(9, 4, 16, 32), dtype=np.uint16)
    dv = rng.integers(0, 1 << 16, size=dk.shape, dtype=np.uint16)
    hk = np.zeros((6,) + dk.shape[1:], np.uint16)
    hv = np.zeros_like(hk)
    out = np.array([[8, 0], [1, 5], [4, 2]])
    hk2, hv2 = swap_blocks(dk, dv, hk, hv, out)
    # the device blocks are reused for something else meanwhile
    dk_reused, dv_reused = dk.copy(), dv.copy()
    dk_reused[[8, 1, 4]] = 7
    dv_reused[[8, 1, 4]] = 9
    back = out[:, ::-1]
    k, v = swap_blocks(hk2, hv2, dk_reused, dv_reused, back)
    assert np.array_equal(k, dk) and np.array_equal(v, dv)
    # host blocks that took no part stay zero
    for b in (1, 3, 4):
        assert not hk2[b].any() and not hv2[b].any()


def test_same_pool_equals_copy_blocks():
    rng = np.random.default_rng(4)
    k = rng.integers(0, 1 << 16, size=(7, 2, 16, 8), dtype=np.uint16)
    v = rng.integers(0, 1 << 16, size=k.shape, dtype=np.uint16)
    pairs = [[0, 3], [1, 5], [2, 6]]   # no destination is a source
    a = swap_blocks(k, v, k, v, pairs)
    b = copy_blocks(k, v, pairs)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_rules():
    dk, dv = filled(3, 0)
    hk, hv = filled(2, 0)
    with pytest.raises(CopyBlocksError):
        swap_blocks(dk, dv, hk, hv, [[3, 0]])          # source outside
    with pytest.raises(CopyBlocksError):
        swap_blocks(dk, dv, hk, hv, [[0, 2]])          # destination outside
    with pytest.raises(CopyBlocksError):
        swap_blocks(dk, dv, hk, hv, [[0, 1], [2, 1]])  # repeated destination
    # a source may repeat (one block saved twice) and the empty list is a no-op
    k, v = swap_blocks(dk, dv, hk, hv, [[1, 0], [1, 1]])
    assert np.all(k == 1) and np.all(v == 1001)
    k, v = swap_blocks(dk, dv, hk, hv, np.zeros((0, 2), np.int64))
    assert np.array_equal(k, hk) and np.array_equal(v, hv)
