"""Plant plausible mistakes in the block-manager oracle and check that its pins
catch each one (the pins are only worth something if they fail on a wrong
manager).  Each mutant replaces one method of ``oracle.KvManager`` for the
duration of one test."""
from __future__ import annotations

from collections import OrderedDict

import pytest

import oracle.kv_manager as km
import test_kv_manager_oracle as pins


def _no_cow_append(self, sid, tokens):
    s = self._seq(sid)
    slots = []
    L = s["len"]
    for t in tokens:
        if L % self.bs == 0:
            s["table"].append(self._alloc())
        slots.append(s["table"][L // self.bs] * self.bs + L % self.bs)
        s["tokens"].append(int(t))
        L += 1
    s["len"] = L
    return slots, []


def _leaky_release(self, b):
    self.ref[b] -= 1


def _fork_without_retain(self, parent, child):
    p = self._seq(parent)
    self.seqs[child] = {"table": list(p["table"]), "len": p["len"], "tokens": list(p["tokens"])}


def _uncache_only_itself(self, b):
    p = self.prefix_of.pop(b)
    del self.cache[p]


def _free_head_first(self, sid):
    s = self._seq(sid)
    for b in s["table"]:
        self._release(b)
    del self.seqs[sid]


def _register_any_prefix(self, b, prefix):
    if self.prefix_caching:
        self.cache[prefix] = b          # overwrites an existing entry
        self.prefix_of[b] = prefix


MUTANTS = {
    "append never copies a shared block": ("append_tokens", _no_cow_append),
    "released blocks never return to the pool": ("_release", _leaky_release),
    "fork does not raise reference counts": ("fork", _fork_without_retain),
    "eviction keeps prefixes that ran through the block": ("_uncache", _uncache_only_itself),
    "free releases the first block first": ("free_sequence", _free_head_first),
    "a full block replaces an existing cache entry": ("_register", _register_any_prefix),
}

# the pins that run against every mutant: the hand-made scenarios and a few
# seeded random streams
SCENARIOS = [
    pins.test_on_demand_allocation_uses_every_block_but_the_last,
    pins.test_outputs_of_one_prompt_share_its_blocks_and_the_first_writers_copy,
    pins.test_full_block_tail_needs_no_copy,
    pins.test_share_prefix_and_share_blocks,
    pins.test_prefix_cache_reuses_whole_blocks_from_position_zero,
    pins.test_prefix_cache_survives_free_and_blocks_filled_by_decode_are_cached,
    pins.test_eviction_takes_the_longest_unreferenced_and_its_extensions,
    pins.test_evicting_a_block_drops_the_prefixes_through_it,
    pins.test_operations_are_all_or_nothing,
] + [(lambda s=s, pc=pc: pins.test_random_streams_keep_every_sequence_readable(s, pc))
     for s in range(6) for pc in (False, True)]


def _some_pin_fails():
    for f in SCENARIOS:
        try:
            f()
        except Exception:   # noqa: BLE001 -- any failure of a pin counts
            return True
    return False


@pytest.mark.parametrize("name", list(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(km.KvManager, attr, fn)
    assert _some_pin_fails(), f"no pin caught: {name}"


def test_unmutated_oracle_passes_every_pin():
    assert not _some_pin_fails()
    assert isinstance(km.KvManager(4, 4, True).evictable, OrderedDict)
