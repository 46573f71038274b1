"""CPU oracle for paged attention over a block-paged KV pool.

TEST INFRASTRUCTURE ONLY.  This package is the plain, slow, obviously correct
definition of what the CUDA library computes, in NumPy float64.  Only the tests,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs
of ``bench.py`` may import it.  It shares no code with the CUDA path and imports
nothing from it; the only thing both sides share is the seeded input generator
in ``workloads``.

The attention functions are pinned by ``tests/test_oracle_pins.py`` against
closed forms, invariants the pages state, a brute-force scalar implementation
and the pages' own worked numbers; the block manager by
``tests/test_kv_manager_oracle.py``, the sampler by ``tests/test_sampler_oracle.py``
and the block swap by ``tests/test_swap_oracle.py``.  Each docstring names the
passage it follows.
"""
from .paged_attention import (  # noqa: F401
    bf16_bits_to_f64,
    f64_to_bf16_bits,
    slot_of,
    gather_kv,
    attend,
    decode,
    chunked_prefill,
    reshape_and_cache,
    copy_blocks,
    swap_blocks,
    CopyBlocksError,
)
from .kv_manager import KvManager, KvManagerError, NoBlocks  # noqa: F401,E402
from . import sampler  # noqa: F401,E402
