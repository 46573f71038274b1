"""Full-size parity: each named workload at its full size, run the way bench.py
runs it (default kernel choice and partitioning), with sampled sequences
checked against the oracle (all their q heads; every query row of a sampled
prefill chunk) and whole-batch properties (finite outputs, no device error)."""
import numpy as np
import pytest

from workloads import synth

import gpu_helpers as H

pytestmark = pytest.mark.gpu


def _samples(lay, rows, k_random=6, seed=0):
    """First, last, longest, shortest and a few random rows of `rows`; where
    rows share their first physical block (samples of one prompt, which the
    plan may lay out side by side), every row sharing it with the first and
    the last row too."""
    rows = list(rows)
    if not rows:
        return []
    lens = lay.context_lens[rows]
    pick = {rows[0], rows[-1], rows[int(np.argmax(lens))], rows[int(np.argmin(lens))]}
    rng = np.random.default_rng(seed)
    pick.update(int(x) for x in rng.choice(rows, size=min(k_random, len(rows)), replace=False))
    first = {int(lay.block_tables[r, 0]) for r in (rows[0], rows[-1]) if lay.context_lens[r] > 0}
    pick.update(r for r in rows if lay.context_lens[r] > 0 and int(lay.block_tables[r, 0]) in first)
    return sorted(pick)


@pytest.mark.parametrize("name", ["llama7b_decode", "llama13b_sampling", "gqa70b_long",
                                  "mixed_qwen32b"])
def test_full_size_sampled(name):
    import paged_kv_cache_454_b200 as pa
    lay = synth.CONFIGS[name]()
    rows = _samples(lay, lay.decode_rows())
    pf = list(lay.prefill_rows())
    if pf:  # two prefill chunks: the one on the longest cache and the first
        rows = sorted(set(rows) | {pf[int(np.argmax(lay.context_lens[pf]))], pf[0]})
    step = H.FullStep(lay, rows)
    res = step.run_gpu()
    assert pa.pa_get_device_error() == 0
    step.check(res, what=name)


def test_tiny_config_all_outputs():
    lay = synth.tiny()
    step = H.FullStep(lay, range(lay.num_seqs))
    step.check(step.run_gpu(), what="tiny")
