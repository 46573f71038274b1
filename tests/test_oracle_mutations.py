"""Plant plausible mistakes in the oracle (on the CPU) and show the pins catch them.

Each mutant is the oracle function's own source with one edit (a dropped term, a
wrong index, a swapped operand, an off-by-one), compiled in the oracle module's
namespace and patched in for the duration of the test.  The test passes when at
least one pin in ``test_oracle_pins.ALL_CHECKS`` fails on the mutant.
"""
import inspect
import textwrap

import pytest

import oracle
from oracle import paged_attention as pa

import test_oracle_pins as pins

MUTANTS = [
    # (function, original text, mutated text, what goes wrong)
    ("attend", "x = scale * (K @ q)", "x = K @ q", "scale dropped"),
    ("attend", "(w @ V) / z", "(w @ K) / z", "K used in place of V"),
    ("attend", "m + np.log(z)", "np.log(z)", "max dropped from the log-sum-exp"),
    ("attend", "w = np.exp(x - m)", "w = np.exp(x)", "max shift dropped from the weights only"),
    ("_kv_head_of", "h // (num_q_heads // num_kv_heads)", "h % num_kv_heads",
     "interleaved instead of contiguous GQA groups"),
    ("gather_kv", "p = int(block_table_row[b])", "p = b", "block table ignored"),
    ("gather_kv", "n = min(bs, L - b * bs)", "n = min(bs, L - b * bs - 1)",
     "last token of every block dropped"),
    ("gather_kv", "k_pool[p, :, :n, :]", "k_pool[p, :, bs - n:, :]",
     "tokens taken from the end of a partial block"),
    ("chunked_prefill", "limit = c + i + 1", "limit = c + i", "query does not see itself"),
    ("chunked_prefill", "limit = c + i + 1", "limit = c + i + 2", "query sees the next token"),
    ("slot_of", "* int(block_size) + offset", "* int(block_size) - offset", "wrong slot sign"),
    ("reshape_and_cache", "k[b, :, o, :] = key[t]", "k[b, :, o, :] = value[t]",
     "value written into the K pool"),
    ("reshape_and_cache", "if slot < 0:\n            continue", "if slot < -1:\n            continue",
     "padding slot not skipped"),
    ("copy_blocks", "k[d] = k_pool[s]", "k[s] = k_pool[d]", "copy direction reversed"),
    ("bf16_bits_to_f64", "<< 16", "<< 15", "wrong widening shift"),
]


def _mutant(name, old, new):
    src = textwrap.dedent(inspect.getsource(getattr(pa, name)))
    assert old in src, f"mutation anchor not found in {name}: {old!r}"
    ns = dict(vars(pa))
    exec(compile(src.replace(old, new, 1), f"<mutant {name}>", "exec"), ns)
    return ns[name]


@pytest.mark.parametrize("name,old,new,why", MUTANTS, ids=[m[3] for m in MUTANTS])
def test_pins_catch_mutant(monkeypatch, name, old, new, why):
    fn = _mutant(name, old, new)
    monkeypatch.setattr(pa, name, fn)
    if hasattr(oracle, name):
        monkeypatch.setattr(oracle, name, fn)
    failed = []
    for check in pins.ALL_CHECKS:
        try:
            check()
        except Exception as e:  # an assertion, or an error the mutant raises
            failed.append((check.__name__, type(e).__name__))
            break
    assert failed, f"no pin caught the mutant: {why}"


def test_unmutated_oracle_passes_every_pin():
    for check in pins.ALL_CHECKS:
        check()
