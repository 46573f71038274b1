"""Helpers for the GPU parity tests: move the seeded inputs to the device, run
one batch step through the library, run the same step through the oracle, and
compare.  The oracle always works on host copies of the inputs taken before any
library call touched them."""
from __future__ import annotations

import numpy as np

import oracle
from workloads import synth

ATOL = 2e-3
RTOL = 1e-2
LSE_ATOL = 1e-3


def torch():
    import torch as t
    return t


def dev_bf16(bits):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(t.bfloat16)


def dev_i32(a):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(np.asarray(a, np.int32))).cuda()


def dev_i64(a):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(np.asarray(a, np.int64))).cuda()


def host_bits(x) -> np.ndarray:
    t = torch()
    return x.contiguous().view(t.int16).cpu().numpy().view(np.uint16)


def host_f64(x) -> np.ndarray:
    return x.float().cpu().numpy().astype(np.float64)


def assert_close(got, want, atol=ATOL, rtol=RTOL, what=""):
    """Element passes if |got - want| <= atol or <= rtol * |want|."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    diff = np.abs(got - want)
    ok = (diff <= atol) | (diff <= rtol * np.abs(want))
    if not ok.all():
        bad = np.argwhere(~ok)
        i = tuple(bad[0])
        big = np.abs(want) > atol
        rel = (diff[big] / np.abs(want[big])).max() if big.any() else 0.0
        raise AssertionError(
            f"{what}: {len(bad)} of {ok.size} elements out of tolerance; first at {i}: "
            f"got {got[i]!r} want {want[i]!r}; max abs {diff.max():.3e}, max rel {rel:.3e}")
    return float(diff.max())


def assert_lse_close(got, want, what=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    inf = np.isinf(want)
    assert np.array_equal(np.isinf(got), inf), f"{what}: -inf pattern differs"
    if (~inf).any():
        d = np.abs(got[~inf] - want[~inf]).max()
        assert d <= LSE_ATOL, f"{what}: lse max abs diff {d:.3e}"


# ----------------------------------------------------------------------------
# One batch step
# ----------------------------------------------------------------------------
class Step:
    """Device copies of a step's inputs plus the host copies the oracle uses."""

    def __init__(self, layout: synth.Layout, host: dict):
        t = torch()
        self.layout = layout
        self.host = host  # bf16 bit patterns (NumPy) as generated
        self.k_pool = dev_bf16(host["k_pool"])
        self.v_pool = dev_bf16(host["v_pool"])
        self.q = dev_bf16(host["q"])
        self.key = dev_bf16(host["key"])
        self.value = dev_bf16(host["value"])
        self.slot_mapping = dev_i64(layout.slot_mapping())
        self.tables = dev_i32(layout.block_tables)
        self.lens = dev_i32(layout.context_lens)
        self.device = t.device("cuda")

    @classmethod
    def from_host(cls, layout, seed=None, poison=True):
        return cls(layout, synth.fill_host(layout, seed=seed, poison=poison))

    def rows_tensor(self, rows):
        return torch().as_tensor(np.asarray(rows, np.int64), device="cuda")

    def run_gpu(self, kernel=0, partition=0, want_lse=True, exact_weights=False):
        """copy_blocks -> reshape_and_cache -> decode (decode rows) and chunked
        prefill (prefill rows).  Returns dict of outputs keyed 'decode'/'prefill'."""
        import paged_kv_cache_454_b200 as pa
        lay = self.layout
        res = {}
        if lay.copy_pairs.size:
            pa.pa_copy_blocks(self.k_pool, self.v_pool, lay.copy_pairs)
        pa.pa_reshape_and_cache(self.key, self.value, self.k_pool, self.v_pool, self.slot_mapping)
        dec = lay.decode_rows()
        if len(dec):
            r = self.rows_tensor(dec)
            qi = self.rows_tensor(synth.token_rows(lay, dec))
            out, lse = pa.pa_decode(self.q.index_select(0, qi), self.k_pool, self.v_pool,
                                    self.tables.index_select(0, r).contiguous(),
                                    self.lens.index_select(0, r).contiguous(), lay.scale,
                                    kernel=kernel, partition_tokens=partition, want_lse=want_lse)
            res["decode"] = (out, lse)
        pf = lay.prefill_rows()
        if len(pf):
            r = self.rows_tensor(pf)
            qi = self.rows_tensor(synth.token_rows(lay, pf))
            cu = dev_i32(lay.cu_q_lens(pf))
            out, lse = pa.pa_chunked_prefill(self.q.index_select(0, qi), cu,
                                             int(lay.q_lens[pf].max()), self.k_pool, self.v_pool,
                                             self.tables.index_select(0, r).contiguous(),
                                             self.lens.index_select(0, r).contiguous(), lay.scale,
                                             want_lse=want_lse, exact_weights=exact_weights)
            res["prefill"] = (out, lse)
        torch().cuda.synchronize()
        return res

    def run_oracle(self):
        lay = self.layout
        h = self.host
        kp, vp = h["k_pool"], h["v_pool"]
        if lay.copy_pairs.size:
            kp, vp = oracle.copy_blocks(kp, vp, lay.copy_pairs)
        kp, vp = oracle.reshape_and_cache(kp, vp, h["key"], h["value"], lay.slot_mapping())
        res = {"pools": (kp, vp)}
        dec = lay.decode_rows()
        if len(dec):
            qi = synth.token_rows(lay, dec)
            res["decode"] = oracle.decode(h["q"][qi], kp, vp, lay.block_tables[dec],
                                          lay.context_lens[dec], lay.scale)
        pf = lay.prefill_rows()
        if len(pf):
            qi = synth.token_rows(lay, pf)
            res["prefill"] = oracle.chunked_prefill(h["q"][qi], lay.cu_q_lens(pf), kp, vp,
                                                    lay.block_tables[pf], lay.context_lens[pf],
                                                    lay.scale)
        return res


def compare_step(gpu: dict, ref: dict, what=""):
    worst = 0.0
    for key in ("decode", "prefill"):
        if key in ref:
            out, lse = gpu[key]
            worst = max(worst, assert_close(host_f64(out), ref[key][0], what=f"{what} {key} out"))
            if lse is not None:
                assert_lse_close(lse.cpu().numpy(), ref[key][1], what=f"{what} {key} lse")
    return worst


# ----------------------------------------------------------------------------
# Full-size steps (pools drawn on the device), checked on sampled sequences
# ----------------------------------------------------------------------------
class FullStep:
    """A full-size batch step on the device.  Before any library call, host
    copies of the sampled sequences' blocks and tokens are taken for the oracle
    (through ``synth.subset``)."""

    def __init__(self, layout: synth.Layout, sample_rows, seed=None):
        t = torch()
        self.layout = layout
        self.dev = t.device("cuda")
        self.t = synth.fill_device(layout, self.dev, seed=seed)
        self.sample_rows = [int(r) for r in sample_rows]
        self.sub, blocks = synth.subset(layout, self.sample_rows)
        idx = t.as_tensor(blocks, device=self.dev)
        tok = t.as_tensor(synth.token_rows(layout, self.sample_rows), device=self.dev)
        self.host = {
            "k_pool": host_bits(self.t["k_pool"].index_select(0, idx)),
            "v_pool": host_bits(self.t["v_pool"].index_select(0, idx)),
            "q": host_bits(self.t["q"].index_select(0, tok)),
            "key": host_bits(self.t["key"].index_select(0, tok)),
            "value": host_bits(self.t["value"].index_select(0, tok)),
        }

    def run_gpu(self):
        """The step as bench.py runs it: block copies, cache write, chunked
        prefill of the prefill rows, decode of the decode rows (default kernel
        choice and partitioning)."""
        import paged_kv_cache_454_b200 as pa
        t = torch()
        lay, d = self.layout, self.t
        tens = lambda a, dt: t.as_tensor(np.ascontiguousarray(a), dtype=dt, device=self.dev)
        if lay.copy_pairs.size:
            pa.pa_copy_blocks(d["k_pool"], d["v_pool"], lay.copy_pairs)
        pa.pa_reshape_and_cache(d["key"], d["value"], d["k_pool"], d["v_pool"],
                                tens(lay.slot_mapping(), t.int64))
        res = {}
        pf = lay.prefill_rows()
        if len(pf):
            q = d["q"][tens(synth.token_rows(lay, pf), t.int64)].contiguous()
            res["prefill"] = pa.pa_chunked_prefill(
                q, tens(lay.cu_q_lens(pf), t.int32), int(lay.q_lens[pf].max()), d["k_pool"],
                d["v_pool"], tens(lay.block_tables[pf], t.int32),
                tens(lay.context_lens[pf], t.int32), lay.scale, want_lse=True)
            res["prefill_rows"] = pf
        dec = lay.decode_rows()
        if len(dec):
            q = d["q"][tens(synth.token_rows(lay, dec), t.int64)].contiguous()
            res["decode"] = pa.pa_decode(q, d["k_pool"], d["v_pool"],
                                         tens(lay.block_tables[dec], t.int32),
                                         tens(lay.context_lens[dec], t.int32), lay.scale,
                                         want_lse=True)
            res["decode_rows"] = dec
        t.cuda.synchronize()
        return res

    def check(self, res, what=""):
        """Sampled sequences against the oracle, plus whole-batch properties."""
        lay, sub, h = self.layout, self.sub, self.host
        kp, vp = h["k_pool"], h["v_pool"]
        if sub.copy_pairs.size:
            kp, vp = oracle.copy_blocks(kp, vp, sub.copy_pairs)
        kp, vp = oracle.reshape_and_cache(kp, vp, h["key"], h["value"], sub.slot_mapping())
        starts = np.concatenate([[0], np.cumsum(sub.q_lens)])
        for kind in ("decode", "prefill"):
            if kind not in res:
                continue
            out, lse = res[kind]
            outf = out.float()
            assert bool(torch().isfinite(outf).all()), f"{what} {kind}: non-finite output"
            rows = list(res[kind + "_rows"])
            # packed token offsets of each row of this call
            ql = lay.q_lens[rows]
            offs = dict(zip(rows, np.concatenate([[0], np.cumsum(ql)])[:-1]))
            for i, s in enumerate(self.sample_rows):
                if s not in offs:
                    continue
                n = int(lay.q_lens[s])
                qs = h["q"][starts[i]:starts[i] + n]
                if kind == "decode":
                    ref_o, ref_l = oracle.decode(qs, kp, vp, sub.block_tables[i:i + 1],
                                                 sub.context_lens[i:i + 1], lay.scale)
                else:
                    ref_o, ref_l = oracle.chunked_prefill(qs, np.array([0, n]), kp, vp,
                                                          sub.block_tables[i:i + 1],
                                                          sub.context_lens[i:i + 1], lay.scale)
                o0 = int(offs[s])
                assert_close(host_f64(out[o0:o0 + n]), ref_o, what=f"{what} {kind} seq {s}")
                assert_lse_close(lse[o0:o0 + n].cpu().numpy(), ref_l, what=f"{what} {kind} seq {s}")
