"""Strength of the oracle's pins: plant a plausible mistake in a copy of the oracle
(on the CPU) and check that at least one pin rejects it."""
import math
import os
import types

import numpy as np
import pytest

import oracle as real_oracle
from oracle import brute
from tests.test_oracle_pins import (brute_decode, brute_prefill, pools_after_store, tiny_decode,
                                    tiny_prefill)

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle",
                   "paged_attention.py")

MUTANTS = {
    "scale dropped": ("z = scale * (K @ q)", "z = (K @ q)"),
    "gqa head map": ("            g = h // G\n            out[s, h]", "            g = h % Hkv\n            out[s, h]"),
    "prefill gqa head map": ("            g = h // G\n            Z =", "            g = h % Hkv\n            Z ="),
    "causal off by one": ("<= pos[:, None]", "< pos[:, None]"),
    "position offset": ("first = ctx - n_new", "first = 0"),
    "row index": ("return block * block_size + pos % block_size",
                  "return block * block_size + pos // block_size"),
    "normalisation": ("w = w / w.sum()", "w = w / w.max()"),
    "prefill K/V swapped": ("@ Kc[:, g, :].T)", "@ Vc[:, g, :].T)"),
    "decode transposed operand": ("return w @ V", "return w @ K"),
    "store ignores skip": ("        if slot < 0:\n            continue\n", ""),
    "no max subtraction": ("z = z - z.max()", "z = z - z.min()"),
    "prefill scale dropped": ("Z = scale * (qf", "Z = (qf"),
    "copy direction": ("        kc[b] = k_cache[a]\n        vc[b] = v_cache[a]",
                       "        kc[a] = k_cache[b]\n        vc[a] = v_cache[b]"),
    "copy only K": ("        vc[b] = v_cache[a]\n", ""),
}


def _mutant(old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique/found: {old!r}"
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


def _pins(m):
    """Run a compact set of the oracle pins against module m; return names that failed."""
    failed = []

    def check(name, fn):
        try:
            ok = fn()
        except Exception:
            ok = False
        if not ok:
            failed.append(name)

    def decode_brute():
        w = tiny_decode(G=2, bs=4, D=8, seed=301)
        kc, vc = pools_after_store(w, m)
        got = m.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale)
        return np.max(np.abs(got - brute_decode(w))) < 1e-12

    def prefill_brute():
        w = tiny_prefill(G=2, bs=4, seed=302)
        kc, vc = pools_after_store(w, m)
        got = m.prefill(w.q, kc, vc, w.block_tables, w.cu_seqlens_q, w.context_lens, w.scale)
        return np.max(np.abs(got - brute_prefill(w))) < 1e-12

    def peaked():
        w = tiny_decode(G=2, bs=4, D=16, q_factor=400.0, seed=5)
        kc, vc = pools_after_store(w, m)
        got = m.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale)
        return np.all(np.isfinite(got)) and np.max(np.abs(got - brute_decode(w))) < 1e-9

    def store_exact():
        w = tiny_decode(G=1, bs=4, D=8, lens=(5, 9), seed=41)
        slots = w.setup_slots.copy()
        slots[-1] = -1                      # the last token is skipped
        k = w.setup_k
        kc, _ = m.store_kvcache(w.empty_pool(), w.empty_pool(), k, w.setup_v, slots)
        flat = kc.reshape(-1, w.num_kv_heads, w.head_dim)
        for r in range(flat.shape[0]):
            hits = np.where(slots == r)[0]
            want = k[hits[-1]] if len(hits) else np.full_like(flat[r], 0xFFC1)
            if not np.array_equal(flat[r], want):
                return False
        return True

    def two_key_closed_form():
        from tests.test_oracle_pins import _manual
        import oracle
        saved = oracle.decode, oracle.store_kvcache
        try:
            oracle.decode, oracle.store_kvcache = m.decode, m.store_kvcache
            out = _manual([1.0, 0.0], [[0.0, 0.0], [2.0, 0.0]], [[1.0, 0.0], [0.0, 1.0]], scale=0.5)
        finally:
            oracle.decode, oracle.store_kvcache = saved
        e = math.e
        return np.allclose(out, [1 / (1 + e), e / (1 + e)], atol=1e-14)

    check("decode brute", decode_brute)
    check("prefill brute", prefill_brute)
    check("peaked", peaked)
    check("store exact", store_exact)
    check("two-key closed form", two_key_closed_form)

    def cow_append():
        from tests.test_oracle_pins import cow_workload, run_cow_decode
        _, (w2, src, dst) = cow_workload(seed=311)
        out, _ = run_cow_decode(w2, src, dst, m)
        return np.max(np.abs(out - brute_decode(w2))) < 1e-12

    check("copy-on-write append", cow_append)
    return failed


def test_real_oracle_passes_the_compact_pins():
    assert _pins(real_oracle.paged_attention) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_each_planted_mistake_is_caught(name):
    old, new = MUTANTS[name]
    failed = _pins(_mutant(old, new))
    assert failed, f"mutant '{name}' passed every pin"
