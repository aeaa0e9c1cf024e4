"""Strength of the fp8 oracle's pins: plant a plausible mistake in a copy of
oracle/fp8.py (on the CPU) and check that at least one pin rejects it."""
import math
import os
import types

import numpy as np
import pytest
import torch

import oracle
from oracle import fp8 as real_fp8
from workloads import build_workload, f32_to_bf16_bits

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "fp8.py")

MUTANTS = {
    "exponent bias": ("return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)",
                      "return sign * (1.0 + m / 8.0) * 2.0 ** (e - 8)"),
    "subnormal step": ("return sign * m * 2.0 ** -9", "return sign * m * 2.0 ** -8"),
    "ties away from zero": ("r = round(a / 2.0 ** e * 8.0)", "r = math.floor(a / 2.0 ** e * 8.0 + 0.5)"),
    "truncation": ("r = round(a / 2.0 ** e * 8.0)", "r = math.floor(a / 2.0 ** e * 8.0)"),
    "saturates to NaN": ("    if a >= E4M3_MAX:\n        return sign | 0x7E",
                         "    if a >= E4M3_MAX:\n        return sign | 0x7F"),
    "sign dropped": ("sign = 0x80 if (y < 0 or (y == 0 and math.copysign(1.0, y) < 0)) else 0",
                     "sign = 0"),
    "scale inverted": ("scales[i] = amax / np.float32(E4M3_MAX)",
                       "scales[i] = np.float32(E4M3_MAX) / amax"),
    "quantiser range": ("inv = np.float32(E4M3_MAX) / amax", "inv = np.float32(240.0) / amax"),
    "store offset transposed": ("b, o = divmod(slot, bs)", "o, b = divmod(slot, bs)"),
    "store ignores skip": ("        if slot < 0:\n            continue\n", ""),
    "V read with K scales": ("vf = dequantize(v_codes, v_scales)", "vf = dequantize(v_codes, k_scales)"),
    "GQA head map": ("Kc[:, h // G, :], Vc[:, h // G, :]", "Kc[:, h % Hkv, :], Vc[:, h % Hkv, :]"),
}


def _mutant(old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique/found: {old!r}"
    src = src.replace(old, new).replace("from .paged_attention import", "from oracle.paged_attention import")
    mod = types.ModuleType("fp8_mutant")
    exec(compile(src, "fp8_mutant", "exec"), mod.__dict__)
    return mod


def _pow2_rows(rng, shape, grid):
    """bf16 rows whose values are e4m3 values times a power of two chosen per row, with
    the row's largest magnitude at 448 times that power: quantising them is exact and
    the row's scale is the power of two."""
    k = rng.integers(-6, 5, size=shape[:-1] + (1,)).astype(np.float64)
    x = rng.choice(grid, size=shape) * rng.choice([-1.0, 1.0], size=shape)
    x[..., 0] = 448.0 * np.where(rng.random(shape[:-1]) < 0.5, -1.0, 1.0)
    return f32_to_bf16_bits((x * 2.0 ** k).astype(np.float32))


def _pins(m):
    failed = []

    def check(name, fn):
        try:
            ok = fn()
        except Exception:
            ok = False
        if not ok:
            failed.append(name)

    def round_trip():
        for c in range(256):
            v = m.e4m3_to_float(c)
            if c in (0x7F, 0xFF):
                if not math.isnan(v):
                    return False
                continue
            if m.float_to_e4m3(v) != c:
                return False
        return True

    def hand_codes():
        cases = [(1.0, 0x38), (448.0, 0x7E), (-448.0, 0xFE), (2.0 ** -9, 0x01), (2.0 ** -6, 0x08),
                 (-3.0, 0xC4), (1.0625, 0x38), (1.1875, 0x3A), (1.5 * 2.0 ** -9, 0x02), (464.0, 0x7E),
                 (1e6, 0x7E), (-1e6, 0xFE)]
        return all(m.float_to_e4m3(x) == c for x, c in cases)

    def hand_values():
        return (m.e4m3_to_float(0x38) == 1.0 and m.e4m3_to_float(0x7E) == 448.0
                and m.e4m3_to_float(0x01) == 2.0 ** -9 and m.e4m3_to_float(0xC4) == -3.0)

    def against_torch():
        rng = np.random.default_rng(91)
        x = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.uniform(-4, 2.6, 3000),
                            rng.uniform(-463.9, 463.9, 1000)]).astype(np.float32)
        x = x[np.abs(x) < 464.0]
        want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        got = np.array([m.float_to_e4m3(v) for v in x.astype(np.float64)], dtype=np.uint8)
        return np.array_equal(got, want)

    def quantiser_bound():
        rng = np.random.default_rng(92)
        x = f32_to_bf16_bits(rng.standard_normal((16, 2, 32)).astype(np.float32))
        codes, scales = m.quantize_rows(x)
        xf = oracle.bf16_bits_to_f64(x)
        amax = np.max(np.abs(xf), axis=-1)
        if not np.array_equal(scales, (amax / 448.0).astype(np.float32)):
            return False
        err = np.abs(m.dequantize(codes, scales) - xf)
        return bool(np.all(err <= 2.0 ** -4 * np.abs(xf) + 0.5 * 2.0 ** -9 * scales[..., None] + 1e-12))

    def exact_rows_decode():
        # per-row power-of-two scales, different for K and V: the fp8 decode must equal
        # the bf16 decode of the same values
        lens = np.array([5, 17, 1, 40, 0, 9])
        w = build_workload(kind="decode", context_lens=lens, new_lens=(lens > 0).astype(int),
                           num_q_heads=4, num_kv_heads=2, head_dim=8, block_size=4, seed=93)
        rng = np.random.default_rng(94)
        grid = np.array([real_fp8.e4m3_to_float(c) for c in range(0x08, 0x7E)])
        w.src_k[:] = _pow2_rows(rng, w.src_k.shape, grid)
        w.src_v[:] = _pow2_rows(rng, w.src_v.shape, grid)
        kc, vc = w.empty_pool(), w.empty_pool()
        kc, vc = oracle.store_kvcache(kc, vc, w.setup_k, w.setup_v, w.setup_slots)
        kc, vc = oracle.store_kvcache(kc, vc, w.new_k, w.new_v, w.new_slots)
        ref = oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale)
        shape = (w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim)
        z8, zs = np.full(shape, 0x7F, np.uint8), np.full(shape[:3], np.nan, np.float32)
        k8, v8, ks, vs = m.store_kvcache_fp8(z8, z8, zs, zs, w.setup_k, w.setup_v, w.setup_slots)
        k8, v8, ks, vs = m.store_kvcache_fp8(k8, v8, ks, vs, w.new_k, w.new_v, w.new_slots)
        got = m.decode_fp8(w.q, k8, v8, ks, vs, w.block_tables, w.context_lens, w.scale)
        return bool(np.all(np.isfinite(got)) and np.max(np.abs(got - ref)) < 1e-12)

    def store_placement():
        # token t lands in block slot // bs, row slot % bs; a slot of -1 writes nothing
        nb, bs, hkv, d = 3, 4, 2, 8
        rng = np.random.default_rng(95)
        k = f32_to_bf16_bits(rng.standard_normal((5, hkv, d)).astype(np.float32))
        slots = np.array([0, 5, 11, -1, 6])   # a mistaken -1 would land on row 11
        z8, zs = np.full((nb, bs, hkv, d), 0x7F, np.uint8), np.full((nb, bs, hkv), -1.0, np.float32)
        k8, v8, ks, vs = m.store_kvcache_fp8(z8, z8, zs, zs, k, k, slots)
        qc, qs = m.quantize_rows(k)
        for t, slot in enumerate(slots):
            if slot < 0:
                continue
            b_, o = divmod(int(slot), bs)
            if not (np.array_equal(k8[b_, o], qc[t]) and np.array_equal(ks[b_, o], qs[t])):
                return False
        written = {int(x) for x in slots if x >= 0}
        for r in range(nb * bs):
            if r not in written and not (np.all(k8.reshape(-1, hkv, d)[r] == 0x7F)
                                         and np.all(ks.reshape(-1, hkv)[r] == -1.0)):
                return False
        return True

    check("store placement", store_placement)
    check("round trip", round_trip)
    check("hand-worked codes", hand_codes)
    check("hand-worked values", hand_values)
    check("against torch", against_torch)
    check("quantiser bound", quantiser_bound)
    check("exact rows decode", exact_rows_decode)
    return failed


def test_real_fp8_oracle_passes_the_compact_pins():
    assert _pins(real_fp8) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_each_planted_fp8_mistake_is_caught(name):
    old, new = MUTANTS[name]
    failed = _pins(_mutant(old, new))
    assert failed, f"mutant '{name}' passed every pin"
