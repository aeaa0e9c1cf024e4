"""Pins of the oracle's fp8 (e4m3) KV-cache pieces against things other than itself:
the exhaustive code table, hand-worked ties, torch's own float8_e4m3fn conversion
(an independent implementation) inside the finite range, the quantiser's error bound,
and decode over exactly representable rows reducing to the bf16 decode."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import fp8
from workloads import build_workload, f32_to_bf16_bits


def test_every_code_round_trips():
    for c in range(256):
        v = fp8.e4m3_to_float(c)
        if math.isnan(v):
            assert c in (0x7F, 0xFF)
            continue
        assert fp8.float_to_e4m3(v) == c, hex(c)


@pytest.mark.parametrize("x,code", [
    (1.0, 0x38), (448.0, 0x7E), (-448.0, 0xFE), (2.0 ** -9, 0x01), (2.0 ** -6, 0x08),
    (-3.0, 0xC4), (0.0, 0x00), (-0.0, 0x80),
    (1.0625, 0x38),          # tie between 1.0 and 1.125: to the even code
    (1.1875, 0x3A),          # tie between 1.125 and 1.25: to the even code
    (0.5 * 2.0 ** -9, 0x00), (1.5 * 2.0 ** -9, 0x02), (7.5 * 2.0 ** -9, 0x08),
    (464.0, 0x7E), (1e6, 0x7E), (-1e6, 0xFE),   # saturation at +-448
])
def test_hand_worked_codes(x, code):
    assert fp8.float_to_e4m3(x) == code


def test_encoder_matches_torch_inside_the_finite_range():
    rng = np.random.default_rng(81)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.uniform(-4, 2.6, 20000),
                        rng.uniform(-463.9, 463.9, 5000)]).astype(np.float32)
    x = x[np.abs(x) < 464.0]        # beyond that torch gives NaN, the kernels saturate
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([fp8.float_to_e4m3(v) for v in x.astype(np.float64)], dtype=np.uint8)
    assert np.array_equal(got, want)


def test_quantize_rows_scale_amax_and_error_bound():
    rng = np.random.default_rng(82)
    x = f32_to_bf16_bits(rng.standard_normal((64, 4, 128)).astype(np.float32))
    codes, scales = fp8.quantize_rows(x)
    xf = oracle.bf16_bits_to_f64(x)
    amax = np.max(np.abs(xf), axis=-1)
    assert np.allclose(scales, (amax / 448.0).astype(np.float32), rtol=0, atol=0)
    # the largest element of each row maps to +-448
    idx = np.argmax(np.abs(xf), axis=-1)
    top = np.take_along_axis(codes, idx[..., None], axis=-1)[..., 0]
    assert np.all((top == 0x7E) | (top == 0xFE))
    # e4m3 keeps 3 mantissa bits: |error| <= 2^-4 |x| for normals, plus half a subnormal step
    err = np.abs(fp8.dequantize(codes, scales) - xf)
    bound = 2.0 ** -4 * np.abs(xf) + 0.5 * 2.0 ** -9 * scales[..., None] + 1e-12
    assert np.all(err <= bound)
    zero_codes, zero_scales = fp8.quantize_rows(np.zeros((2, 8), np.uint16))
    assert np.all(zero_codes == 0) and np.all(zero_scales == 0)


def test_quantize_rows_at_the_fp32_overflow_edge():
    """448 / amax overflows fp32 below amax = 448 / FLT_MAX (~1.3166e-36): such rows
    store zeros; just above it the row quantises normally, its scale an fp32
    subnormal, and reads back within the error bound."""
    flt_max = float(np.finfo(np.float32).max)
    edge = 448.0 / flt_max
    tiny = f32_to_bf16_bits(np.array([[0.5 * edge, -0.25 * edge, 0.0, 1e-40]], np.float32))
    codes, scales = fp8.quantize_rows(tiny)
    assert np.all(codes == 0) and np.all(scales == 0)
    row = np.array([[2.0 * edge, -edge, 0.5 * edge, 0.0]], np.float32)
    bits = f32_to_bf16_bits(row)
    codes, scales = fp8.quantize_rows(bits)
    xf = oracle.bf16_bits_to_f64(bits)
    assert codes[0, 0] == 0x7E and codes[0, 3] == 0
    assert 0 < scales[0] < np.finfo(np.float32).tiny          # subnormal fp32 scale
    assert abs(float(scales[0]) - np.max(np.abs(xf)) / 448.0) <= 2.0 ** -149
    err = np.abs(fp8.dequantize(codes, scales) - xf)
    assert np.all(err <= 2.0 ** -4 * np.abs(xf) + 2.0 ** -149 * 448)


def test_decode_of_exactly_representable_rows_equals_bf16_decode():
    """Rows whose values are e4m3 values times a power of two scale survive quantising
    exactly, so the fp8 decode must equal the bf16 decode of the same rows."""
    lens = np.array([5, 17, 1, 40])
    w = build_workload(kind="decode", context_lens=lens, new_lens=np.ones(4, int), num_q_heads=4,
                       num_kv_heads=2, head_dim=8, block_size=4, seed=83)
    rng = np.random.default_rng(84)
    grid = np.array([fp8.e4m3_to_float(c) for c in range(0x38, 0x70)], dtype=np.float32)  # 1 .. 240

    def representable(shape):
        v = rng.choice(grid, size=shape) * rng.choice([-1, 1], size=shape)
        v[..., 0] = 448.0 * np.sign(v[..., 0])    # amax = 448 in every row: scale 1
        return f32_to_bf16_bits(v.astype(np.float32))

    src_k, src_v = representable(w.src_k.shape), representable(w.src_v.shape)
    w.src_k[:], w.src_v[:] = src_k, src_v
    kc, vc = w.empty_pool(), w.empty_pool()
    kc, vc = oracle.store_kvcache(kc, vc, w.setup_k, w.setup_v, w.setup_slots)
    kc, vc = oracle.store_kvcache(kc, vc, w.new_k, w.new_v, w.new_slots)
    ref = oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale)
    shape = (w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim)
    z8, zs = np.zeros(shape, np.uint8), np.zeros(shape[:3], np.float32)
    k8, v8, ks, vs = fp8.store_kvcache_fp8(z8, z8, zs, zs, w.setup_k, w.setup_v, w.setup_slots)
    k8, v8, ks, vs = fp8.store_kvcache_fp8(k8, v8, ks, vs, w.new_k, w.new_v, w.new_slots)
    assert np.all(ks[ks != 0] == 1.0)
    got = fp8.decode_fp8(w.q, k8, v8, ks, vs, w.block_tables, w.context_lens, w.scale)
    assert np.max(np.abs(got - ref)) < 1e-12
