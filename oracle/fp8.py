"""fp8 (e4m3) KV cache: the codec, the row quantiser, and decode over dequantised pools.

TEST INFRASTRUCTURE ONLY (like the rest of this package).

The pages list quantisation of the KV cache only as an extension; the readings here:
  * values are stored as OCP fp8 e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa
    bits; no infinities; the largest finite value is 448; subnormals are m * 2**-9);
  * every (position, kv head) row of D values has its own fp32 scale: a decode step
    writes one row at a time into a block, so a scale per row can be chosen when the
    row is written (a per-block scale could not, before the block is full);
  * quantising a row x (bf16 values, finite): amax = max |x|; in fp32 with
    round-to-nearest, inv = 448 / amax; if inv is not a finite fp32 (amax == 0, or
    amax below 448 / FLT_MAX, about 1.3e-36, where the quotient overflows) the codes
    and the scale are 0; otherwise y_i = x_i * inv, code_i = e4m3(y_i) rounded to
    nearest even and saturated to +-448, and scale = amax / 448. A value is read back
    as e4m3(code) * scale.
The quantiser's integer decisions are taken in fp32, the precision the kernels use.
"""
from __future__ import annotations

import math

import numpy as np

E4M3_MAX = 448.0


def e4m3_to_float(code: int) -> float:
    """Exact value of one e4m3 code (NaN for the two NaN codes)."""
    c = int(code) & 0xFF
    sign = -1.0 if c & 0x80 else 1.0
    e = (c >> 3) & 0xF
    m = c & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * m * 2.0 ** -9
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def float_to_e4m3(y: float) -> int:
    """Round a finite value to the nearest e4m3 code (ties to even), saturating to
    +-448. Exact: y is taken as a float64 holding an fp32 value."""
    y = float(y)
    sign = 0x80 if (y < 0 or (y == 0 and math.copysign(1.0, y) < 0)) else 0
    a = abs(y)
    if a == 0.0:
        return sign
    if a >= E4M3_MAX:
        return sign | 0x7E
    e = math.floor(math.log2(a))
    # guard the float log2 near powers of two
    while 2.0 ** e > a:
        e -= 1
    while 2.0 ** (e + 1) <= a:
        e += 1
    if e < -6:                                   # subnormal range: multiples of 2**-9
        r = round(a / 2.0 ** -9)                 # Python rounds ties to even
        if r >= 8:
            return sign | (1 << 3)               # rounds up to the smallest normal
        return sign | r
    r = round(a / 2.0 ** e * 8.0)                # in [8, 16], ties to even
    if r == 16:
        e += 1
        r = 8
    if e > 8 or (e == 8 and r - 8 > 6):
        return sign | 0x7E                       # beyond 448: saturate
    return sign | ((e + 7) << 3) | (r - 8)


def quantize_rows(x_bits: np.ndarray):
    """Rows of bf16 bits [..., D] -> (uint8 codes [..., D], float32 scales [...])."""
    x = np.asarray(x_bits, dtype=np.uint16)
    xf = (x.astype(np.uint32) << np.uint32(16)).view(np.float32)
    flat = xf.reshape(-1, xf.shape[-1])
    codes = np.zeros(flat.shape, dtype=np.uint8)
    scales = np.zeros(flat.shape[0], dtype=np.float32)
    for i, row in enumerate(flat):
        amax = np.float32(np.max(np.abs(row)))
        with np.errstate(over="ignore", divide="ignore"):
            inv = np.float32(E4M3_MAX) / amax
        if not np.isfinite(inv):
            continue
        y = (row * inv).astype(np.float32)
        codes[i] = [float_to_e4m3(v) for v in y.astype(np.float64)]
        scales[i] = amax / np.float32(E4M3_MAX)
    return codes.reshape(x.shape), scales.reshape(x.shape[:-1])


def dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """float64 values code * scale (exact: 4 significant bits times an fp32)."""
    lut = np.array([e4m3_to_float(c) for c in range(256)], dtype=np.float64)
    return lut[np.asarray(codes, dtype=np.uint8)] * np.asarray(scales, dtype=np.float64)[..., None]


def store_kvcache_fp8(k_codes, v_codes, k_scales, v_scales, k, v, slot_mapping):
    """Copies of the fp8 pools with row slot_mapping[t] replaced by the quantised k[t] /
    v[t] (negative slot: skipped). Pools: codes uint8 [num_blocks, bs, Hkv, D], scales
    float32 [num_blocks, bs, Hkv]; k, v: bf16 bits [T, Hkv, D]."""
    kc, vc = np.array(k_codes, copy=True), np.array(v_codes, copy=True)
    ks, vs = np.array(k_scales, copy=True), np.array(v_scales, copy=True)
    nb, bs, hkv, d = kc.shape
    qk, sk = quantize_rows(k)
    qv, sv = quantize_rows(v)
    for t, slot in enumerate(np.asarray(slot_mapping)):
        slot = int(slot)
        if slot < 0:
            continue
        if slot >= nb * bs:
            raise IndexError(f"slot {slot} outside a pool of {nb * bs} rows")
        b, o = divmod(slot, bs)
        kc[b, o], vc[b, o], ks[b, o], vs[b, o] = qk[t], qv[t], sk[t], sv[t]
    return kc, vc, ks, vs


def decode_fp8(q, k_codes, v_codes, k_scales, v_scales, block_tables, context_lens, scale):
    """Paged decode over the dequantised pools: the textbook fp64 attention of the
    values the pools hold (nothing else changes from the bf16 decode)."""
    from .paged_attention import bf16_bits_to_f64, softmax_attention
    kf = dequantize(k_codes, k_scales)
    vf = dequantize(v_codes, v_scales)
    B, Hq, D = q.shape
    nb, bs, Hkv, _ = kf.shape
    G = Hq // Hkv
    qf = bf16_bits_to_f64(q)
    scale = float(np.float32(scale))
    out = np.zeros((B, Hq, D), dtype=np.float64)
    for s in range(B):
        ctx = int(context_lens[s])
        if ctx <= 0:
            continue
        pos = np.arange(ctx)
        rows = block_tables[s, pos // bs].astype(np.int64) * bs + pos % bs
        Kc = kf.reshape(nb * bs, Hkv, D)[rows]
        Vc = vf.reshape(nb * bs, Hkv, D)[rows]
        for h in range(Hq):
            out[s, h] = softmax_attention(qf[s, h], Kc[:, h // G, :], Vc[:, h // G, :], scale)
    return out
