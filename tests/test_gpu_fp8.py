"""GPU parity of the fp8 (e4m3) KV cache.

Store: codes and scales bit-exact against the oracle's quantiser (both take every
decision in fp32 with round-to-nearest). Decode: within the decode bar of
tests/gpu_helpers.py against the oracle's fp64 attention of the exact values the pools
hold (code * scale). The kernel's tensor cores read the codes themselves (exact); q
reaches them as three e4m3 terms (about 2^-13 relative per element) and the
probabilities as two (about 2^-8 relative, of the size of the bf16 rounding of P that
the bf16 decode carries).
"""
import numpy as np
import pytest
import torch

from oracle import fp8
import paged_kv_cache_442_b200 as pa
from tests.gpu_helpers import assert_close, bf16_dev, i32_dev, to_f64
from workloads import CONFIGS, build_workload, f32_to_bf16_bits, generate

pytestmark = pytest.mark.gpu

NAN_CODE = 0x7F  # what unwritten rows of the code pools hold in these tests


def scales_to_device_layout(s, nb, bs, hkv):
    """oracle scales [nb, bs, Hkv] -> the library's [Hkv, nb * bs]."""
    return np.ascontiguousarray(np.asarray(s, np.float32).reshape(nb * bs, hkv).T)


def f32_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def u8_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def rows_with_edges(rng, t, hkv, d):
    """bf16 rows of varied magnitude plus the quantiser's special rows."""
    mag = 10.0 ** rng.uniform(-3, 3, size=(t, hkv, 1))
    x = (rng.standard_normal((t, hkv, d)) * mag).astype(np.float32)
    edge = 448.0 / float(np.finfo(np.float32).max)
    x[0, 0] = 0.0                                   # all zeros
    x[1, 0] = 0.0
    x[1, 0, 3] = -2.5                               # one non-zero value
    x[2, 0] = 0.4 * edge                            # 448 / amax overflows: stored as zeros
    x[3, 0] = rng.uniform(-1, 1, d) * 3 * edge      # just above the edge: subnormal scale
    x[4, 0] = rng.uniform(-1, 1, d) * 1e-39         # bf16 subnormals
    x[5, 0] = rng.uniform(-1, 1, d) * 3e38          # near the top of the range
    x[6, 0, :] = 1.0                                # every value at amax
    x[7, 0] = np.round(rng.standard_normal(d) * 4) / 4  # many ties after scaling
    return f32_to_bf16_bits(x)


@pytest.mark.parametrize("d,hkv,bs", [(128, 8, 16), (128, 2, 256), (64, 4, 64)])
def test_fp8_store_codes_and_scales_bit_exact(d, hkv, bs):
    rng = np.random.default_rng(d + hkv + bs)
    nb, t = 48, 300
    k = rows_with_edges(rng, t, hkv, d)
    v = rows_with_edges(rng, t, hkv, d)[::-1].copy()
    slots = rng.permutation(nb * bs)[:t].astype(np.int32)
    slots[[9, 50]] = -1                             # skipped tokens
    z8 = np.full((nb, bs, hkv, d), NAN_CODE, np.uint8)
    zs = np.zeros((nb, bs, hkv), np.float32)
    want = fp8.store_kvcache_fp8(z8, z8, zs, zs, k, v, slots)
    kc, vc = u8_dev(z8), u8_dev(z8)
    ks, vs = f32_dev(scales_to_device_layout(zs, nb, bs, hkv)), f32_dev(scales_to_device_layout(zs, nb, bs, hkv))
    pa.pa_store_kvcache_fp8(bf16_dev(k), bf16_dev(v), kc, vc, ks, vs, i32_dev(slots))
    torch.cuda.synchronize()
    assert np.array_equal(kc.cpu().numpy(), want[0])
    assert np.array_equal(vc.cpu().numpy(), want[1])
    assert np.array_equal(ks.cpu().numpy().view(np.uint32),
                          scales_to_device_layout(want[2], nb, bs, hkv).view(np.uint32))
    assert np.array_equal(vs.cpu().numpy().view(np.uint32),
                          scales_to_device_layout(want[3], nb, bs, hkv).view(np.uint32))


def test_fp8_store_flags_a_slot_past_the_pool():
    rng = np.random.default_rng(5)
    nb, bs, hkv, d = 8, 16, 2, 128
    k = rows_with_edges(rng, 12, hkv, d)
    slots = np.arange(12, dtype=np.int32)
    slots[4] = nb * bs + 3
    kc = torch.zeros((nb, bs, hkv, d), dtype=torch.uint8, device="cuda")
    vc = torch.zeros_like(kc)
    ks = torch.zeros((hkv, nb * bs), dtype=torch.float32, device="cuda")
    vs = torch.zeros_like(ks)
    pa.pa_set_debug_checks(True)
    with pytest.raises(pa.PAError) as e:
        pa.pa_store_kvcache_fp8(bf16_dev(k), bf16_dev(k), kc, vc, ks, vs, i32_dev(slots))
    assert e.value.status == 3
    assert pa.pa_check_device_errors() == 0
    # the other tokens were stored
    z8 = np.zeros((nb, bs, hkv, d), np.uint8)
    zs = np.zeros((nb, bs, hkv), np.float32)
    ok = slots.copy()
    ok[4] = -1
    want = fp8.store_kvcache_fp8(z8, z8, zs, zs, k, k, ok)
    assert np.array_equal(kc.cpu().numpy(), want[0])


class Fp8Pools:
    """A decode workload's rows quantised by the oracle into e4m3 pools (unwritten rows:
    NaN codes and NaN scales), on the host and on the device."""

    def __init__(self, w):
        shape = (w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim)
        z8 = np.full(shape, NAN_CODE, np.uint8)
        zs = np.full(shape[:3], np.nan, np.float32)
        k8, v8, ks, vs = fp8.store_kvcache_fp8(z8, z8, zs, zs, w.setup_k, w.setup_v, w.setup_slots)
        if len(w.new_slots):
            k8, v8, ks, vs = fp8.store_kvcache_fp8(k8, v8, ks, vs, w.new_k, w.new_v, w.new_slots)
        self.host = (k8, v8, ks, vs)
        nb, bs, hkv = shape[:3]
        self.k8, self.v8 = u8_dev(k8), u8_dev(v8)
        self.ks = f32_dev(scales_to_device_layout(ks, nb, bs, hkv))
        self.vs = f32_dev(scales_to_device_layout(vs, nb, bs, hkv))


def gpu_decode_fp8(w, pools, partition_size=0):
    q = bf16_dev(w.q)
    out = torch.empty_like(q)
    ws, P = pa.decode_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                w.max_context_len, partition_size)
    pa.pa_decode_fp8(out, q, pools.k8, pools.v8, pools.ks, pools.vs, i32_dev(w.block_tables),
                     i32_dev(w.context_lens), w.scale, w.max_context_len, P, ws)
    return to_f64(out)


def oracle_decode_fp8(w, host, seqs=None):
    k8, v8, ks, vs = host
    if seqs is None:
        return fp8.decode_fp8(w.q, k8, v8, ks, vs, w.block_tables, w.context_lens, w.scale)
    seqs = np.asarray(seqs)
    return fp8.decode_fp8(w.q[seqs], k8, v8, ks, vs, w.block_tables[seqs], w.context_lens[seqs],
                          w.scale)


@pytest.mark.parametrize("g,bs,parts", [(4, 16, 128), (4, 16, 0), (1, 64, 256), (2, 256, 128),
                                        (8, 32, 512)])
def test_fp8_decode_matches_oracle_ragged(g, bs, parts):
    lens = np.array([1, 127, 128, 129, 300, 0, 1000, 17, 640, 255, 2048, 3])
    hkv = 2
    w = build_workload(kind="decode", context_lens=lens, new_lens=(lens > 0).astype(int),
                       num_q_heads=hkv * g, num_kv_heads=hkv, head_dim=128, block_size=bs,
                       seed=700 + g + bs)
    pools = Fp8Pools(w)
    got = gpu_decode_fp8(w, pools, parts)
    ref = oracle_decode_fp8(w, pools.host)
    assert_close(got, ref, f"fp8 decode g={g} bs={bs} P={parts}")
    assert np.all(got[lens == 0] == 0)


def test_fp8_store_then_decode_on_the_gpu():
    """The library's own store feeds its decode: equal to the oracle's store + decode."""
    lens = np.array([5, 129, 700, 1, 64, 2000])
    w = build_workload(kind="decode", context_lens=lens, new_lens=np.ones(6, int), num_q_heads=16,
                       num_kv_heads=4, head_dim=128, block_size=64, seed=811)
    host = Fp8Pools(w)
    shape = (w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim)
    k8 = torch.full(shape, NAN_CODE, dtype=torch.uint8, device="cuda")
    v8 = torch.full_like(k8, NAN_CODE)
    ks = torch.full((w.num_kv_heads, w.num_blocks * w.block_size), float("nan"), device="cuda")
    vs = torch.full_like(ks, float("nan"))
    for kk, vv, ss in ((w.setup_k, w.setup_v, w.setup_slots), (w.new_k, w.new_v, w.new_slots)):
        pa.pa_store_kvcache_fp8(bf16_dev(kk), bf16_dev(vv), k8, v8, ks, vs, i32_dev(ss))

    class Dev:
        pass
    dev = Dev()
    dev.k8, dev.v8, dev.ks, dev.vs = k8, v8, ks, vs
    got = gpu_decode_fp8(w, dev, 256)
    assert np.array_equal(k8.cpu().numpy(), host.host[0])
    assert_close(got, oracle_decode_fp8(w, host.host), "store + decode")


def compact(w, seqs, k8, v8, ks, vs):
    """The blocks the sampled sequences read, renumbered into a small pool (pure data
    movement, so the oracle sees the same bytes)."""
    bs = w.block_size
    used, tables = [], []
    for s in seqs:
        nblk = -(-int(w.context_lens[s]) // bs)
        ids = w.block_tables[s, :nblk]
        tables.append(np.arange(len(used), len(used) + nblk))
        used.extend(ids.tolist())
    used = np.array(used, dtype=np.int64)
    bt = np.full((len(seqs), max(len(t) for t in tables)), -1, np.int32)
    for i, t in enumerate(tables):
        bt[i, :len(t)] = t
    hkv = w.num_kv_heads
    ks_b = ks.reshape(hkv, w.num_blocks, bs)[:, used].transpose(1, 2, 0)
    vs_b = vs.reshape(hkv, w.num_blocks, bs)[:, used].transpose(1, 2, 0)
    return k8[used], v8[used], ks_b, vs_b, bt


@pytest.mark.parametrize("name", ["decode_b64", "long_ctx_decode"])
def test_fp8_decode_full_size_sampled(name):
    """The full configuration with seeded random codes and scales as the pools (any
    codes are valid decode inputs), checked on sampled sequences."""
    w = generate(CONFIGS[name])
    rng = np.random.default_rng(91)
    shape = (w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim)
    k8 = rng.integers(0, 256, size=shape, dtype=np.uint8)
    v8 = rng.integers(0, 256, size=shape, dtype=np.uint8)
    k8[(k8 & 0x7F) == 0x7F] ^= 1                        # no NaN codes
    v8[(v8 & 0x7F) == 0x7F] ^= 1
    slots = w.num_blocks * w.block_size
    ks = (rng.uniform(0.5, 2.0, size=(w.num_kv_heads, slots)) * (3.0 / 448)).astype(np.float32)
    vs = (rng.uniform(0.5, 2.0, size=(w.num_kv_heads, slots)) * (3.0 / 448)).astype(np.float32)

    class Dev:
        pass
    dev = Dev()
    dev.k8, dev.v8, dev.ks, dev.vs = u8_dev(k8), u8_dev(v8), f32_dev(ks), f32_dev(vs)
    got = gpu_decode_fp8(w, dev)
    seqs = rng.choice(w.num_seqs, size=min(4 if name == "decode_b64" else 2, w.num_seqs),
                      replace=False)
    ck8, cv8, cks, cvs, bt = compact(w, seqs, k8, v8, ks, vs)
    ref = fp8.decode_fp8(w.q[seqs], ck8, cv8, cks, cvs, bt, w.context_lens[seqs], w.scale)
    assert_close(got[seqs], ref, f"{name} fp8 sampled")
    assert np.all(np.isfinite(got))


def test_fp8_decode_agrees_with_bf16_decode_on_exact_rows():
    """Rows that are e4m3 values times a power of two survive quantising exactly, and
    their dequantised values are exact in bf16: the fp8 and bf16 decodes then attend
    over the same numbers. They round differently on the way (the fp8 kernel feeds q
    to the tensor cores as three e4m3 terms and the probabilities as two, the bf16
    kernel rounds the probabilities to bf16), so both are checked against the oracle
    and against each other to a tight norm."""
    lens = np.array([40, 300, 1, 129])
    w = build_workload(kind="decode", context_lens=lens, new_lens=np.ones(4, int), num_q_heads=8,
                       num_kv_heads=2, head_dim=128, block_size=16, seed=812)
    rng = np.random.default_rng(813)
    grid = np.array([fp8.e4m3_to_float(c) for c in range(0x30, 0x70)], dtype=np.float32)

    def representable(shape):
        x = rng.choice(grid, size=shape) * rng.choice([-1, 1], size=shape)
        x[..., 0] = 448.0
        return f32_to_bf16_bits((x / 256.0).astype(np.float32))   # amax 1.75: scale 2^-8

    w.src_k[:], w.src_v[:] = representable(w.src_k.shape), representable(w.src_v.shape)
    pools = Fp8Pools(w)
    got8 = gpu_decode_fp8(w, pools, 128)
    from tests.gpu_helpers import DeviceWorkload, oracle_decode
    got16 = to_f64(DeviceWorkload(w).decode(128))
    ref = oracle_decode(w)
    assert_close(got8, ref, "fp8 on exact rows")
    assert_close(got16, ref, "bf16 on exact rows")
    assert np.linalg.norm(got8 - got16) / np.linalg.norm(got16) < 5e-3
    assert np.array_equal(got8[lens == 1], got16[lens == 1])   # one position: its V row


@pytest.mark.parametrize("q_factor", [8.0, 24.0])
def test_fp8_decode_peaked_queries(q_factor):
    """Peaked softmax (q scaled up): a few positions carry almost all the weight and the
    rest are tiny; the two-term probabilities keep both within the bar."""
    lens = np.array([2048, 700, 129, 1, 1500, 300])
    w = build_workload(kind="decode", context_lens=lens, new_lens=np.ones(6, int), num_q_heads=16,
                       num_kv_heads=4, head_dim=128, block_size=64, seed=820, q_factor=q_factor)
    pools = Fp8Pools(w)
    for P in (0, 256):
        got = gpu_decode_fp8(w, pools, P)
        assert_close(got, oracle_decode_fp8(w, pools.host), f"fp8 peaked x{q_factor} P={P}")


def test_fp8_decode_sixteen_query_heads_per_kv_head():
    lens = np.array([5, 128, 129, 1000, 3000])
    w = build_workload(kind="decode", context_lens=lens, new_lens=np.ones(5, int), num_q_heads=32,
                       num_kv_heads=2, head_dim=128, block_size=16, seed=821)
    pools = Fp8Pools(w)
    for P in (0, 256, 2048):
        assert_close(gpu_decode_fp8(w, pools, P), oracle_decode_fp8(w, pools.host), f"G=16 P={P}")


def test_fp8_decode_zero_rows_and_zero_queries():
    """All-zero rows quantise to codes 0 with scale 0: a V scale of 0 must give that
    position weight in the sum but nothing in the output, a whole first tile of them
    must not poison the reference of later tiles, and q = 0 (a zero q scale) gives the
    mean of V."""
    lens = np.array([400, 129, 300, 1])
    w = build_workload(kind="decode", context_lens=lens, new_lens=np.ones(4, int), num_q_heads=8,
                       num_kv_heads=2, head_dim=128, block_size=64, seed=822)
    rows0 = w.logical_rows[0]
    w.src_v[rows0[:200]] = 0                      # sequence 0: its first 200 V rows are zero
    w.src_k[w.logical_rows[2][::3]] = 0           # sequence 2: every third K row is zero
    w.src_v[w.logical_rows[3]] = 0                # sequence 3: its one V row is zero
    w.q[1] = 0                                    # sequence 1: q = 0 (the mean of V)
    pools = Fp8Pools(w)
    for P in (0, 128):
        got = gpu_decode_fp8(w, pools, P)
        assert_close(got, oracle_decode_fp8(w, pools.host), f"zero rows P={P}")
        assert np.all(got[3] == 0)


def test_fp8_decode_many_one_tile_items():
    """e4m3 pools, 640 sequences of at most 130 positions over 8 kv heads: an item
    boundary at almost every tile for the issuer, the scheduler's q terms and the
    K-scale ring."""
    rng = np.random.default_rng(65)
    lens = rng.integers(1, 131, size=640)
    lens[:6] = [1, 2, 127, 128, 129, 130]
    w = build_workload(kind="decode", context_lens=lens, new_lens=np.ones_like(lens),
                       num_q_heads=16, num_kv_heads=8, head_dim=128, block_size=16, seed=6500)
    pools = Fp8Pools(w)
    got = gpu_decode_fp8(w, pools, 128)
    assert_close(got, oracle_decode_fp8(w, pools.host), "fp8 one-tile items")
