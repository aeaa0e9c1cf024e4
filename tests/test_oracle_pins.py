"""Pins of the CPU oracle against things other than itself: brute force over the
contiguous rows the generator drew, closed forms, invariants of the method (the
pool layout must not matter), and the cached-equals-recompute property of the
mini-vllm page's benchmark ("性能评估与基准测试")."""
import math

import numpy as np
import pytest

import oracle
from oracle import brute
from workloads import build_workload, relabel_blocks

TOL = 1e-12


def pools_after_store(w, oracle_mod=oracle):
    """Empty (sentinel) pools, setup rows stored, then the step's new rows stored."""
    kc, vc = w.empty_pool(), w.empty_pool()
    kc, vc = oracle_mod.store_kvcache(kc, vc, w.setup_k, w.setup_v, w.setup_slots)
    kc, vc = oracle_mod.store_kvcache(kc, vc, w.new_k, w.new_v, w.new_slots)
    return kc, vc


def run_decode(w, oracle_mod=oracle):
    kc, vc = pools_after_store(w, oracle_mod)
    return oracle_mod.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale)


def run_prefill(w, oracle_mod=oracle):
    kc, vc = pools_after_store(w, oracle_mod)
    return oracle_mod.prefill(w.q, kc, vc, w.block_tables, w.cu_seqlens_q, w.context_lens, w.scale)


def brute_decode(w):
    ks = [w.logical_k(s).tolist() for s in range(w.num_seqs)]
    vs = [w.logical_v(s).tolist() for s in range(w.num_seqs)]
    return np.array(brute.decode_contiguous(w.q.tolist(), ks, vs, w.scale))


def brute_prefill(w):
    ks = [w.logical_k(s).tolist() for s in range(w.num_seqs)]
    vs = [w.logical_v(s).tolist() for s in range(w.num_seqs)]
    return np.array(brute.prefill_contiguous(w.q.tolist(), w.cu_seqlens_q.tolist(), ks, vs, w.scale))


def tiny_decode(G=2, bs=4, D=8, Hkv=2, lens=(1, 7, 40, 13, 0, 16), new=1, seed=11, **kw):
    lens = np.asarray(lens)
    return build_workload(kind="decode", context_lens=lens,
                          new_lens=np.where(lens > 0, new, 0), num_q_heads=G * Hkv,
                          num_kv_heads=Hkv, head_dim=D, block_size=bs, seed=seed, **kw)


def tiny_prefill(G=2, bs=4, D=8, Hkv=2, lens=(9, 23, 5), new=(4, 23, 1), seed=12, **kw):
    return build_workload(kind="prefill", context_lens=np.asarray(lens), new_lens=np.asarray(new),
                          num_q_heads=G * Hkv, num_kv_heads=Hkv, head_dim=D, block_size=bs,
                          seed=seed, **kw)


# ---------------------------------------------------------------- brute force
@pytest.mark.parametrize("G", [1, 2, 4])
@pytest.mark.parametrize("bs", [1, 4, 16])
@pytest.mark.parametrize("D", [4, 16])
def test_decode_oracle_equals_brute_force(G, bs, D):
    w = tiny_decode(G=G, bs=bs, D=D, seed=100 + G * 10 + bs + D)
    got = run_decode(w)
    ref = brute_decode(w)
    assert np.max(np.abs(got - ref)) < TOL


@pytest.mark.parametrize("G", [1, 4])
@pytest.mark.parametrize("bs", [1, 4, 16])
def test_prefill_oracle_equals_brute_force(G, bs):
    w = tiny_prefill(G=G, bs=bs, seed=200 + G + bs)
    got = run_prefill(w)
    ref = brute_prefill(w)
    assert np.max(np.abs(got - ref)) < TOL


def test_peaked_scores_are_stable():
    # large scores: exp without subtracting the max would overflow
    w = tiny_decode(G=2, bs=4, D=16, q_factor=400.0, seed=5)
    got = run_decode(w)
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got - brute_decode(w))) < 1e-9


# ---------------------------------------------------------------- closed forms
def _manual(q, K, V, scale=1.0, Hkv=None):
    """Tiny hand-built case straight into the pool (bs=2, one sequence)."""
    from workloads.gen import f32_to_bf16_bits
    K = np.asarray(K, np.float32)
    V = np.asarray(V, np.float32)
    q = np.asarray(q, np.float32)
    n, D = K.shape
    bs = 2
    nb = -(-n // bs) + 1
    kc = np.full((nb, bs, 1, D), 0xFFC1, np.uint16)
    vc = kc.copy()
    kb = f32_to_bf16_bits(K).reshape(n, 1, D)
    vb = f32_to_bf16_bits(V).reshape(n, 1, D)
    # blocks placed in reverse order to exercise the table
    table = np.array([nb - 1 - i for i in range(nb)], np.int32)
    slots = np.array([table[p // bs] * bs + p % bs for p in range(n)], np.int32)
    kc, vc = oracle.store_kvcache(kc, vc, kb, vb, slots)
    qb = f32_to_bf16_bits(q).reshape(1, 1, D)
    return oracle.decode(qb, kc, vc, table[None, :], np.array([n], np.int32), scale)[0, 0]


def test_single_key_returns_its_value_exactly():
    out = _manual([0.3, -1.0], [[2.0, 5.0]], [[1.5, -0.25]], scale=0.7)
    assert np.array_equal(out, [1.5, -0.25])


def test_zero_query_gives_mean_of_values():
    V = [[1.0, 2.0], [3.0, -4.0], [0.5, 0.25], [8.0, 1.0], [-2.0, 0.0]]
    K = [[1.0, 3.0], [-2.0, 1.0], [0.5, 0.5], [4.0, 4.0], [0.0, 1.0]]
    out = _manual([0.0, 0.0], K, V)
    assert np.allclose(out, np.mean(np.array(V), axis=0), atol=1e-14)


def test_equal_keys_give_mean_of_values():
    V = [[1.0, 2.0], [3.0, -4.0], [0.5, 0.25]]
    out = _manual([1.0, -2.0], [[0.5, 1.0]] * 3, V, scale=3.0)
    assert np.allclose(out, np.mean(np.array(V), axis=0), atol=1e-14)


def test_constant_values_give_that_constant():
    out = _manual([1.0, 2.0], [[1.0, 0.0], [0.0, 1.0], [2.0, 2.0], [-1.0, 3.0]], [[0.75, -3.0]] * 4)
    assert np.allclose(out, [0.75, -3.0], atol=1e-14)


def test_dominant_key_selects_its_value():
    K = [[0.0, 0.0], [64.0, 0.0], [0.0, 1.0]]
    V = [[1.0, 1.0], [-5.0, 2.0], [3.0, 3.0]]
    out = _manual([16.0, 0.0], K, V, scale=1.0)     # score 1024 vs 0
    assert np.allclose(out, [-5.0, 2.0], atol=1e-14)


def test_two_key_softmax_closed_form_with_scale():
    # q.k = (0, 2), scale 0.5 -> z = (0, 1): weights 1/(1+e), e/(1+e)
    out = _manual([1.0, 0.0], [[0.0, 0.0], [2.0, 0.0]], [[1.0, 0.0], [0.0, 1.0]], scale=0.5)
    e = math.e
    assert np.allclose(out, [1 / (1 + e), e / (1 + e)], atol=1e-14)


def test_empty_context_is_zero():
    w = tiny_decode(lens=(0, 3))
    out = run_decode(w)
    assert np.all(out[0] == 0.0)


# ---------------------------------------------------------------- invariants
def test_gqa_equals_mha_on_replicated_kv_heads():
    G, Hkv = 4, 2
    w = tiny_decode(G=G, Hkv=Hkv, D=8, bs=4, seed=9)
    got = run_decode(w)
    # replicate every kv head G times -> an Hq = Hkv*G multi-head problem
    kc, vc = pools_after_store(w)
    kr = np.repeat(kc, G, axis=2)
    vr = np.repeat(vc, G, axis=2)
    ref = oracle.decode(w.q, kr, vr, w.block_tables, w.context_lens, w.scale)
    assert np.array_equal(got, ref)


def test_block_permutation_invariance():
    w = tiny_decode(G=2, bs=4, seed=21)
    perm = np.random.default_rng(2).permutation(w.num_blocks)
    a = run_decode(w)
    b = run_decode(relabel_blocks(w, perm))
    assert np.array_equal(a, b)
    wp = tiny_prefill(G=2, bs=4, seed=22)
    permp = np.random.default_rng(3).permutation(wp.num_blocks)
    assert np.array_equal(run_prefill(wp), run_prefill(relabel_blocks(wp, permp)))


def test_prefix_sharing_invariance():
    lens = np.array([3, 20, 33, 17, 40, 8])
    kw = dict(kind="decode", context_lens=lens, new_lens=np.zeros_like(lens), num_q_heads=4,
              num_kv_heads=2, head_dim=8, block_size=4, seed=31, shared_prefix_len=16)
    shared = build_workload(**kw)
    private = build_workload(**kw, share_prefix=False)
    assert shared.num_blocks < private.num_blocks
    assert np.array_equal(run_decode(shared), run_decode(private))


def test_store_writes_exactly_the_mapped_rows():
    w = tiny_decode(G=1, bs=4, D=8, lens=(5, 9), seed=41)
    kc0, vc0 = w.empty_pool(), w.empty_pool()
    k = w.setup_k
    slots = w.setup_slots.copy()
    slots[-1] = -1                                 # skipped token (the last one)
    kc, vc = oracle.store_kvcache(kc0, vc0, k, w.setup_v, slots)
    flat = kc.reshape(-1, w.num_kv_heads, w.head_dim)
    written = set(int(s) for s in slots if s >= 0)
    for r in range(flat.shape[0]):
        if r in written:
            t = int(np.where(slots == r)[0][0])
            assert np.array_equal(flat[r], k[t])
        else:
            assert np.all(flat[r] == 0xFFC1)
    with pytest.raises(IndexError):
        oracle.store_kvcache(kc0, vc0, k[:1], w.setup_v[:1], np.array([kc0.shape[0] * 4]))


def test_gather_reconstructs_logical_rows_bit_exactly():
    for w in (tiny_decode(G=2, bs=4, seed=51), tiny_prefill(G=1, bs=16, seed=52),
              build_workload(kind="decode", context_lens=np.array([5, 30, 12]),
                             new_lens=np.zeros(3, int), num_q_heads=2, num_kv_heads=1,
                             head_dim=4, block_size=4, seed=53, shared_prefix_len=8)):
        kc, vc = pools_after_store(w)
        for s in range(w.num_seqs):
            ctx = int(w.context_lens[s])
            assert np.array_equal(oracle.gather_sequence(kc, w.block_tables[s], ctx), w.logical_k(s))
            assert np.array_equal(oracle.gather_sequence(vc, w.block_tables[s], ctx), w.logical_v(s))


# ------------------------------------------- cached decode == full recompute
def _as_full_prefill(w):
    """The same sequences with every position treated as a new query token."""
    return build_workload(kind="prefill", context_lens=w.context_lens,
                          new_lens=w.context_lens, num_q_heads=w.num_q_heads,
                          num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                          block_size=w.block_size, seed=0)


def test_decode_equals_last_row_of_full_causal_recompute():
    w = tiny_decode(G=2, bs=4, D=8, lens=(6, 19, 1), seed=61)
    dec = run_decode(w)
    full = _as_full_prefill(w)
    # put the decode query at the last position of each sequence, reuse the decode K/V
    kc, vc = pools_after_store(w)
    Tq = int(full.cu_seqlens_q[-1])
    rng = np.random.default_rng(0)
    q = rng.integers(0, 2 ** 16, size=(Tq, w.num_q_heads, w.head_dim)).astype(np.uint16)
    q = np.where((q & 0x7F80) == 0x7F80, q & 0x3FFF, q)          # no inf/NaN patterns
    for s in range(w.num_seqs):
        q[int(full.cu_seqlens_q[s + 1]) - 1] = w.q[s]
    pre = oracle.prefill(q, kc, vc, w.block_tables, full.cu_seqlens_q, w.context_lens, w.scale)
    for s in range(w.num_seqs):
        assert np.max(np.abs(pre[int(full.cu_seqlens_q[s + 1]) - 1] - dec[s])) < TOL


def test_chunked_prefill_rows_equal_full_prefill_rows():
    lens = np.array([11, 24, 7])
    new = np.array([3, 24, 7])
    w = build_workload(kind="prefill", context_lens=lens, new_lens=lens, num_q_heads=4,
                       num_kv_heads=2, head_dim=8, block_size=4, seed=71)
    full = run_prefill(w)
    kc, vc = pools_after_store(w)
    cu = np.zeros(len(lens) + 1, np.int32)
    cu[1:] = np.cumsum(new)
    rows = np.concatenate([np.arange(int(w.cu_seqlens_q[s + 1]) - int(new[s]),
                                     int(w.cu_seqlens_q[s + 1])) for s in range(len(lens))])
    part = oracle.prefill(w.q[rows], kc, vc, w.block_tables, cu, lens, w.scale)
    assert np.max(np.abs(part - full[rows])) < TOL


def test_one_token_prefill_equals_decode():
    w = tiny_decode(G=4, bs=4, D=8, lens=(9, 1, 30), seed=81)
    dec = run_decode(w)
    kc, vc = pools_after_store(w)
    cu = np.arange(w.num_seqs + 1, dtype=np.int32)
    pre = oracle.prefill(w.q, kc, vc, w.block_tables, cu, w.context_lens, w.scale)
    assert np.max(np.abs(pre - dec)) < TOL


def test_compare_reports_both_norms():
    r = np.array([[1.0, 0.0], [0.0, 1.0]])
    c = oracle.compare(r + np.array([[0.0, 0.1], [0.0, 0.0]]), r)
    assert math.isclose(c["max_abs"], 0.1) and math.isclose(c["norm_rel"], 0.1 / math.sqrt(2))


# ---------------------------------------------------------------- copy-on-write
def test_copy_blocks_copies_exactly_the_pairs():
    rng = np.random.default_rng(51)
    kc = rng.integers(0, 1 << 16, size=(9, 4, 2, 8), dtype=np.uint16)
    vc = rng.integers(0, 1 << 16, size=(9, 4, 2, 8), dtype=np.uint16)
    src, dst = np.array([3, 0, 7]), np.array([5, 8, 1])
    k2, v2 = oracle.copy_blocks(kc, vc, src, dst)
    for b in range(9):
        i = np.where(dst == b)[0]
        want_k = kc[src[i[0]]] if len(i) else kc[b]
        want_v = vc[src[i[0]]] if len(i) else vc[b]
        assert np.array_equal(k2[b], want_k) and np.array_equal(v2[b], want_v)
    assert np.array_equal(kc[5], kc[5])             # inputs are not modified
    with pytest.raises(ValueError):
        oracle.copy_blocks(kc, vc, np.array([1, 2]), np.array([4, 4]))     # duplicate destination
    with pytest.raises(ValueError):
        oracle.copy_blocks(kc, vc, np.array([1, 2]), np.array([2, 3]))     # destination is a source
    with pytest.raises(IndexError):
        oracle.copy_blocks(kc, vc, np.array([9]), np.array([1]))


def cow_workload(seed=61, bs=4):
    from workloads import copy_on_write_append
    lens = np.array([3, 20, 14, 17, 40, 8, 16, 6])
    w = build_workload(kind="decode", context_lens=lens, new_lens=np.zeros_like(lens), num_q_heads=4,
                       num_kv_heads=2, head_dim=8, block_size=bs, seed=seed, shared_prefix_len=16)
    return w, copy_on_write_append(w)


def run_cow_decode(w2, src, dst, oracle_mod=oracle):
    """Pools as the sequences left them, shared blocks copied, last rows appended, decode."""
    kc, vc = w2.empty_pool(), w2.empty_pool()
    kc, vc = oracle_mod.store_kvcache(kc, vc, w2.setup_k, w2.setup_v, w2.setup_slots)
    kc, vc = oracle_mod.copy_blocks(kc, vc, src, dst)
    kc, vc = oracle_mod.store_kvcache(kc, vc, w2.new_k, w2.new_v, w2.new_slots)
    return oracle_mod.decode(w2.q, kc, vc, w2.block_tables, w2.context_lens, w2.scale), (kc, vc)


def test_copy_on_write_append_equals_brute_force_and_keeps_sharers_intact():
    w, (w2, src, dst) = cow_workload()
    assert len(src) > 0                                # some last positions were in shared blocks
    out, (kc, vc) = run_cow_decode(w2, src, dst)
    assert np.max(np.abs(out - brute_decode(w2))) < TOL
    # no block is read by one sequence and written in the step by another
    bs = w2.block_size
    written = {int(s) // bs for s in w2.new_slots}
    for s in range(w2.num_seqs):
        ctx = int(w2.context_lens[s])
        mine = int(w2.new_slots[np.where(np.nonzero(w2.new_lens)[0] == s)[0][0]]) // bs
        for b in w2.block_tables[s, :-(-ctx // bs)]:
            assert int(b) not in written or int(b) == mine
    # appending without the copies would put rows in blocks other sequences read
    shared_slots = []
    for s in range(w.num_seqs):
        last = int(w.context_lens[s]) - 1
        shared_slots.append(int(w.block_tables[s, last // bs]) * bs + last % bs)
    assert len(set(np.array(shared_slots) // bs)) < len(shared_slots)


# ---------------------------------------------------------------- chained block hashes
def test_block_hashes_against_golden_and_the_recursive_rule():
    import os
    from workloads import compute_hash
    golden = os.path.join(os.path.dirname(__file__), "golden", "rolling_hash.txt")
    for line in open(golden):
        if line.startswith("#") or not line.strip():
            continue
        pre, toks, want = [x.strip() for x in line.split(";")]
        toks = [int(t) for t in toks.split()] if toks else []
        if int(pre) == 0 and toks:
            # a seed of 0 is the first block: the closed form over the whole block
            assert int(oracle.block_hashes(toks, len(toks))[0]) == int(want)
    rng = np.random.default_rng(71)
    for bs in (1, 3, 16):
        toks = rng.integers(0, 1 << 31, size=5 * bs + (bs - 1)).tolist()   # 5 full blocks + a tail
        got = oracle.block_hashes(toks, bs)
        assert len(got) == 5
        h = 0
        for b in range(5):
            h = compute_hash(toks[b * bs:(b + 1) * bs], h)
            assert int(got[b]) == h
