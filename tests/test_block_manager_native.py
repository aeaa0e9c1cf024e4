"""The library's host block manager (pa_bm_*) against the test fixture's BlockManager:
the same stream of requests, finishes and decode appends must give the same block
tables, slots, copy-on-write pairs and reference counts after every step. Host-only:
no GPU needed."""
import numpy as np
import pytest

import oracle
import paged_kv_cache_442_b200 as pa
from paged_kv_cache_442_b200 import build as pa_build
from workloads import BlockManager


@pytest.fixture(scope="module", autouse=True)
def _lib():
    pa_build.build()
    pa.load_library()


def make_requests(rng, n, prefixes, vocab=50):
    reqs = []
    for _ in range(n):
        p = prefixes[rng.integers(len(prefixes))] if rng.random() < 0.7 else []
        tail = rng.integers(1, vocab, size=rng.integers(0, 14)).tolist()
        toks = list(p) + tail
        if not toks:
            toks = [int(rng.integers(1, vocab))]
        reqs.append(toks)
    return reqs


@pytest.mark.parametrize("bs,seed", [(1, 1), (2, 2), (4, 3), (4, 4), (8, 5)])
def test_native_matches_fixture_on_a_random_stream(bs, seed):
    rng = np.random.default_rng(seed)
    nb = 1536 // bs + 64
    order = rng.permutation(nb)
    py = BlockManager(nb, bs, free_order=order)
    nat = pa.BlockManager(nb, bs, free_order=order)
    prefixes = [rng.integers(1, 50, size=rng.integers(1, 20)).tolist() for _ in range(4)]
    live = {}          # id -> (python table, native table, tokens)
    steps = 0
    for toks in make_requests(rng, 400, prefixes):
        op = rng.random()
        if op < 0.45 or not live:
            try:
                t_py = py.allocate(toks)
            except MemoryError:
                with pytest.raises(pa.PAError) as e:
                    nat.allocate(toks)
                assert e.value.status == 6
                break                    # the fixture keeps partial state on failure: stop here
            t_nat = nat.allocate(toks)
            assert t_nat == t_py
            live[steps] = (t_py, list(t_nat), list(toks))
        elif op < 0.85:
            k = list(live)[rng.integers(len(live))]
            t_py, t_nat, _ = live.pop(k)
            py.free_table(t_py)
            nat.free(t_nat)
        else:
            k = list(live)[rng.integers(len(live))]
            t_py, t_nat, seq = live[k]
            pos, tok = len(seq), int(rng.integers(1, 50))
            try:
                r_py = py.append(t_py, pos, tok)
            except MemoryError:
                with pytest.raises(pa.PAError) as e:
                    nat.append(t_nat, pos, tok)
                assert e.value.status == 6
                break
            r_nat = nat.append(t_nat, pos, tok)
            assert r_nat == r_py and t_nat == t_py
            seq.append(tok)
        assert nat.num_used() == py.num_used()
        assert np.array_equal(nat.ref_counts(), np.array(py.ref_counts()))
        steps += 1
    assert steps > 50
    # everything finishes: the pool is empty again
    for t_py, t_nat, _ in live.values():
        py.free_table(t_py)
        nat.free(t_nat)
    assert nat.num_used() == 0 and py.num_used() == 0


def test_native_shares_prefix_blocks_and_uses_given_hashes():
    bs = 4
    nat = pa.BlockManager(32, bs)
    sys_prompt = list(range(1, 13))                 # 3 full blocks
    a = nat.allocate(sys_prompt + [40, 41])
    b = nat.allocate(sys_prompt + [50])
    assert a[:3] == b[:3] and a[3] != b[3]
    rc = nat.ref_counts()
    assert all(rc[x] == 2 for x in a[:3])
    # hashes supplied by the caller (as the GPU computes them) give the same table
    nat2 = pa.BlockManager(32, bs)
    a2 = nat2.allocate(sys_prompt + [40, 41], block_hashes=oracle.block_hashes(sys_prompt + [40, 41], bs))
    b2 = nat2.allocate(sys_prompt + [50], block_hashes=oracle.block_hashes(sys_prompt + [50], bs))
    assert (a2, b2) == (a, b)


def test_native_errors():
    nat = pa.BlockManager(4, 2)
    t = nat.allocate([1, 2, 3, 4, 5, 6])
    with pytest.raises(pa.PAError) as e:
        nat.allocate([9, 9, 9])                      # 2 blocks needed, 1 free
    assert e.value.status == 6
    assert nat.num_used() == 3                       # the failed request holds nothing
    with pytest.raises(pa.PAError):
        nat.free([t[0], t[0]])                       # released twice
    assert nat.num_used() == 3                       # and nothing changed
    with pytest.raises(pa.PAError):
        nat.free([7])
    with pytest.raises(ValueError):
        pa.BlockManager(4, 2, free_order=[0, 1, 1, 2])


def test_native_append_cases_match_fixture():
    """Fresh block, private block, shared block (copy-on-write) and a private block
    still registered under a hash, on both managers."""
    order = [3, 1, 4, 0, 5, 2, 6, 7]
    py, nat = BlockManager(8, 2, free_order=order), pa.BlockManager(8, 2, free_order=order)
    ops = [("alloc", [1, 2, 3]), ("append", 0, 3, 9), ("append", 0, 4, 5), ("alloc", [1, 2, 7]),
           ("alloc", [1]), ("append", 2, 1, 8), ("free", 1), ("alloc", [1, 2]), ("free", 0),
           ("alloc", [1]), ("append", 4, 1, 6)]
    tp, tn = [], []
    for op in ops:
        if op[0] == "alloc":
            tp.append(py.allocate(op[1]))
            tn.append(nat.allocate(op[1]))
            assert tn[-1] == tp[-1]
        elif op[0] == "free":
            py.free_table(tp[op[1]])
            nat.free(tn[op[1]])
            tp[op[1]], tn[op[1]] = [], []
        else:
            r1 = py.append(tp[op[1]], op[2], op[3])
            r2 = nat.append(tn[op[1]], op[2], op[3])
            assert r1 == r2 and tp[op[1]] == tn[op[1]]
        assert np.array_equal(nat.ref_counts(), np.array(py.ref_counts()))


@pytest.mark.parametrize("bs,seed", [(1, 11), (4, 12), (16, 13)])
def test_batch_allocation_equals_one_call_per_request(bs, seed):
    """pa_bm_allocate_batch gives the tables and reference counts of allocating the same
    requests one call at a time, with and without precomputed block hashes."""
    rng = np.random.default_rng(seed)
    nb = 4096 // bs + 64
    order = rng.permutation(nb)
    prefixes = [rng.integers(1, 50, size=rng.integers(1, 40)).tolist() for _ in range(3)]
    reqs = make_requests(rng, 120, prefixes)
    one = pa.BlockManager(nb, bs, free_order=order)
    want = [one.allocate(r) for r in reqs]
    for hashes in (None, [oracle.block_hashes(r, bs) for r in reqs]):
        batch = pa.BlockManager(nb, bs, free_order=order)
        got = batch.allocate_batch(reqs, block_hashes=hashes)
        assert got == want
        assert np.array_equal(batch.ref_counts(), one.ref_counts())
        # and the tables free cleanly
        for t in got:
            batch.free(t)
        assert batch.num_used() == 0


def test_batch_allocation_stops_at_the_first_request_that_does_not_fit():
    bs = 4
    reqs = [list(range(1, 9)), list(range(20, 33)), list(range(40, 60)), [7, 7]]
    bm = pa.BlockManager(6, bs)           # 2 + 4 blocks fit, the third request does not
    with pytest.raises(pa.PAError) as e:
        bm.allocate_batch(reqs)
    assert e.value.status == 6 and e.value.done == 2
    assert [len(t) for t in e.value.tables] == [2, 4]
    ref = pa.BlockManager(6, bs)
    ref.allocate(reqs[0])
    ref.allocate(reqs[1])
    assert np.array_equal(bm.ref_counts(), ref.ref_counts())   # request 2 holds nothing


def test_batch_allocation_argument_checks():
    import ctypes
    bm = pa.BlockManager(16, 4)
    lib = pa.load_library()
    toks = np.arange(1, 11, dtype=np.int32)
    cu = np.array([0, 6, 10], dtype=np.int32)
    out = np.zeros(8, dtype=np.int32)
    done = ctypes.c_int32(-1)
    # hash offsets that disagree with the lengths (6 tokens = 1 full block, not 2)
    hs = np.zeros(3, dtype=np.uint32)
    cub = np.array([0, 2, 3], dtype=np.int32)
    st = lib.pa_bm_allocate_batch(bm.h, toks.ctypes.data, cu.ctypes.data, 2, hs.ctypes.data,
                                  cub.ctypes.data, out.ctypes.data, ctypes.byref(done))
    assert st == 1 and done.value == 0 and bm.num_used() == 0
    bad_cu = np.array([1, 6, 10], dtype=np.int32)
    st = lib.pa_bm_allocate_batch(bm.h, toks.ctypes.data, bad_cu.ctypes.data, 2, None, None,
                                  out.ctypes.data, ctypes.byref(done))
    assert st == 1 and bm.num_used() == 0
    st = lib.pa_bm_allocate_batch(bm.h, toks.ctypes.data, cu.ctypes.data, 0, None, None,
                                  out.ctypes.data, ctypes.byref(done))
    assert st == 0 and done.value == 0


def test_batch_allocation_rejects_a_negative_token_before_taking_blocks():
    """A negative token id in a later request fails the whole call up front: the
    requests before it do not keep any block."""
    import ctypes
    bm = pa.BlockManager(16, 4)
    lib = pa.load_library()
    toks = np.arange(1, 11, dtype=np.int32)
    toks[7] = -3                                   # inside the second request
    cu = np.array([0, 6, 10], dtype=np.int32)
    out = np.zeros(8, dtype=np.int32)
    done = ctypes.c_int32(-1)
    st = lib.pa_bm_allocate_batch(bm.h, toks.ctypes.data, cu.ctypes.data, 2, None, None,
                                  out.ctypes.data, ctypes.byref(done))
    assert st == 1 and done.value == 0 and bm.num_used() == 0
