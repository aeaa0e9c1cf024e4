"""Batched chained block hashes on the GPU (pa_block_hashes), bit-exact against the
oracle's closed form on small ragged batches, against the recursive rule at full
size, and feeding the host block manager the same tables as host hashing."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_442_b200 as pa
from workloads import CONFIGS, compute_hash, generate

pytestmark = pytest.mark.gpu


def gpu_hashes(seqs, bs):
    toks = np.concatenate([np.asarray(s, dtype=np.int32) for s in seqs]) if seqs else np.zeros(0, np.int32)
    lens = np.array([len(s) for s in seqs], dtype=np.int64)
    cu_t = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    cu_b = np.concatenate([[0], np.cumsum(lens // bs)]).astype(np.int32)
    d_t = torch.from_numpy(toks).cuda() if len(toks) else torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.zeros(max(1, int(cu_b[-1])), dtype=torch.int32, device="cuda")
    pa.pa_block_hashes(d_t, torch.from_numpy(cu_t).cuda(), torch.from_numpy(cu_b).cuda(), bs, out)
    h = out.cpu().numpy().view(np.uint32)
    return [h[cu_b[i]:cu_b[i + 1]] for i in range(len(seqs))]


def recursive(seq, bs):
    out, h = [], 0
    for b in range(len(seq) // bs):
        h = compute_hash(seq[b * bs:(b + 1) * bs], h)
        out.append(h)
    return np.array(out, dtype=np.uint32)


@pytest.mark.parametrize("bs,max_len", [(1, 90), (4, 300), (16, 600), (64, 700)])
def test_block_hashes_match_closed_form(bs, max_len):
    rng = np.random.default_rng(bs)
    lens = rng.integers(0, max_len, size=40)
    lens[:4] = [0, bs - 1, bs, 33 * bs + 1]          # empty, no full block, one block, > 32 blocks
    seqs = [rng.integers(0, 1 << 31, size=int(n)).tolist() for n in lens]
    got = gpu_hashes(seqs, bs)
    for s, g in zip(seqs, got):
        assert np.array_equal(g, oracle.block_hashes(s, bs))


def test_block_hashes_full_size_against_recursive_rule():
    cfg = CONFIGS["prefix_share_decode"]
    w = generate(cfg)
    rng = np.random.default_rng(3)
    prefix = rng.integers(1, 1 << 20, size=1024).tolist()
    seqs = [prefix[:n] + rng.integers(1, 1 << 20, size=max(0, int(n) - 1024)).tolist()
            for n in w.context_lens]
    got = gpu_hashes(seqs, cfg.block_size)
    for s, g in zip(seqs, got):
        assert np.array_equal(g, recursive(s, cfg.block_size))


def test_gpu_hashes_give_the_same_tables():
    bs = 16
    rng = np.random.default_rng(4)
    prefix = rng.integers(1, 500, size=100).tolist()
    seqs = [prefix[:int(rng.integers(1, 100))] + rng.integers(1, 500, size=int(rng.integers(0, 60))).tolist()
            for _ in range(64)]
    hs = gpu_hashes(seqs, bs)
    host, dev = pa.BlockManager(2048, bs), pa.BlockManager(2048, bs)
    for s, h in zip(seqs, hs):
        assert dev.allocate(s, block_hashes=h) == host.allocate(s)
    assert np.array_equal(dev.ref_counts(), host.ref_counts())


def test_block_offsets_past_the_tokens_are_clamped_and_reported():
    """cu_blocks claiming one block more than a sequence's tokens hold: nothing is read
    past the sequence (the token buffer is padded so that even an unclamped read would
    stay inside it), the mismatch is reported, and every in-range hash is unchanged."""
    bs = 16
    rng = np.random.default_rng(12)
    seqs = [rng.integers(0, 1 << 31, size=n).tolist() for n in (70, 33, 100)]
    want = [oracle.block_hashes(s, bs) for s in seqs]
    toks = np.concatenate([np.asarray(s, np.int32) for s in seqs] + [np.zeros(4 * bs, np.int32)])
    lens = np.array([len(s) for s in seqs])
    cu_t = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    nblk = lens // bs
    nblk[1] += 1                                   # sequence 1 claims 3 blocks, has 2
    cu_b = np.concatenate([[0], np.cumsum(nblk)]).astype(np.int32)
    sentinel = 0x5A5A5A5A
    out = torch.full((int(cu_b[-1]),), sentinel, dtype=torch.int32, device="cuda")
    with pytest.raises(pa.PAError) as e:
        pa.pa_block_hashes(torch.from_numpy(toks).cuda(), torch.from_numpy(cu_t).cuda(),
                           torch.from_numpy(cu_b).cuda(), bs, out)
    assert e.value.status == 3
    h = out.cpu().numpy().view(np.uint32)
    assert np.array_equal(h[cu_b[0]:cu_b[1]], want[0])
    assert np.array_equal(h[cu_b[1]:cu_b[1] + 2], want[1])
    assert h[cu_b[1] + 2] == sentinel               # the claimed third block is not written
    assert np.array_equal(h[cu_b[2]:cu_b[3]], want[2])
