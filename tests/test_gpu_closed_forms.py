"""Closed forms of attention on the GPU (head dim 128, the tensor-core paths).

Each case is a special input whose softmax attention has a plain answer, checked
through pa_decode (single and split contexts) and pa_prefill against both the fp64
oracle and the closed form itself:
  * q = 0: every visible position has the same score, so the output is the mean of
    the visible V rows;
  * all keys of a sequence equal: same, the mean of V;
  * V the same row c at every position: the weights sum to one, so the output is c;
  * one key that is a large multiple of the (shared) query: its weight is ~1 and the
    output is its V row.
The kernels round the probabilities to bf16 before the value product, so results are
compared within the decode bar, not bit for bit.
"""
import numpy as np
import pytest

from tests.gpu_helpers import (DeviceWorkload, assert_close, oracle_decode, oracle_prefill,
                               to_f64)
from workloads import build_workload
from workloads.gen import f32_to_bf16_bits

pytestmark = pytest.mark.gpu

CASES = ["q_zero", "equal_keys", "constant_v", "dominant_key"]


def bf16_to_f64(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def decode_workload(seed):
    lens = np.array([1, 127, 300, 1000, 2500, 64])
    return build_workload(kind="decode", context_lens=lens, new_lens=np.ones(len(lens), int),
                          num_q_heads=16, num_kv_heads=8, head_dim=128, block_size=64, seed=seed)


def prefill_workload(seed):
    ctx = np.array([700, 129, 300])
    new = np.array([200, 129, 1])
    return build_workload(kind="prefill", context_lens=ctx, new_lens=new, num_q_heads=8,
                          num_kv_heads=2, head_dim=128, block_size=64, seed=seed)


def shape_case(w, case):
    """Rewrite the workload's source rows / queries in place; returns a function
    (sequence, q head, visible positions) -> the closed-form output, float64 [D]."""
    G = w.num_q_heads // w.num_kv_heads
    rng = np.random.default_rng(17)
    if case == "q_zero":
        w.q[:] = 0
    elif case == "equal_keys":
        for s in range(w.num_seqs):
            rows = w.logical_rows[s]
            w.src_k[rows] = w.src_k[rows[0]]
    elif case == "constant_v":
        c = f32_to_bf16_bits(rng.standard_normal((w.num_kv_heads, w.head_dim)).astype(np.float32))
        w.src_v[:] = c
    elif case == "dominant_key":
        # every query head of a group (and, in prefill, every new token of a sequence)
        # gets the same vector u; the key at one chosen position is 4 u, so its score
        # is 4 |u|^2 / sqrt(D) (~45) against ~N(0, 1) for the others
        chosen = {}
        for s in range(w.num_seqs):
            rows = w.logical_rows[s]
            ctx = len(rows)
            q0, q1 = int(w.cu_seqlens_q[s]), int(w.cu_seqlens_q[s + 1])
            j = 0 if w.kind == "prefill" else ctx // 2     # position 0 is visible to all
            for g in range(w.num_kv_heads):
                u = w.q[q0, g * G].copy()
                w.q[q0:q1, g * G:(g + 1) * G] = u
                w.src_k[rows[j], g] = f32_to_bf16_bits(4.0 * bf16_to_f64(u).astype(np.float32))
            chosen[s] = rows[j]
    else:
        raise ValueError(case)

    def closed(s, h, npos):
        rows = w.logical_rows[s][:npos]
        g = h // G
        if case in ("q_zero", "equal_keys"):
            return bf16_to_f64(w.src_v[rows, g]).mean(axis=0)
        if case == "constant_v":
            return bf16_to_f64(w.src_v[rows[0], g])
        return bf16_to_f64(w.src_v[chosen[s], g])
    return closed


@pytest.mark.parametrize("case", CASES)
def test_decode_closed_forms(case):
    w = decode_workload(seed=300 + CASES.index(case))
    closed = shape_case(w, case)
    ref = oracle_decode(w)
    want = np.stack([np.stack([closed(s, h, int(w.context_lens[s]))
                               for h in range(w.num_q_heads)]) for s in range(w.num_seqs)])
    # the oracle itself reaches the closed form (to fp64 rounding)
    assert np.max(np.abs(ref - want)) <= 1e-9 * max(1.0, np.max(np.abs(want)))
    dw = DeviceWorkload(w)
    for P in (0, 256):
        got = to_f64(dw.decode(partition_size=P))
        assert_close(got, ref, f"decode {case} P={P}")
        assert_close(got, want, f"decode {case} P={P} vs closed form")


@pytest.mark.parametrize("case", CASES)
def test_prefill_closed_forms(case):
    w = prefill_workload(seed=400 + CASES.index(case))
    closed = shape_case(w, case)
    ref = oracle_prefill(w)
    rows = []
    for s in range(w.num_seqs):
        n = int(w.cu_seqlens_q[s + 1] - w.cu_seqlens_q[s])
        first = int(w.context_lens[s]) - n
        for i in range(n):
            rows.append(np.stack([closed(s, h, first + i + 1) for h in range(w.num_q_heads)]))
    want = np.stack(rows)
    assert np.max(np.abs(ref - want)) <= 1e-9 * max(1.0, np.max(np.abs(want)))
    got = to_f64(DeviceWorkload(w).prefill())
    assert_close(got, ref, f"prefill {case}")
    assert_close(got, want, f"prefill {case} vs closed form")
