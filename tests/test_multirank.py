"""The benchmark's multi-rank path on CPU: two gloo ranks (world size 2) run the same
host logic the NCCL ranks run on GPUs. Each rank draws its own batch of the same
configuration (weak scaling, no data exchange), and the whole-job number is the
bytes of all ranks over the slowest rank's time. No GPU needed."""
import datetime
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    try:
        sys.path.insert(0, ROOT)
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        import torch
        import torch.distributed as dist
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=60))
        import bench
        from workloads import CONFIGS
        cfg = CONFIGS["tiny_decode"]
        w = bench.rank_workload(cfg, rank)
        shape = (w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size)
        shapes = [None] * world
        dist.all_gather_object(shapes, shape)
        lens = [None] * world
        dist.all_gather_object(lens, w.context_lens.tolist())
        step_ms = 1.0 + rank                                  # rank 1 is the slowest
        mx = bench.max_over_ranks(step_ms, dist, torch, "cpu")
        nbytes = bench.decode_bytes(w) + bench.store_bytes(w)
        tot = bench.sum_over_ranks(nbytes, dist, torch, "cpu")
        allb = [None] * world
        dist.all_gather_object(allb, nbytes)
        dist.barrier()
        dist.destroy_process_group()
        out.put((rank, {"shapes": shapes, "lens": lens, "max": mx, "sum": tot, "all_bytes": allb,
                        "value": bench.job_gbps(tot, mx)}))
    except Exception as e:  # report instead of hanging the parent
        out.put((rank, {"error": repr(e)}))


def test_two_gloo_ranks_weak_scaling_and_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        r, d = q.get(timeout=240)
        res[r] = d
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(2):
        assert "error" not in res[r], res[r]
    a, b = res[0], res[1]
    # same configuration shape on every rank, different sequences (independent batches)
    assert a["shapes"][0] == a["shapes"][1]
    assert a["lens"][0] != a["lens"][1]
    # every rank agrees on the slowest time and on the job's bytes
    assert a["max"] == b["max"] == 2.0
    assert a["sum"] == b["sum"] == float(sum(a["all_bytes"]))
    assert a["value"] == pytest.approx(sum(a["all_bytes"]) / 2.0e-3 / 1e9)


def test_single_rank_helpers_and_rank0_batch():
    sys.path.insert(0, ROOT)
    import bench
    from workloads import CONFIGS, generate
    cfg = CONFIGS["tiny_decode"]
    assert np.array_equal(bench.rank_workload(cfg, 0).context_lens, generate(cfg).context_lens)
    assert bench.max_over_ranks(3.5, None, None, "cpu") == 3.5
    assert bench.job_gbps(2e9, 1000.0) == pytest.approx(2.0)


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3",
                                      "--workload", "tiny_decode"])
    bench.main()
    assert capsys.readouterr().out == ""          # other ranks exit without work or output
