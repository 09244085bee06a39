"""The multi-rank path on CPU: two `gloo` ranks run the benchmark's rank logic.

Every rank processes its own independent batch (weak scaling, no collective on the data path);
the only collective is the max over ranks of the timing.  Each rank's batch is checked with the
fp64 oracle on a small case, so the test also shows the shards are independent problems.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import kda_inputs as KI
import oracle


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = bench.rank_workload(KI.Workload("mr", (40, 23), 2, 64, 64, seed=5), rank)
        inp = KI.make_inputs(w, "cpu")
        h = lambda t: None if t is None else t.double().numpy()
        out, SF = oracle.kda_fwd(h(inp["q"]), h(inp["k"]), h(inp["v"]), h(inp["a"]), h(inp["beta"]),
                                 h(inp["A_log"]), inp["cu_seqlens"].numpy(), gate=h(inp["gate"]),
                                 n_threads=1)
        # a fake per-rank time: the job is as slow as its slowest rank
        ms = bench.max_over_ranks(1.0 + rank, world, "cpu")
        rate = bench.whole_job_rate(w.total_tokens, world, ms)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), out=out, SF=SF, ms=ms, rate=rate,
                 seed=w.seed, q=h(inp["q"]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    r = [np.load(tmp_path / f"rank{i}.npz") for i in range(world)]
    # the max over ranks reached both ranks
    assert float(r[0]["ms"]) == float(r[1]["ms"]) == 2.0
    # whole-job throughput: both ranks' tokens over the slowest rank's time
    assert float(r[0]["rate"]) == pytest.approx(2 * 63 / 2e-3)
    # independent batches (different seeds, different data), each self-consistent
    assert int(r[0]["seed"]) != int(r[1]["seed"])
    assert not np.array_equal(r[0]["q"], r[1]["q"])
    for x in r:
        assert np.isfinite(x["out"]).all() and np.isfinite(x["SF"]).all()


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_rate(8192, 1, 1.0) == pytest.approx(8192e3)
    w = KI.PREFILL_8K
    assert bench.rank_workload(w, 0) == w and bench.rank_workload(w, 3).seed == w.seed + 3


def test_reference_arm_runs_on_rank0_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    import argparse
    ns = argparse.Namespace(impl="reference", gpus=2, steps=1, warmup=0,
                            workload="pr1_ref_B1_H2_T256_d64")
    assert bench.run_reference(ns) == 0   # returns at once, no work, no output
