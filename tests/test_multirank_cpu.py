"""The bench's multi-rank path on CPU: two gloo ranks. The path shards into
independent replicas (no data exchange), so what the ranks share is the
timing: every rank ends with the slowest rank's figures, and the reference
arm runs on rank 0 alone (the other ranks return without work)."""
import json
import os
import socket

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, ws: int, port: int, out_dir: str):
    import datetime
    import sys
    import time

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist

    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        sys.path.insert(0, ROOT)
        import bench
        import workloads as W

        # rank r's timings (ms): the job's are the per-entry maxima
        vals = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 0.5 * rank], dist, "cpu")
        ref_s = None
        if rank != 0:

            class Args:
                steps, warmup, cpu_seconds = 1, 0, 1.0

            t0 = time.time()
            assert bench.run_reference(Args, W.spec("tiny"), ws, rank) is None
            ref_s = time.time() - t0
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"vals": vals, "ref_s": ref_s}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_timing(tmp_path):
    mp.start_processes(_rank, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    for g in got:
        assert g["vals"] == [2.0, 10.0, 0.5]
    assert got[1]["ref_s"] is not None and got[1]["ref_s"] < 5.0  # rank 1 did no oracle work


def test_single_rank_keeps_its_values():
    import sys

    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks([3, 1.5], None, "cpu") == [3.0, 1.5]
