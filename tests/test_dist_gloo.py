"""Host logic of the multi-rank benchmark, on two gloo ranks on the CPU.

Each rank draws its own batch (weak scaling, no data-path collective); the
timed region's duration is the maximum over ranks; the reference arm prints
only on rank 0.
"""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import bench
    from linear_attention_recurrent_decode_b200 import workloads

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # max over ranks
        local = 10.0 + rank * 5.0
        got = bench.reduce_max(local)
        # per-rank batches: same shapes, different draws
        w = workloads.config("n1_t1_hv8", seed=bench.rank_seed(0, rank))
        digest = float(w.q.float().sum() + w.state.sum())
        # reference arm: only rank 0 prints
        buf = io.StringIO()
        with redirect_stdout(buf):
            bench.main(["--impl", "reference", "--gpus", str(world), "--steps", "2", "--warmup", "3",
                        "--config", "n1_t1_hv8", "--reference-budget-s", "5"])
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max": got, "digest": digest, "stdout": buf.getvalue()}, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert [r["max"] for r in res] == [15.0, 15.0]
    assert res[0]["digest"] != res[1]["digest"], "ranks must draw different batches"
    line = json.loads(res[0]["stdout"].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["unit"] == "us/call"
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert res[1]["stdout"] == ""


def test_replica_count_exceeds_twice_l2():
    sys.path.insert(0, ROOT)
    import bench

    l2 = 126 * 2 ** 20
    for touched in (1 << 20, 17 << 20, 68 << 20, 600 << 20):
        r = bench.choose_replicas(touched, l2)
        assert (r - 1) * touched >= 2 * l2 or r == 2 and touched >= 2 * l2
