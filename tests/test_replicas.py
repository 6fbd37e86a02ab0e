"""The several-GPU path on CPU: two gloo ranks run the replica bookkeeping the benchmark
uses (barrier, slowest-rank time, whole-job throughput, per-replica input streams)."""
import json
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime
    import torch.distributed as dist
    from streaming_video_attention_b200 import replicas

    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        assert replicas.world() == (rank, world, rank)
        replicas.barrier()
        # rank r took (r + 1) seconds for 100 units
        value, slow = replicas.job_throughput(100, float(rank + 1))
        cfg = replicas.replica_config(synth.CONFIGS["tiny_fp32"], rank)
        q = synth.chunk_q(cfg, 0, 0)
        replicas.barrier()
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"value": value, "slow": slow, "seed": cfg.seed, "q0": float(q.ravel()[0]),
                       "q_sum": float(np.sum(q))}, f)
    finally:
        dist.destroy_process_group()


def test_two_replicas_report_slowest_rank_and_distinct_streams(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    r = [json.load(open(tmp_path / f"r{i}.json")) for i in range(world)]
    for x in r:
        assert x["slow"] == 2.0                       # max over ranks, seen by every rank
        assert x["value"] == pytest.approx(2 * 100 / 2.0)
    assert r[0]["seed"] != r[1]["seed"]
    assert r[0]["q_sum"] != r[1]["q_sum"]             # replicas draw their own inputs
    # rank 0 keeps the configuration's own stream
    base = synth.chunk_q(synth.CONFIGS["tiny_fp32"], 0, 0)
    assert r[0]["q0"] == float(base.ravel()[0])


def test_single_process_needs_no_process_group():
    from streaming_video_attention_b200 import replicas
    replicas.barrier()
    assert replicas.job_throughput(50, 2.0) == (25.0, 2.0)
