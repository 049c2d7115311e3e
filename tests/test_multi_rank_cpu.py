"""World-size-2 checks of the multi-GPU host logic on CPU (gloo): each rank runs
its own independent batch (no collective on the data path), the step time is
the max over ranks, and the whole-job value counts every rank's units."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    from gated_linear_attention_local_b200.workloads import make_workload
    args = bench.parse_args([])
    w_size, r, _ = bench.dist_setup(args)
    assert (w_size, r) == (world, rank)
    # per-rank time: rank 1 is slower; every rank must see the max
    t = bench.max_over_ranks(10.0 + 5.0 * rank, world, torch.device("cpu"))
    # per-rank inputs differ (independent batches), shapes agree
    w = make_workload("tiny_fp32", seed=args.seed + 1000 * rank)
    digest = torch.tensor([float(w["q"].double().sum())])
    gathered = [torch.zeros(1) for _ in range(world)]
    dist.all_gather(gathered, digest)
    out[rank] = (t, [float(x) for x in gathered])
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_timing_and_sharding():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    assert sorted(out.keys()) == [0, 1]
    for rank in range(world):
        t, digests = out[rank]
        assert t == 15.0
        assert digests[0] != digests[1]


def test_whole_job_value_counts_all_ranks():
    import bench
    from gated_linear_attention_local_b200.workloads import make_workload
    w = make_workload("tiny_fp32")
    c = bench.algorithmic_counts(w)
    assert c["tokens"] == 256
    # value = world * units / max time
    ms = 2.0
    assert 4 * c["tokens"] / (ms * 1e-3) == pytest.approx(512000.0)
