"""N > 1 path on CPU: world_size-2 gloo process group exercising the replica logic bench.py uses
under torchrun (disjoint sequence sets, max-over-ranks timing, whole-job throughput).  The
sampling path shards by sequence with no data exchange, so only these host-side pieces run
multi-rank."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import synth
from masked_discrete_diffusion_sparse_b200.replicas import (aggregate_throughput,
                                                            replica_sequence_ids,
                                                            slowest_time_ms)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, batch):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ids = replica_sequence_ids(rank, batch)
        all_ids = [None] * world
        dist.all_gather_object(all_ids, ids)
        flat = [i for r in all_ids for i in r]
        assert sorted(flat) == list(range(world * batch)), flat   # disjoint and complete
        # each rank draws its own prompts and decoding orders from its sequence ids
        wl = synth.WORKLOADS["C"]
        firsts = [tuple(synth.make_plan(wl, i).order[:8].tolist()) for i in ids]
        all_firsts = [None] * world
        dist.all_gather_object(all_firsts, firsts)
        assert len({f for r in all_firsts for f in r}) == world * batch
        # timing: the job ends with its slowest replica
        ms = 10.0 + 5.0 * rank
        ms_max = slowest_time_ms(ms, world, dist)
        assert ms_max == 10.0 + 5.0 * (world - 1)
        v = aggregate_throughput(4096 * batch, world, ms_max)
        assert abs(v - 4096 * batch * world / (ms_max / 1e3)) < 1e-6
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("batch", [1, 4])
def test_replicas_world2_gloo(batch):
    mp.spawn(_worker, args=(2, _free_port(), batch), nprocs=2, join=True)


def test_replica_helpers_single_process():
    assert replica_sequence_ids(0, 3) == [0, 1, 2]
    assert replica_sequence_ids(2, 3) == [6, 7, 8]
    assert slowest_time_ms(12.5, 1) == 12.5
    assert aggregate_throughput(4096, 1, 50.0) == pytest.approx(81920.0)
    with pytest.raises(ValueError):
        replica_sequence_ids(-1, 1)
    with pytest.raises(ValueError):
        aggregate_throughput(1, 1, 0.0)
