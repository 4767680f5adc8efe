"""Host-side logic of the multi-GPU benchmark path on two CPU ranks (gloo).

The operator shards by independent (batch, head) work with no data-path
collective; what spans ranks is only the timing protocol: a barrier around
the timed region, the maximum of the per-rank device times, and the
whole-job throughput computed from it.  These run here as two gloo
processes, without a GPU."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    r, w, lr = bench.dist_env()
    assert (r, w, lr) == (rank, world, rank)
    bench.barrier(world)
    # each rank reports a different local time; every rank sees the maximum
    mx = bench.max_over_ranks(10.0 + rank, world, torch.device("cpu"))
    # per-rank seeds of the weak-scaling workload differ
    from differential_attention_sm_b200 import inputs as I
    w2 = I.WORKLOADS["v1_prefill_bf16"]
    x = I.v1_inputs(1, 8, 2, 4, 8, w2.seed + 1000 * rank)
    first = float(x["q"].float().reshape(-1)[0])
    gathered = [None] * world
    dist.all_gather_object(gathered, first)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, mx, gathered))


def test_two_rank_timing_protocol():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, gathered in res:
        assert mx == 11.0                      # max over ranks, seen by every rank
        assert gathered[0] != gathered[1]      # ranks draw different batches


def test_whole_job_throughput_scales_with_ranks():
    import bench
    B, N, H = 4, 4096, 16
    flops = bench.prefill_pairs(B, N, H) * bench.v1_flops_per_pair(64, 128)
    assert flops == 537001984 * 768
    # value = world * per-rank work / max time
    for world in (1, 2, 8):
        v = world * flops * 10 / (5.0e-3) / 1e12
        assert v == pytest.approx(world * flops * 2000 / 1e12)
