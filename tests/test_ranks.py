"""World-size-2 gloo tests of the replica plumbing (CPU, no GPU)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_diffusion_attention_b200 import ranks, synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, wsz, local = ranks.rank_env()
        assert (r, wsz, local) == (rank, world, rank)
        # each rank's "elapsed time" differs; the job time is the slowest rank's
        got = ranks.max_over_ranks(1.5 + rank)
        ranks.barrier(device_sync=False)
        w = ranks.replica_workload(synth.WORKLOADS["tiny_fp32"], rank)
        q = synth.block_base(w, 0)[0]
        rate = ranks.whole_job_rate(16 * 10, wsz, got)
        out[rank] = (got, float(q.sum()), rate)
    finally:
        dist.destroy_process_group()


def test_replicas_gloo_world2():
    ctx = mp.get_context("spawn")
    port = _free_port()
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(2, port, out), nprocs=2, start_method="spawn", join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 2.5          # max over ranks
    assert res[0][1] != res[1][1]                  # replicas draw different inputs
    assert res[0][2] == res[1][2] == pytest.approx(2 * 160 / 2.5)


def test_single_process_identity():
    assert ranks.max_over_ranks(3.25) == 3.25
    w = synth.WORKLOADS["lm_gqa"]
    assert ranks.replica_workload(w, 0) is w
    assert ranks.replica_workload(w, 2).wid == w.wid + 2000
