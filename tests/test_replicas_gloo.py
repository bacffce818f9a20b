"""The multi-GPU path is independent replicas; its only cross-rank steps are a
barrier and a max-reduction of the ranks' times.  Checked here with two gloo
ranks on the CPU."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from paged_fp8_gated_b200 import replicas, workloads as W


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    r, w, lr = replicas.rank_info()
    replicas.barrier(w)
    local_time = 1.0 + r          # rank 1 is the slow one
    slowest = replicas.max_over_ranks(local_time, w)
    rate = replicas.job_rate(100.0, w, slowest)
    spec = W.Spec("rep", B=2, ctx=50, seed=replicas.replica_seed(7, r))
    qkv_sum = float(W.make_inputs(spec)["qkv"].float().sum())
    out[rank] = (r, w, lr, slowest, rate, qkv_sum)
    replicas.barrier(w)
    dist.destroy_process_group()


def test_two_gloo_ranks_reduce_to_the_slowest():
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0][:3] == (0, 2, 0) and res[1][:3] == (1, 2, 1)
    for r in range(2):
        assert res[r][3] == 2.0                  # max over ranks
        assert res[r][4] == pytest.approx(100.0)  # 2 ranks x 100 units / 2 s
    assert res[0][5] != res[1][5]                # replicas draw different inputs


def test_single_process_defaults():
    assert replicas.max_over_ranks(3.5, 1) == 3.5
    assert replicas.job_rate(10.0, 1, 2.0) == 5.0
