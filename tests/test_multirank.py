"""The multi-rank path of the benchmark on CPU (gloo, world size 2).

On N GPUs every rank runs its own sequences against replicated weights; the
step has no collective.  The job time is the slowest rank's (max over ranks)
and the job throughput counts every rank's revealed tokens.  These tests run
two gloo ranks as processes and check exactly that host-side logic.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    import dllm_synth as SY
    r, w, l = bench.dist_env()
    assert (r, w, l) == (rank, world, rank)
    # the job time is the slowest rank's
    t = bench.max_over_ranks(10.0 + 5.0 * rank, world)
    bench.barrier(world)
    # each rank draws its own sequences; weights are identical on every rank
    shape = SY.with_(SY.TINY, batch=2)
    tok = bench.rank_inputs(shape, rank, device="cpu")
    W = SY.model_weights(shape, seed=0, device="cpu")
    wsum = torch.tensor([float(W["layers"][0]["wq"].double().sum())], dtype=torch.float64)
    tsum = torch.tensor([float(tok.double().sum())], dtype=torch.float64)
    ws = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
    ts = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
    dist.all_gather(ws, wsum)
    dist.all_gather(ts, tsum)
    value = bench.job_tokens_per_s(world, shape.batch * shape.n_unmask, t)
    out[rank] = (t, [x.item() for x in ws], [x.item() for x in ts], value)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_sharded_inputs():
    port = _free_port()
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    for rank in range(world):
        t, wsums, tsums, value = res[rank]
        assert t == 15.0                           # max over ranks
        assert wsums[0] == wsums[1]                # replicated weights
        assert tsums[0] != tsums[1]                # different sequences per rank
        assert value == pytest.approx(world * 2 * 8 * 1000.0 / 15.0)
