"""Host logic of the multi-GPU (weak scaling over tokens) benchmark, run as two
gloo ranks on the CPU: the job time is the max over ranks, the value counts
every rank's FLOPs, and ranks draw different tokens against the same weights."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import sys
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from synth import WORKLOADS, make_inputs
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    local_ms = 10.0 + 5.0 * rank
    m = bench.max_over_ranks(local_ms, world, "cpu")
    layer = WORKLOADS["tiny_fp8"].layers[0]
    inp = make_inputs(layer, seed=bench.rank_seed(rank), w_seed=0)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, m, inp["x"][:2, :8].copy(), inp["w"][:2, :8].copy()))


@pytest.mark.parametrize("world", [2])
def test_gloo_max_over_ranks_and_rank_inputs(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort(key=lambda t: t[0])
    assert all(r[1] == 15.0 for r in res)                 # every rank sees the slowest time
    assert not np.array_equal(res[0][2], res[1][2])        # own tokens per rank
    assert np.array_equal(res[0][3], res[1][3])            # same weights on every rank


def test_weak_scaling_value():
    import bench
    # 2 ranks x 10 steps x 1e12 FLOP in 100 ms (slowest rank) = 200 TFLOP/s
    assert bench.weak_scaling_tflops(1e12, 2, 10, 100.0) == pytest.approx(200.0)
    assert bench.max_over_ranks(3.5, 1) == 3.5
