"""Host logic of the N-replica benchmark on CPU: two `gloo` ranks take the
max of their step times and report the whole-job rate over the slowest
rank (no GPU; the same helpers run over NCCL on GPUs)."""
import datetime
import os
import socket

import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        step_ms = [3.0, 5.0][rank]   # rank 1 is the slow one
        e2e_ms = [2.5, 1.5][rank]    # rank 0 is the slow one here
        m = bench.max_over_ranks(step_ms)
        e = bench.max_over_ranks(e2e_ms)
        q.put((rank, m, e, bench.job_rate(world, 1e9, m), bench.job_rate(world, 64, m)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_single_process():
    assert bench.max_over_ranks(4.25) == 4.25
    assert bench.job_rate(1, 1e9, 4.0) == 1e9 / 4e-3


def test_two_gloo_ranks_take_the_slowest_step():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = sorted(q.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.terminate()
    assert [r[0] for r in res] == [0, 1]
    for _, m, e, rate, tok in res:
        assert m == 5.0 and e == 2.5          # every rank sees the same maxima
        assert rate == 2 * 1e9 / 5e-3         # both ranks' bytes over the slowest time
        assert tok == 2 * 64 / 5e-3
    assert all(p.exitcode == 0 for p in procs)
