"""The N > 1 path of the bench is N independent replicas: the only
collectives are barriers and the reductions of the timings.  Checked here
with two gloo ranks on CPU."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        bench.barrier(ws)
        slow = bench.max_over_ranks(1.0 + rank, ws, "cpu")          # rank 1 is the slow one
        tput = bench.replica_throughput(64, 2.0 + rank, ws, "cpu")   # 64 tokens per replica
        q.put((rank, slow, tput))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_replicas_reduce_timings():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, slow, tput in res:
        assert slow == 2.0                       # max over ranks
        assert tput == pytest.approx(128 / 3.0)  # all tokens / slowest rank's seconds


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr("sys.argv", ["bench.py", "--impl", "reference"])
    bench.main()
    assert capsys.readouterr().out == ""
