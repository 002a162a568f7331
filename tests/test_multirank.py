"""The multi-process host logic of bench.py on CPU: world_size-2 gloo ranks.

Every rank of a bench run is an independent replica of the decode (the path
has no exchange between GPUs), so the only cross-rank steps are the barrier
and the max over ranks of each timed duration; the reported value is the
whole job's rate.  These run the same helpers bench.py uses, on gloo."""
import datetime
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, durations, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        t = bench.max_over_ranks(durations[rank], dist, torch.device("cpu"))
        dist.barrier()
        out_q.put((rank, t))
    finally:
        dist.destroy_process_group()


def _run_ranks(durations):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, len(durations), port, durations, q))
             for r in range(len(durations))]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in procs:
            r, t = q.get(timeout=120)
            got[r] = t
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    return got


@pytest.mark.parametrize("durations", [[1.25, 2.5], [3.0, 0.75]])
def test_max_over_ranks_on_gloo(durations):
    got = _run_ranks(durations)
    assert got == {0: max(durations), 1: max(durations)}


def test_single_process_keeps_its_own_time():
    assert bench.max_over_ranks(1.75, None, torch.device("cpu")) == 1.75


def test_whole_job_rate_is_weak_scaling():
    # every rank decodes its own replica: N ranks in the same time do N times the work
    assert bench.whole_job_rate(1, 146.0e9, 0.16) == pytest.approx(146.0e9 / 0.16e-3)
    assert bench.whole_job_rate(8, 146.0e9, 0.16) == pytest.approx(8 * 146.0e9 / 0.16e-3)


def test_reference_arm_runs_on_rank_0_only(capsys, monkeypatch):
    """Under torchrun the oracle arm runs and prints on rank 0; other ranks exit without work."""
    monkeypatch.setenv("RANK", "1")

    class Args:
        steps, warmup, gpus = 1, 3, 2
    assert bench.run_reference(Args(), bench.W.WORKLOADS["tiny"]) is None
    assert capsys.readouterr().out == ""


def test_l2_note_is_truthful():
    assert bench.l2_note(604e6).startswith("inputs larger than L2")
    assert "fits in L2" in bench.l2_note(75.5e6)
