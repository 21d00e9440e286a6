"""The multi-rank host logic of bench.py on CPU: two processes over gloo (127.0.0.1).
Each rank is an independent replica; the only cross-rank steps are the barrier, the
element-wise maximum of the durations, and rank 0 alone printing (and, for the reference
arm, alone doing the work)."""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import datetime
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        # rank r took (1 + r) ms for the step and 10 - r ms for the decode part
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 3.5], torch.device("cpu"), world)
        torch.distributed.barrier()

        class Args:
            steps, warmup = 1, 0
        ref = bench.run_reference(Args, rank, world) if rank != 0 else "skipped"
        q.put((rank, got, ref))
    finally:
        torch.distributed.destroy_process_group()


def test_two_ranks_agree_on_the_max_and_only_rank0_reports():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict()
    for _ in range(world):
        rank, got, ref = q.get(timeout=120)
        res[rank] = (got, ref)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(world):
        assert res[rank][0] == [2.0, 10.0, 3.5]
    assert res[1][1] is None   # the reference arm does no work on rank 1


def test_whole_job_rate_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    # two replicas, each 4e12 FLOP in at most 2 s: 4 TFLOP/s for the job
    assert bench.whole_job_rate(4e12, 2, 2.0) == pytest.approx(4e12)
    assert bench.max_over_ranks([1.5, 2.5], torch.device("cpu"), 1) == [1.5, 2.5]


def test_traffic_staleness_ignores_comments_only():
    sys.path.insert(0, ROOT)
    import bench
    src = "int a = 1;  // one\n/* block\n comment */\nint b = 2;\n"
    assert bench._code_only(src) == bench._code_only("int a = 1;\n// other words\nint b = 2;  /* x */\n")
    assert bench._code_only(src) != bench._code_only("int a = 2;\nint b = 2;\n")


def test_paged_layout_maps_every_row_once():
    """The bench's paged copy: row r of sequence b sits at row r % P of page table[b][r // P],
    every cache row appears exactly once, and the rest of each last page is empty."""
    sys.path.insert(0, ROOT)
    import bench
    lens, P = [5, 64, 65, 1, 130], 16
    offs = [0]
    for n in lens:
        offs.append(offs[-1] + n)
    table, src = bench.paged_layout(lens, offs, P)
    for b, n in enumerate(lens):
        for r in range(n):
            assert int(src[int(table[b, r // P]) * P + r % P]) == offs[b] + r
    used = src[src >= 0]
    assert sorted(used.tolist()) == list(range(offs[-1]))
    assert (table[0, :1] >= 0).all() and int(table[0, 1]) == -1
