"""The multi-rank host logic of bench.py on CPU: two gloo ranks set up the group the way
bench.py does under torchrun, take the max over ranks of their timings, pass the barrier,
and draw different batches (weak scaling)."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    from state_space_sequence_chunked_b200 import inputs

    got_ws, got_rank, _ = bench.dist_setup("gloo")
    timing = 1.0 + rank  # this rank's "device time"
    bench.barrier(got_ws)
    m = bench.reduce_max(timing, got_ws, device="cpu")
    wl = inputs.WORKLOADS["tiny_fp32"]
    x = inputs.draw(wl, seed=bench.rank_seed(wl, got_rank))["x"].bits
    out.put((got_rank, got_ws, m, float(x.ravel()[0])))
    bench.barrier(got_ws)
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_draw_their_own_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1] and all(r[1] == 2 for r in res)
    assert all(r[2] == pytest.approx(2.0) for r in res)  # max over ranks, seen by both
    assert res[0][3] != res[1][3]                          # different batches per rank


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench

    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        os.environ.pop(k, None)
    assert bench.dist_setup("gloo") == (1, 0, 0)
    assert bench.reduce_max(3.5, 1) == 3.5
