"""The N > 1 host path of bench.py on CPU: two gloo ranks on 127.0.0.1.

bench.py runs one independent replica per GPU; the only collectives are the
barriers around the timed region and the max over ranks of the device time.
These run here with the gloo backend (no GPU): both ranks must agree on the
maximum, and a rank count that does not match --gpus must stop the run.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    r, w, local, pg = bench.dist_setup(world)
    try:
        bench.barrier(pg)
        # each rank's "device time" differs; every rank must see the largest
        got = bench.max_over_ranks(pg, 10.0 + 7.5 * rank)
        bench.barrier(pg)
        out.put((r, w, local, got))
    finally:
        pg.destroy_process_group()


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="the gloo path is the CPU one; with a GPU, bench.py uses NCCL, one rank per GPU")
def test_two_ranks_take_the_max_over_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    results = [out.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    results.sort()
    assert [r[:3] for r in results] == [(0, 2, 0), (1, 2, 1)]
    assert all(r[3] == 17.5 for r in results)


def test_rank_count_must_match_gpus(monkeypatch):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("RANK", "0")
    with pytest.raises(SystemExit):
        bench.dist_setup(2)


def test_single_rank_needs_no_process_group(monkeypatch):
    import bench
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.delenv("RANK", raising=False)
    rank, world, local, pg = bench.dist_setup(1)
    assert (rank, world, pg) == (0, 1, None)
    assert bench.max_over_ranks(pg, 3.25) == 3.25
