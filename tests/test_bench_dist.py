"""The benchmark's multi-rank path on CPU: two real processes joined by a gloo
process group, as torchrun starts them (RANK / WORLD_SIZE / LOCAL_RANK /
MASTER_* in the environment).  The layers are independent replicas, so the
only collective is the max over ranks of the measured times; these tests
check that every rank ends with the slowest rank's time, that rank 0 scales
the throughput by the number of replicas, and that the reference arm does no
work on the other ranks."""
import multiprocessing as mp
import os
import socket
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    try:
        sys.path.insert(0, ROOT)
        os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                           "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
        import datetime

        import torch
        import torch.distributed as dist

        import bench
        args = types.SimpleNamespace(gpus=world, steps=4, warmup=3)
        w, r, lr = bench.dist_setup(args)
        dist.init_process_group("gloo", rank=r, world_size=w,
                                timeout=datetime.timedelta(seconds=60))
        cpu = torch.device("cpu")
        # per-rank "timed region" and "e2e" times: rank r is slower on one,
        # faster on the other, so a max taken over the wrong axis shows
        mine = [10.0 + 5.0 * r, 7.0 - 2.0 * r]
        got = bench.max_over_ranks(dist, mine, cpu)
        # a second collective in the same order on every rank
        got2 = bench.max_over_ranks(dist, [float(r)], cpu)
        dist.barrier()
        dist.destroy_process_group()
        ref = bench.time_reference(args) if r != 0 else "skipped"
        q.put((r, {"got": got, "got2": got2, "world": w, "local": lr,
                   "ref": ref, "oracle_loaded": "oracle.oracle" in sys.modules}))
    except BaseException as e:  # report instead of hanging the parent
        q.put((rank, {"error": repr(e)}))


def _run(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    try:
        for _ in range(world):
            r, res = q.get(timeout=180)
            out[r] = res
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
    return out


def test_two_rank_max_over_ranks_and_reference_arm():
    out = _run(2)
    for r in range(2):
        assert "error" not in out[r], out[r]
        assert out[r]["world"] == 2 and out[r]["local"] == r
        # both ranks hold the slowest rank's time for each quantity
        assert out[r]["got"] == [15.0, 7.0]
        assert out[r]["got2"] == [1.0]
    # the reference arm runs on rank 0 alone; rank 1 returns without work
    # and without loading the oracle
    assert out[1]["ref"] is None
    assert out[1]["oracle_loaded"] is False


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(None, [3.5, 2], None) == [3.5, 2.0]


def test_replica_throughput_scales_with_world():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.replica_gbs(1, 4096 * 4096 * 2, 0.04)
    assert one == pytest.approx(4096 * 4096 * 2 / 0.04e-3 / 1e9)
    # N replicas each moving the same bytes, timed by the slowest rank
    assert bench.replica_gbs(8, 4096 * 4096 * 2, 0.04) == pytest.approx(8 * one)
    assert bench.replica_gbs(2, 4096 * 4096 * 2, 0.08) == pytest.approx(one)


def test_gpus_flag_must_match_world(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "4")
    monkeypatch.setenv("RANK", "2")
    monkeypatch.setenv("LOCAL_RANK", "2")
    assert bench.dist_setup(types.SimpleNamespace(gpus=4)) == (4, 2, 2)
    with pytest.raises(SystemExit):
        bench.dist_setup(types.SimpleNamespace(gpus=2))
