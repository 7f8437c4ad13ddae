"""The multi-GPU host logic of bench.py on the CPU, as world_size-2 gloo ranks.

The path shards by sequence: every rank runs its own prefill with no data-path
collective, and the only cross-rank steps are a barrier and a MAX all-reduce of
the step time.  These tests run exactly those steps (bench.reduce_max,
bench.job_throughput) on gloo, check that the reference arm does no work on
ranks other than 0, and that a rank which leaves before a collective makes the
other rank's collective fail with an error instead of waiting for ever.
"""
import datetime
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port, timeout_s):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=timeout_s))


def _timing_worker(rank, world, port, q):
    _init(rank, world, port, 60)
    import bench
    try:
        ms = bench.reduce_max(10.0 + 5.0 * rank, world, "cpu")   # rank 1 is the slow one
        ms2 = bench.reduce_max(3.0 - rank, world, "cpu")         # a second step, same order
        value = bench.job_throughput(200000, world, ms)
        dist.barrier()
        q.put((rank, ms, ms2, value))
    finally:
        dist.destroy_process_group()


def test_step_time_is_the_max_over_ranks_and_throughput_is_whole_job():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_timing_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, *_ in out] == [0, 1]
    for _, ms, ms2, value in out:
        assert ms == 15.0 and ms2 == 3.0
        assert value == pytest.approx(2 * 200000 / 0.015)   # both ranks' tokens / slowest rank


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert not dist.is_initialized()
    assert bench.reduce_max(7.5, 1, "cpu") == 7.5
    assert bench.job_throughput(1000, 1, 2.0) == pytest.approx(500000.0)


def _leaver_worker(rank, world, port, q):
    _init(rank, world, port, 10)
    import bench
    if rank == 1:
        # leaves between steps: nothing in flight, no collective joined
        _put_and_exit(q, (rank, "left"))
    try:
        bench.reduce_max(1.0, world, "cpu")
        msg = "no error"
    except Exception as e:  # the collective must end with an error
        msg = "error: %s" % type(e).__name__
    _put_and_exit(q, (rank, msg))


def _put_and_exit(q, item):
    q.put(item)
    q.close()
    q.join_thread()  # the queue's feeder thread must flush before the process ends
    os._exit(0)


def test_a_rank_that_leaves_makes_the_collective_fail_not_hang():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_leaver_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert res[1] == "left"
    assert res[0].startswith("error"), res[0]


def test_reference_arm_does_no_work_on_other_ranks():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


# ------------------------------------------------------------------ sharding one prefill
def test_zigzag_plan_covers_every_row_once_and_balances_the_causal_work():
    sys.path.insert(0, ROOT)
    from sparse_attention_indexer_sum_b200.sharding import causal_pairs, zigzag_row_ranges
    for L, W in ((200000, 8), (200000, 2), (1000, 3), (7, 4), (5, 1)):
        covered = []
        work = []
        for r in range(W):
            rr = zigzag_row_ranges(L, W, r)
            covered += [t for r0, n in rr for t in range(r0, r0 + n)]
            work.append(sum(causal_pairs(r0, n) for r0, n in rr))
        assert sorted(covered) == list(range(L))
        assert sum(work) == L * (L + 1) // 2
        if L >= 1000:
            assert max(work) / min(work) < 1.01, (L, W, work)
    # contiguous ranges would not balance: the last of 8 ranks has 15x the first's work
    assert causal_pairs(175000, 25000) > 14 * causal_pairs(0, 25000)
    with pytest.raises(ValueError):
        zigzag_row_ranges(10, 2, 2)


def _plan_worker(rank, world, port, q):
    _init(rank, world, port, 60)
    import torch
    from sparse_attention_indexer_sum_b200.sharding import zigzag_row_ranges
    try:
        mine = torch.tensor(zigzag_row_ranges(200000, world, rank), dtype=torch.int64)
        got = [torch.empty_like(mine) for _ in range(world)]
        dist.all_gather(got, mine)       # every rank sees the whole plan
        q.put((rank, [t.tolist() for t in got]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_a_plan_that_tiles_the_rows():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_plan_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out[0] == out[1]
    rows = sorted(t for rr in out[0] for r0, n in rr for t in (r0, r0 + n))
    assert rows == [0, 50000, 50000, 100000, 100000, 150000, 150000, 200000]
