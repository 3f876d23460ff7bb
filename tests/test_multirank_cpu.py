"""The bench's multi-rank plumbing on CPU ranks (gloo, world size 2): the
timing reduction takes the max over ranks, the job value counts every
rank's bytes, and barriers pair up."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import sys
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        assert bench.dist_env() == (world, rank, rank)
        bench.barrier()
        m = bench.max_over_ranks(1.5 + rank)          # rank 1 is the slow one
        v = bench.weak_scaling_value(10**9, world, 4, m)
        bench.barrier()
        out.put((rank, m, v))
    finally:
        dist.destroy_process_group()


def test_two_cpu_ranks_max_timing_and_weak_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, m, v in res:
        assert m == 2.5
        assert v == pytest.approx(2 * 1e9 * 4 / 2.5 / 1e9)


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.weak_scaling_value(2 * 10**9, 1, 2, 4.0) == 1.0


def test_rotation_sets_exceed_twice_l2():
    import bench
    for step in (131072, 9_191_424, 47_742_976, 300_000_000, 700_000_000):
        R = bench.rotation_sets(step)
        assert R == 1 and step >= 4 * bench.L2_BYTES or (R - 1) * step > 2 * bench.L2_BYTES


def test_step_bytes_match_the_workload_formulas():
    import bench
    decode = sum(bench.call_bytes(c) for c in bench.workload_calls("decode"))
    assert decode == 2 * sum(114688 * T + 16384 for T in (1, 2, 4, 8, 16, 32, 64, 80))
    (tiny,) = [bench.call_bytes(c) for c in bench.workload_calls("tiny")]
    assert tiny == 663552
    (pre,) = [bench.call_bytes(c) for c in bench.workload_calls("prefill")]
    assert pre == 671096832
    fp8 = [bench.call_bytes(c) for c in bench.workload_calls("fp8")]
    assert fp8[0] == 76960 + 10240 and fp8[-1] == 32768 * 76960 + 10240
    qk = [bench.call_bytes(c) for c in bench.workload_calls("qk")]
    assert qk == [28672 * T + 14336 for T in (1, 64, 2048)]
