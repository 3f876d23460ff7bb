"""The rank form's handle path on a real GPU, without any cross-rank kernel:
two processes on one GPU each create a communicator, exchange the 128-byte
handle records over gloo, check them and map each other's region through
CUDA IPC (ar_comm_open), then meet and free (ar_comm_destroy).

No exchange kernel runs here.  Ranks whose kernels wait on one another are
never run as separate processes on one GPU: nothing guarantees that their
kernels are resident at the same time.  The exchange protocol itself is
covered by the one-launch groups of test_comm_gpu.py, which run every rank's
part in one cooperative launch."""
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
    import torch
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from tensor_allreduce_residual_ar_b200 import comm as C
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        c = C.Comm(1 << 16)              # create, handle, exchange, check, open
        algo = c.algo(1, 4096)           # host-side query of the opened communicator
        dist.barrier()                   # both ranks have mapped each other's region
        c.close()                        # synchronise, unmap the peer, free its own region
        dist.barrier()
        out.put((rank, f"ok:{algo}:{c.world}"))
    except Exception as e:               # reported to the test, never hidden
        out.put((rank, f"error:{type(e).__name__}:{str(e)[:200]}"))
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
def test_two_processes_map_each_others_regions(lib):
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        res = dict(q.get(timeout=300) for _ in range(world))
    finally:
        for p in procs:
            p.join(timeout=120)
            if p.is_alive():
                p.kill()
    assert res == {0: "ok:oneshot:2", 1: "ok:oneshot:2"}, res
