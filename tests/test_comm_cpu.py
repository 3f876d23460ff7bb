"""Host side of the multi-GPU form, without a GPU: the library's handle
record check, argument rejection before any device work, and the record
exchange over torch.distributed on CPU ranks (gloo, world size 2),
including a rank that never joins."""
import ctypes
import os
import socket
import struct

import pytest
import torch.multiprocessing as mp

from tensor_allreduce_residual_ar_b200 import build as arbuild

EINVAL = 1
MAGIC = 0x41524331


def record(rank, world, max_elems=1 << 20, region=123456, sms=148):
    head = struct.pack("<Iiiiqq", MAGIC, rank, world, sms, max_elems, region)
    return head + bytes(32) + bytes(range(64))


@pytest.fixture(scope="module")
def clib():
    lib = ctypes.CDLL(arbuild.build())
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    lib.ar_comm_check_handles.argtypes = [P, i32]
    lib.ar_comm_create.argtypes = [i32, i32, i64, ctypes.POINTER(ctypes.c_void_p)]
    lib.ar_comm_create_group.argtypes = [i32, i64, ctypes.POINTER(ctypes.c_void_p)]
    for name in ("ar_comm_destroy",):
        getattr(lib, name).argtypes = [P]
    lib.ar_comm_set_timeout.argtypes = [P, ctypes.c_uint64]
    lib.ar_comm_status.argtypes = [P, i32]
    lib.ar_comm_open.argtypes = [P, P]
    lib.ar_comm_handle.argtypes = [P, P]
    lib.ar_comm_test_withhold.argtypes = [P, i32]
    return lib


def test_record_check(clib):
    good = b"".join(record(r, 4) for r in range(4))
    assert clib.ar_comm_check_handles(good, 4) == 0
    swapped = record(1, 4) + record(0, 4) + record(2, 4) + record(3, 4)
    assert clib.ar_comm_check_handles(swapped, 4) == EINVAL
    assert clib.ar_comm_check_handles(b"".join(record(r, 3) for r in range(3)) + record(3, 4), 4) == EINVAL
    assert clib.ar_comm_check_handles(b"".join(record(r, 2, max_elems=8 << r) for r in range(2)), 2) == EINVAL
    assert clib.ar_comm_check_handles(b"".join(record(r, 2, sms=148 - r) for r in range(2)), 2) == EINVAL
    bad_magic = bytearray(good)
    bad_magic[128] ^= 1
    assert clib.ar_comm_check_handles(bytes(bad_magic), 4) == EINVAL
    assert clib.ar_comm_check_handles(None, 4) == EINVAL
    assert clib.ar_comm_check_handles(good, 0) == EINVAL


def test_arguments_rejected_before_device_work(clib):
    out = ctypes.c_void_p()
    assert clib.ar_comm_create(2, 2, 1 << 20, ctypes.byref(out)) == EINVAL
    assert clib.ar_comm_create(0, 0, 1 << 20, ctypes.byref(out)) == EINVAL
    assert clib.ar_comm_create(0, 17, 1 << 20, ctypes.byref(out)) == EINVAL
    assert clib.ar_comm_create(0, 2, 4, ctypes.byref(out)) == EINVAL
    assert clib.ar_comm_create(0, 2, 1 << 20, None) == EINVAL
    assert clib.ar_comm_create_group(0, 1 << 20, ctypes.byref(out)) == EINVAL
    assert clib.ar_comm_destroy(None) == 0
    assert clib.ar_comm_set_timeout(None, 10**9) == EINVAL
    assert clib.ar_comm_status(None, 1) == EINVAL
    assert clib.ar_comm_open(None, None) == EINVAL
    assert clib.ar_comm_handle(None, None) == EINVAL
    assert clib.ar_comm_test_withhold(None, 0) == EINVAL


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, mode, out):
    import datetime
    import sys
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from tensor_allreduce_residual_ar_b200 import comm as C
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    try:
        if mode == "absent" and rank == 1:
            out.put((rank, "left"))
            return
        rec = bytes([rank]) * C.HANDLE_BYTES
        try:
            blob = C.exchange_records(rec, None)
        except Exception as e:          # the missing rank shows as a failure, not a hang
            out.put((rank, "error:" + type(e).__name__))
            return
        out.put((rank, blob))
    finally:
        if not (mode == "absent"):
            dist.destroy_process_group()


def _marker_worker(rank, world, port, out):
    import datetime
    import sys
    import types
    import torch
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from tensor_allreduce_residual_ar_b200 import comm as C
    from tensor_allreduce_residual_ar_b200 import fx_patterns as FX
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        # the marker needs only the communicator's world size and group
        C._REGISTRY[5] = types.SimpleNamespace(world=world, group=None)
        x = torch.full((3, 8), float(rank + 1))
        y = FX.tp_all_reduce_reference(x, 5)
        out.put((rank, (float(x[0, 0]), y.tolist())))
    finally:
        dist.destroy_process_group()


def test_tensor_parallel_marker_all_reduces_over_the_group():
    """The unfused program's all-reduce marker sums the ranks' partials
    through torch.distributed (gloo, world size 2) and leaves its input
    untouched."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_marker_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    for r in range(world):
        x0, y = res[r]
        assert x0 == r + 1
        assert y == [[3.0] * 8] * 3


def _run(mode):
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, mode, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    return res


def test_records_gathered_in_rank_order():
    res = _run("ok")
    want = bytes([0]) * 128 + bytes([1]) * 128
    assert res[0] == want and res[1] == want


def test_rank_that_never_joins_is_an_error_not_a_hang():
    res = _run("absent")
    assert res[1] == "left"
    assert isinstance(res[0], str) and res[0].startswith("error:")


def test_oneshot_limit_from_measured_rows():
    from tensor_allreduce_residual_ar_b200.comm import oneshot_limit
    rows = [[1, 5.0, 7.0], [8, 6.0, 7.5], [64, 9.0, 8.0], [512, 30.0, 20.0]]
    assert oneshot_limit(rows, 8192) == 8 * 8192 * 2
    assert oneshot_limit([[1, 9.0, 8.0], [8, 5.0, 7.0]], 4096) == 0      # first loss ends it
    assert oneshot_limit([[1, 5.0, 5.0], [2, 5.0, 6.0]], 1024) == 2 * 1024 * 2   # ties go one-shot
