"""Failure of a rank between expert-parallel steps, on the CPU (gloo, two ranks, no GPU).

Each step of the expert-parallel block ends with the reduce-scatter of the partial routed
sums (sparse_moe_ffn_gemv_b200.ep.reduce_scatter_routed). A rank that leaves between steps
(here: raises before its second step) must not leave the other rank waiting for good: its
next collective ends with an error within the process group's timeout, which the host
reports. The failure is made on the host; nothing faults or hangs a device.
"""
import multiprocessing as mp
import os
import socket
import sys
import time

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from sparse_moe_ffn_gemv_b200 import ep as EP
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    rows, K = EP.shard_rows(21, world), 16
    partial = torch.full((rows * world, K), float(rank + 1), dtype=torch.float32)
    shard = EP.reduce_scatter_routed(partial, world)  # step 1: both ranks take part
    ok1 = bool(torch.all(shard == sum(r + 1 for r in range(world))))
    if rank == 1:
        q.put((rank, ok1, "left"))
        q.close()
        q.join_thread()  # the message is out before the process goes
        os._exit(3)  # leaves between steps, with nothing of its own in flight
    t0 = time.time()
    try:
        EP.reduce_scatter_routed(partial, world)  # step 2: the peer never joins
        q.put((rank, ok1, "no error"))
    except Exception as exc:  # the collective reports the missing rank
        q.put((rank, ok1, f"error after {time.time() - t0:.1f} s: {type(exc).__name__}"))
    q.close()
    q.join_thread()
    os._exit(0)


@pytest.mark.timeout(120)
def test_a_rank_that_leaves_between_steps_ends_the_others_next_collective_with_an_error():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict((r, (ok, msg)) for r, ok, msg in (q.get(timeout=90) for _ in procs))
    for p in procs:
        p.join(timeout=30)
    assert out[0][0] and out[1][0]                  # the first step summed correctly
    assert out[1][1] == "left" and procs[1].exitcode == 3
    assert out[0][1].startswith("error after"), out[0][1]
    assert float(out[0][1].split()[2]) < 30.0       # within the process group's timeout bound
