"""The multi-GPU path of bench.py is replicas only: each rank streams its own
synthetic inputs with no collective on the data path, and the ranks meet
only to time (a barrier around the timed region, the maximum of the device
times over ranks). This runs that rank logic with world size 2 on the gloo
backend, on CPU."""
import datetime
import os
import socket

import torch.multiprocessing as mp

import swa_workloads as W


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    import torch.distributed as tdist

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    tdist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # each rank's own "device time"; every rank takes part in the reduction
        t_max = bench.max_over_ranks(10.0 + 5.0 * rank, True, device="cpu")
        tdist.barrier()
        seeds = [bench.layer_seed_base(W.STREAM, l, bench.replica_seed_offset(rank)) for l in range(W.STREAM.layers)]
        ref = bench.run_reference(None, rank, world) if rank != 0 else "skipped"
        out.put((rank, t_max, seeds, ref))
    finally:
        tdist.destroy_process_group()


def test_replicas_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(2):
            rank, t_max, seeds, ref = q.get(timeout=120)
            got[rank] = (t_max, seeds, ref)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    # the slowest rank's time, seen by both
    assert got[0][0] == got[1][0] == 15.0
    # independent streams: no seed shared between the ranks' layers
    assert len(set(got[0][1]) | set(got[1][1])) == 2 * W.STREAM.layers
    # the reference arm runs on rank 0 alone; other ranks return nothing
    assert got[1][2] is None


def test_single_process_max_is_identity():
    import bench
    assert bench.max_over_ranks(3.25, False) == 3.25

