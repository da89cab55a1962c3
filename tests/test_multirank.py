"""The replicas-only multi-GPU plumbing of bench.py (one process per GPU,
every rank decoding its own batch, no collective on the data path), run as two
gloo ranks on the host: the barrier, the max over ranks that timings take, the
whole-job throughput, and the reference arm, which only rank 0 runs."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import argparse
    import torch.distributed as dist
    import bench
    try:
        r, w, _ = bench.dist_setup(argparse.Namespace(gpus=world))
        assert (r, w) == (rank, world) and dist.get_backend() == "gloo"
        bench.barrier(w)
        ms = bench.max_over_ranks(1.0 + rank, w)          # rank 1 is the slow one
        gbs = bench.whole_job_gbs(w, 1e9, ms)
        # only rank 0 runs the reference arm; the others return at once
        ref = bench.run_reference(argparse.Namespace(steps=1, warmup=0, workload="tiny")) \
            if rank != 0 else "skipped"
        bench.barrier(w)
        q.put((rank, ms, gbs, ref))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_gloo_ranks():
    if torch.cuda.is_available():
        pytest.skip("host-only test of the multi-rank plumbing")
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, ms, gbs, ref in got:
        assert ms == 2.0                                   # the slower rank's time on both
        assert gbs == pytest.approx(2 * 1e9 / 2e-3 / 1e9)  # both ranks' bytes / that time
    assert got[1][3] is None                               # rank 1 did no reference work
