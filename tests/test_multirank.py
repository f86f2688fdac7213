"""The multi-rank plumbing of bench.py on CPU with gloo, world size 2.

Under torchrun every rank decodes its own batch (weak scaling, no collective on
the data path); the only cross-rank operation is the max of the timed region.
These tests run that host logic in two gloo processes."""
import os
import socket
import sys

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from compressed_kv_cache_gva_b200.synth import make_decode_inputs
        r, w, loc = bench.dist_env()
        wl = bench.rank_workload("tiny_fp32_t64", r)
        di = make_decode_inputs(wl)
        checksum = float(di.V.double().sum())
        ms_max = bench.reduce_max(1.5 + r)           # rank r "took" 1.5 + r ms
        value = bench.job_value(1000, 10, w, ms_max)
        ref = None
        if r != 0:
            class A:                                 # the reference arm's arguments
                workload, steps, warmup = "tiny_fp32_t64", 1, 0
            ref = bench.run_reference(A, r, w)
        gathered = [None] * w
        dist.all_gather_object(gathered, (r, w, loc, wl.seed, checksum, ms_max, value, ref))
        if r == 0:
            q.put(gathered)
    finally:
        dist.destroy_process_group()


def test_weak_scaling_plumbing_world_size_2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out = sorted(out)
    (r0, w0, l0, s0, c0, m0, v0, ref0), (r1, w1, l1, s1, c1, m1, v1, ref1) = out
    assert (r0, r1, w0, w1, l0, l1) == (0, 1, 2, 2, 0, 1)
    # each rank has its own batch: different seeds, different data
    assert s0 != s1 and c0 != c1
    # the timed region is the slowest rank's, on every rank
    assert m0 == m1 == 2.5
    # whole-job value: both ranks' bytes over the slowest time
    assert np.isclose(v0, 2 * 10 * 1000 / 2.5e-3 / 1e9) and v0 == v1
    # the reference arm runs on rank 0 only; other ranks return without work
    assert ref1 is None
