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


def _split_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from compressed_kv_cache_gva_b200 import seqsplit
        from compressed_kv_cache_gva_b200.synth import WORKLOADS, as_f64, make_decode_inputs
        wl = WORKLOADS["350m_b8_t4096"]
        L = np.array([5, 64, 1, 33])
        di = make_decode_inputs(wl, lengths=L)
        V_r, K_r, off_r, len_r, start = seqsplit.shard_cache(di.V, di.k_rope, di.seq_offset,
                                                             di.seq_len, world, rank)
        out_r, lse_r = oracle.gva_decode(as_f64(di.q), as_f64(di.M), di.q_pos.numpy(), as_f64(V_r),
                                         as_f64(K_r), off_r.numpy(), len_r.numpy(), wl.d_n,
                                         wl.d_r, wl.rope_base)
        outs = [torch.zeros(out_r.shape, dtype=torch.float64) for _ in range(world)]
        lses = [torch.zeros(lse_r.shape, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(outs, torch.from_numpy(out_r))
        dist.all_gather(lses, torch.from_numpy(lse_r))
        if rank == 0:
            q.put((np.stack([o.numpy() for o in outs]), np.stack([l.numpy() for l in lses])))
    finally:
        dist.destroy_process_group()


def test_sequence_split_exchange_world_size_2():
    """Each rank decodes its part of every sequence (oracle on CPU), the parts
    are all-gathered in rank order and merged by the softmax decomposition; the
    result equals the oracle on the whole cache."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    outs, lses = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    sys.path.insert(0, ROOT)
    import oracle
    from compressed_kv_cache_gva_b200 import seqsplit
    from compressed_kv_cache_gva_b200.synth import WORKLOADS, as_f64, make_decode_inputs
    wl = WORKLOADS["350m_b8_t4096"]
    L = np.array([5, 64, 1, 33])
    di = make_decode_inputs(wl, lengths=L)
    ref, ref_lse = oracle.gva_decode(as_f64(di.q), as_f64(di.M), di.q_pos.numpy(), as_f64(di.V),
                                     as_f64(di.k_rope), di.seq_offset.numpy(), L, wl.d_n, wl.d_r,
                                     wl.rope_base)
    # the parts partition the positions
    s0, c0 = seqsplit.shard_ranges(L, 2, 0)
    s1, c1 = seqsplit.shard_ranges(L, 2, 1)
    assert np.array_equal(s0, 0 * L) and np.array_equal(s1, c0) and np.array_equal(c0 + c1, L)
    mx = np.max(lses, axis=0)
    w = np.where(np.isneginf(lses), 0.0, np.exp(lses - mx))
    merged = (w[..., None] * np.nan_to_num(outs)).sum(0) / w.sum(0)[..., None]
    assert np.max(np.abs(merged - ref)) < 1e-12
    assert np.max(np.abs(mx + np.log(w.sum(0)) - ref_lse)) < 1e-12
