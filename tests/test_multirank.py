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
        from compressed_kv_cache_gva_b200 import gva, seqsplit
        from compressed_kv_cache_gva_b200.synth import (WORKLOADS, make_append_inputs,
                                                        make_decode_inputs)
        wl = WORKLOADS["350m_b8_t4096"]
        L = np.array([5, 64, 1, 33, 0])
        di = make_decode_inputs(wl, extra_slots=1, lengths=L)
        slots = (di.seq_offset.numpy() + L).astype(np.int32)
        ap = make_append_inputs(wl, slots, L.astype(np.int32))
        V_r, K_r, off_r, len_r, app_r, start = seqsplit.shard_step_inputs(
            di.V, di.k_rope, di.seq_offset, L, (ap.v_new, ap.kpe_new, ap.slot, ap.pos), world, rank)
        # the product's exchange on host buffers: each rank's part is a recognisable
        # function of its rank, gathered into every rank's outs / lses in rank order
        sh = gva.make_shape(len(L), wl.H, wl.G, wl.d_h, wl.d_n, wl.d_r)
        m = seqsplit.SequenceSplitMerge(sh, world, "cpu")
        m.out_part.copy_(torch.arange(m.out_part.numel(), dtype=torch.float32).view_as(m.out_part)
                         + 1000 * rank)
        m.lse_part.fill_(-float(rank))
        m.exchange()
        q.put((rank, start, len_r.numpy(), off_r.numpy(), V_r.float().numpy(), K_r.float().numpy(),
               [t.float().numpy() if t.is_floating_point() else t.numpy() for t in app_r],
               m.outs.numpy(), m.lses.numpy()))
    finally:
        dist.destroy_process_group()


def test_sequence_split_shards_and_exchange_world_size_2():
    """The sequence split's host logic on two gloo ranks: shard_step_inputs cuts
    every sequence's step (history + the appended token) into two parts that
    partition its positions, only the rank holding position L appends the new
    token (at the right slot of its shard), and SequenceSplitMerge.exchange gives
    every rank all parts in rank order.  (The merge arithmetic and the per-rank
    decodes run on the GPU: tests/test_gpu_seqsplit_ranks.py.)"""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=180) for _ in range(2)], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    sys.path.insert(0, ROOT)
    from compressed_kv_cache_gva_b200.synth import (WORKLOADS, make_append_inputs,
                                                    make_decode_inputs)
    wl = WORKLOADS["350m_b8_t4096"]
    L = np.array([5, 64, 1, 33, 0])
    di = make_decode_inputs(wl, extra_slots=1, lengths=L)
    ap = make_append_inputs(wl, (di.seq_offset.numpy() + L).astype(np.int32), L.astype(np.int32))
    V = di.V.float().numpy()
    KR = di.k_rope.float().numpy()
    off = di.seq_offset.numpy()
    owners = np.zeros(len(L), dtype=int)
    for rank, start, cnt, off_r, V_r, K_r, (v_new, kpe_new, slot_r, pos_r), outs, lses in res:
        # parts of the step's L + 1 positions: rank 0 from 0, rank 1 from rank 0's end
        assert np.array_equal(start, ((L + 1) * rank) // 2)
        for b in range(len(L)):
            rows = np.arange(off[b] + start[b], off[b] + start[b] + cnt[b])
            assert np.array_equal(V_r[off_r[b]:off_r[b] + cnt[b]], V[rows])
            assert np.array_equal(K_r[off_r[b]:off_r[b] + cnt[b]], KR[rows])
        own = (L >= start) & (L < start + cnt)
        owners += own
        assert np.array_equal(slot_r, (off_r + L - start)[own])
        assert np.array_equal(pos_r, L[own])
        assert np.array_equal(v_new, ap.v_new.float().numpy()[own])
        assert np.array_equal(kpe_new, ap.kpe_new.float().numpy()[own])
        # every rank holds every part, in rank order
        part = np.arange(outs[0].size, dtype=np.float32).reshape(outs[0].shape)
        assert np.array_equal(outs[0], part) and np.array_equal(outs[1], part + 1000)
        assert np.all(lses[0] == 0) and np.all(lses[1] == -1)
    assert np.all(owners == 1)               # each new token is appended exactly once
    total = sum(r[2] for r in res)
    assert np.array_equal(total, L + 1)
