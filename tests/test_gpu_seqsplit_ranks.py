"""The sequence split across ranks, end to end through the product's code, on
one GPU: two gloo processes each take their part of every sequence
(seqsplit.shard_step_inputs, as bench.py --split sequence does), run
gva_decode_step on it (the rank holding position L appends the new token), and
SequenceSplitMerge.merge all-gathers the parts and merges them with
gva_merge_states.  The merged output must equal the float64 oracle's append +
decode on the whole cache.  The ranks' kernels never wait on one another: the
only cross-rank step is the host-side gloo all-gather between launches."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu

CASES = [("350m_b8_t4096", [4096, 77, 1, 0, 300]), ("d128_b1_t131072", [3001])]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, name, lengths, q):
    sys.path.insert(0, ROOT)
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        from compressed_kv_cache_gva_b200 import gva, seqsplit
        from compressed_kv_cache_gva_b200.synth import (WORKLOADS, make_append_inputs,
                                                        make_decode_inputs)
        torch.cuda.set_device(0)
        wl = WORKLOADS[name]
        L = np.array(lengths)
        B = len(L)
        di = make_decode_inputs(wl, extra_slots=1, lengths=L)
        ap = make_append_inputs(wl, (di.seq_offset.numpy() + L).astype(np.int32), L.astype(np.int32))
        V_r, K_r, off_r, len_r, app_r, _ = seqsplit.shard_step_inputs(
            di.V, di.k_rope, di.seq_offset, L, (ap.v_new, ap.kpe_new, ap.slot, ap.pos), world, rank)
        d = lambda t: t.to("cuda").contiguous()
        sh = gva.make_shape(B, wl.H, wl.G, wl.d_h, wl.d_n, wl.d_r, cache_dtype=wl.torch_dtype,
                            rope_base=wl.rope_base)
        total = max(int(len_r.sum()), 1)
        ws = gva.new_workspace(sh, total)
        q_abs = torch.empty(B, wl.H, wl.d_h + wl.d_r, dtype=torch.float32, device="cuda")
        merger = seqsplit.SequenceSplitMerge(sh, world, "cuda")
        out = torch.empty(B, wl.H, wl.d_h, dtype=torch.float32, device="cuda")
        lse = torch.empty(B, wl.H, dtype=torch.float32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        gva.decode_step(sh, d(di.q), d(di.M), d(torch.from_numpy(L.astype(np.int32))),
                        *(d(t) for t in app_r), d(V_r), d(K_r), d(off_r), d(len_r), total, q_abs,
                        merger.out_part, merger.lse_part, err, ws)
        merger.merge(out, lse)
        torch.cuda.synchronize()
        q.put((rank, out.cpu().numpy(), lse.cpu().numpy(), gva.workspace_status(ws),
               int(err.item())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name,lengths", CASES)
def test_sequence_split_two_ranks_match_oracle(name, lengths):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, name, lengths, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=600) for _ in range(2)], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    sys.path.insert(0, ROOT)
    import oracle
    from compressed_kv_cache_gva_b200.synth import (WORKLOADS, as_f64, make_append_inputs,
                                                    make_decode_inputs)
    from gpu_helpers import assert_close, lse_close
    wl = WORKLOADS[name]
    L = np.array(lengths)
    di = make_decode_inputs(wl, extra_slots=1, lengths=L)
    slots = (di.seq_offset.numpy() + L).astype(np.int32)
    ap = make_append_inputs(wl, slots, L.astype(np.int32))
    V_ref, K_ref, _ = oracle.append_cache(as_f64(di.V), as_f64(di.k_rope), as_f64(ap.v_new),
                                          as_f64(ap.kpe_new), slots, L, wl.rope_base, wl.dtype)
    ref, ref_lse = oracle.gva_decode(as_f64(di.q), as_f64(di.M), L, V_ref, K_ref,
                                     di.seq_offset.numpy(), L + 1, wl.d_n, wl.d_r, wl.rope_base)
    for rank, out, lse, st, err in res:
        assert st == 0 and err == 0
        assert_close(out, ref, wl.dtype, f"rank {rank} merged output")
        lse_close(lse, ref_lse, f"rank {rank} merged lse")
    assert np.array_equal(res[0][1], res[1][1])       # every rank holds the same merged result
