"""Benchmark of one GVA decode step on synthetic caches.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole decode path over one batch: absorb the queries
(q M^T + query RoPE), append each sequence's new token (value copy + rotated
positional key), then decode attention over the history plus the new token.
Every step reads a different copy of the cache (copies rotate; together they
exceed 3x the L2), so no step starts with its cache in L2.

Printed: ONE JSON line on rank 0.  value = cache GB/s of the whole job (algorithmic
cache bytes of all steps on all ranks / max-over-ranks device time).  Under
torchrun every rank runs its own batch (weak scaling, no collective on the data
path).  `--impl reference` times the float64 CPU oracle on the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from compressed_kv_cache_gva_b200 import gva  # noqa: E402
from compressed_kv_cache_gva_b200.synth import (WORKLOADS, make_append_inputs,  # noqa: E402
                                                make_decode_inputs, make_gqa_inputs,
                                                make_multi_queries)

METRIC = "GVA decode cache GB/s & %HBM peak (1xB200); decode steps/s vs same-shape GQA"
DEFAULT_WORKLOAD = "350m_b8_t4096"
L2_BYTES = 126 * 1024 * 1024
NOMINAL_HBM_GBS = 8000.0


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20000)
    p.add_argument("--warmup", type=int, default=200)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--fma", action="store_true", help="decode on the CUDA-core FMA path")
    p.add_argument("--ctas-per-sm", type=int, default=0)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-prefill", action="store_true", help="skip the chunked-prefill timing")
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    p.add_argument("--split", default="batch", choices=["batch", "sequence"],
                   help="batch: one independent batch per GPU (weak scaling, default); "
                        "sequence: one batch, every sequence's cache split across the GPUs "
                        "(strong scaling, NCCL all-gather + merge)")
    return p.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def rank_workload(name, rank):
    """Weak scaling: every rank decodes its own batch of the named workload,
    drawn from its own seed (seed + rank); no data crosses ranks."""
    wl = WORKLOADS[name]
    return wl.scaled(seed=wl.seed + rank)


def reduce_max(value, device=None):
    """Max of a float over all ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(bytes_per_step_per_rank, steps, world, ms_max):
    """Whole-job GB/s: bytes all ranks processed over the slowest rank's time."""
    return world * steps * bytes_per_step_per_rank / (ms_max * 1e-3) / 1e9


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def load_peak_record():
    """The whole measured-peaks record, or None (the bf16 figure falls back to the
    pool's earlier 1590 TFLOP/s burst measurement)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except Exception:
        return {"bf16_tflops": 1590.0}


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 50 ms in a thread."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.samples = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.index), "-lms", "50"], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 10:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        win = [s for t, s in self.samples if t0 <= t <= t1]
        label = "timed"
        if len(win) < 3:
            return None
        def num(x):
            try:
                return float(x)
            except ValueError:
                return float("nan")
        sm = [num(s[2]) for s in win]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for s in win:
            for n, v in zip(names, s[6:10]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": float(np.nanmedian(sm)), "sm_max_mhz": num(win[0][3]),
                "reasons": sorted(reasons), "samples": len(win), "window": label,
                "power_w_median": float(np.nanmedian([num(s[4]) for s in win]))}


# ----------------------------------------------------------------------------- our arm

def cache_row_bytes(wl):
    return (wl.G * wl.d_h + wl.d_r) * wl.elem_bytes


# Sources of the kernels behind the roofline figure (split kernel, combine), their
# device helpers and their grid choice; the recorded ncu traffic is valid while
# these are unchanged.
ROOFLINE_SOURCES = ("common.cuh", "decode_mma.cuh", "decode_mma.cu", "combine.cu")


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "compressed_kv_cache_gva_b200", "csrc")
    for f in ROOFLINE_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[workload][kernel_key]
        if e.get("source_hash") != kernel_source_hash():
            return None
        return float(e["dram_bytes_per_launch"])
    except Exception:
        return None


def run_ours(args, rank, world, local):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    split_seq = args.split == "sequence"
    # sequence split: every rank holds a part of the same batch
    wl = WORKLOADS[args.workload] if split_seq else rank_workload(args.workload, rank)
    di = make_decode_inputs(wl, extra_slots=1)
    B, H, G, d_h, d_r = len(di.seq_len), wl.H, wl.G, wl.d_h, wl.d_r
    L = di.seq_len.numpy().astype(np.int64)
    row_bytes = cache_row_bytes(wl)
    step_tokens = int((L + 1).sum())                       # history + the appended token
    step_cache_bytes = step_tokens * row_bytes             # this rank's batch (or whole batch)
    slots_np = (di.seq_offset.numpy() + L).astype(np.int32)
    ap = make_append_inputs(wl, slots_np, L.astype(np.int32), seed=7 + (0 if split_seq else rank))
    app_host = [ap.v_new, ap.kpe_new, ap.slot, ap.pos]
    V_src, K_src, soff_src = di.V, di.k_rope, di.seq_offset
    slen_src = torch.from_numpy((L + 1).astype(np.int32))
    if split_seq:
        from compressed_kv_cache_gva_b200 import seqsplit
        V_src, K_src, soff_src, slen_src, start = seqsplit.shard_cache(
            di.V, di.k_rope, di.seq_offset, slen_src, world, rank)
        cnt = slen_src.numpy().astype(np.int64)
        own = (L >= start) & (L < start + cnt)            # new token of sequence b lands here
        sl = (soff_src.numpy().astype(np.int64) + L - start)[own].astype(np.int32)
        app_host = [ap.v_new[torch.from_numpy(own)].contiguous(),
                    ap.kpe_new[torch.from_numpy(own)].contiguous(),
                    torch.from_numpy(sl), ap.pos[torch.from_numpy(own)].contiguous()]
    part_tokens = int(slen_src.to(torch.int64).sum())
    cache_bytes = max(1, V_src.shape[0]) * row_bytes
    R = max(2, math.ceil(3 * L2_BYTES / cache_bytes))
    flags = gva.FLAG_FMA_PATH if args.fma else 0
    sh = gva.make_shape(B, H, G, d_h, wl.d_n, d_r, cache_dtype=wl.torch_dtype, rope_base=wl.rope_base,
                        flags=flags, ctas_per_sm=args.ctas_per_sm)

    d = lambda t: t.to(dev).contiguous()
    Vs = [d(V_src) for _ in range(R)]
    KRs = [d(K_src) for _ in range(R)]
    q, M = d(di.q), d(di.M)
    soff = d(soff_src)
    slen_step = d(slen_src)
    qpos = d(di.seq_len)                                    # new token at position L_b
    v_new, kpe_new, slot, pos = (d(t) for t in app_host)
    q_abs = torch.empty(B, H, d_h + d_r, dtype=torch.float32, device=dev)
    out = torch.empty(B, H, d_h, dtype=torch.float32, device=dev)
    max_total = max(part_tokens, 1)
    ws = gva.new_workspace(sh, max_total, device=dev)
    merger = None
    if split_seq:
        merger = seqsplit.SequenceSplitMerge(sh, world, dev)
    dec_out = merger.out_part if split_seq else out
    dec_lse = merger.lse_part if split_seq else None

    def finish():
        if split_seq:
            merger.merge(out)

    def step(c, qq=None, app=None, o=None):
        vv, kk, ss, pp = app if app is not None else (v_new, kpe_new, slot, pos)
        gva.decode_step(sh, q if qq is None else qq, M, qpos, vv, kk, ss, pp, Vs[c], KRs[c], soff,
                        slen_step, max_total, q_abs, dec_out if o is None else o, dec_lse, None, ws)
        finish()

    def step_separate(c):
        gva.append_cache(sh, v_new, kpe_new, slot, pos, Vs[c], KRs[c])
        gva.absorb_query(sh, q, M, qpos, q_abs)
        gva.decode_attention(sh, q_abs, Vs[c], KRs[c], soff, slen_step, max_total, dec_out, dec_lse,
                             ws)
        finish()

    def decode_only(c):
        gva.decode_attention(sh, q_abs, Vs[c], KRs[c], soff, slen_step, max_total, dec_out, dec_lse,
                             ws)
        finish()

    # eager warm-up (initialises the library and the launch attributes)
    for c in range(R):
        step(c)
    torch.cuda.synchronize()

    def capture(fn, n, first=0):
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                for i in range(n):
                    fn((first + i) % R)
        torch.cuda.current_stream().wait_stream(s)
        return g

    CHUNK = 256

    def graphs_for(fn, K):
        gs = []
        done = 0
        while done < K:
            n = min(CHUNK, K - done)
            gs.append((capture(fn, n, done), n))
            done += n
        return gs

    def replay(gs):
        for g, _ in gs:
            g.replay()

    def timed(gs, K, sampler_window=None):
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        st = torch.cuda.current_stream()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0 = time.time()
        e0.record(st)
        replay(gs)
        e1.record(st)
        torch.cuda.synchronize()
        t1 = time.time()
        if world > 1:
            torch.distributed.barrier()
        ms = reduce_max(e0.elapsed_time(e1), device=dev)
        return ms, t0, t1

    K, W = args.steps, args.warmup
    g_warm = graphs_for(step, max(W, 1))
    g_time = graphs_for(step, K)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.2)
    tw0 = time.time()
    replay(g_warm)
    torch.cuda.synchronize()
    ms, t0, t1 = timed(g_time, K)
    clocks = sampler.summary(tw0, t1)
    if clocks is None:
        # timed region too short for 50 ms sampling: keep the same graphs running
        # (untimed) for about a second and report the clocks seen under that load
        s0 = time.time()
        while time.time() - s0 < 1.2:
            replay(g_time)
            torch.cuda.synchronize()
        clocks = sampler.summary(tw0, time.time())
        if clocks is not None:
            clocks["window"] = "warm-up + timed + untimed soak of the same step graphs"
    sampler.stop()
    assert gva.workspace_status(ws) == 0, "device status word set"

    # the same step as three separate calls (no early cache streaming), for reference
    g_sep = graphs_for(step_separate, K)
    replay(g_sep)
    ms_sep, _, _ = timed(g_sep, K)
    del g_sep

    # decode-only timing (roofline of the dominant kernel) and the GQA comparison
    g_dec = graphs_for(decode_only, K)
    replay(g_dec)
    ms_dec, _, _ = timed(g_dec, K)
    prefill = None
    if not args.fma and not split_seq and not args.no_prefill:
        ms_pf, pf_flops = time_prefill(wl, di, 512, graphs_for, replay, timed, d, dev, K)
        peaks = load_peak_record()
        tf_peak = peaks.get("bf16_tflops") if peaks else None
        tf = pf_flops / (ms_pf * 1e-3) / 1e12
        prefill = {"n_query": 512, "call": "gva_decode_attention_multi (tcgen05 kernel)",
                   "tokens_per_sequence": "history + 512",
                   "us_per_call": round(ms_pf * 1e3, 2), "alg_tflop_per_call": round(pf_flops / 1e12, 4),
                   "roofline": {"bound": "tensor", "achieved": round(tf, 1),
                                "peak": tf_peak,
                                "peak_kind": "measured bf16 burst" if os.path.exists(
                                    os.path.join(ROOT, "MEASURED_PEAKS.json")) else "fallback",
                                "unit": "TFLOP/s",
                                "frac": round(tf / tf_peak, 4) if tf_peak else None,
                                "flops": "2*(2*d_h + d_r) per (query row, visible key); the kernel "
                                         "issues ~1.6x that (bf16 hi + lo query halves)"}}
    multi = None
    if not args.fma and not split_seq and (H // G) * 2 in (4, 8):
        multi = time_multi_token(sh, wl, di, 2, Vs, KRs, soff, slen_step, max_total, M, R, d,
                                 graphs_for, replay, timed, K, dev, row_bytes, part_tokens, ms_dec)
    ms_gqa = None
    if not split_seq:
        ms_gqa, gqa_bytes, ms_kv = run_gqa_comparison(args, wl, B, H, G, d_h, R, flags, d,
                                                      graphs_for, replay, timed, dev)

    # end to end through the public API with host buffers: every step copies its
    # inputs (q, new value, new positional key, slot, position) from one pinned
    # host buffer into one device staging buffer, runs the step on views of it,
    # and reads the output back into pinned host memory
    parts = [di.q] + app_host
    offs_b, nb = [], 0
    for t in parts:
        offs_b.append(nb)
        nb += (t.numel() * t.element_size() + 255) // 256 * 256
    h_stage = torch.zeros(nb, dtype=torch.uint8).pin_memory()
    d_stage = torch.zeros(nb, dtype=torch.uint8, device=dev)

    def view(buf, i):
        t = parts[i]
        n = t.numel() * t.element_size()
        return buf[offs_b[i]:offs_b[i] + n].view(t.dtype).view(t.shape)

    for i, t in enumerate(parts):
        view(h_stage, i).copy_(t)
    eq, ev, ek, es, ep = (view(d_stage, i) for i in range(5))
    h_out = torch.empty(B, H, d_h, dtype=torch.float32).pin_memory()
    h2d = nb
    d2h = h_out.numel() * h_out.element_size()

    def e2e_step(c):
        d_stage.copy_(h_stage, non_blocking=True)
        step(c, qq=eq, app=(ev, ek, es, ep))
        h_out.copy_(out, non_blocking=True)

    g_e2e = graphs_for(e2e_step, K)
    replay(g_e2e)
    ms_e2e_serial, _, _ = timed(g_e2e, K)
    del g_e2e
    ms_e2e = ms_e2e_serial
    e2e_mode = "serial: copy in, step, copy out, one after the other on one stream"
    if not split_seq:
        ms_e2e = time_e2e_pipelined(step, parts, h_stage, nb, view, B, H, d_h, R, K, dev, timed)
        e2e_mode = ("pipelined: every step copies its inputs host->device and its output "
                    "device->host on two copy streams, through two staging and output buffers, "
                    "so the copies of one step overlap the compute of its neighbours")

    hbm_peak, peak_kind = load_peaks()
    ms_step = ms / K
    job_ranks = 1 if split_seq else world      # sequence split: one batch for all ranks
    value = job_value(step_cache_bytes, K, job_ranks, ms)
    dec_s = ms_dec / K * 1e-3
    alg_dec_bytes = part_tokens * row_bytes + B * H * (d_h + d_r) * 4 + B * H * d_h * 4
    achieved = alg_dec_bytes / dec_s / 1e9
    kernel_key = "gva_decode_attention" + ("_fma" if args.fma else "")
    res = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": round(ms_step, 6), "higher_is_better": True,
        "scaling": "strong" if split_seq else "weak",
        "vs_baseline": None, "dtype": "bf16" if wl.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": wl.name, "B": B, "H": H, "G": G, "d_h": d_h, "d_n": wl.d_n, "d_r": d_r,
                   "T": wl.T, "ragged": wl.ragged, "rope_base": wl.rope_base,
                   "tokens_per_step": step_tokens, "cache_bytes_per_step": step_cache_bytes,
                   "l2": f"inputs larger than L2: {R} rotating cache copies, "
                         f"{R * cache_bytes / 2**20:.0f} MiB",
                   "parallelism": (f"sequence split: each sequence's cache over {world} GPU(s), "
                                   "NCCL all-gather of (out, lse) + merge") if split_seq else
                                  f"weak: {world} independent batch(es), one per GPU",
                   "step": "gva_decode_step: append + absorb (one kernel), decode (split + combine)",
                   "graphs": "CUDA graphs",
                   "decode_path": "fma" if args.fma else "tensor"},
        "steps_per_s": round(world * K / (ms * 1e-3), 1),
        "ms_per_step_separate_calls": round(ms_sep / K, 6),
        "pct_hbm_peak": {"of_measured": round(value / world / hbm_peak, 4),
                         "of_nominal_8TBs": round(value / world / NOMINAL_HBM_GBS, 4)},
        "gqa_comparison": None if ms_gqa is None else {
            "gva_decode_steps_per_s": round(K / (ms_dec * 1e-3), 1),
            "gqa_decode_steps_per_s": round(K / (ms_gqa * 1e-3), 1),
            "decode_speedup_vs_gqa": round(ms_gqa / ms_dec, 4),
            "gva_cache_bytes": step_cache_bytes, "gqa_cache_bytes": gqa_bytes,
            "cache_ratio": round(step_cache_bytes / gqa_bytes, 6),
            "gqa_cache_GBs": round(gqa_bytes / (ms_gqa / K * 1e-3) / 1e9, 2),
            "shared_kv_decode_steps_per_s": round(K / (ms_kv * 1e-3), 1),
            "shared_kv_speedup_vs_gqa": round(ms_gqa / ms_kv, 4),
            "shared_kv_cache_GBs": round(gqa_bytes / 2 / (ms_kv / K * 1e-3) / 1e9, 2)},
        "roofline": {"bound": "hbm",
                     "kernel": ("decode_simt_kernel" if args.fma else "decode_mma_kernel")
                               + " + combine_kernel (one gva_decode_attention call)",
                     "achieved": round(achieved, 2), "peak": hbm_peak, "peak_kind": peak_kind,
                     "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                     "alg_bytes_per_launch": alg_dec_bytes, "us_per_launch": round(dec_s * 1e6, 3),
                     "traffic": ncu_traffic(kernel_key, wl.name)},
        "e2e": {"value": round(job_value(step_cache_bytes, K, job_ranks, ms_e2e), 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(ms_e2e / K, 6), "mode": e2e_mode,
                "serial": {"value": round(job_value(step_cache_bytes, K, job_ranks, ms_e2e_serial), 2),
                           "ms_per_step": round(ms_e2e_serial / K, 6)}},
        "multi_token": multi,
        "prefill": prefill,
        "gpu_launches": (4 if split_seq else 3) * K,
        "clocks": clocks,
    }
    return res, di


def time_e2e_pipelined(step, parts, h_stage, nb, view, B, H, d_h, R, K, dev, timed):
    """End-to-end steps with double-buffered host<->device copies.

    Step i copies its inputs (one pinned host buffer -> device staging buffer i % 2)
    on one copy stream, runs gva_decode_step on the compute stream once that copy
    has landed, and copies its output (device buffer i % 2 -> pinned host buffer
    i % 2) on a second copy stream.  A staging buffer is refilled only after the
    step that read it has finished, and an output buffer is rewritten only after
    its previous copy-out has finished, so every step reads its own inputs and every
    output reaches the host."""
    NBUF = 2
    d_st = [torch.zeros(nb, dtype=torch.uint8, device=dev) for _ in range(NBUF)]
    o_dev = [torch.empty(B, H, d_h, dtype=torch.float32, device=dev) for _ in range(NBUF)]
    o_host = [torch.empty(B, H, d_h, dtype=torch.float32).pin_memory() for _ in range(NBUF)]
    vw = [[view(d_st[k], i) for i in range(len(parts))] for k in range(NBUF)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def capture(n, first):
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream())
        ev_in = [torch.cuda.Event() for _ in range(n)]
        ev_done = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event() for _ in range(n)]
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                for i in range(n):
                    k = i % NBUF
                    if i < NBUF:
                        s_in.wait_stream(s)
                    else:
                        s_in.wait_event(ev_done[i - NBUF])
                    with torch.cuda.stream(s_in):
                        d_st[k].copy_(h_stage, non_blocking=True)
                        ev_in[i].record(s_in)
                    s.wait_event(ev_in[i])
                    if i >= NBUF:
                        s.wait_event(ev_out[i - NBUF])
                    step((first + i) % R, qq=vw[k][0], app=tuple(vw[k][1:]), o=o_dev[k])
                    ev_done[i].record(s)
                    s_out.wait_event(ev_done[i])
                    with torch.cuda.stream(s_out):
                        o_host[k].copy_(o_dev[k], non_blocking=True)
                        ev_out[i].record(s_out)
                for i in range(max(0, n - NBUF), n):
                    s.wait_event(ev_out[i])
        torch.cuda.current_stream().wait_stream(s)
        return g

    gs, done = [], 0
    while done < K:
        n = min(256, K - done)
        gs.append((capture(n, done), n))
        done += n
    for g, _ in gs:
        g.replay()
    torch.cuda.synchronize()
    ms, _, _ = timed(gs, K)
    # every output that reached the host equals a plain step's output (the steps
    # repeat the same inputs, and the decode is deterministic)
    o_chk = torch.empty(B, H, d_h, dtype=torch.float32, device=dev)
    step(0, o=o_chk)
    torch.cuda.synchronize()
    for k in range(NBUF):
        assert torch.equal(o_host[k], o_chk.cpu()), "pipelined end-to-end output differs"
    return ms


def time_multi_token(sh, wl, di, Q, Vs, KRs, soff, slen, max_total, M, R, d, graphs_for, replay,
                     timed, K, dev, row_bytes, part_tokens, ms_dec):
    """Q new tokens per sequence decoded together (causal among them), as in
    speculative-decoding verification: one gva_decode_attention_multi call on the
    same caches, timed like the single-token decode."""
    B, H, d_h, d_r = len(di.seq_len), wl.H, wl.d_h, wl.d_r
    q = make_multi_queries(wl, B, Q)
    L = di.seq_len.numpy().astype(np.int64) + 1
    qpos = torch.from_numpy(np.stack([L - Q + i for i in range(Q)], 1).astype(np.int32))
    sh_q = gva.make_shape(B * Q, H, wl.G, d_h, wl.d_n, d_r, cache_dtype=wl.torch_dtype,
                          rope_base=wl.rope_base)
    q_abs = torch.empty(B, Q, H, d_h + d_r, dtype=torch.float32, device=dev)
    gva.absorb_query(sh_q, d(q.reshape(B * Q, H, -1)), M, d(qpos.reshape(-1)), q_abs)
    ws = torch.zeros(gva.decode_workspace_size_multi(sh, Q, max_total), dtype=torch.uint8,
                     device=dev)
    out = torch.empty(B, Q, H, d_h, dtype=torch.float32, device=dev)

    def call(c):
        gva.decode_attention_multi(sh, Q, q_abs, Vs[c], KRs[c], soff, slen, max_total, out, None, ws)

    for c in range(R):
        call(c)
    gs = graphs_for(call, K)
    replay(gs)
    ms, _, _ = timed(gs, K)
    assert gva.workspace_status(ws) == 0, "device status word set"
    s = ms / K * 1e-3
    alg = part_tokens * row_bytes + B * Q * H * (d_h + d_r) * 4 + B * Q * H * d_h * 4
    return {"n_query": Q, "call": "gva_decode_attention_multi", "us_per_call": round(s * 1e6, 3),
            "alg_GBs": round(alg / s / 1e9, 2), "time_vs_single_token_decode": round(ms / ms_dec, 4)}


def time_prefill(wl, di, Q, graphs_for, replay, timed, d, dev, steps):
    """Chunked prefill: Q new tokens appended to every sequence of the batch
    (positions L .. L+Q-1, causal among them), one gva_decode_attention_multi
    call on the tcgen05 kernel.  Returns the call time and its algorithmic
    tensor work: per (query row, visible key) 2*(2*d_h + d_r) flops, the scores
    q~.v + q_r.k_rope and the output p*v."""
    L = di.seq_len.numpy().astype(np.int64) + Q
    B, H = len(L), wl.H
    dq = make_decode_inputs(wl, extra_slots=0, lengths=L)
    q = make_multi_queries(wl, B, Q)
    qpos = torch.from_numpy(np.stack([L - Q + i for i in range(Q)], 1).astype(np.int32))
    sh_q = gva.make_shape(B * Q, H, wl.G, wl.d_h, wl.d_n, wl.d_r, cache_dtype=wl.torch_dtype,
                          rope_base=wl.rope_base)
    q_abs = torch.empty(B, Q, H, wl.d_h + wl.d_r, dtype=torch.float32, device=dev)
    gva.absorb_query(sh_q, d(q.reshape(B * Q, H, -1)), d(dq.M), d(qpos.reshape(-1)), q_abs)
    sh = gva.make_shape(B, H, wl.G, wl.d_h, wl.d_n, wl.d_r, cache_dtype=wl.torch_dtype,
                        rope_base=wl.rope_base)
    tot = int(L.sum())
    cb = dq.V.numel() * dq.V.element_size() + dq.k_rope.numel() * dq.k_rope.element_size()
    R = max(2, math.ceil(3 * L2_BYTES / cb))
    Vs = [d(dq.V) for _ in range(R)]
    Ks = [d(dq.k_rope) for _ in range(R)]
    soff, slen = d(dq.seq_offset), d(dq.seq_len)
    ws = torch.zeros(gva.decode_workspace_size_multi(sh, Q, tot), dtype=torch.uint8, device=dev)
    out = torch.empty(B, Q, H, wl.d_h, dtype=torch.float32, device=dev)

    def call(c):
        c %= R   # graphs_for counts copies of the step's cache
        gva.decode_attention_multi(sh, Q, q_abs, Vs[c], Ks[c], soff, slen, tot, out, None, ws)

    for c in range(R):
        call(c)
    n = max(10, min(steps, 200))
    gs = graphs_for(call, n)
    replay(gs)
    ms, _, _ = timed(gs, n)
    assert gva.workspace_status(ws) == 0, "device status word set"
    keys = int(sum(Q * (int(l) - Q) + Q * (Q + 1) // 2 for l in L))
    flops = keys * H * 2 * (2 * wl.d_h + wl.d_r)
    return ms / n, flops


def run_gqa_comparison(args, wl, B, H, G, d_h, R, flags, d, graphs_for, replay, timed, dev):
    """Same-shape GQA decode (K and V cache) timed like the GVA decode."""
    gi = make_gqa_inputs(wl, extra_slots=1)
    Kq = [d(gi.K) for _ in range(R)]
    Vq = [d(gi.V) for _ in range(R)]
    sh_q = gva.make_shape(B, H, G, d_h, d_h, 0, cache_dtype=wl.torch_dtype, flags=flags,
                          ctas_per_sm=args.ctas_per_sm)
    qg = d(gi.q)
    slen_q = d(torch.from_numpy((gi.seq_len.numpy() + 1).astype(np.int32)))
    soff_q = d(gi.seq_offset)
    tot_q = int(gi.seq_len.numpy().astype(np.int64).sum()) + B
    ws_q = gva.new_workspace(sh_q, tot_q, device=dev)
    out_q = torch.empty(B, H, d_h, dtype=torch.float32, device=dev)

    def gqa_decode(c):
        gva.gqa_decode_attention(sh_q, qg, Kq[c], Vq[c], soff_q, slen_q, tot_q, out_q, None, ws_q)

    for c in range(R):
        gqa_decode(c)
    g_gqa = graphs_for(gqa_decode, args.steps)
    replay(g_gqa)
    ms_gqa, _, _ = timed(g_gqa, args.steps)
    del g_gqa

    # shared keys and values (K = V, the pages' first design): the same batch
    # with the value cache only, through gva_shared_kv_decode_attention
    sh_kv = gva.make_shape(B, H, G, d_h, d_h, 0, cache_dtype=wl.torch_dtype, flags=flags,
                           ctas_per_sm=args.ctas_per_sm)
    ws_kv = gva.new_workspace(sh_kv, tot_q, device=dev)

    def kv_decode(c):
        gva.shared_kv_decode_attention(sh_kv, qg, Vq[c], soff_q, slen_q, tot_q, out_q, None, ws_kv)

    for c in range(R):
        kv_decode(c)
    g_kv = graphs_for(kv_decode, args.steps)
    replay(g_kv)
    ms_kv, _, _ = timed(g_kv, args.steps)
    assert gva.workspace_status(ws_kv) == 0, "device status word set"
    return ms_gqa, tot_q * 2 * G * d_h * wl.elem_bytes, ms_kv


# ----------------------------------------------------------------------------- oracle arm

def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def time_oracle(wl, di, budget_s, max_units=None):
    """Oracle decode on (sequence, head) pairs until the time budget is spent.
    Returns (cache bytes attended per second, description)."""
    import oracle
    from compressed_kv_cache_gva_b200.synth import as_f64
    q, M = as_f64(di.q), as_f64(di.M)
    V, KR = as_f64(di.V), as_f64(di.k_rope)
    L = di.seq_len.numpy()
    pairs = [(b, h) for b in range(len(L)) for h in range(wl.H)]
    done, nbytes = 0, 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s and (max_units is None or done < max_units):
        b, h = pairs[done % len(pairs)]
        oracle.gva_decode(q, M, di.q_pos.numpy(), V, KR, di.seq_offset.numpy(), L, wl.d_n, wl.d_r,
                          wl.rope_base, pairs=[(b, h)])
        # one (b, h) pair attends L_b rows; H pairs of a sequence cover its whole cache row
        nbytes += int(L[b]) * cache_row_bytes(wl) / wl.H
        done += 1
    dt = time.perf_counter() - t0
    return nbytes / dt / 1e9, f"{done} (sequence, head) pairs of the full-size cache, {dt:.1f} s", dt, done


def cpu_baseline(wl, di, seconds):
    gbs, desc, dt, n = time_oracle(wl, di, seconds)
    return {"value": round(gbs, 6), "unit": "GB/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": desc}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    wl = WORKLOADS[args.workload]
    di = make_decode_inputs(wl, extra_slots=1)
    total_steps = args.steps + args.warmup
    per_step = max(0.002, min(2.0, 150.0 / total_steps))
    import oracle  # noqa: F401
    for _ in range(args.warmup):
        time_oracle(wl, di, per_step, max_units=1)
    t0 = time.perf_counter()
    nbytes_rate = []
    for _ in range(args.steps):
        g, _, dt, n = time_oracle(wl, di, per_step, max_units=None if per_step > 0.01 else 1)
        nbytes_rate.append((g, dt))
    elapsed = time.perf_counter() - t0
    total_bytes = sum(g * 1e9 * dt for g, dt in nbytes_rate)
    value = total_bytes / elapsed / 1e9
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(elapsed / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "step": "float64 CPU oracle, non-absorbed route, "
                                                  "bounded sample of (sequence, head) pairs per step"},
        "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": oracle_threads(),
                         "kind": "oracle",
                         "sample": f"each step: oracle decode of (sequence, head) pairs for "
                                   f"~{per_step * 1e3:.0f} ms"},
        "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    res, di = run_ours(args, rank, world, local)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        wl = WORKLOADS[args.workload]
        res["cpu_baseline"] = cpu_baseline(wl, di, args.cpu_seconds)
    elif rank == 0:
        res["cpu_baseline"] = None
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
