"""Benchmark of one GVA decode step on synthetic caches.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--workloads NAME,NAME|none] [--impl ours|reference]

A step is one pass of the whole decode path over one batch: append each
sequence's new token (value copy + rotated positional key), absorb the queries
(q M^T + query RoPE), then decode attention over the history plus the new token.
Every step reads a different copy of the cache (copies rotate; together they
exceed 3x the L2), so no step starts with its cache in L2.

Timing: K steps are captured in CUDA graphs; after W warm-up steps the K-step
pass is replayed back to back until at least 0.2 s (and at least 20 passes) have
run, with a CUDA event between passes, and the median pass over K is the time
per step (max over ranks).  The driver's short runs (small K) so measure the same
steady state as long ones.

Printed: ONE JSON line on rank 0.  value = cache GB/s of the whole job (algorithmic
cache bytes of all steps on all ranks / max-over-ranks device time).  Under
torchrun every rank runs its own batch (weak scaling, no collective on the data
path).  `--impl reference` times the float64 CPU oracle on the same workload.
"""
from __future__ import annotations

import argparse
import gc
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
                                                make_decode_inputs, make_gqa_append_inputs,
                                                make_gqa_inputs, make_multi_queries)

METRIC = "GVA decode cache GB/s & %HBM peak (1xB200); decode steps/s vs same-shape GQA"
DEFAULT_WORKLOAD = "350m_b8_t4096"
# the long-context workloads of the study, measured in the same run (compact form)
EXTRA_WORKLOADS = ("dr24_b4_t32768", "ragged_b64_1k_16k", "d128_b1_t131072")
L2_BYTES = 126 * 1024 * 1024
NOMINAL_HBM_GBS = 8000.0
MIN_TIMED_S = 0.2      # every timed measurement replays its K-step pass this long ...
MIN_PASSES = 20        # ... and at least this many times
MAX_PASSES = 100000
CHUNK = 256            # steps per captured graph


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=1000)
    p.add_argument("--warmup", type=int, default=50)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    p.add_argument("--workloads", default=",".join(EXTRA_WORKLOADS),
                   help="comma-separated workloads also measured (decode, step and GQA "
                        "comparison), or 'none'")
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
    return p.parse_args(argv)


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


def passes_for(t_pass_s, min_s=MIN_TIMED_S, min_passes=MIN_PASSES, max_passes=MAX_PASSES):
    """Number of back-to-back passes of the timed region: at least `min_passes`
    and at least `min_s` seconds of work."""
    n = max(min_passes, math.ceil(min_s / max(t_pass_s, 1e-9)))
    return int(min(n, max_passes))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def load_peak_record():
    """The whole measured-peaks record, or the pool's earlier 1590 TFLOP/s bf16
    burst measurement when it is absent."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured bf16 burst"
    except Exception:
        return {"bf16_tflops": 1590.0}, "fallback"


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
                "reasons": sorted(reasons), "samples": len(win), "window": "timed",
                "power_w_median": float(np.nanmedian([num(s[4]) for s in win]))}


# ----------------------------------------------------------------------------- graphs + timing

class GraphTimer:
    """Captures K calls of a step function in CUDA graphs (chunks of CHUNK) and
    times them: the K-step pass is replayed back to back, with an event between
    passes, for at least MIN_TIMED_S and MIN_PASSES passes; the result is the
    median pass (max over ranks).  Step i of a pass reads cache copy i mod R."""

    def __init__(self, dev, world):
        self.dev, self.world = dev, world
        self.windows = []          # (t0, t1) host times of every timed region

    def capture(self, fn, n, first, R):
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream(device=self.dev)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                for i in range(n):
                    fn((first + i) % R)
        torch.cuda.current_stream().wait_stream(s)
        return g

    def graphs(self, fn, K, R):
        gs, done = [], 0
        while done < K:
            n = min(CHUNK, K - done)
            gs.append((self.capture(fn, n, done, R), n))
            done += n
        return gs

    @staticmethod
    def replay(gs):
        for g, _ in gs:
            g.replay()

    def barrier(self):
        if self.world > 1:
            torch.distributed.barrier()

    def timed(self, gs):
        """Median device ms of one pass over `gs` (max over ranks), the number of
        passes and the host window."""
        st = torch.cuda.current_stream()
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        self.replay(gs)                            # the first replays run slower
        c0.record(st)
        for _ in range(8):                         # calibration passes (untimed)
            self.replay(gs)
        c1.record(st)
        torch.cuda.synchronize()
        # 25% margin: the timed passes may run faster than the calibration ones
        n = passes_for(c0.elapsed_time(c1) / 8 * 1e-3, min_s=1.25 * MIN_TIMED_S)
        n = int(reduce_max(n, device=self.dev))    # the same count on every rank
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
        self.barrier()
        torch.cuda.synchronize()
        t0 = time.time()
        ev[0].record(st)
        for i in range(n):
            self.replay(gs)
            ev[i + 1].record(st)
        torch.cuda.synchronize()
        t1 = time.time()
        self.barrier()
        per = sorted(ev[i].elapsed_time(ev[i + 1]) for i in range(n))
        med = per[n // 2] if n % 2 else 0.5 * (per[n // 2 - 1] + per[n // 2])
        self.windows.append((t0, t1))
        return reduce_max(med, device=self.dev), n, (t0, t1)

    def time_fn(self, fn, K, R, warm=True):
        """Capture K steps of fn, warm up, and time them: (ms per step, passes, window)."""
        gs = self.graphs(fn, K, R)
        if warm:
            self.replay(gs)
        ms, n, win = self.timed(gs)
        del gs
        return ms / K, n, win


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


def copies_for(nbytes):
    """Cache copies whose total exceeds 3x the L2."""
    return max(2, math.ceil(3 * L2_BYTES / max(nbytes, 1)))


class GQAStep:
    """The same-shape GQA baseline of a workload: K and V caches (R copies, one
    free slot per sequence), its decode and its full step (query rotation +
    append of the new key and value + decode)."""

    def __init__(self, wl, B, flags, ctas_per_sm, dev):
        d = lambda t: t.to(dev).contiguous()
        self.gi = gi = make_gqa_inputs(wl, extra_slots=1)
        L = gi.seq_len.numpy().astype(np.int64)
        self.B, self.wl = B, wl
        self.bytes_per_step = int((L + 1).sum()) * 2 * wl.G * wl.d_h * wl.elem_bytes
        self.R = copies_for(self.bytes_per_step)
        self.K = [d(gi.K) for _ in range(self.R)]
        self.V = [d(gi.V) for _ in range(self.R)]
        kw = dict(cache_dtype=wl.torch_dtype, rope_base=wl.rope_base, flags=flags,
                  ctas_per_sm=ctas_per_sm)
        self.sh = gva.make_shape(B, wl.H, wl.G, wl.d_h, wl.d_h, 0, **kw)
        self.sh_f = gva.make_shape(B, wl.H, wl.G, wl.d_h, wl.d_h, 0, q_dtype=torch.float32, **kw)
        self.q = d(gi.q)
        self.q_pos = d(gi.seq_len)
        self.soff = d(gi.seq_offset)
        self.slen = d(torch.from_numpy((L + 1).astype(np.int32)))
        self.total = int((L + 1).sum())
        ap = make_gqa_append_inputs(wl, (gi.seq_offset.numpy() + L).astype(np.int32),
                                    L.astype(np.int32))
        self.k_new, self.v_new, self.slot, self.pos = d(ap.k_new), d(ap.v_new), d(ap.slot), d(ap.pos)
        self.q_rot = torch.empty(B, wl.H, wl.d_h, dtype=torch.float32, device=dev)
        self.out = torch.empty(B, wl.H, wl.d_h, dtype=torch.float32, device=dev)
        self.ws = gva.new_workspace(self.sh, self.total, device=dev)

    def decode(self, c):
        gva.gqa_decode_attention(self.sh, self.q, self.K[c], self.V[c], self.soff, self.slen,
                                 self.total, self.out, None, self.ws)

    def step(self, c):
        gva.gqa_decode_step(self.sh, self.q, self.q_pos, self.k_new, self.v_new, self.slot,
                            self.pos, self.K[c], self.V[c], self.soff, self.slen, self.total,
                            self.q_rot, self.out, None, None, self.ws)

    def shared_kv(self, c):
        gva.shared_kv_decode_attention(self.sh, self.q, self.V[c], self.soff, self.slen,
                                       self.total, self.out, None, self.ws)


class GVAStep:
    """Buffers and calls of one GVA decode step over one rank's batch."""

    def __init__(self, wl, args, world, rank, dev, split_seq=False):
        self.wl, self.dev = wl, dev
        d = lambda t: t.to(dev).contiguous()
        self.di = di = make_decode_inputs(wl, extra_slots=1)
        B, H, G, d_h, d_r = len(di.seq_len), wl.H, wl.G, wl.d_h, wl.d_r
        self.B = B
        L = di.seq_len.numpy().astype(np.int64)
        self.row_bytes = cache_row_bytes(wl)
        self.step_tokens = int((L + 1).sum())                 # history + the appended token
        self.step_cache_bytes = self.step_tokens * self.row_bytes
        slots_np = (di.seq_offset.numpy() + L).astype(np.int32)
        ap = make_append_inputs(wl, slots_np, L.astype(np.int32),
                                seed=7 + (0 if split_seq else rank))
        app_host = (ap.v_new, ap.kpe_new, ap.slot, ap.pos)
        V_src, K_src, soff_src = di.V, di.k_rope, di.seq_offset
        slen_src = torch.from_numpy((L + 1).astype(np.int32))
        if split_seq:
            from compressed_kv_cache_gva_b200 import seqsplit
            V_src, K_src, soff_src, slen_src, app_host, _ = seqsplit.shard_step_inputs(
                di.V, di.k_rope, di.seq_offset, L, app_host, world, rank)
        self.app_host = list(app_host)
        self.part_tokens = int(slen_src.to(torch.int64).sum())
        cache_bytes = max(1, V_src.shape[0]) * self.row_bytes
        self.R = copies_for(cache_bytes)
        self.l2_note = (f"inputs larger than L2: {self.R} rotating cache copies, "
                        f"{self.R * cache_bytes / 2**20:.0f} MiB")
        flags = gva.FLAG_FMA_PATH if args.fma else 0
        self.flags = flags
        self.sh = gva.make_shape(B, H, G, d_h, wl.d_n, d_r, cache_dtype=wl.torch_dtype,
                                 rope_base=wl.rope_base, flags=flags, ctas_per_sm=args.ctas_per_sm)
        self.Vs = [d(V_src) for _ in range(self.R)]
        self.KRs = [d(K_src) for _ in range(self.R)]
        self.q, self.M = d(di.q), d(di.M)
        self.soff = d(soff_src)
        self.slen = d(slen_src)
        self.qpos = d(di.seq_len)                              # new token at position L_b
        self.v_new, self.kpe_new, self.slot, self.pos = (d(t) for t in self.app_host)
        self.q_abs = torch.empty(B, H, d_h + d_r, dtype=torch.float32, device=dev)
        self.out = torch.empty(B, H, d_h, dtype=torch.float32, device=dev)
        self.max_total = max(self.part_tokens, 1)
        self.ws = gva.new_workspace(self.sh, self.max_total, device=dev)
        self.merger = None
        if split_seq:
            from compressed_kv_cache_gva_b200 import seqsplit
            self.merger = seqsplit.SequenceSplitMerge(self.sh, world, dev)
        self.dec_out = self.merger.out_part if split_seq else self.out
        self.dec_lse = self.merger.lse_part if split_seq else None
        # decode-call bytes: cache of this rank + absorbed queries + output
        self.alg_dec_bytes = (self.part_tokens * self.row_bytes + B * H * (d_h + d_r) * 4
                              + B * H * d_h * 4)

    def finish(self):
        if self.merger is not None:
            self.merger.merge(self.out)

    def step(self, c, qq=None, app=None, o=None):
        vv, kk, ss, pp = app if app is not None else (self.v_new, self.kpe_new, self.slot, self.pos)
        gva.decode_step(self.sh, self.q if qq is None else qq, self.M, self.qpos, vv, kk, ss, pp,
                        self.Vs[c], self.KRs[c], self.soff, self.slen, self.max_total, self.q_abs,
                        self.dec_out if o is None else o, self.dec_lse, None, self.ws)
        self.finish()

    def step_separate(self, c):
        gva.append_cache(self.sh, self.v_new, self.kpe_new, self.slot, self.pos, self.Vs[c],
                         self.KRs[c])
        gva.absorb_query(self.sh, self.q, self.M, self.qpos, self.q_abs)
        gva.decode_attention(self.sh, self.q_abs, self.Vs[c], self.KRs[c], self.soff, self.slen,
                             self.max_total, self.dec_out, self.dec_lse, self.ws)
        self.finish()

    def decode_only(self, c):
        gva.decode_attention(self.sh, self.q_abs, self.Vs[c], self.KRs[c], self.soff, self.slen,
                             self.max_total, self.dec_out, self.dec_lse, self.ws)
        self.finish()


def decode_figures(st, ms_dec, hbm_peak):
    """GB/s and roofline fraction of one decode call from its time per call."""
    s = ms_dec * 1e-3
    ach = st.alg_dec_bytes / s / 1e9
    return {"decode_us": round(s * 1e6, 3), "decode_alg_GBs": round(ach, 2),
            "frac_of_measured": round(ach / hbm_peak, 4),
            "frac_of_nominal_8TBs": round(ach / NOMINAL_HBM_GBS, 4)}


def measure_extra(name, args, timer, sampler, dev, hbm_peak, K):
    """Compact figures of one more workload: the fused step, the decode call and
    the same-shape GQA decode and step, each timed like the main workload."""
    wl = WORKLOADS[name]
    st = GVAStep(wl, args, 1, 0, dev)
    for c in range(st.R):
        st.step(c)
    torch.cuda.synchronize()
    t_start = time.time()
    ms_step, n_step, _ = timer.time_fn(st.step, K, st.R)
    ms_dec, n_dec, _ = timer.time_fn(st.decode_only, K, st.R)
    assert gva.workspace_status(st.ws) == 0, f"{name}: device status word set"
    res = {"B": st.B, "tokens_per_step": st.step_tokens, "cache_bytes_per_step": st.step_cache_bytes,
           "l2": st.l2_note,
           "step_us": round(ms_step * 1e3, 3),
           "step_GBs": round(st.step_cache_bytes / (ms_step * 1e-3) / 1e9, 2),
           "step_frac_of_measured": round(st.step_cache_bytes / (ms_step * 1e-3) / 1e9 / hbm_peak, 4)}
    res.update(decode_figures(st, ms_dec, hbm_peak))
    B = st.B
    del st
    gc.collect()
    torch.cuda.empty_cache()
    if not args.fma:
        gq = GQAStep(wl, B, 0, args.ctas_per_sm, dev)
        for c in range(gq.R):
            gq.step(c)
        ms_gd, _, _ = timer.time_fn(gq.decode, K, gq.R)
        ms_gs, _, _ = timer.time_fn(gq.step, K, gq.R)
        assert gva.workspace_status(gq.ws) == 0, f"{name}: GQA status word set"
        res.update({"gqa_decode_us": round(ms_gd * 1e3, 3),
                    "decode_speedup_vs_gqa": round(ms_gd / ms_dec, 4),
                    "gqa_step_us": round(ms_gs * 1e3, 3),
                    "step_speedup_vs_gqa": round(ms_gs / ms_step, 4),
                    "gqa_cache_bytes_per_step": gq.bytes_per_step})
        del gq
        gc.collect()
        torch.cuda.empty_cache()
    res["passes"] = {"step": n_step, "decode": n_dec}
    res["clocks"] = sampler.summary(t_start, time.time())
    return res


def run_ours(args, rank, world, local):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    split_seq = args.split == "sequence"
    # sequence split: every rank holds a part of the same batch
    wl = WORKLOADS[args.workload] if split_seq else rank_workload(args.workload, rank)
    st = GVAStep(wl, args, world, rank, dev, split_seq=split_seq)
    B, H, G, d_h, d_r = st.B, wl.H, wl.G, wl.d_h, wl.d_r
    R = st.R
    timer = GraphTimer(dev, world)
    K, W = args.steps, max(args.warmup, 3)

    # eager warm-up (initialises the library and every cache copy)
    for c in range(R):
        st.step(c)
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.2)
    g_warm = timer.graphs(st.step, W, R)
    g_time = timer.graphs(st.step, K, R)
    tw0 = time.time()
    timer.replay(g_warm)
    torch.cuda.synchronize()
    ms_pass, n_pass, (t0, t1) = timer.timed(g_time)
    clocks = sampler.summary(tw0, t1)
    del g_warm, g_time
    assert gva.workspace_status(st.ws) == 0, "device status word set"
    ms_step = ms_pass / K

    # the same step as three separate calls (no early cache streaming), for reference
    ms_sep, _, _ = timer.time_fn(st.step_separate, K, R)
    # decode-only timing (roofline of the dominant kernel)
    ms_dec, n_dec, _ = timer.time_fn(st.decode_only, K, R)

    hbm_peak, peak_kind = load_peaks()
    prefill = None
    if not args.fma and not split_seq and not args.no_prefill:
        ms_pf, pf_flops = time_prefill(wl, st.di, 512, timer, dev, K)
        peaks, pk_kind = load_peak_record()
        tf_peak = peaks.get("bf16_tflops")
        tf = pf_flops / (ms_pf * 1e-3) / 1e12
        prefill = {"n_query": 512, "call": "gva_decode_attention_multi (tcgen05 kernel)",
                   "tokens_per_sequence": "history + 512",
                   "us_per_call": round(ms_pf * 1e3, 2), "alg_tflop_per_call": round(pf_flops / 1e12, 4),
                   "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": tf_peak,
                                "peak_kind": pk_kind, "unit": "TFLOP/s",
                                "frac": round(tf / tf_peak, 4) if tf_peak else None,
                                "flops": "2*(2*d_h + d_r) per (query row, visible key); the kernel "
                                         "issues ~1.6x that (bf16 hi + lo query halves)"}}
    multi = None
    if not args.fma and not split_seq and (H // G) * 2 <= 8:
        multi = time_multi_token(st, 2, timer, K, dev, ms_dec)
    gqa_cmp = None
    if not split_seq and not args.fma:
        gq = GQAStep(wl, B, 0, args.ctas_per_sm, dev)
        for c in range(gq.R):
            gq.step(c)
        ms_gd, _, _ = timer.time_fn(gq.decode, K, gq.R)
        ms_gs, _, _ = timer.time_fn(gq.step, K, gq.R)
        ms_kv, _, _ = timer.time_fn(gq.shared_kv, K, gq.R)
        assert gva.workspace_status(gq.ws) == 0, "GQA status word set"
        gb = gq.bytes_per_step
        gqa_cmp = {
            "gva_decode_steps_per_s": round(1e3 / ms_dec, 1),
            "gqa_decode_steps_per_s": round(1e3 / ms_gd, 1),
            "decode_speedup_vs_gqa": round(ms_gd / ms_dec, 4),
            "gva_full_steps_per_s": round(1e3 / ms_step, 1),
            "gqa_full_steps_per_s": round(1e3 / ms_gs, 1),
            "full_step_speedup": round(ms_gs / ms_step, 4),
            "gqa_full_step": "gqa_decode_step: query rotation + append of key and value (one "
                             "kernel), GQA decode (split + combine)",
            "gva_cache_bytes": st.step_cache_bytes, "gqa_cache_bytes": gb,
            "cache_ratio": round(st.step_cache_bytes / gb, 6),
            "gqa_cache_GBs": round(gb / (ms_gd * 1e-3) / 1e9, 2),
            "shared_kv_decode_steps_per_s": round(1e3 / ms_kv, 1),
            "shared_kv_speedup_vs_gqa": round(ms_gd / ms_kv, 4),
            "shared_kv_cache_GBs": round(gb / 2 / (ms_kv * 1e-3) / 1e9, 2)}
        del gq
        gc.collect()
        torch.cuda.empty_cache()

    # end to end through the public API with host buffers: every step copies its
    # inputs (q, new value, new positional key, slot, position) from one pinned
    # host buffer into one device staging buffer, runs the step on views of it,
    # and reads the output back into pinned host memory
    parts = [st.di.q] + st.app_host
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
        st.step(c, qq=eq, app=(ev, ek, es, ep))
        h_out.copy_(st.out, non_blocking=True)

    ms_e2e_serial, _, _ = timer.time_fn(e2e_step, K, R)
    ms_e2e = ms_e2e_serial
    e2e_mode = "serial: copy in, step, copy out, one after the other on one stream"
    if not split_seq:
        ms_e2e = time_e2e_pipelined(st, parts, h_stage, nb, view, K, dev, timer)
        e2e_mode = ("pipelined: every step copies its inputs host->device and its output "
                    "device->host on two copy streams, through two staging and output buffers, "
                    "so the copies of one step overlap the compute of its neighbours")

    workloads = {}
    extra = [] if (args.workloads in ("", "none") or split_seq or world > 1) else \
        [w for w in args.workloads.split(",") if w and w != wl.name]
    for name in extra:
        workloads[name] = measure_extra(name, args, timer, sampler, dev, hbm_peak, K)
    sampler.stop()

    job_ranks = 1 if split_seq else world      # sequence split: one batch for all ranks
    value = job_value(st.step_cache_bytes, 1, job_ranks, ms_step)
    dec = decode_figures(st, ms_dec, hbm_peak)
    kernel_key = "gva_decode_attention" + ("_fma" if args.fma else "")
    launches_per_step = 4 if split_seq else 3
    res = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": round(ms_step, 6), "higher_is_better": True,
        "scaling": "strong" if split_seq else "weak",
        "vs_baseline": None, "dtype": "bf16" if wl.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": wl.name, "B": B, "H": H, "G": G, "d_h": d_h, "d_n": wl.d_n, "d_r": d_r,
                   "T": wl.T, "ragged": wl.ragged, "rope_base": wl.rope_base,
                   "tokens_per_step": st.step_tokens, "cache_bytes_per_step": st.step_cache_bytes,
                   "l2": st.l2_note,
                   "parallelism": (f"sequence split: each sequence's cache over {world} GPU(s), "
                                   "NCCL all-gather of (out, lse) + merge") if split_seq else
                                  f"weak: {world} independent batch(es), one per GPU",
                   "step": "gva_decode_step: append + absorb (one kernel), decode (split + combine)",
                   "graphs": "CUDA graphs of the K steps; the K-step pass replayed back to back, "
                             "median pass",
                   "decode_path": "fma" if args.fma else "tensor"},
        "timing": {"passes": n_pass, "timed_region_s": round(t1 - t0, 3),
                   "ms_per_pass_median": round(ms_pass, 6), "min_timed_s": MIN_TIMED_S,
                   "min_passes": MIN_PASSES},
        "steps_per_s": round(world * 1e3 / ms_step, 1),
        "ms_per_step_separate_calls": round(ms_sep, 6),
        "pct_hbm_peak": {"of_measured": round(value / world / hbm_peak, 4),
                         "of_nominal_8TBs": round(value / world / NOMINAL_HBM_GBS, 4)},
        "gqa_comparison": gqa_cmp,
        "roofline": {"bound": "hbm",
                     "kernel": ("decode_simt_kernel" if args.fma else "decode_mma_kernel")
                               + " + combine_kernel (one gva_decode_attention call)",
                     "achieved": dec["decode_alg_GBs"], "peak": hbm_peak, "peak_kind": peak_kind,
                     "unit": "GB/s", "frac": dec["frac_of_measured"],
                     "alg_bytes_per_launch": st.alg_dec_bytes, "us_per_launch": dec["decode_us"],
                     "passes": n_dec, "traffic": ncu_traffic(kernel_key, wl.name)},
        "e2e": {"value": round(job_value(st.step_cache_bytes, 1, job_ranks, ms_e2e), 2),
                "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(ms_e2e, 6), "mode": e2e_mode,
                "serial": {"value": round(job_value(st.step_cache_bytes, 1, job_ranks,
                                                    ms_e2e_serial), 2),
                           "ms_per_step": round(ms_e2e_serial, 6)}},
        "multi_token": multi,
        "prefill": prefill,
        "workloads": workloads,
        "gpu_launches": launches_per_step * K * n_pass,
        "clocks": clocks,
    }
    return res, st.di


E2E_BUFFERS = 2   # staging / output buffers of the pipelined end-to-end loop


def time_e2e_pipelined(st, parts, h_stage, nb, view, K, dev, timer, nbuf=None):
    """End-to-end steps with multi-buffered host<->device copies, ms per step.

    Step i copies its inputs (one pinned host buffer -> device staging buffer
    i % NBUF) on one copy stream, runs gva_decode_step on the compute stream once
    that copy has landed, and copies its output (device buffer i % NBUF -> pinned
    host buffer i % NBUF) on a second copy stream.  A staging buffer is refilled
    only after the step that read it has finished, and an output buffer is
    rewritten only after its previous copy-out has finished, so every step reads
    its own inputs and every output reaches the host."""
    NBUF = nbuf or E2E_BUFFERS
    B, H, d_h, R = st.B, st.wl.H, st.wl.d_h, st.R
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
                    st.step((first + i) % R, qq=vw[k][0], app=tuple(vw[k][1:]), o=o_dev[k])
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
        n = min(CHUNK, K - done)
        gs.append((capture(n, done), n))
        done += n
    timer.replay(gs)
    torch.cuda.synchronize()
    ms, _, _ = timer.timed(gs)
    # every output that reached the host equals a plain step's output (the steps
    # repeat the same inputs, and the decode is deterministic)
    o_chk = torch.empty(B, H, d_h, dtype=torch.float32, device=dev)
    st.step(0, o=o_chk)
    torch.cuda.synchronize()
    for k in range(NBUF):
        assert torch.equal(o_host[k], o_chk.cpu()), "pipelined end-to-end output differs"
    return ms / K


def time_multi_token(st, Q, timer, K, dev, ms_dec):
    """Q new tokens per sequence decoded together (causal among them), as in
    speculative-decoding verification: one gva_decode_attention_multi call on the
    same caches, timed like the single-token decode."""
    wl, di = st.wl, st.di
    B, H, d_h, d_r = st.B, wl.H, wl.d_h, wl.d_r
    d = lambda t: t.to(dev).contiguous()
    q = make_multi_queries(wl, B, Q)
    L = di.seq_len.numpy().astype(np.int64) + 1
    qpos = torch.from_numpy(np.stack([L - Q + i for i in range(Q)], 1).astype(np.int32))
    sh_q = gva.make_shape(B * Q, H, wl.G, d_h, wl.d_n, d_r, cache_dtype=wl.torch_dtype,
                          rope_base=wl.rope_base)
    q_abs = torch.empty(B, Q, H, d_h + d_r, dtype=torch.float32, device=dev)
    gva.absorb_query(sh_q, d(q.reshape(B * Q, H, -1)), st.M, d(qpos.reshape(-1)), q_abs)
    ws = torch.zeros(gva.decode_workspace_size_multi(st.sh, Q, st.max_total), dtype=torch.uint8,
                     device=dev)
    out = torch.empty(B, Q, H, d_h, dtype=torch.float32, device=dev)

    def call(c):
        gva.decode_attention_multi(st.sh, Q, q_abs, st.Vs[c], st.KRs[c], st.soff, st.slen,
                                   st.max_total, out, None, ws)

    for c in range(st.R):
        call(c)
    ms, _, _ = timer.time_fn(call, K, st.R)
    assert gva.workspace_status(ws) == 0, "device status word set"
    s = ms * 1e-3
    alg = st.part_tokens * st.row_bytes + B * Q * H * (d_h + d_r) * 4 + B * Q * H * d_h * 4
    return {"n_query": Q, "call": "gva_decode_attention_multi", "us_per_call": round(s * 1e6, 3),
            "alg_GBs": round(alg / s / 1e9, 2), "time_vs_single_token_decode": round(ms / ms_dec, 4)}


def time_prefill(wl, di, Q, timer, dev, steps):
    """Chunked prefill: Q new tokens appended to every sequence of the batch
    (positions L .. L+Q-1, causal among them), one gva_decode_attention_multi
    call on the tcgen05 kernel.  Returns the call time (ms) and its algorithmic
    tensor work: per (query row, visible key) 2*(2*d_h + d_r) flops, the scores
    q~.v + q_r.k_rope and the output p*v."""
    d = lambda t: t.to(dev).contiguous()
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
    R = copies_for(cb)
    Vs = [d(dq.V) for _ in range(R)]
    Ks = [d(dq.k_rope) for _ in range(R)]
    soff, slen = d(dq.seq_offset), d(dq.seq_len)
    ws = torch.zeros(gva.decode_workspace_size_multi(sh, Q, tot), dtype=torch.uint8, device=dev)
    out = torch.empty(B, Q, H, wl.d_h, dtype=torch.float32, device=dev)

    def call(c):
        gva.decode_attention_multi(sh, Q, q_abs, Vs[c], Ks[c], soff, slen, tot, out, None, ws)

    for c in range(R):
        call(c)
    n = max(10, min(steps, 200))
    ms, _, _ = timer.time_fn(call, n, R)
    assert gva.workspace_status(ws) == 0, "device status word set"
    keys = int(sum(Q * (int(l) - Q) + Q * (Q + 1) // 2 for l in L))
    flops = keys * H * 2 * (2 * wl.d_h + wl.d_r)
    return ms, flops


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
    Returns (cache bytes attended per second, description, seconds, pairs)."""
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
