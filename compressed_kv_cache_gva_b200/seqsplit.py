"""One batch decoded by several GPUs that each hold a part of every sequence's cache.

Rank r of `world` keeps positions [L*r/world, L*(r+1)/world) of each sequence
(with its own compact slot layout), decodes them with the ordinary split-KV
kernels, then the ranks exchange their normalised outputs and log-sum-exps with
one NCCL all-gather and each rank merges them with gva_merge_states.  The stored
positional keys carry their absolute positions (they were rotated at append
time) and the query position is absolute, so a part needs no re-indexing.

Only the exchange is collective; the arithmetic stays in the CUDA kernels.
"""
from __future__ import annotations

import numpy as np
import torch

from . import gva


def shard_ranges(lengths, world: int, rank: int):
    """(start, count) per sequence of the positions rank `rank` keeps."""
    L = np.asarray(lengths, dtype=np.int64)
    start = (L * rank) // world
    stop = (L * (rank + 1)) // world
    return start, stop - start


def shard_cache(V, k_rope, seq_offset, seq_len, world: int, rank: int, extra_slots: int = 0):
    """Gather this rank's rows of a full cache into a compact shard (host or device
    tensors); returns (V_r, k_rope_r, seq_offset_r, seq_len_r, start)."""
    L = seq_len.cpu().numpy().astype(np.int64)
    off = seq_offset.cpu().numpy().astype(np.int64)
    start, count = shard_ranges(L, world, rank)
    cap = count + extra_slots
    offs_r = np.concatenate([[0], np.cumsum(cap)[:-1]]).astype(np.int64)
    rows = np.concatenate([np.arange(off[b] + start[b], off[b] + start[b] + count[b])
                           for b in range(len(L))] + [np.zeros(0, dtype=np.int64)])
    dst = np.concatenate([np.arange(offs_r[b], offs_r[b] + count[b]) for b in range(len(L))]
                         + [np.zeros(0, dtype=np.int64)])
    S_r = max(int(cap.sum()), 1)
    V_r = torch.zeros((S_r,) + tuple(V.shape[1:]), dtype=V.dtype, device=V.device)
    K_r = torch.zeros((S_r,) + tuple(k_rope.shape[1:]), dtype=k_rope.dtype, device=k_rope.device)
    if len(rows):
        ri = torch.from_numpy(rows).to(V.device)
        di = torch.from_numpy(dst).to(V.device)
        V_r[di] = V[ri]
        K_r[di] = k_rope[ri]
    return (V_r, K_r, torch.from_numpy(offs_r.astype(np.int32)),
            torch.from_numpy(count.astype(np.int32)), start)


def shard_step_inputs(V, k_rope, seq_offset, hist_len, append, world: int, rank: int):
    """This rank's part of one decode step whose every sequence is split across
    `world` ranks.  The step attends hist_len[b] + 1 rows (the history plus the
    token appended in this step); rank r keeps positions
    [(L+1)*r/world, (L+1)*(r+1)/world) of them, so exactly one rank holds the new
    token's position L = hist_len[b] and appends it there.

    V, k_rope, seq_offset: the full cache (host tensors), with a free slot after
    each sequence's history; append = (v_new, kpe_new, slot, pos) of the B new
    tokens.  Returns (V_r, k_rope_r, seq_offset_r, seq_len_r, append_r, start):
    the compact shard, its step lengths, and the append inputs of the tokens that
    land on this rank with their slots in the shard's layout."""
    L = np.asarray(hist_len, dtype=np.int64)
    step_len = torch.from_numpy((L + 1).astype(np.int32))
    V_r, K_r, off_r, len_r, start = shard_cache(V, k_rope, seq_offset, step_len, world, rank)
    cnt = len_r.numpy().astype(np.int64)
    own = (L >= start) & (L < start + cnt)
    sel = torch.from_numpy(own)
    v_new, kpe_new, _, pos = append
    slot_r = (off_r.numpy().astype(np.int64) + L - start)[own].astype(np.int32)
    append_r = (v_new[sel].contiguous(), kpe_new[sel].contiguous(), torch.from_numpy(slot_r),
                pos[sel].contiguous())
    return V_r, K_r, off_r, len_r, append_r, start


class SequenceSplitMerge:
    """Buffers and calls for the exchange + merge of one decode step.

    `out_part`/`lse_part` receive this rank's normalised output and lse (pass
    them to the decode); `merge()` all-gathers them over `group` (NCCL) and
    writes the merged result into `out`/`lse` with gva_merge_states."""

    def __init__(self, shape: gva.Shape, world: int, device, group=None):
        B, H, d_h = shape.B, shape.H, shape.d_h
        self.shape, self.world, self.group = shape, world, group
        self.outs = torch.empty(world, B, H, d_h, dtype=torch.float32, device=device)
        self.lses = torch.empty(world, B, H, dtype=torch.float32, device=device)
        if world == 1:      # nothing to exchange: decode straight into the merge input
            self.out_part, self.lse_part = self.outs[0], self.lses[0]
        else:
            self.out_part = torch.empty(B, H, d_h, dtype=torch.float32, device=device)
            self.lse_part = torch.empty(B, H, dtype=torch.float32, device=device)

    def exchange(self):
        """All-gather every rank's (out_part, lse_part) into outs/lses, in rank
        order.  The buffers are gathered as flat vectors, which NCCL and gloo both
        accept; with gloo, device buffers go through host copies."""
        if self.world == 1:
            return
        import torch.distributed as dist
        pairs = ((self.outs, self.out_part), (self.lses, self.lse_part))
        if dist.get_backend(self.group) == "gloo" and self.outs.is_cuda:
            for full, part in pairs:
                host = torch.empty(full.numel(), dtype=full.dtype)
                dist.all_gather_into_tensor(host, part.reshape(-1).cpu(), group=self.group)
                full.copy_(host.view(full.shape))
            return
        for full, part in pairs:
            dist.all_gather_into_tensor(full.view(-1), part.view(-1), group=self.group)

    def merge(self, out, lse=None):
        self.exchange()
        gva.merge_states(self.shape, self.outs, self.lses, out, lse)
