"""Context-parallel absorbed decode: split-KV across devices, one process per GPU.

Every rank holds a contiguous slice of each sequence's positions in its own latent cache, runs the
absorbed decode (mla_decode_absorbed) over that slice, and the ranks' partial results are merged by
their log-sum-exp (mla_lse_merge): the softmax over the union of disjoint slices, restated from the
per-slice maxima and sums ("ferrox-core src/mla_absorbed.rs", the body of
causal_mla_absorbed_attention: max-subtracted exponentials, their sum, the weighted sum of rows). The
split is worth it where one sequence's cache is long: the cache size does not depend on the head
count and generation is bandwidth-bound ("preacher-1/MLA_tutorial formula.md", Part 3, the note
after the inference form), so each device streams 1/world of the bytes.

Partition (a reading: the pages fix none): sequence b of T_b positions is cut at
floor(r * T_b / world) for r = 1 .. world-1, each cut lowered to at most T_b - n_q, so the last
rank always holds the n_q newest positions, the queries' own. Under the causal rule query j sees
positions t <= T_b - n_q + j: every position of the other ranks is visible to every query, and the
last rank's slice obeys the same rule relative to its own length. Only the last rank therefore
decodes with MLA_DECODE_CAUSAL.

Exchange. ``transport="nccl"``: an all-gather of the partial (out_lat, lse) of every rank
(torch.distributed), then one merge kernel on the gathered copies. ``transport="p2p"``: the partials
live in symmetric memory and the merge kernel loads the peers' partials directly over NVLink (the
merge is the exchange); a device-side barrier before the merge makes the peers' partials complete,
and one after it keeps them from being overwritten while a peer still reads them.

The merged result is the same on every rank (every rank merges all query rows).
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch
import torch.distributed as dist

from . import mla as M


def slice_bounds(seqlens, n_q: int, world: int) -> np.ndarray:
    """Cut points [world + 1, B]: rank r holds positions bounds[r, b] .. bounds[r + 1, b] of sequence b."""
    T = np.asarray(seqlens, dtype=np.int64).reshape(1, -1)
    if world < 1:
        raise ValueError("world must be >= 1")
    if np.any(T < n_q):
        raise ValueError("every sequence must hold its n_q query tokens")
    r = np.arange(world + 1, dtype=np.int64).reshape(-1, 1)
    b = (r * T) // world
    b[1:world] = np.minimum(b[1:world], T - n_q)
    return b


def local_slice(seqlens, n_q: int, world: int, rank: int):
    """(first position, end position, length) per sequence of this rank's slice, and whether the
    rank decodes with the causal rule (the last rank only)."""
    b = slice_bounds(seqlens, n_q, world)
    lo, hi = b[rank], b[rank + 1]
    return lo, hi, hi - lo, rank == world - 1


class ContextParallelDecode:
    """One rank's part of a context-parallel decode step over resident slices of the latent cache.

    cache_slice: this rank's rows, sequence after sequence (the local_slice() lengths, packed).
    ``__call__(q_abs, out_lat, lse)``: q_abs [B * n_q, H, d_c + d_r] (the same on every rank);
    out_lat [B * n_q, H, d_c] fp32 and lse [B * n_q, H] receive the merged result."""

    def __init__(self, d: M.mla_dims, batch: int, n_q: int, seqlens, cache_slice: torch.Tensor,
                 group=None, causal: bool = True, transport: str = "nccl"):
        if transport not in ("nccl", "p2p"):
            raise ValueError("transport is 'nccl' or 'p2p'")
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.d, self.batch, self.n_q, self.causal, self.transport = d, batch, n_q, causal, transport
        lo, hi, lens, last = local_slice(seqlens, n_q, self.world, self.rank)
        self.lens = lens
        self.flags = M.MLA_DECODE_CAUSAL if (causal and last) else 0
        self.max_local = int(lens.max()) if lens.size else 0
        dev = cache_slice.device
        self.cache = cache_slice
        if cache_slice.shape[0] != int(lens.sum()):
            raise ValueError("cache_slice must hold exactly this rank's slice of every sequence")
        self.cu = torch.from_numpy(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)).to(dev)
        nq = batch * n_q
        H, dc = d.n_heads, d.kv_lora_rank
        self.n_o = nq * H * dc
        if transport == "p2p":
            import torch.distributed._symmetric_memory as symm_mem
            self.symm = symm_mem.empty(self.n_o + nq * H, dtype=torch.float32, device=dev)
            self.handle = symm_mem.rendezvous(self.symm, group if group is not None else dist.group.WORLD)
            self.o_part = self.symm[:self.n_o].view(nq, H, dc)
            self.l_part = self.symm[self.n_o:].view(nq, H)
        else:
            self.o_part = torch.empty(nq, H, dc, dtype=torch.float32, device=dev)
            self.l_part = torch.empty(nq, H, dtype=torch.float32, device=dev)
            self.o_all = torch.empty(self.world, nq, H, dc, dtype=torch.float32, device=dev)
            self.l_all = torch.empty(self.world, nq, H, dtype=torch.float32, device=dev)
        self.ws: Optional[torch.Tensor] = None

    # -- the three steps; the CPU tests of the host logic replace the first and the last --------
    def decode_slice(self, q_abs: torch.Tensor) -> None:
        """This rank's slice through the library's decode, into (o_part, l_part)."""
        if self.ws is None:
            self.ws = M.workspace(M.mla_decode_workspace_size(self.d, q_abs.dtype, self.batch, self.n_q,
                                                              self.max_local, self.cache.shape[0], self.flags),
                                  self.cache.device)
        M.mla_decode_absorbed(self.d, q_abs, self.cache, self.cu, self.batch, self.n_q, self.max_local,
                              self.flags, self.o_part, self.l_part, self.ws)

    def exchange(self):
        """Make every rank's partials readable here; returns (out_lat parts, lse parts) as lists whose
        entries are tensors (nccl) or device addresses (p2p), in rank order."""
        if self.transport == "nccl":
            dist.all_gather(list(self.o_all.unbind(0)), self.o_part, group=self.group)
            dist.all_gather(list(self.l_all.unbind(0)), self.l_part, group=self.group)
            return list(self.o_all.unbind(0)), list(self.l_all.unbind(0))
        self.handle.barrier(channel=0)
        ptrs = [int(p) for p in self.handle.buffer_ptrs]
        return ptrs, [p + 4 * self.n_o for p in ptrs]

    def merge(self, o_parts, l_parts, out_lat: torch.Tensor, lse: Optional[torch.Tensor]) -> None:
        M.mla_lse_merge(self.d, o_parts, l_parts, 0, self.batch * self.n_q, out_lat, lse)

    def __call__(self, q_abs: torch.Tensor, out_lat: torch.Tensor, lse: Optional[torch.Tensor] = None):
        self.decode_slice(q_abs)
        o_parts, l_parts = self.exchange()
        self.merge(o_parts, l_parts, out_lat, lse)
        if self.transport == "p2p":
            self.handle.barrier(channel=1)     # peers have finished reading this rank's partials
        return out_lat
