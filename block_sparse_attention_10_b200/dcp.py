"""Indexer decode context parallelism: one long-context decode step over G ranks.

The pages report splitting the decode indexer of a long context over GPUs
("vLLM delivers day-0 support for MiniMax-M3.1-Flash", readmex.ai, TL;DR;
"vLLM Adds Day-0 Support for MiniMax-M3.1-Flash on NVIDIA and AMD GPUs",
ainewsbites.com, "Kernel and serving optimizations").  Rank g of G holds the
contiguous block range ``block_ranges(nbmax, G)[g]`` of every sequence's K, V and
index-K caches.  One step:

    msa_dcp_candidates (own range)  -> all-gather of G x [B, Tq, 16] (score, id)
    msa_dcp_merge (same on every rank) -> msa_dcp_attend (own range)
    -> all-gather of G x ([B, Tq, Hq, D] out, [B, Tq, Hq] lse) -> msa_dcp_combine

Every rank ends with the full output of every query; the selection equals the
single-rank msa_decode selection bit for bit (include/msa.h explains why).  This
module only moves data between ranks: the compute is the C ABI's (``CudaOps``).
The collectives are torch.distributed all-gathers (NCCL on GPUs: one
``all_gather_into_tensor`` per exchanged tensor; any other backend gathers into
a list), so every rank issues the same collectives in the same order.  The step
functions are taken from an ``ops`` object so that the exchange can be exercised
on CPU ranks in tests; the library itself has only ``CudaOps`` and no fallback.
"""
from __future__ import annotations

from typing import List, Optional, Tuple

import torch

from . import msa


def block_ranges(nbmax: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous, non-empty, non-overlapping ranges [n0, n1) covering [0, nbmax), one per rank."""
    if world < 1 or world > nbmax:
        raise ValueError(f"cannot split {nbmax} blocks over {world} ranks")
    return [(nbmax * g // world, nbmax * (g + 1) // world) for g in range(world)]


class CudaOps:
    """The four context-parallel steps as calls of libmsa.so."""

    @staticmethod
    def workspace(p: msa.MsaProblem) -> torch.Tensor:
        return torch.empty(msa.msa_dcp_workspace_size(p), dtype=torch.uint8, device=p.q.device)

    @staticmethod
    def candidates(p, n0, n1, ws, cand_score, cand_id, stream=None):
        msa.msa_dcp_candidates(p, n0, n1, ws, cand_score, cand_id, stream)

    @staticmethod
    def merge(p, cand_score_all, cand_id_all, sel, stream=None):
        msa.msa_dcp_merge(p, cand_score_all, cand_id_all, sel, stream)

    @staticmethod
    def attend(p, n0, n1, sel, part_out, part_lse, stream=None):
        msa.msa_dcp_attend(p, n0, n1, sel, part_out, part_lse, stream)

    @staticmethod
    def combine(p, part_out_all, part_lse_all, out, lse, stream=None):
        msa.msa_dcp_combine(p, part_out_all, part_lse_all, out, lse, stream)


def all_gather(t: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """[world, *t.shape]: every rank's t in rank order."""
    import torch.distributed as dist
    out = torch.empty((world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, t.contiguous(), group=group)
    else:
        dist.all_gather(list(out.unbind(0)), t.contiguous(), group=group)
    return out


class DcpDecoder:
    """This rank's share of context-parallel decode steps for one problem shape.

    ``p`` describes the whole problem (all B sequences and Tq query tokens; queries on
    every rank) with caches of which this rank's block range is read.  Buffers are
    allocated once; ``step`` writes the full output (and lse) on every rank."""

    def __init__(self, p: msa.MsaProblem, rank: int, world: int, group=None, ops=CudaOps):
        self.p, self.rank, self.world, self.group, self.ops = p, rank, world, group, ops
        self.n0, self.n1 = block_ranges(p.nbmax, world)[rank]
        B, Tq, Hq, D = p.q.shape
        dev = p.q.device
        self.ws = ops.workspace(p)
        self.cand_score = torch.empty(B, Tq, msa.MSA_TOPK_BLOCKS, dtype=torch.float32, device=dev)
        self.cand_id = torch.empty(B, Tq, msa.MSA_TOPK_BLOCKS, dtype=torch.int32, device=dev)
        self.sel = torch.empty(B, Tq, msa.MSA_TOPK_BLOCKS, dtype=torch.int32, device=dev)
        self.part_out = torch.empty(B, Tq, Hq, D, dtype=torch.float32, device=dev)
        self.part_lse = torch.empty(B, Tq, Hq, dtype=torch.float32, device=dev)

    def step(self, out: torch.Tensor, lse: Optional[torch.Tensor] = None) -> torch.Tensor:
        """One decode step; returns the merged selection [B, Tq, 16] (this rank's buffer)."""
        p, ops = self.p, self.ops
        ops.candidates(p, self.n0, self.n1, self.ws, self.cand_score, self.cand_id)
        cs = all_gather(self.cand_score, self.world, self.group)
        ci = all_gather(self.cand_id, self.world, self.group)
        ops.merge(p, cs, ci, self.sel)
        ops.attend(p, self.n0, self.n1, self.sel, self.part_out, self.part_lse)
        po = all_gather(self.part_out, self.world, self.group)
        pl = all_gather(self.part_lse, self.world, self.group)
        ops.combine(p, po, pl, out, lse)
        return self.sel


def simulate_ranks(p: msa.MsaProblem, world: int, out: torch.Tensor, lse: Optional[torch.Tensor] = None,
                   ops=CudaOps) -> torch.Tensor:
    """All `world` ranks' steps one after another on the current device, with the
    exchanges done by stacking (no collective and no kernel that waits for another):
    what G ranks compute, for tests and for timing one rank's share.  Returns the
    merged selection."""
    ranges = block_ranges(p.nbmax, world)
    B, Tq, Hq, D = p.q.shape
    dev = p.q.device
    ws = ops.workspace(p)
    cs = torch.empty(world, B, Tq, msa.MSA_TOPK_BLOCKS, dtype=torch.float32, device=dev)
    ci = torch.empty(world, B, Tq, msa.MSA_TOPK_BLOCKS, dtype=torch.int32, device=dev)
    for g, (n0, n1) in enumerate(ranges):
        ops.candidates(p, n0, n1, ws, cs[g], ci[g])
    sel = torch.empty(B, Tq, msa.MSA_TOPK_BLOCKS, dtype=torch.int32, device=dev)
    ops.merge(p, cs, ci, sel)
    po = torch.empty(world, B, Tq, Hq, D, dtype=torch.float32, device=dev)
    pl = torch.empty(world, B, Tq, Hq, dtype=torch.float32, device=dev)
    for g, (n0, n1) in enumerate(ranges):
        ops.attend(p, n0, n1, sel, po[g], pl[g])
    ops.combine(p, po, pl, out, lse)
    return sel
