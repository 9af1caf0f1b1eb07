"""Data-parallel sharding of a packed variable-length batch across ranks.

Every (sequence, head) chain of the gated delta rule is independent (the state is per
sequence and per head), so a batch splits across GPUs by whole sequences with no
exchange step: each rank runs gdn_chunk_fwd on its own sequences and the outputs are
simply placed back. Balance is by token count: a chain's time is proportional to its
length.
"""
from __future__ import annotations

import heapq
from typing import List, Sequence, Tuple

import torch

__all__ = ["balance_sequences", "local_batch", "scatter_rows", "gather_rows"]


def balance_sequences(lengths: Sequence[int], world: int) -> List[List[int]]:
    """Assign sequence indices to `world` ranks, longest first onto the least-loaded
    rank (ties by rank index). Returns one sorted index list per rank."""
    if world <= 0:
        raise ValueError("world must be positive")
    heap = [(0, r) for r in range(world)]
    out: List[List[int]] = [[] for _ in range(world)]
    order = sorted(range(len(lengths)), key=lambda i: (-int(lengths[i]), i))
    for i in order:
        load, r = heapq.heappop(heap)
        out[r].append(i)
        heapq.heappush(heap, (load + int(lengths[i]), r))
    return [sorted(x) for x in out]


def local_batch(cu_seqlens: torch.Tensor, seqs: Sequence[int]) -> Tuple[torch.Tensor, torch.Tensor]:
    """Token indices (into the packed batch) and the local cu_seqlens of the given
    sequences, in the order given."""
    cu = [int(x) for x in cu_seqlens.tolist()]
    idx = [torch.arange(cu[s], cu[s + 1], dtype=torch.int64) for s in seqs]
    tokens = torch.cat(idx) if idx else torch.zeros(0, dtype=torch.int64)
    lens = torch.tensor([cu[s + 1] - cu[s] for s in seqs], dtype=torch.int32)
    local_cu = torch.zeros(len(seqs) + 1, dtype=torch.int32)
    if len(seqs):
        local_cu[1:] = torch.cumsum(lens, 0)
    return tokens, local_cu


def scatter_rows(x: torch.Tensor, tokens: torch.Tensor) -> torch.Tensor:
    """The rows of a packed [N_tok, ...] tensor that belong to one rank."""
    return x.index_select(0, tokens.to(x.device))


def gather_rows(parts: Sequence[torch.Tensor], tokens: Sequence[torch.Tensor], n_tok: int) -> torch.Tensor:
    """Inverse of scatter_rows over all ranks: place each rank's rows back."""
    ref = parts[0]
    out = torch.empty((n_tok,) + tuple(ref.shape[1:]), dtype=ref.dtype, device=ref.device)
    for p, t in zip(parts, tokens):
        out.index_copy_(0, t.to(out.device), p)
    return out
