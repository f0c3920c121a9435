"""Data parallelism over a jagged batch: one process per GPU.

Sequences are independent units of HSTU attention, so a batch shards by
sequence with no exchange in the forward.  The backward has one exchange:
the bias tables are parameters shared by every sequence, so each rank's
table gradients are partial sums that are added across ranks.  This module
holds the host side of that: the split (``hstu_partition_batch`` in the C
library balances visible (query, key) pairs per rank), the rank's local view
of the batch, and the single all-reduce of both table gradients.
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np
import torch

from . import ops


def partition(seq_offsets, world: int, num_candidates=None) -> Tuple[np.ndarray, np.ndarray]:
    """(rank_of_seq [B], visible pairs per rank [world]); deterministic."""
    return ops.partition_batch(seq_offsets, world, num_candidates)


def local_sequences(seq_offsets, world: int, rank: int, num_candidates=None) -> np.ndarray:
    """Indices (ascending) of the sequences `rank` owns."""
    rank_of, _ = partition(seq_offsets, world, num_candidates)
    return np.nonzero(rank_of == rank)[0].astype(np.int64)


def local_batch(seq_offsets, seqs: np.ndarray, num_candidates=None):
    """The rank's local batch: (local offsets [b+1], global token index of
    every local token [t], local candidate counts or None).  Gather any
    per-token array with ``a[tokens]``."""
    off = np.asarray(seq_offsets, np.int64)
    lens = off[1:] - off[:-1]
    seqs = np.asarray(seqs, np.int64)
    loc_off = np.concatenate([[0], np.cumsum(lens[seqs])]).astype(np.int64)
    tokens = (np.concatenate([np.arange(off[s], off[s + 1]) for s in seqs]).astype(np.int64)
              if len(seqs) else np.zeros(0, np.int64))
    nc = None if num_candidates is None else np.asarray(num_candidates, np.int32)[seqs]
    return loc_off, tokens, nc


class RabGrads:
    """Both bias-table gradients in one float32 buffer, so the backward's
    exchange is one collective: ``pos`` and ``time`` are views into it, to be
    passed to hstu_attn_bwd as drab_pos / drab_time (which accumulate)."""

    def __init__(self, pos_shape, time_shape, device):
        n_p = int(np.prod(pos_shape))
        n_t = int(np.prod(time_shape))
        self.flat = torch.zeros(n_p + n_t, dtype=torch.float32, device=device)
        self.pos = self.flat[:n_p].view(*pos_shape)
        self.time = self.flat[n_p:].view(*time_shape)

    def zero_(self) -> "RabGrads":
        self.flat.zero_()
        return self

    def all_reduce(self, group: Optional[object] = None) -> "RabGrads":
        """Sum across ranks (one all-reduce; a no-op without a process group)."""
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
            dist.all_reduce(self.flat, group=group)
        return self
