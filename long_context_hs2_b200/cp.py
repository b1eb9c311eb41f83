"""Context-parallel full attention with token selection across ranks.

A context of a million tokens (the case the HySparse2 pages analyse: dpshk.com
explainer, section 05) can be split across G GPUs: rank r holds a contiguous
slice of every sequence's cache -- `L_local` positions starting at global
position `key_pos0` -- and all queries.  One full-attention layer with its
selection is then five library steps and three exchanges (include/hs2.h,
"Context parallelism"):

  1. hs2_cp_attn_partial            O_r, lse_r over the slice
  2. all-gather lse_r; hs2_cp_lse_combine      the global normaliser lse
  3. hs2_cp_rescale O_r; sum all-reduce of O   the layer output O
  4. hs2_cp_select_local            the slice's top-k candidates and scores
  5. all-gather the lists; hs2_cp_merge_select the global selection idx, n_sel

This module is the orchestration only: buffers, the order of the steps, and
the collectives (torch.distributed: NCCL between GPUs; every rank takes the
same collective steps in the same order).  All arithmetic runs in the
library's kernels -- or, for a host-side test of the orchestration, in the
`ops` object the caller passes (the same five steps, on host tensors).
"""

from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import (hs2_cp_attn_partial, hs2_cp_lse_combine, hs2_cp_merge_select, hs2_cp_rescale,
               hs2_cp_select_local, hs2_cp_workspace)


@dataclass
class CpSlice:
    """This rank's slice of the context and the query positions (global)."""
    B: int
    T: int
    H: int
    D: int
    L_local: int      # positions held by this rank
    key_pos0: int     # global position of this rank's first position
    q_pos0: int       # global position of query 0 (queries at q_pos0 .. q_pos0 + T - 1)
    scale: float
    topk: int = 1024
    window: int = 128


class LibraryOps:
    """The five steps on this rank's GPU (libhs2)."""

    def __init__(self, dt: int):
        self.dt = dt
        self._ws = None

    def workspace(self, s: CpSlice, device):
        n = hs2_cp_workspace(s.B, s.T, s.L_local, s.H, s.D, s.topk, s.window, self.dt)
        if n == 0:
            raise ValueError("unsupported context-parallel slice")
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.empty(n, dtype=torch.uint8, device=device)
        return self._ws, n

    def partial(self, q, kv, s: CpSlice, o, lse):
        ws, n = self.workspace(s, q.device)
        hs2_cp_attn_partial(q, kv, s.B, s.T, s.L_local, s.q_pos0 - s.key_pos0, s.H, s.D, s.scale,
                            self.dt, o, lse, ws, n)

    def lse_combine(self, lse_parts, lse):
        hs2_cp_lse_combine(lse_parts, lse_parts.shape[0], lse.numel(), lse)

    def rescale(self, o, lse_part, lse):
        hs2_cp_rescale(o, lse_part, lse, lse.numel(), o.shape[-1])

    def select_local(self, q, kv, s: CpSlice, lse, cand_score, cand_idx):
        ws, n = self.workspace(s, q.device)
        hs2_cp_select_local(q, kv, s.B, s.T, s.L_local, s.q_pos0 - s.key_pos0, s.key_pos0, s.H, s.D,
                            s.scale, s.topk, s.window, self.dt, lse, cand_score, cand_idx, ws, n)

    def merge_select(self, cand_scores, cand_idxs, s: CpSlice, idx, n_sel):
        hs2_cp_merge_select(cand_scores, cand_idxs, cand_scores.shape[0], s.B, s.T, s.q_pos0,
                            s.topk, s.window, idx, n_sel)


def _all_gather(t, world, group):
    """[world, *t.shape] tensor of every rank's t (rank order)."""
    out = torch.empty((world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
    dist.all_gather(list(out.unbind(0)), t, group=group)
    return out


def cp_full_attn_select(q, kv, s: CpSlice, ops, group=None):
    """One context-parallel full-attention layer with selection on this rank.

    q: this layer's queries [B, T, H, D] (every rank holds all of them); kv:
    this rank's slice in the form `ops` takes.  Returns (O [B, T, H, D],
    lse [B, T, H], idx [B, T, topk + window], n_sel [B, T]), identical on every
    rank.
    """
    world = dist.get_world_size(group)
    dev = q.device
    fdt = getattr(ops, "float_dtype", torch.float32)   # the library's outputs are fp32
    o = torch.empty(s.B, s.T, s.H, s.D, dtype=fdt, device=dev)
    lse_part = torch.empty(s.B, s.T, s.H, dtype=fdt, device=dev)
    ops.partial(q, kv, s, o, lse_part)                                  # 1
    lse = torch.empty_like(lse_part)
    ops.lse_combine(_all_gather(lse_part, world, group), lse)           # 2
    ops.rescale(o, lse_part, lse)                                       # 3
    dist.all_reduce(o, op=dist.ReduceOp.SUM, group=group)
    cand_score = torch.empty(s.B, s.T, s.topk, dtype=fdt, device=dev)
    cand_idx = torch.empty(s.B, s.T, s.topk, dtype=torch.int32, device=dev)
    ops.select_local(q, kv, s, lse, cand_score, cand_idx)               # 4
    idx = torch.empty(s.B, s.T, s.topk + s.window, dtype=torch.int32, device=dev)
    n_sel = torch.empty(s.B, s.T, dtype=torch.int32, device=dev)
    ops.merge_select(_all_gather(cand_score, world, group),             # 5
                     _all_gather(cand_idx, world, group), s, idx, n_sel)
    return o, lse, idx, n_sel
