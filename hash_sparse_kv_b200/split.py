"""Token-split decode step: one long sequence's cache cut across ranks.

Rank r of G holds the contiguous token range [r0, r1) of a sequence of N
tokens (ranks in token order) -- its K, V and key codes -- and a copy of the
query.  One decode step takes two exchanges (all-gathers):

1. every rank encodes the query heads and takes its own top-k over its range
   (hkv_retrieve_topk; every token of the sequence's top-k is in its own
   rank's top-k); the ranks all-gather those candidates (index, distance);
2. every rank keeps its share of the sequence's top-k (hkv_split_select) and
   attends its own rows -- the selected ones plus the part of the sink and of
   the local window it holds (hkv_sparse_attend); the ranks all-gather the
   partial (out, lse) and merge them (hkv_lse_merge_n).

The result equals the single-GPU decode step over the whole sequence: the
same index set, and attention over the same rows up to rounding.  The
collectives run on torch.distributed (NCCL between GPUs).  The arithmetic
runs in the library's kernels; ``ops`` exists so that the exchange protocol
can be exercised with other implementations of the same five steps.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


def token_range(N: int, world: int, rank: int):
    """[r0, r1): rank's contiguous share of N tokens (sizes differ by at most one)."""
    return rank * N // world, (rank + 1) * N // world


def local_window(N: int, n_sink: int, n_local: int, r0: int, r1: int):
    """(sink, local) counts of the range [r0, r1) such that the library's
    window over the range's n = r1 - r0 tokens -- sink [0, sink), candidates
    [sink, n - local), local [n - local, n) -- is the intersection of the
    sequence's window with the range."""
    n = r1 - r0
    sink_end = min(n_sink, N)
    local_start = max(sink_end, N - n_local)
    sink = min(max(sink_end - r0, 0), n)
    local = min(max(r1 - local_start, 0), n)
    return sink, local


class LibraryOps:
    """The five steps in the library's kernels."""

    def __init__(self):
        import hash_sparse_kv_b200 as hkv
        self.hkv = hkv

    def encode_queries(self, h, q, q_codes):
        self.hkv.hkv_encode_keys(h, q.reshape(-1, q.shape[-1]), q_codes.view(-1, q_codes.shape[-1]))

    def retrieve(self, q_codes, k_codes, n, sink, local, idx, dist, ws, status):
        self.hkv.hkv_retrieve_topk(q_codes, k_codes, n, sink, local, idx.shape[-1], idx, dist, ws=ws, status=status)

    def select(self, rank, Hq, code_bits, cand_idx, cand_dist, idx, status):
        self.hkv.hkv_split_select(rank, Hq, code_bits, cand_idx, cand_dist, idx, status=status)

    def attend(self, q, K, V, n, idx, sink, local, out, lse, scale, ws, status):
        self.hkv.hkv_sparse_attend(q, K, V, n, idx, sink, local, out, lse=lse, scale=scale, ws=ws, status=status)

    def merge(self, o, lse, out, lse_out):
        self.hkv.hkv_lse_merge_n(o, lse, out, lse_out)


@dataclasses.dataclass
class SplitState:
    """Per-rank buffers of one shape (reused across steps)."""

    world: int
    rank: int
    q_codes: torch.Tensor    # [B, Hq, W]
    own_idx: torch.Tensor    # [B, Hkv, k] this rank's top-k (local indices)
    own_dist: torch.Tensor   # [B, Hkv, k]
    cand_idx: torch.Tensor   # [G, B, Hkv, k] every rank's top-k
    cand_dist: torch.Tensor  # [G, B, Hkv, k]
    sel_idx: torch.Tensor    # [B, Hkv, k] this rank's share of the sequence's top-k
    part_out: torch.Tensor   # [B, Hq, 128]
    part_lse: torch.Tensor   # [B, Hq]
    all_out: torch.Tensor    # [G, B * Hq, 128]
    all_lse: torch.Tensor    # [G, B * Hq]
    ws_retrieve: Optional[torch.Tensor]
    ws_attend: Optional[torch.Tensor]
    status: Optional[torch.Tensor]

    @staticmethod
    def make(world, rank, B, Hq, Hkv, code_bits, top_k, N, n_sink, n_local, device, workspaces=True):
        """Buffers of rank `rank`; with `workspaces`, the library's workspaces
        for its range and a status word."""
        W = code_bits // 32
        i32 = dict(dtype=torch.int32, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        ws_r = ws_a = status = None
        if workspaces:
            import hash_sparse_kv_b200 as hkv
            r0, r1 = token_range(N, world, rank)
            sink, local = local_window(N, n_sink, n_local, r0, r1)
            ws_r = hkv.workspace(B, Hq, Hkv, r1 - r0, code_bits, top_k, sink, local, device=device)
            ws_a = hkv.workspace(B, Hq, Hkv, r1 - r0, code_bits, top_k, sink, local, device=device)
            status = hkv.status_word(device)
        return SplitState(world, rank, torch.zeros(B, Hq, W, **i32), torch.zeros(B, Hkv, top_k, **i32),
                          torch.zeros(B, Hkv, top_k, **i32), torch.zeros(world, B, Hkv, top_k, **i32),
                          torch.zeros(world, B, Hkv, top_k, **i32), torch.zeros(B, Hkv, top_k, **i32),
                          torch.zeros(B, Hq, 128, **f32), torch.zeros(B, Hq, **f32),
                          torch.zeros(world, B * Hq, 128, **f32), torch.zeros(world, B * Hq, **f32), ws_r, ws_a,
                          status)


def phase_candidates(ops, st: SplitState, q_hash, q, k_codes, N, n_sink, n_local):
    """Step 1 on one rank: query codes and the rank's own top-k."""
    r0, r1 = token_range(N, st.world, st.rank)
    sink, local = local_window(N, n_sink, n_local, r0, r1)
    ops.encode_queries(q_hash, q, st.q_codes)
    ops.retrieve(st.q_codes, k_codes, r1 - r0, sink, local, st.own_idx, st.own_dist, st.ws_retrieve, st.status)


def phase_attend(ops, st: SplitState, q, K, V, N, n_sink, n_local, code_bits, scale):
    """Step 2 on one rank, after the candidates were gathered: its share of
    the selection and its partial attention."""
    r0, r1 = token_range(N, st.world, st.rank)
    sink, local = local_window(N, n_sink, n_local, r0, r1)
    ops.select(st.rank, q.shape[1], code_bits, st.cand_idx, st.cand_dist, st.sel_idx, st.status)
    ops.attend(q, K, V, r1 - r0, st.sel_idx, sink, local, st.part_out, st.part_lse, scale, st.ws_attend, st.status)


def phase_merge(ops, st: SplitState, out, lse=None):
    """Step 3 on one rank, after the partials were gathered."""
    B, Hq, d = out.shape
    ops.merge(st.all_out, st.all_lse, out.view(B * Hq, d), None if lse is None else lse.view(B * Hq))


def decode_step_split(st: SplitState, q_hash, q, k_codes, K, V, N: int, n_sink: int, n_local: int, code_bits: int,
                      out, lse=None, scale: Optional[float] = None, group=None, ops=None) -> None:
    """One decode step of this rank (see the module docstring).  k_codes, K,
    V hold the rank's token range token_range(N, world, rank) from row 0."""
    import torch.distributed as dist
    r0, r1 = token_range(N, st.world, st.rank)
    for name, t in (("k_codes", k_codes), ("K", K), ("V", V)):
        if t.shape[2] < r1 - r0:
            raise ValueError(f"{name} holds {t.shape[2]} tokens; rank {st.rank} of {st.world} owns {r1 - r0} "
                             f"(tokens [{r0}, {r1}) of {N})")
    if st.cand_idx.shape[0] != st.world or tuple(st.own_idx.shape) != tuple(st.cand_idx.shape[1:]):
        raise ValueError("split state was made for another world size or shape")
    ops = ops or LibraryOps()
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    # flat views: every backend takes a 1-D concatenation of the ranks' parts
    phase_candidates(ops, st, q_hash, q, k_codes, N, n_sink, n_local)
    dist.all_gather_into_tensor(st.cand_idx.view(-1), st.own_idx.view(-1), group=group)
    dist.all_gather_into_tensor(st.cand_dist.view(-1), st.own_dist.view(-1), group=group)
    phase_attend(ops, st, q, K, V, N, n_sink, n_local, code_bits, scale)
    dist.all_gather_into_tensor(st.all_out.view(-1), st.part_out.view(-1), group=group)
    dist.all_gather_into_tensor(st.all_lse.view(-1), st.part_lse.view(-1), group=group)
    phase_merge(ops, st, out, lse)
