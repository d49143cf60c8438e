"""Prefill of one long prompt split across GPUs: one token range per rank.

The gated delta rule is affine in its state (Jet-Nemotron paper, section
2.3), so every range can run at once from a zero start; what the ranges
exchange is small and fixed in size:
  1. the conv's halo: each range needs the last three raw V tokens of the
     range before it (all-gathered, [B,3,H,dv] per rank);
  2. each range's end state E [B,H,dv,dk] and transition A [B,H,dk,dk]
     (all-gathered: 1.6 MB per rank at the 2B shapes);
  3. every rank composes all start states from the pairs (the library's
     tensor-core compose, so every rank also holds the final state) and adds
     its range's start-state term to its outputs.
The first range starts from the caller's state for real and skips step 3's
correction. Every rank takes the same collective steps in the same order.

The library's three calls are reached through `LibraryOps`; a test can pass
other ops (e.g. the float64 oracle on CPU tensors with a gloo group) to check
the exchange itself.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import jet_gdn_range_compose, jet_gdn_range_correct, jet_jetblock_prefill_range


class LibraryOps:
    """The library calls of a range (tensors on the rank's GPU)."""

    @staticmethod
    def range_pass(x, W1, W2, q, k, v, g, beta, hist_in, S0, first):
        """-> (o, E, A, Qe); A and Qe are None for the first range."""
        return jet_jetblock_prefill_range(x, W1, W2, q, k, v, g, beta, hist_in, None, S0, first)

    @staticmethod
    def compose(E_all, A_all):
        """E_all [R,B,H,dv,dk], A_all [R,B,H,dk,dk] -> (start states [R,...], final state)."""
        return jet_gdn_range_compose(E_all, A_all)

    @staticmethod
    def correct(Qe, S_start, o):
        return jet_gdn_range_correct(Qe, S_start, o)


def _all_gather(t: torch.Tensor, group) -> torch.Tensor:
    world = dist.get_world_size(group)
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.stack(parts)


def sequence_parallel_prefill(x, W1, W2, q, k, v, g, beta, S0=None, hist_in=None, group=None, ops=LibraryOps):
    """This rank's range of a prompt split across the ranks of `group`, in
    rank order: x [B,T_r,D], q, k [B,T_r,H,dk], v [B,T_r,H,dv] (raw), g, beta
    [B,T_r,H] (ranges may differ in length; each holds at least 3 tokens).
    S0 and hist_in: the sequence's initial state and conv history (read by
    rank 0 only; None = zeros). Returns (o [B,T_r,H,dv] final outputs of the
    range, S [B,H,dv,dk] the state after the whole prompt, hist [B,3,H,dv]
    the conv history after the whole prompt), the last two on every rank."""
    if v.shape[1] < 3:
        raise ValueError("every range needs at least 3 tokens (the conv's reach)")
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    # 1. halo: the last three raw V tokens of every range
    tails = _all_gather(v[:, -3:], group)                       # [R,B,3,H,dv]
    halo = hist_in if rank == 0 else tails[rank - 1]
    # 2. the range from its start (rank 0: the sequence's real start)
    first = rank == 0
    o, E, A, Qe = ops.range_pass(x, W1, W2, q, k, v, g, beta, halo, S0 if first else None, first)
    if world == 1:
        return o, E, tails[-1]
    if A is None:                                              # rank 0 sends a placeholder transition
        B, H, dv, dk = E.shape
        A = torch.zeros((B, H, dk, dk), dtype=E.dtype, device=E.device)
    # 3. the pairs of every range, composed into every start state and the final state
    E_all = _all_gather(E, group)
    A_all = _all_gather(A, group)
    S_start, S_final = ops.compose(E_all, A_all)
    if not first:
        o = ops.correct(Qe, S_start[rank], o)
    return o, S_final, tails[-1]
