"""Sequence (context) parallel forward and backward of the WKV7 recurrence over
a process group.

One long sequence is cut into contiguous stretches, stretch i on rank i (rank
order = time order).  The recurrence S_t = S_{t-1} (diag(w_t) + a_t b_t^T) +
v_t k_t^T is affine in the state, because the transition does not depend on S
(RWKV-7 "Goose" paper review, section "Architecture"): a stretch maps its entry
state to its final state as S_out = S_in M + E.  So each rank

  1. computes the summary [E; M] of its own stretch (wkv7_forward_summary: the
     stretch's segments run side by side, each carrying one state from S = 0
     and one from S = I with v read as 0, and their summaries are chained
     into E and M);
  2. all-gathers the summaries (2 B H N^2 fp32 per rank: 1 MiB for B = 1,
     H = 32, N = 64);
  3. composes the entry state of every stretch (wkv7_compose_states), which
     also yields the final state of the whole sequence on every rank;
  4. runs its stretch from that entry state (wkv7_forward_continue, which
     reuses the segment summaries of step 1 kept in the workspace).

The backward takes the same steps in reverse.  The state gradient is affine in
dL/dS_out too, dL/dS_in = dL/dS_out M^T + F with F the stretch's own part, so
each rank

  1. sweeps its stretch for F (wkv7_state_gradient with dL/dS_out = 0: a
     reverse pass over r, w, a, b and dy alone);
  2. all-gathers the F's (B H N^2 fp32 per rank);
  3. composes dL/dS after every stretch from the forward's summaries, last
     stretch first (wkv7_compose_adjoints);
  4. runs its stretch's backward from its entry state with that dL/dS_out.

Each exchange is one small all-gather, latency-bound whatever carries it, so it
goes through the process group's collective (NCCL over NVLink on GPUs, gloo on
CPU in tests).  The per-rank compute is injectable (``ops``) so the host
logic can be tested on CPU against a reference implementation.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Optional

import torch
import torch.distributed as dist


@dataclass
class StretchOps:
    """The per-rank computations the orchestration needs.  Forward:

    summary(r, w, k, v, a, b) -> ([2, B, H, N, N] fp32 [E; M], ctx)
    compose(summaries [n, 2, B, H, N, N], s0 or None) -> states [n + 1, B, H, N, N]
    forward(r, w, k, v, a, b, s_in, ctx) -> y [B, T, H, N]

    ``ctx`` is whatever summary() keeps for forward() (the CUDA path's
    workspace with the segment summaries).  Backward (optional):

    state_gradient(r, w, a, b, dy) -> F [B, H, N, N] (dL/dS_in at dL/dS_out = 0)
    compose_adjoints(summaries, F [n, B, H, N, N], dsT or None)
        -> adj [n + 1, B, H, N, N], adj[k] = dL/dS before stretch k
    backward(r, w, k, v, a, b, s_in, dy, ds_out) -> (dr, dw, dk, dv, da, db, ds_in)
    """
    summary: Callable
    compose: Callable
    forward: Callable
    state_gradient: Optional[Callable] = None
    compose_adjoints: Optional[Callable] = None
    backward: Optional[Callable] = None


def cuda_ops(y_dtype: Optional[torch.dtype] = None, grad_dtype: torch.dtype = torch.float32,
             stream=None) -> StretchOps:
    """The library's kernels (through the C ABI) on the current CUDA device."""
    from . import wkv7

    def summary(r, w, k, v, a, b):
        B, T, H, N = r.shape
        nbytes = wkv7.forward_summary_workspace_size(B, T, H, N)
        ws = torch.empty(nbytes, dtype=torch.uint8, device=r.device) if nbytes else None
        return wkv7.forward_summary(r, w, k, v, a, b, workspace=ws, stream=stream), ws

    def forward(r, w, k, v, a, b, s_in, ws):
        return wkv7.forward_continue(r, w, k, v, a, b, s_in, workspace=ws, y_dtype=y_dtype, stream=stream)

    def backward(r, w, k, v, a, b, s_in, dy, ds_out):
        return wkv7.backward(r, w, k, v, a, b, s_in, dy, ds_out, grad_dtype=grad_dtype, stream=stream)

    return StretchOps(summary=summary, compose=lambda sums, s0: wkv7.compose_states(sums, s0, stream=stream),
                      forward=forward,
                      state_gradient=lambda r, w, a, b, dy: wkv7.state_gradient(r, w, a, b, dy, stream=stream),
                      compose_adjoints=lambda sums, F, dsT: wkv7.compose_adjoints(sums, F, dsT, stream=stream),
                      backward=backward)


def _gather(x, world, group):
    """[world, *x.shape]: every rank's x in rank order (x itself at world 1)."""
    x = x.contiguous()
    if world == 1:
        return x[None]
    parts = [torch.empty_like(x) for _ in range(world)]
    dist.all_gather(parts, x, group=group)
    return torch.stack(parts)


def _world_rank(group):
    if not dist.is_initialized():
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


def forward_context_parallel(r, w, k, v, a, b, s0=None, *, ops: Optional[StretchOps] = None, group=None,
                             return_summaries: bool = False):
    """Forward of this rank's stretch [B, T_i, H, N] of a sequence split over the
    ranks of ``group`` in rank order.

    ``s0`` is the state before the first token of the whole sequence; pass the
    same tensor (or None for zeros) on every rank.  Stretch lengths may differ
    between ranks, including 0.  Returns (y of this stretch, the entry state of
    this stretch, the final state of the whole sequence), and with
    ``return_summaries`` also every stretch's summary [world, 2, B, H, N, N]
    (what backward_context_parallel needs).
    """
    ops = ops or cuda_ops()
    world, rank = _world_rank(group)
    summary, ctx = ops.summary(r, w, k, v, a, b)
    summaries = _gather(summary, world, group)
    states = ops.compose(summaries, s0)
    s_in = states[rank].contiguous()
    y = ops.forward(r, w, k, v, a, b, s_in, ctx)
    if return_summaries:
        return y, s_in, states[world], summaries
    return y, s_in, states[world]


def backward_context_parallel(r, w, k, v, a, b, s_in, summaries, dy, dsT=None, *,
                              ops: Optional[StretchOps] = None, group=None):
    """Gradients for this rank's stretch of a sequence split over ``group`` in
    rank order, of L = sum(dy * y) over the whole sequence + sum(dsT * S_T)
    (S_T the state after the last token; ``dsT`` the same tensor or None on
    every rank).

    ``s_in`` and ``summaries`` are what forward_context_parallel returned on
    this rank (the stretch's entry state; all stretches' summaries).  Returns
    (dr, dw, dk, dv, da, db of this stretch, dL/dS_0 of the whole sequence)
    where S_0 is the state before its first token: the same on every rank.
    """
    ops = ops or cuda_ops()
    world, rank = _world_rank(group)
    if summaries.shape[0] != world:
        raise ValueError(f"{summaries.shape[0]} summaries for {world} ranks")
    F = _gather(ops.state_gradient(r, w, a, b, dy), world, group)
    adj = ops.compose_adjoints(summaries, F, dsT)
    grads = ops.backward(r, w, k, v, a, b, s_in, dy, adj[rank + 1].contiguous())
    return (*grads[:6], adj[0])


def split_lengths(T: int, world: int, chunk: int = 32) -> list:
    """Stretch lengths for ``world`` ranks: whole chunks of ``chunk`` tokens,
    as even as possible (earlier ranks take the extra chunks), with the ragged
    tail in the last non-empty stretch."""
    chunks = -(-T // chunk)
    base, extra = divmod(chunks, world)
    ends, c = [], 0
    for i in range(world):
        c += base + (1 if i < extra else 0)
        ends.append(min(T, c * chunk))
    return [e - s for s, e in zip([0] + ends[:-1], ends)]
