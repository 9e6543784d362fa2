"""Context-parallel KDA prefill: each rank holds one span of the sequences.

aiblin.ru, "Kimi K3 -- открытая модель, которая обошла закрытых лидеров
рынка", section "Как распараллелили последовательное обновление": a span of
tokens acts on its incoming state as an affine map, S_out = M S_in + B (a local
state plus a token-dependent transition matrix), whose size does not depend on
the span's length.  So every GPU computes the map of its own span, one
all-gather shares the maps, and a prefix scan over them gives each GPU the
true state entering its span; the forward pass over the span then needs
nothing more from the others.  Communication per rank is one (M, B) pair per
(sequence, head) -- 128 KiB in fp32 at d = 128 -- whatever the length.

Layout: B sequences split along T into equal, contiguous spans, span r on
rank r of ``group`` (the caller slices; ``[B, T/W, H, *]`` tensors on every
rank).  Every rank passes the same ``initial_state`` (the state entering span
0, or None).  Each rank gets its span's outputs and the state at the end of
its span; on the last rank that is the sequences' final state.

The collective is a plain ``torch.distributed.all_gather`` (NCCL between GPUs);
the kernels are the library's: :func:`kda_span_transition`, then
:func:`kda_apply_transitions` on the gathered maps of the ranks before this
one, then :func:`kda_span_forward` from that state, which reuses the
transition step's per-segment work.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable


@dataclass
class SpanOps:
    """The three per-rank steps.  ``transition(q, k, v, log_alpha, beta)`` returns
    (one tensor to exchange, all ranks the same shape; a context the forward
    step may reuse); ``apply(prior, initial_state)`` takes the stack of the
    earlier ranks' tensors ([r, ...], r may be 0); ``forward(q, k, v,
    log_alpha, beta, s_in, out_gate, context)`` returns (out, end state)."""
    transition: Callable
    apply: Callable
    forward: Callable


def library_ops() -> SpanOps:
    """The library's kernels.  The transition step keeps its segment transitions
    and every chunk's output-pass operands in a workspace, so the forward step
    does not compute them again (kda_span_transition / kda_span_forward)."""
    from . import kda_apply_transitions, kda_span_forward, kda_span_transition, span_workspace

    def transition(q, k, v, log_alpha, beta):
        ws = span_workspace(k)
        return kda_span_transition(q, k, v, log_alpha, beta, ws), ws

    def forward(q, k, v, log_alpha, beta, s_in, out_gate, ws):
        return kda_span_forward(q, k, v, log_alpha, beta, ws, s_in, out_gate=out_gate)

    return SpanOps(transition=transition,
                   apply=lambda prior, s0: kda_apply_transitions(prior, s0),
                   forward=forward)


def cp_prefill(q, k, v, log_alpha, beta, initial_state=None, group=None, out_gate=None,
               ops: SpanOps | None = None):
    """Forward pass of this rank's span; returns (out, state at the span's end)."""
    import torch
    import torch.distributed as dist

    ops = ops or library_ops()
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    trans, ctx = ops.transition(q, k, v, log_alpha, beta)
    gathered = [torch.empty_like(trans) for _ in range(world)]
    dist.all_gather(gathered, trans.contiguous(), group=group)
    prior = torch.stack(gathered[:rank]) if rank else trans.new_empty((0,) + tuple(trans.shape))
    s_in = ops.apply(prior, initial_state)
    return ops.forward(q, k, v, log_alpha, beta, s_in, out_gate, ctx)
