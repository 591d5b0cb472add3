"""Sequence-sharded evaluation of the GLA layer: one contiguous segment of the
sequence per rank, rank order = sequence order.

The state recurrence S_t = diag(alpha_t) S_{t-1} + k_t^T v_t is affine in the
entering state, so a segment maps an entering state X to diag(a) X + U, with
a = exp(sum of log alpha over the segment) per key channel and U the segment's
end state from a zero start. Each rank computes its summary (a, U) with the
library's kernels, the summaries are all-gathered (NCCL over NVLink into every
GPU's own memory on a GPU process group; gloo on CPU), and the library's
combine kernel gives each rank the state entering its segment; the forward then
runs once more from that state. The backward mirrors it: (a, W) with W the
gradient a segment sends to its entering state when nothing arrives at its end,
combined in reverse order into the gradient arriving at each segment's end.
The pages carry the recurrent state across training segments ("Gated Linear
Attention Transformers with Hardware-Efficient Training", atlas.scime.ai
summary, "Measured effects": truncated BPTT over 2K segments); here the
segments are shards of one sequence on different devices.

Every arithmetic step runs in the library's kernels (gla_fwd_final_state and
gla_bwd_initial_grad for the summaries where the tensor-core path serves them,
else gla_fwd and gla_bwd; gla_segment_decay; gla_state_combine); this module
moves tensors and calls the collective. The phases are separate functions so that a caller (or a test) can
run several shards on one device in turn.
"""
from __future__ import annotations

import ctypes
from typing import Callable, List, Optional, Sequence

import torch

from . import _lib, gla_bwd, gla_bwd_initial_grad, gla_fwd, gla_fwd_final_state, gate_shape, make_desc
from ._lib import load

__all__ = ["segment_decay", "state_combine", "summary_fwd", "finish_fwd", "summary_bwd", "finish_bwd",
           "SeqShard"]


def _stream(dev):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def segment_decay(log_a: torch.Tensor, B: int, H: int, L: int, Dk: int, gate: str = "channel", tau: float = 0.0,
                  out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """a[B,H,Dk] = exp(sum over the L steps of log alpha) for the gate argument of kind `gate`."""
    lib = load()
    dev = log_a.device
    if tuple(log_a.shape) != tuple(gate_shape(gate, B, H, L, Dk)) or log_a.dtype != torch.float32:
        raise ValueError("log_a has shape %s, expected %s fp32" % (tuple(log_a.shape), gate_shape(gate, B, H, L, Dk)))
    if out is None:
        out = torch.empty(B, H, Dk, dtype=torch.float32, device=dev)
    desc = make_desc(B, H, L, Dk, 4, "bf16", gate=gate, tau=tau)
    with torch.cuda.device(dev):
        st = lib.gla_segment_decay(ctypes.byref(desc), ctypes.c_void_p(log_a.data_ptr()),
                                   ctypes.c_void_p(out.data_ptr()), _stream(dev))
    if st != _lib.GLA_OK:
        raise _lib.GlaError(st, "gla_segment_decay")
    return out


def state_combine(a_all: torch.Tensor, U_all: torch.Tensor, r: int, init: Optional[torch.Tensor] = None,
                  reverse: bool = False, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The state entering segment r (reverse=False) or the gradient arriving at its end (reverse=True)
    from the G summaries a_all [G,B,H,Dk] and U_all [G,B,H,Dk,Dv] (fp32, contiguous)."""
    lib = load()
    G, B, H, Dk = a_all.shape
    Dv = U_all.shape[-1]
    if tuple(U_all.shape) != (G, B, H, Dk, Dv) or not (a_all.is_contiguous() and U_all.is_contiguous()):
        raise ValueError("summaries must be contiguous [G,B,H,Dk] and [G,B,H,Dk,Dv]")
    if init is not None and (tuple(init.shape) != (B, H, Dk, Dv) or not init.is_contiguous()):
        raise ValueError("init must be a contiguous [B,H,Dk,Dv] tensor")
    if out is None:
        out = torch.empty(B, H, Dk, Dv, dtype=torch.float32, device=a_all.device)
    dev = a_all.device
    with torch.cuda.device(dev):
        st = lib.gla_state_combine(G, B * H, Dk, Dv, ctypes.c_void_p(a_all.data_ptr()),
                                   ctypes.c_void_p(U_all.data_ptr()),
                                   None if init is None else ctypes.c_void_p(init.data_ptr()), int(r),
                                   1 if reverse else 0, ctypes.c_void_p(out.data_ptr()), _stream(dev))
    if st != _lib.GLA_OK:
        raise _lib.GlaError(st, "gla_state_combine")
    return out


# ---- the phases of one rank ---------------------------------------------------------------------
def summary_fwd(q, k, v, log_a, gate="channel", tau=0.0, **kw):
    """(a, U) of this segment: its decay and its end state from a zero start (the state walk alone where
    the library has it, else a full forward)."""
    B, H, L, Dk = q.shape
    try:
        U = gla_fwd_final_state(q, k, v, log_a, None, gate=gate, tau=tau, **kw)
    except _lib.GlaError as e:
        if e.status != _lib.GLA_ERR_UNSUPPORTED:
            raise
        _, U = gla_fwd(q, k, v, log_a, None, gate=gate, tau=tau, **kw)
    return segment_decay(log_a, B, H, L, Dk, gate, tau), U


def finish_fwd(q, k, v, log_a, a_all, U_all, r, h0=None, gate="channel", tau=0.0, **kw):
    """This segment's forward from the state the earlier segments hand it. Returns (o, hT, h0_r)."""
    h0_r = state_combine(a_all, U_all, r, init=h0)
    o, hT = gla_fwd(q, k, v, log_a, h0_r, gate=gate, tau=tau, **kw)
    return o, hT, h0_r


def summary_bwd(q, k, v, log_a, dO, gate="channel", tau=0.0, **kw):
    """(a, W) of this segment: its decay and the gradient it sends to its entering state when nothing
    arrives at its end (that gradient does not depend on the entering state)."""
    B, H, L, Dk = q.shape
    try:
        W = gla_bwd_initial_grad(q, k, v, log_a, dO, None, gate=gate, tau=tau, **kw)
    except _lib.GlaError as e:
        if e.status != _lib.GLA_ERR_UNSUPPORTED:
            raise
        W = gla_bwd(q, k, v, log_a, dO, None, None, gate=gate, tau=tau, **kw)["dh0"]
    return segment_decay(log_a, B, H, L, Dk, gate, tau), W


def finish_bwd(q, k, v, log_a, dO, h0_r, a_all, W_all, r, dhT=None, gate="channel", tau=0.0, **kw):
    """This segment's backward with the gradient the later segments send to its end state. Returns the
    gradient dict; segment 0's dh0 is the sequence's."""
    dhT_r = state_combine(a_all, W_all, r, init=dhT, reverse=True)
    return gla_bwd(q, k, v, log_a, dO, h0_r, dhT_r, gate=gate, tau=tau, **kw)


# ---- the collective wrapper ---------------------------------------------------------------------
def _all_gather_stack(group):
    import torch.distributed as dist

    def gather(t: torch.Tensor) -> torch.Tensor:
        world = dist.get_world_size(group)
        parts: List[torch.Tensor] = [torch.empty_like(t) for _ in range(world)]
        dist.all_gather(parts, t.contiguous(), group=group)
        return torch.stack(parts)

    return gather


class SeqShard:
    """One rank's share of a sequence split along L over the ranks of `group` (rank i holds the i-th
    contiguous segment). `gather(t)` returns the G ranks' tensors stacked along a new first axis; the
    default all-gathers over `group`. `ops` supplies the per-segment computations (default: this
    library's kernels); every rank must call forward/backward together."""

    def __init__(self, group=None, gather: Optional[Callable] = None, rank: Optional[int] = None, ops=None):
        import torch.distributed as dist

        self.group = group
        self.rank = dist.get_rank(group) if rank is None else rank
        self.gather = gather or _all_gather_stack(group)
        self.ops = ops or _LibOps()

    def forward(self, q, k, v, log_a, h0=None, **kw):
        """(o, hT, h0_r) of this rank's segment: the last rank's hT is the sequence's final state; keep
        h0_r for the backward. Every rank passes the same h0 (or None)."""
        a, U = self.ops.summary_fwd(q, k, v, log_a, **kw)
        a_all, U_all = self.gather(a), self.gather(U)
        return self.ops.finish_fwd(q, k, v, log_a, a_all, U_all, self.rank, h0, **kw)

    def backward(self, q, k, v, log_a, dO, h0_r, dhT=None, **kw):
        """Gradients of this rank's segment; rank 0's dh0 is the sequence's. Every rank passes the same
        dhT (the gradient arriving at the sequence's final state, or None)."""
        a, W = self.ops.summary_bwd(q, k, v, log_a, dO, **kw)
        a_all, W_all = self.gather(a), self.gather(W)
        return self.ops.finish_bwd(q, k, v, log_a, dO, h0_r, a_all, W_all, self.rank, dhT, **kw)


class _LibOps:
    summary_fwd = staticmethod(summary_fwd)
    finish_fwd = staticmethod(finish_fwd)
    summary_bwd = staticmethod(summary_bwd)
    finish_bwd = staticmethod(finish_bwd)


def split_lengths(L: int, world: int) -> Sequence[int]:
    """Segment lengths of a sequence of L steps over `world` ranks (the first L % world get one more)."""
    base, extra = divmod(L, world)
    return [base + (1 if i < extra else 0) for i in range(world)]
