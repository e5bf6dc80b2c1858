"""Scan of a batch of sequences split along its tokens across ranks.

Rank r holds the contiguous segment r of every batch row (tokens
``[L_r, L_{r+1})``) and runs one process per GPU.  The scan element
``(exp(delta*A), h)`` composes associatively with seed ``(1, h0)`` ("Adding
Initial Value Support to Selective Scan Forward Kernel", state-spaces/mamba
issue 285), so every rank scans its segment at the same time from a zero state
and two small exchanges join the segments:

1. conv tails: rank r's conv input history is the last K-1 raw conv inputs of
   segment r-1 (all-gather of ``[b, conv_dim, K-1]``, before the scans);
2. segment pairs: every rank's ``(sum of delta, end state from zero)``
   (one all-gather of ``b*U + b*state`` fp32), after the scans.

Each rank then folds the pairs of the segments before it into the state that
enters its own segment and adds that state's contribution to its y.  All
arithmetic runs in ``libssm.so`` (``ssm_split_*`` and ``ssm_scan_fwd``); this
module only orders the calls and the exchanges.  Every segment must hold at
least K-1 tokens.

Exchanges go through ``torch.distributed`` (NCCL over NVLink between GPUs)
unless an ``all_gather`` callable is given: it receives this rank's tensor and
returns the ``[R, ...]`` stack of every rank's tensor, in rank order.
"""
from __future__ import annotations

import torch

from . import ops


def dist_all_gather(group=None):
    """An ``all_gather`` over a torch.distributed process group."""
    import torch.distributed as dist

    def gather(t: torch.Tensor) -> torch.Tensor:
        parts = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
        dist.all_gather(parts, t.contiguous(), group=group)
        return torch.stack(parts)
    return gather


class SegmentScan:
    """One rank's part of a split scan, phase by phase.

    ``tail()`` -> tensor for exchange 1; ``scan(tails)`` -> packed pair for
    exchange 2; ``join(pairs)`` -> ``(y, h_out, conv_state_out)``.  The packed
    pair is ``[sum_delta (b*U) | pad | h_loc (b*state) | pad]`` fp32 with both
    parts starting on a 4-element boundary, so ``join`` reads the gathered
    ``[R, pack]`` buffer in place.  ``h_out``
    is the state after this rank's segment (the last rank's is the
    sequences' final state), ``conv_state_out`` the segment's conv tail.
    """

    def __init__(self, mode, rank, nranks, x, dt, A, B, C_, *, D=None, z=None, dt_bias=None, h0=None, conv_w=None,
                 conv_b=None, conv_state_in=None, delta_softplus=True, backend=ops, stream=None):
        if not 0 <= rank < nranks:
            raise ValueError("rank out of range")
        self.mode, self.rank, self.nranks, self.be, self.stream = mode, rank, nranks, backend, stream
        self.K = 0 if conv_w is None else conv_w.shape[1]
        if self.K > 1 and x.shape[1] < self.K - 1:
            raise ValueError("every segment needs at least K-1 tokens")
        self.t = dict(x=x, dt=dt, A=A, B=B, C_=C_)
        self.kw = dict(D=D, z=z, dt_bias=dt_bias, conv_w=conv_w, conv_b=conv_b, delta_softplus=delta_softplus)
        self.h0 = h0 if rank == 0 else None         # the true h0 enters at segment 0 only
        self.conv_state_in = conv_state_in if rank == 0 else None
        self.y = self.h_loc = self.conv_out = self.cum = None

    def _args(self):
        t = self.t
        return (self.mode, t["x"], t["dt"], t["A"], t["B"], t["C_"])

    def _layout(self):
        """``(b, U, state shape, offset of h_loc, pack length)`` of the packed pair."""
        x, A, B = self.t["x"], self.t["A"], self.t["B"]
        b, U = x.shape[0], x.shape[2]
        state = (b,) + tuple(A.shape) if x.dim() == 3 else (b, x.shape[2], x.shape[3], B.shape[3])
        off = (b * U + 3) // 4 * 4
        return b, U, state, off, off + (self._nhl(state) + 3) // 4 * 4

    def pack_size(self):
        """Elements of this rank's packed pair."""
        return self._layout()[4]

    def tail(self):
        """This segment's last K-1 raw conv inputs (None without a conv of width > 1)."""
        if self.K < 2:
            return None
        return self.be.split_conv_tail(*self._args(), conv_state_in=self.conv_state_in, stream=self.stream,
                                       **self.kw)

    def scan(self, tails=None, out=None):
        """Scan the segment from zero (rank 0: from h0); return the packed
        ``(sum_delta, h_loc)``, written straight into ``out`` (fp32, ``pack_size()``
        elements: this rank's block of the exchange buffer) when given."""
        if self.rank > 0 and tails is not None:
            self.conv_state_in = tails[self.rank - 1]
        b, U, state, off, n = self._layout()
        x = self.t["x"]
        dtype = getattr(self.be, "PACK_DTYPE", torch.float32)     # the backend's state precision
        if out is None:
            out = torch.empty(n, dtype=dtype, device=x.device)
        elif out.dtype != dtype or out.numel() != n or not out.is_contiguous():
            raise ValueError(f"out must be a contiguous {dtype} tensor of {n} elements")
        h_loc = out[off:off + self._nhl(state)].view(state)
        self.y, self.h_loc, self.conv_out = self.be.scan_fwd(*self._args(), h0=self.h0, h_final=h_loc,
                                                             conv_state_in=self.conv_state_in,
                                                             stream=self.stream, **self.kw)
        kw = {k: self.kw[k] for k in ("dt_bias", "delta_softplus")}
        self.cum, _ = self.be.split_cum_delta(*self._args(), cum=self.rank > 0, sum_delta=out[:b * U].view(b, U),
                                              stream=self.stream, **kw)
        return out

    @staticmethod
    def _nhl(state):
        n = 1
        for v in state:
            n *= v
        return n

    def join(self, pairs):
        """Fold the gathered pairs ``[R, b*U + b*state]`` and fix up y: ``(y, h_out, conv_state_out)``."""
        R = pairs.shape[0]
        if R != self.nranks:
            raise ValueError("expected one pair per rank")
        b, U, state, off, n = self._layout()
        if pairs.dim() != 2 or pairs.shape[1] != n:
            raise ValueError(f"expected [R, {n}] packed pairs")
        # views of the gathered buffer: each rank's block is contiguous
        sd_all = pairs[:, :b * U].unflatten(1, (b, U))
        hl_all = pairs[:, off:off + self._nhl(state)].unflatten(1, state)
        h_in, h_out = self.be.split_combine(self.mode, self.t["A"], sd_all, hl_all, self.rank, stream=self.stream)
        if self.rank > 0:
            self.be.split_fixup(*self._args(), self.y, self.cum, h_in, conv_state_in=self.conv_state_in,
                                stream=self.stream, **self.kw)
        return self.y, h_out, self.conv_out


def scan_fwd_seq_split(mode, x, dt, A, B, C_, *, rank, nranks, all_gather=None, group=None, **kw):
    """This rank's segment of a split scan: ``(y, h_out, conv_state_out)`` (see :class:`SegmentScan`)."""
    if all_gather is None:
        import torch.distributed as dist
        if dist.get_world_size(group) != nranks or dist.get_rank(group) != rank:
            raise ValueError("rank / nranks do not match the process group")
    gather = all_gather if all_gather is not None else dist_all_gather(group)
    seg = SegmentScan(mode, rank, nranks, x, dt, A, B, C_, **kw)
    tail = seg.tail()
    tails = gather(tail) if tail is not None else None
    pairs = gather(seg.scan(tails))
    return seg.join(pairs)


__all__ = ["SegmentScan", "scan_fwd_seq_split", "dist_all_gather"]
