"""Sequence-parallel prefill across ranks (one process per GPU).

Rank r of a group of P holds segment r of every sequence: tokens
[r L, (r + 1) L) of q, k, v and the gates, [B, L, H, *] on its own GPU.  The
recurrence is affine in the state, so over a segment S_out = M S_in + N; the
one exchange step of the method is the all-gather of the segments' (M, N).
Then every rank scans them for the state at the start of its own segment,
runs its segment from there, and ends with the final state of the whole
sequence.  Long-sequence scaling is what the FG^2-GDN page (gist.science
2604.19021) reports in section 4 "Experimental results" (efficiency).

The three compute steps are libgdr.so calls (api.segment_maps,
api.segment_scan, api.forward_chunked); the collective is torch.distributed's
all_gather (NCCL over NVLink on GPUs).  No TMA multicast or peer-memory
access is involved.  ``ops`` exists so that the CPU tests can drive the same
exchange over gloo with other implementations of the three steps.
"""

from __future__ import annotations

from typing import Optional, Tuple

import torch


class LibOps:
    """The library's CUDA calls for the three compute steps."""

    @staticmethod
    def maps(q, k, v, a, b, w, fg2=False):
        from . import api
        return api.segment_maps(q, k, v, a, b, w, fg2=fg2)

    @staticmethod
    def scan(m_all, n_all, s0):
        from . import api
        return api.segment_scan(m_all, n_all, s0)

    @staticmethod
    def forward(q, k, v, a, b, w, s_start, fg2=False):
        from . import api
        chunk = 64 if q.dtype == torch.bfloat16 else 32
        o, _ = api.forward_chunked(q, k, v, a, b, w, s_start, chunk=chunk, return_final=False,
                                   fg2=fg2)
        return o


def prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
            a: Optional[torch.Tensor] = None, b: Optional[torch.Tensor] = None,
            w: Optional[torch.Tensor] = None, s0: Optional[torch.Tensor] = None, *,
            group=None, ops=None, fg2: bool = False) -> Tuple[torch.Tensor, torch.Tensor]:
    """This rank's segment of the prefill.  Returns (o of this rank's tokens,
    S_T of the whole sequence, the same on every rank).  s0 [B, H, dk, dv]
    is the state before segment 0 and must be the same on every rank (or None
    everywhere).  Every rank takes the same collective steps in the same
    order."""
    import torch.distributed as dist
    ops = ops or LibOps
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    m, n = ops.maps(q, k, v, a, b, w, fg2=fg2)
    m_list = [torch.empty_like(m) for _ in range(world)]
    n_list = [torch.empty_like(n) for _ in range(world)]
    dist.all_gather(m_list, m.contiguous(), group=group)
    dist.all_gather(n_list, n.contiguous(), group=group)
    s_start, s_final = ops.scan(torch.stack(m_list), torch.stack(n_list), s0)
    o = ops.forward(q, k, v, a, b, w, s_start[rank].contiguous(), fg2=fg2)
    return o, s_final
