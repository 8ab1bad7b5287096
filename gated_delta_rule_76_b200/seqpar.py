"""Sequence split along time over the ranks of a process group, one GPU per rank.

Rank r of the group holds segment r of every sequence (consecutive tokens, in rank order) with
the same batch and heads on every rank.  A segment acts on the state as an affine map
S -> M S + N (each token's update is affine in the state: GDN-2 summary, «Méthodologie» §1; the
state has a fixed size whatever the context: mkdocs chapter «Gated DeltaNet», «L'état, en
mémoire»).  The exchange is one all-gather of the maps; every rank then composes the maps of the
segments before it (an exclusive scan) to get the state entering its own segment, and re-runs its
segment from that state.  The backward is the same in reverse: one all-gather of each segment's
own contribution to the gradient of its entering state, then the transposed maps carry the
gradient of the final state back across the later segments.

This module is host logic only: the collective is torch.distributed (NCCL between GPUs, gloo for
the CPU tests) and every arithmetic step runs in the library's kernels through ``ops``
(``DeviceOps``: gdn_segment_map, gdn_state_compose, gdn_chunk_fwd, gdn_chunk_bwd).  The work per
rank is two forward passes (the map, the re-run) against one for a single GPU.
"""
from __future__ import annotations

from typing import Dict, List, Optional

import torch
import torch.distributed as dist

from . import gdn


class DeviceOps:
    """The library's kernels on the caller's device.  ``out_f32``: the forward writes its output in
    fp32 (the unrounded accumulator) instead of the input dtype."""

    def __init__(self, out_f32: bool = False):
        self.out_f32 = out_f32

    def segment_map(self, x: Dict[str, torch.Tensor]):
        return gdn.gdn_segment_map(x["q"], x["k"], x["v"], x["alpha"], b=x.get("b"), w=x.get("w"),
                                   beta=x.get("beta"), head_map=x.get("head_map"))

    def compose(self, M, N, S, transpose: bool = False):
        return gdn.gdn_state_compose(M, N, S, transpose=transpose)

    def forward(self, x: Dict[str, torch.Tensor], h0, scale: float):
        return gdn.gdn_chunk_fwd(x["q"], x["k"], x["v"], x["alpha"], b=x.get("b"), w=x.get("w"),
                                 beta=x.get("beta"), h0=h0, head_map=x.get("head_map"), scale=scale,
                                 out_f32=self.out_f32)

    def backward(self, x: Dict[str, torch.Tensor], h0, grad_o, grad_ht, scale: float):
        return gdn.gdn_chunk_bwd(x["q"], x["k"], x["v"], x["alpha"], b=x.get("b"), w=x.get("w"),
                                 beta=x.get("beta"), h0=h0, head_map=x.get("head_map"), scale=scale,
                                 grad_o=grad_o, grad_ht=grad_ht)


def entering_state(Ms, Ns, h0, rank: int, ops):
    """The state entering segment `rank`: the maps of segments 0 .. rank-1 applied to h0."""
    s = h0 if h0 is not None else torch.zeros_like(Ns[0])
    for r in range(rank):
        s = ops.compose(Ms[r], Ns[r], s)
    return s


def final_state(Ms, Ns, ht_local, rank: int, ops):
    """The state after the last segment, from the state after segment `rank`."""
    s = ht_local
    for r in range(rank + 1, len(Ms)):
        s = ops.compose(Ms[r], Ns[r], s)
    return s


def leaving_grad(Ms, Gs, grad_ht, rank: int, ops):
    """The gradient of the state leaving segment `rank`: the final state's gradient carried back
    across segments len-1 .. rank+1 (M_r^T d + G_r, G_r a segment's own contribution)."""
    d = grad_ht if grad_ht is not None else torch.zeros_like(Gs[0])
    for r in range(len(Ms) - 1, rank, -1):
        d = ops.compose(Ms[r], Gs[r], d, transpose=True)
    return d


def _all_gather(t: torch.Tensor, group) -> List[torch.Tensor]:
    out = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
    dist.all_gather(out, t.contiguous(), group=group)
    return out


def forward(x: Dict[str, torch.Tensor], h0: Optional[torch.Tensor] = None, scale: float = 1.0,
            group=None, ops=None):
    """Forward of this rank's segment.  ``x``: q, k, v, alpha and b, w or beta (and optionally
    head_map) of the segment; ``h0``: the state entering the whole sequence (the same on every
    rank, or None for zeros).  Returns a dict: o (this segment's output), ht (the final state of the
    whole sequence, on every rank), s_in (the state entering this segment) and maps (every rank's
    M, for the backward)."""
    ops = ops or DeviceOps()
    rank = dist.get_rank(group)
    M, N = ops.segment_map(x)
    Ms, Ns = _all_gather(M, group), _all_gather(N, group)
    s_in = entering_state(Ms, Ns, h0, rank, ops)
    o, ht_local = ops.forward(x, s_in, scale)
    return {"o": o, "ht": final_state(Ms, Ns, ht_local, rank, ops), "s_in": s_in, "maps": Ms}


def backward(x: Dict[str, torch.Tensor], fwd: Dict[str, object], grad_o: torch.Tensor,
             grad_ht: Optional[torch.Tensor] = None, scale: float = 1.0, group=None, ops=None):
    """Backward of this rank's segment, given forward()'s result ``fwd``, the gradient of this
    segment's output and (optionally, the same on every rank) the gradient of the whole sequence's
    final state.  Returns the gradients of this segment's inputs; dh0 is the gradient of the state
    entering this segment (on rank 0: the gradient of h0)."""
    ops = ops or DeviceOps()
    rank = dist.get_rank(group)
    Ms = fwd["maps"]
    # this segment's own contribution to the gradient of its entering state (final-state gradient 0)
    own = ops.backward(x, fwd["s_in"], grad_o, None, scale)["dh0"]
    Gs = _all_gather(own, group)
    return ops.backward(x, fwd["s_in"], grad_o, leaving_grad(Ms, Gs, grad_ht, rank, ops), scale)
