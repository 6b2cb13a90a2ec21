"""Context-parallel prefill: one long sequence split across the ranks of a process group.

The state after a segment is affine in the state before it (Qwen3.5 page, section 5: each
token maps S to alpha S (I - beta k k^T) + beta v k^T). For a segment of tokens,

    S_out = S_in P + S_loc,   P = prod_t alpha_t (I - beta_t k_t k_t^T)   (token order),

where S_loc is the segment's final state from a zero state and P (dk x dk per value head) is
the final state of the same segment run with v = 0 from the identity state, so both come from
the ordinary prefill kernels. Each rank computes (S_loc, P) for its own segment, the ranks
exchange them in one all-gather, every rank folds the segments before it into its incoming
state, and a second pass over the segment from that state gives its outputs. The fold also
yields the whole sequence's final state on every rank.

The per-segment prefill defaults to ``gdn_chunk_prefill`` (the CUDA library); the fold is two
small batched GEMMs per preceding segment.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Tuple

import torch
import torch.distributed as dist

# prefill(q, k, v, g, beta, initial_state) -> (o [T, Hv, dv], final_state [1, Hv, dv, dk])
PrefillFn = Callable[..., Tuple[torch.Tensor, torch.Tensor]]


def _library_prefill(scale: float, qk_l2norm: bool) -> PrefillFn:
    from ._lib import gdn_chunk_prefill

    def run(q, k, v, g, beta, initial_state):
        Hv, dv, dk = v.shape[1], v.shape[2], q.shape[2]
        fin = torch.empty((1, Hv, dv, dk), dtype=torch.float32, device=q.device)
        o = gdn_chunk_prefill(q, k, v, g, beta, None, initial_state, fin, scale, qk_l2norm)
        return o, fin
    return run


def segment_summary(q, k, v, g, beta, prefill: PrefillFn) -> Tuple[torch.Tensor, torch.Tensor]:
    """(S_loc, P) of one segment: its final state from zero, and its transition (the final
    state with v = 0 from the identity), both [1, Hv, d, d] fp32."""
    Hv, dv, dk = v.shape[1], v.shape[2], q.shape[2]
    if dv != dk:
        raise ValueError("context-parallel prefill needs dk == dv (the transition is dk x dk)")
    zero = torch.zeros((1, Hv, dv, dk), dtype=torch.float32, device=q.device)
    eye = torch.eye(dk, dtype=torch.float32, device=q.device).expand(1, Hv, dk, dk).contiguous()
    _, s_loc = prefill(q, k, v, g, beta, zero)
    _, P = prefill(q, k, torch.zeros_like(v), g, beta, eye)
    return s_loc, P


def fold(summaries: List[Tuple[torch.Tensor, torch.Tensor]], s0: torch.Tensor) -> List[torch.Tensor]:
    """States entering each segment and leaving the last: [S_in_0 = s0, S_in_1, ..., S_out]."""
    states = [s0]
    s = s0
    for s_loc, P in summaries:
        s = torch.matmul(s, P) + s_loc
        states.append(s)
    return states


def cp_prefill(q, k, v, g, beta, initial_state: Optional[torch.Tensor] = None, scale: float = 1.0,
               qk_l2norm: bool = True, group=None,
               prefill: Optional[PrefillFn] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Prefill of one sequence whose tokens are split across the ranks of ``group`` in rank
    order: this rank holds q, k [T_r, Hk, d], v [T_r, Hv, d], g, beta [T_r, Hv] (T_r may
    differ per rank). Returns (o [T_r, Hv, d] of this rank's tokens, the whole sequence's
    final state [1, Hv, d, d] fp32, the same on every rank). ``initial_state`` (the state
    before the first rank's tokens) must be given identically on every rank, or None.
    One all-gather of 2 x Hv x d x d fp32 per rank crosses the group."""
    prefill = prefill or _library_prefill(scale, qk_l2norm)
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    s_loc, P = segment_summary(q, k, v, g, beta, prefill)
    packed = torch.stack([s_loc[0], P[0]])                      # [2, Hv, d, d]
    gathered = [torch.empty_like(packed) for _ in range(world)]
    dist.all_gather(gathered, packed, group=group)
    s0 = (initial_state.to(s_loc.dtype) if initial_state is not None
          else torch.zeros_like(s_loc))
    states = fold([(t[0:1], t[1:2]) for t in gathered], s0)
    o, _ = prefill(q, k, v, g, beta, states[rank].contiguous())
    return o, states[-1]
