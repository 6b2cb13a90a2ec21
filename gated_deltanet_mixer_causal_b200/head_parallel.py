"""Head-group split of the mixer across the ranks of a process group (tensor parallel).

Key head j serves value heads j*G .. j*G + G - 1 (G = Hv / Hk), and the state, the conv
channels and the recurrence of one key-head group never read another group's ("Inside
Qwen3.5", config footnote: 16 key / 48 value heads of 128; section 5: one state per value
head). So N ranks split the layer by key-head groups: rank r takes key heads
[r*Hk/N, (r+1)*Hk/N) with their value heads, and the conv channels that feed them,

    q channels  [hk0*d, hk1*d)     k channels  Hk*d + [hk0*d, hk1*d)
    v channels  2*Hk*d + [hv0*d, hv1*d)

and runs the ordinary entry points on that slice. Nothing crosses ranks inside the mixer
(the out-projection's reduction after it is not part of the mixer). In a model the
column-parallel in-projection already produces each rank's slice; ``shard_*`` cut it from
whole-layer tensors, and ``gather_heads`` reassembles per-rank results along the head axis
(one all-gather, for checking or for a caller that wants the whole layer on every rank).
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist


def head_range(Hk: int, Hv: int, rank: int, world: int) -> Tuple[int, int, int, int]:
    """(hk0, hk1, hv0, hv1): the key heads and value heads of ``rank``."""
    if Hk % world != 0:
        raise ValueError(f"{Hk} key heads do not split over {world} ranks")
    if Hv % Hk != 0:
        raise ValueError(f"Hv = {Hv} is not a multiple of Hk = {Hk}")
    G = Hv // Hk
    per = Hk // world
    hk0, hk1 = rank * per, (rank + 1) * per
    return hk0, hk1, hk0 * G, hk1 * G


def channel_index(Hk: int, Hv: int, d: int, rank: int, world: int,
                  device: Optional[torch.device] = None) -> torch.Tensor:
    """Indices of ``rank``'s conv channels in the [q | k | v] order of the whole layer, in
    the same order for the slice ([q_r | k_r | v_r])."""
    hk0, hk1, hv0, hv1 = head_range(Hk, Hv, rank, world)
    q = torch.arange(hk0 * d, hk1 * d)
    k = Hk * d + q
    v = torch.arange(2 * Hk * d + hv0 * d, 2 * Hk * d + hv1 * d)
    return torch.cat([q, k, v]).to(device)


def shard_prefill_inputs(x, conv_w, g, beta, Hk, Hv, d, rank, world, initial_state=None,
                         conv_state=None):
    """Slices of a whole-layer prefill batch for ``rank``: x [T, Cc_r], conv_w [Cc_r, 4],
    g, beta [T, Hv_r], initial_state [N, Hv_r, d, d], conv_state [N, 3, Cc_r] (copies)."""
    _, _, hv0, hv1 = head_range(Hk, Hv, rank, world)
    ch = channel_index(Hk, Hv, d, rank, world, x.device)
    out = [x.index_select(1, ch).contiguous(), conv_w.index_select(0, ch).contiguous(),
           g[:, hv0:hv1].contiguous(), beta[:, hv0:hv1].contiguous(),
           None if initial_state is None else initial_state[:, hv0:hv1].contiguous(),
           None if conv_state is None else conv_state.index_select(2, ch).contiguous()]
    return out


def shard_decode_inputs(x, conv_w, conv_state, g, beta, state, Hk, Hv, d, rank, world):
    """Slices of a whole-layer decode batch for ``rank``: x [B, Cc_r] (or [B, n, Cc_r]),
    conv_w, conv_state [B, 3, Cc_r], g, beta [B, Hv_r] (or [B, n, Hv_r]), state
    [B, Hv_r, d, d] (copies; the caller keeps each rank's conv and recurrent states)."""
    _, _, hv0, hv1 = head_range(Hk, Hv, rank, world)
    ch = channel_index(Hk, Hv, d, rank, world, x.device)
    return (x.index_select(x.dim() - 1, ch).contiguous(), conv_w.index_select(0, ch).contiguous(),
            conv_state.index_select(2, ch).contiguous(), g[..., hv0:hv1].contiguous(),
            beta[..., hv0:hv1].contiguous(), state[:, hv0:hv1].contiguous())


def head_parallel_prefill(x, conv_w, g, beta, Hk, Hv, d, rank, world, cu_seqlens=None,
                          initial_state=None, prefill=None):
    """This rank's part of a whole-layer prefill: returns (o [T, Hv_r, d], final state
    [N, Hv_r, d, d] fp32). ``prefill(x, w, g, beta, Hk_r, Hv_r, d, cu, init)`` defaults to the
    library's conv + chunked prefill (``prefill_layer``)."""
    xs, ws, gs, bs, s0, _ = shard_prefill_inputs(x, conv_w, g, beta, Hk, Hv, d, rank, world,
                                                 initial_state)
    hk0, hk1, hv0, hv1 = head_range(Hk, Hv, rank, world)
    if prefill is None:
        from . import prefill_layer

        def prefill(x_, w_, g_, b_, hk_, hv_, d_, cu_, init_):
            n = 1 if cu_ is None else cu_.numel() - 1
            fin = torch.empty((n, hv_, d_, d_), dtype=torch.float32, device=x_.device)
            o = prefill_layer(x_, w_, g_, b_, hk_, hv_, d_, cu_, init_, final_state=fin)
            return o, fin
    return prefill(xs, ws, gs, bs, hk1 - hk0, hv1 - hv0, d, cu_seqlens, s0)


def gather_heads(t: torch.Tensor, dim: int, group=None) -> torch.Tensor:
    """Concatenate every rank's head slice along ``dim`` (rank order = head order)."""
    world = dist.get_world_size(group)
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.cat(parts, dim=dim)
