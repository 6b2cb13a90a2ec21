"""B200-native (sm_100a) Gated DeltaNet token mixer.

The compute runs in ``libgdn.so`` (hand-written CUDA, C ABI in ``include/gdn.h``); this
package marshals torch tensors into it. The library is loaded on first use and a missing
library raises -- there is no fallback.

Entry points (same names as the C ABI): ``gdn_conv1d_silu``, ``gdn_chunk_prefill`` (states at
block boundaries on request), ``gdn_chunk_prefill_workspace_size``,
``gdn_chunk_prefill_noalloc``, ``gdn_decode_step`` and ``gdn_decode_tokens`` (fp32 or bf16
states, taken from the state tensor); ``prefill_layer`` chains the conv and the chunked
prefill over one packed batch without copies.
"""
from __future__ import annotations

from typing import Optional

import torch

from ._lib import (GDNError, LIB_PATH, gdn_chunk_prefill, gdn_chunk_prefill_noalloc,
                   gdn_chunk_prefill_path, gdn_chunk_prefill_launches, gdn_chunk_prefill_workspace_size, gdn_conv1d_silu, gdn_decode_step,
                   gdn_decode_tokens, gdn_prefill_noalloc_status, gdn_prefill_status, lib)

__all__ = ["GDNError", "LIB_PATH", "lib", "gdn_conv1d_silu", "gdn_chunk_prefill",
           "gdn_chunk_prefill_workspace_size", "gdn_chunk_prefill_noalloc", "gdn_chunk_prefill_path", "gdn_chunk_prefill_launches", "gdn_decode_step",
           "gdn_decode_tokens", "gdn_prefill_status", "gdn_prefill_noalloc_status",
           "prefill_layer", "qkv_views"]


def qkv_views(y: torch.Tensor, Hk: int, Hv: int, d: int):
    """q, k, v as strided views of a conv output y [T, Cc] in channel order
    [q: Hk*d | k: Hk*d | v: Hv*d] (no copy)."""
    T, Cc = y.shape
    q = y.as_strided((T, Hk, d), (Cc, d, 1), y.storage_offset())
    k = y.as_strided((T, Hk, d), (Cc, d, 1), y.storage_offset() + Hk * d)
    v = y.as_strided((T, Hv, d), (Cc, d, 1), y.storage_offset() + 2 * Hk * d)
    return q, k, v


def prefill_layer(x: torch.Tensor, conv_w: torch.Tensor, g: torch.Tensor, beta: torch.Tensor,
                  Hk: int, Hv: int, d: int, cu_seqlens: Optional[torch.Tensor] = None,
                  initial_state: Optional[torch.Tensor] = None,
                  conv_state_in: Optional[torch.Tensor] = None,
                  final_state: Optional[torch.Tensor] = None,
                  conv_state_out: Optional[torch.Tensor] = None, scale: float = 1.0,
                  y: Optional[torch.Tensor] = None, o: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The mixer core over one packed batch: conv + SiLU, then the chunked gated delta
    rule with q/k L2 norm. Returns o [T, Hv, d]; fills final_state / conv_state_out when
    given."""
    y = gdn_conv1d_silu(x, conv_w, cu_seqlens, conv_state_in, conv_state_out, y)
    q, k, v = qkv_views(y, Hk, Hv, d)
    return gdn_chunk_prefill(q, k, v, g, beta, cu_seqlens, initial_state, final_state, scale,
                             True, o, workspace)
