"""gdn_chunk_prefill_noalloc against gdn_chunk_prefill.

The no-allocation entry point is for callers that cannot allocate device memory -- a
plugin inside a host application that owns all GPU memory through its own pool, or a
latency-critical loop where cudaMalloc is not acceptable. It runs the same chunked
prefill with its scratch in an array the library reserves statically on each GPU. These
tests call it through the C ABI twice in a row, on different inputs, and check that it
agrees with the regular entry point (given a caller-allocated workspace) within the bf16
tolerance the parity tests use; and that sizes beyond its scratch are refused before any
launch. The file sorts last so that a run stopping at the first failure has run every
other test first; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import gated_deltanet_mixer_causal_b200 as gdn
from gated_deltanet_mixer_causal_b200 import _lib
from gated_deltanet_mixer_causal_b200 import workloads as W
from gated_deltanet_mixer_causal_b200.build import build
from parity import BF16_TOL, np64, worst_head_o, worst_head_state

pytestmark = pytest.mark.gpu


def _prepared(seed, lengths, dev):
    p = W.make_prefill(W.QWEN35_9B, 0, seed=seed, g_low=-0.5, init_std=0.02, lengths=lengths)
    sh = p.shape
    cu = p.cu_seqlens.to(dev)
    y = gdn.gdn_conv1d_silu(p.x.to(dev), p.conv_w.to(dev), cu)
    q, k, v = gdn.qkv_views(y, sh.Hk, sh.Hv, sh.dk)
    return p, cu, q, k, v


def test_noalloc_matches_workspace_entry_point(cuda_device):
    build()
    dev = cuda_device
    for seed, lengths in [(61, [300, 400]), (62, [1000, 17, 130])]:
        p, cu, q, k, v = _prepared(seed, lengths, dev)
        sh = p.shape
        g, beta, init = p.g.to(dev), p.beta.to(dev), p.initial_state.to(dev)
        need = gdn.gdn_chunk_prefill_workspace_size(p.T, p.n_seq, sh.Hk, sh.Hv, sh.dk, sh.dv, q.dtype)
        assert 0 < need <= 64 << 20          # exercises the scratch, within its limit
        fin_ref = torch.empty_like(init)
        o_ref = gdn.gdn_chunk_prefill(q, k, v, g, beta, cu, init, fin_ref)
        fin = torch.full_like(init, float("nan"))
        o = torch.full((p.T, sh.Hv, sh.dv), float("nan"), dtype=q.dtype, device=dev)
        gdn.gdn_chunk_prefill_noalloc(q, k, v, g, beta, cu, init, fin, o=o)
        gdn.gdn_prefill_noalloc_status(dev)   # every bounded wait of the call completed
        torch.cuda.synchronize()
        cu_np = p.cu_seqlens.numpy()
        assert worst_head_o(np64(o), np64(o_ref), cu_np) <= BF16_TOL
        assert worst_head_state(np64(fin), np64(fin_ref)) <= BF16_TOL


def test_noalloc_refuses_sizes_beyond_its_scratch():
    build()
    L = _lib.lib()
    fake = 0x7f0000000000    # aligned, never dereferenced: the call is refused first
    T, Hk, Hv, d = 1 << 20, 16, 48, 128
    assert L.gdn_chunk_prefill_workspace_size(T, 1, Hk, Hv, d, d, _lib.GDN_BF16) > (64 << 20)
    st = L.gdn_chunk_prefill_noalloc(fake, fake + (1 << 34), fake + (2 << 34), fake + (3 << 34),
                                     fake + (4 << 34), fake + (5 << 34), _lib.GDN_BF16, T, Hk, Hv,
                                     d, d, 0, 0, None, 1, None, None, 1.0, 1, None)
    assert st == _lib.GDN_ERR_WORKSPACE
    assert "needed" in L.gdn_last_error().decode()
