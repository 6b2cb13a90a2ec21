"""gdn_chunk_prefill_noalloc against gdn_chunk_prefill.

The no-allocation entry point is for callers that cannot allocate device memory -- a
plugin inside a host application that owns all GPU memory through its own pool, or a
latency-critical loop where cudaMalloc is not acceptable. It runs the same prefill with
its scratch in an array the library reserves statically on each GPU. These tests call it
through the C ABI twice in a row, on different inputs, and check that it gives exactly the
bytes the regular entry point (given a caller-allocated workspace) gives: both run the
same kernels on the same inputs, so any difference would mean a stale or misplaced scratch
read. They also cover the paths that need no scratch, and the refusal of sizes beyond the
scratch, which must launch nothing. The file sorts last so that a run stopping at the
first failure has run every other test first; it also passes on its own in a fresh
process.
"""
import numpy as np
import pytest
import torch

import gated_deltanet_mixer_causal_b200 as gdn
from gated_deltanet_mixer_causal_b200 import _lib
from gated_deltanet_mixer_causal_b200 import workloads as W
from gated_deltanet_mixer_causal_b200.build import build

pytestmark = pytest.mark.gpu

SCRATCH = 64 << 20


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
        assert 0 < need <= SCRATCH          # exercises the scratch, within its limit
        fin_ref = torch.empty_like(init)
        o_ref = gdn.gdn_chunk_prefill(q, k, v, g, beta, cu, init, fin_ref)
        fin = torch.full_like(init, float("nan"))
        o = torch.full((p.T, sh.Hv, sh.dv), float("nan"), dtype=q.dtype, device=dev)
        gdn.gdn_chunk_prefill_noalloc(q, k, v, g, beta, cu, init, fin, o=o)
        gdn.gdn_prefill_noalloc_status(dev)   # every bounded wait of the call completed
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref)
        assert torch.equal(fin, fin_ref)


@pytest.mark.parametrize("case", ["bf16_d128_no_l2norm", "fp32_d16"])
def test_noalloc_paths_without_scratch(cuda_device, case):
    """Shapes on the token-recurrent path need no scratch: the call runs them as the regular
    entry point does (bit for bit) and its status call reports that call, not an older one."""
    build()
    dev = cuda_device
    if case == "fp32_d16":
        r = W.make_recurrence(W.LayerShape(2, 4, 16, 16), 0, seed=63, dtype=torch.float32,
                              init_std=0.1, lengths=[40, 90])
        l2 = True
    else:
        r = W.make_recurrence(W.LayerShape(2, 4, 128, 128), 0, seed=64, dtype=torch.float32,
                              init_std=0.02, lengths=[100, 150])
        r.q = (r.q / np.sqrt(128)).to(torch.bfloat16)
        r.k = (r.k / np.sqrt(128)).to(torch.bfloat16)
        r.v = r.v.to(torch.bfloat16)
        l2 = False
    sh = r.shape
    assert gdn.gdn_chunk_prefill_path(r.q.dtype, sh.Hk, sh.Hv, sh.dk, sh.dv, l2) == "recurrent"
    args = [t.to(dev) for t in (r.q, r.k, r.v, r.g, r.beta, r.cu_seqlens)]
    init = r.initial_state.to(dev)
    fin_ref = torch.empty_like(init)
    o_ref = gdn.gdn_chunk_prefill(*args, init, fin_ref, 1.0, l2)
    for _ in range(2):
        fin = torch.full_like(init, float("nan"))
        o = gdn.gdn_chunk_prefill_noalloc(*args, init, fin, 1.0, l2)
        gdn.gdn_prefill_noalloc_status(dev)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref)
        assert torch.equal(fin, fin_ref)


def test_noalloc_size_limit_follows_the_path(cuda_device):
    """3,000 tokens of 48 value heads: the tensor-core path would need more than the scratch,
    so with the L2 norm on the call is refused before any launch (o stays untouched); with
    the norm off it takes the token-recurrent path, which needs no scratch, and runs."""
    build()
    dev = cuda_device
    sh = W.LayerShape(16, 48, 128, 128)
    T = 3000
    assert gdn.gdn_chunk_prefill_workspace_size(T, 1, sh.Hk, sh.Hv, sh.dk, sh.dv,
                                                torch.bfloat16) > SCRATCH
    r = W.make_recurrence(sh, T, seed=65, dtype=torch.float32)
    q = (r.q / np.sqrt(128)).to(torch.bfloat16).to(dev)
    k = (r.k / np.sqrt(128)).to(torch.bfloat16).to(dev)
    v = r.v.to(torch.bfloat16).to(dev)
    g, beta = r.g.to(dev), r.beta.to(dev)
    o = torch.full((T, sh.Hv, sh.dv), float("nan"), dtype=torch.bfloat16, device=dev)
    with pytest.raises(gdn.GDNError) as e:
        gdn.gdn_chunk_prefill_noalloc(q, k, v, g, beta, o=o)
    assert e.value.status == _lib.GDN_ERR_WORKSPACE
    assert "nothing was launched" in str(e.value)
    torch.cuda.synchronize()
    assert torch.isnan(o.float()).all()
    o2 = gdn.gdn_chunk_prefill_noalloc(q, k, v, g, beta, qk_l2norm=False, o=o)
    gdn.gdn_prefill_noalloc_status(dev)
    o_ref = gdn.gdn_chunk_prefill(q, k, v, g, beta, qk_l2norm=False)
    torch.cuda.synchronize()
    assert torch.equal(o2, o_ref)


def test_noalloc_refuses_sizes_beyond_its_scratch():
    build()
    L = _lib.lib()
    fake = 0x7f0000000000    # aligned, never dereferenced: the call is refused first
    T, Hk, Hv, d = 1 << 20, 16, 48, 128
    assert L.gdn_chunk_prefill_workspace_size(T, 1, Hk, Hv, d, d, _lib.GDN_BF16) > SCRATCH
    st = L.gdn_chunk_prefill_noalloc(fake, fake + (1 << 34), fake + (2 << 34), fake + (3 << 34),
                                     fake + (4 << 34), fake + (5 << 34), _lib.GDN_BF16, T, Hk, Hv,
                                     d, d, 0, 0, None, 1, None, None, 1.0, 1, None)
    assert st == _lib.GDN_ERR_WORKSPACE
    assert "needed" in L.gdn_last_error().decode() or "need" in L.gdn_last_error().decode()


def test_noalloc_wrapper_checks_devices_and_dtypes(cuda_device):
    """The Python wrapper refuses, before any launch, a host cu_seqlens, an int64 cu_seqlens
    and a v whose dtype differs from q's."""
    build()
    dev = cuda_device
    r = W.make_recurrence(W.LayerShape(2, 4, 128, 128), 0, seed=66, dtype=torch.bfloat16,
                          lengths=[30, 40])
    q, k, v, g, b = (t.to(dev) for t in (r.q, r.k, r.v, r.g, r.beta))
    with pytest.raises(ValueError):
        gdn.gdn_chunk_prefill_noalloc(q, k, v, g, b, r.cu_seqlens)               # host array
    with pytest.raises(ValueError):
        gdn.gdn_chunk_prefill_noalloc(q, k, v, g, b, r.cu_seqlens.long().to(dev))
    with pytest.raises(ValueError):
        gdn.gdn_chunk_prefill_noalloc(q, k, v.float(), g, b, r.cu_seqlens.to(dev))
