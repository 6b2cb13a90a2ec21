"""A long single sequence is prefilled in pieces: the intra-chunk work of the later pieces
runs beside the chain of the current one, and the state passes from one chain piece to the
next in fp32. Parity against the oracle across the piece boundaries (output, final state and
block states, fp32 and bf16 state storage), and bit-equality with the same sequence split by
the caller at the same chunk boundaries."""
import math

import numpy as np
import pytest
import torch

import gated_deltanet_mixer_causal_b200 as gdn
from gated_deltanet_mixer_causal_b200 import workloads as W
import oracle
from parity import BF16_TOL, check, np64, worst_head_o, worst_head_state

pytestmark = pytest.mark.gpu

SHAPE = W.LayerShape(2, 6, 128, 128)   # 12 chain CTAs: the pieces path
T = 33000                              # 516 chunks: eight pieces, the last one ragged
BLOCK = 4096


def _piece_bounds(n_tok):
    """The library's split: eight pieces of at least 64 chunks each."""
    n_chunks = math.ceil(n_tok / 64)
    per = max(64, math.ceil(n_chunks / 8))
    pieces = math.ceil(n_chunks / per)
    return [min(i * per * 64, n_tok) for i in range(pieces)] + [n_tok]


def _inputs(seed):
    return W.make_recurrence(SHAPE, T, seed=seed, dtype=torch.bfloat16, init_std=0.02)


@pytest.mark.parametrize("state_dtype", [torch.float32, torch.bfloat16])
def test_pieces_against_oracle(cuda_device, state_dtype):
    dev = cuda_device
    r = _inputs(91)
    sh = r.shape
    s0 = r.initial_state.numpy()
    if state_dtype == torch.bfloat16:
        s0 = oracle.round_bf16(s0)
    n_blocks = T // BLOCK
    fin = torch.empty((1, sh.Hv, sh.dv, sh.dk), dtype=state_dtype, device=dev)
    bs = torch.full((n_blocks + 1, sh.Hv, sh.dv, sh.dk), float("nan"), dtype=state_dtype, device=dev)
    o = gdn.gdn_chunk_prefill(r.q.to(dev), r.k.to(dev), r.v.to(dev), r.g.to(dev), r.beta.to(dev),
                              None, torch.from_numpy(s0).to(state_dtype).to(dev), fin,
                              block_tokens=BLOCK, block_states=bs,
                              block_rows=torch.zeros(1, dtype=torch.int32, device=dev), check=True)
    torch.cuda.synchronize()
    q, k, v = (t.float().numpy() for t in (r.q, r.k, r.v))
    g, beta = r.g.numpy(), r.beta.numpy()
    o_r, f_r = oracle.recurrence(q, k, v, g, beta, None, s0)
    rnd = oracle.round_bf16 if state_dtype == torch.bfloat16 else (lambda x: x)
    case = f"test_pieces_against_oracle[{str(state_dtype).split('.')[-1]}]"
    check(case, "o per head", worst_head_o(np64(o), o_r, None), BF16_TOL)
    check(case, "state per head", worst_head_state(np64(fin), rnd(f_r)), BF16_TOL)
    # block states: the oracle chained block by block from the same initial state
    got, s, worst = np64(bs), s0, 0.0
    for m in range(n_blocks):
        a, b = m * BLOCK, (m + 1) * BLOCK
        _, s = oracle.recurrence(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], None, s)
        worst = max(worst, worst_head_state(got[m:m + 1], rnd(s)))
    check(case, "block states", worst, BF16_TOL)
    assert np.isnan(got[n_blocks]).all()


@pytest.mark.parametrize("form", ["initial_state", "zero_state_and_cu_seqlens"])
def test_pieces_equal_the_caller_split(cuda_device, form):
    """The pieces path computes exactly what consecutive calls over the same chunk ranges
    compute, each from the previous one's fp32 final state: with an initial state, and
    from zeros with the one sequence given through cu_seqlens."""
    dev = cuda_device
    r = _inputs(92)
    sh = r.shape
    q, k, v, g, beta = (t.to(dev) for t in (r.q, r.k, r.v, r.g, r.beta))
    fin = torch.empty((1, sh.Hv, sh.dv, sh.dk), dtype=torch.float32, device=dev)
    if form == "initial_state":
        s0, cu = r.initial_state.to(dev), None
    else:
        s0, cu = None, torch.tensor([0, T], dtype=torch.int32, device=dev)
    o = gdn.gdn_chunk_prefill(q, k, v, g, beta, cu, s0, fin, check=True)
    bounds = _piece_bounds(T)
    assert len(bounds) == 9                      # eight pieces
    parts, state = [], s0
    for a, b in zip(bounds[:-1], bounds[1:]):
        assert b - a < 8 * 64 * 64               # each part alone takes the one-pass path
        nxt = torch.empty_like(fin)
        parts.append(gdn.gdn_chunk_prefill(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], None, state,
                                           nxt, check=True))
        state = nxt
    torch.cuda.synchronize()
    assert torch.equal(o, torch.cat(parts, 0))
    assert torch.equal(fin, state)


@pytest.mark.parametrize("T_call", [16384, 65536])
def test_launch_count_is_what_runs(cuda_device, T_call):
    """gdn_chunk_prefill_launches, which the benchmark reports as its kernel count, equals the
    number of this library's kernels one call runs (CUPTI trace): one pass at 16,384 tokens
    of the 27B layer, the up-front, beside-the-chain and chain launches at 65,536."""
    from torch.profiler import ProfilerActivity, profile
    dev = cuda_device
    sh = W.QWEN35_27B
    gen = torch.Generator(device="cpu").manual_seed(5)
    q = torch.randn((T_call, sh.Hk, sh.dk), generator=gen).to(torch.bfloat16).to(dev)
    k = torch.randn((T_call, sh.Hk, sh.dk), generator=gen).to(torch.bfloat16).to(dev)
    v = torch.randn((T_call, sh.Hv, sh.dv), generator=gen).to(torch.bfloat16).to(dev)
    g = (-0.3 * torch.rand((T_call, sh.Hv), generator=gen)).to(dev)
    beta = torch.sigmoid(torch.randn((T_call, sh.Hv), generator=gen)).to(dev)
    fin = torch.empty((1, sh.Hv, sh.dv, sh.dk), device=dev)
    o = torch.empty((T_call, sh.Hv, sh.dv), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(gdn.gdn_chunk_prefill_workspace_size(T_call, 1, sh.Hk, sh.Hv, sh.dk, sh.dv, torch.bfloat16),
                     dtype=torch.uint8, device=dev)
    run = lambda: gdn.gdn_chunk_prefill(q, k, v, g, beta, None, None, fin, 1.0, True, o, ws)
    run()
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        run()
        torch.cuda.synchronize()
    ours = [e.name for e in prof.events()
            if e.device_type == torch.autograd.DeviceType.CUDA and "chunk_" in e.name]
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    expect = gdn.gdn_chunk_prefill_launches(T_call, 1, sh.Hk, sh.Hv, sh.dk, sh.dv, torch.bfloat16, sms)
    assert len(ours) == expect, ours
    assert sum("chunk_plan" in n for n in ours) == 1
    assert sum("chunk_chain" in n for n in ours) == (1 if expect == 3 else 8)
