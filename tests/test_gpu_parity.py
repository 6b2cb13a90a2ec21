"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the same
seeded inputs.

Small cases are compared element by element and span several chunks and a ragged tail;
the full-size workloads run in the benchmark's launch configuration and are compared on
sampled heads/sequences that the oracle computes on its own.
"""
import numpy as np
import pytest
import torch

import gated_deltanet_mixer_causal_b200 as gdn
from gated_deltanet_mixer_causal_b200 import workloads as W
import oracle
from parity import (BF16_TOL, FP32_TOL, check, frob_rel, max_rel, np64, oracle_layer_heads,
                    worst_head_o, worst_head_state)

pytestmark = pytest.mark.gpu

_CACHE = {}


def cached(name, fn):
    """Large seeded workloads are generated once per session."""
    if name not in _CACHE:
        _CACHE[name] = fn()
    return _CACHE[name]


def to_dev(t, dev):
    return None if t is None else t.to(dev)


def run_layer(p, dev, conv_state_in=None, want_conv_state=False):
    sh = p.shape
    x = p.x.to(dev)
    cu = to_dev(p.cu_seqlens, dev)
    init = to_dev(p.initial_state, dev)
    fin = torch.empty((p.n_seq, sh.Hv, sh.dv, sh.dk), dtype=torch.float32, device=dev)
    cs_out = (torch.empty((p.n_seq, 3, sh.conv_channels), dtype=x.dtype, device=dev)
              if want_conv_state else None)
    o = gdn.prefill_layer(x, p.conv_w.to(dev), p.g.to(dev), p.beta.to(dev), sh.Hk, sh.Hv, sh.dk,
                          cu, init, to_dev(conv_state_in, dev), fin, cs_out)
    torch.cuda.synchronize()
    return o, fin, cs_out


# ------------------------------------------------------------------ fp32 tiny gate

def test_tiny_recurrence_fp32(cuda_device):
    r = W.tiny_recurrence()
    o_ref, f_ref = oracle.recurrence(r.q.numpy(), r.k.numpy(), r.v.numpy(), r.g.numpy(),
                                     r.beta.numpy())
    fin = torch.empty((1, 2, 16, 16), device=cuda_device)
    o = gdn.gdn_chunk_prefill(r.q.to(cuda_device), r.k.to(cuda_device), r.v.to(cuda_device),
                              r.g.to(cuda_device), r.beta.to(cuda_device), final_state=fin)
    check("test_tiny_recurrence_fp32", "max rel o", max_rel(np64(o), o_ref), FP32_TOL)
    check("test_tiny_recurrence_fp32", "max rel state", max_rel(np64(fin), f_ref), FP32_TOL)


def test_tiny_layer_fp32(cuda_device):
    p = W.tiny_layer()
    sh = p.shape
    o_ref, f_ref, cs_ref = oracle.layer_prefill(p.x.numpy(), p.conv_w.numpy(), p.g.numpy(),
                                                p.beta.numpy(), sh.Hk, sh.Hv, sh.dk, sh.dv)
    o, fin, cs = run_layer(p, cuda_device, want_conv_state=True)
    check("test_tiny_layer_fp32", "max rel o", max_rel(np64(o), o_ref), FP32_TOL)
    check("test_tiny_layer_fp32", "max rel state", max_rel(np64(fin), f_ref), FP32_TOL)
    np.testing.assert_array_equal(np64(cs), cs_ref)


# ----------------------------------------------------------------------------- conv

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_conv_varlen_edges(cuda_device, dtype):
    """Empty, 1-, 2-, 3-token sequences, run boundaries (31/32/33) and a ragged tail,
    with carried taps in and out."""
    rng = np.random.default_rng(21)
    lengths = [0, 1, 2, 3, 31, 32, 33, 0, 100, 5]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    T, Cc = int(cu[-1]), 96
    x = torch.from_numpy(rng.standard_normal((T, Cc), dtype=np.float32)).to(dtype)
    w = torch.from_numpy(rng.standard_normal((Cc, 4), dtype=np.float32) * 0.5).to(dtype)
    s_in = torch.from_numpy(rng.standard_normal((len(lengths), 3, Cc), dtype=np.float32)).to(dtype)
    y_ref, s_ref = oracle.conv1d_silu(np64(x), np64(w), cu, np64(s_in), return_state=True)
    s_out = torch.empty_like(s_in, device=cuda_device)
    y = gdn.gdn_conv1d_silu(x.to(cuda_device), w.to(cuda_device),
                            torch.from_numpy(cu).to(cuda_device), s_in.to(cuda_device), s_out)
    torch.cuda.synchronize()
    rtol = 2.0 ** -8 if dtype == torch.bfloat16 else 1e-5
    np.testing.assert_allclose(np64(y), y_ref, rtol=rtol, atol=1e-6)
    np.testing.assert_array_equal(np64(s_out), s_ref)


def test_conv_full_27b_rows(cuda_device):
    """The 27B-shaped conv at T=65536 in the benchmark's configuration; the oracle checks
    sampled token rows (each row needs only its three predecessors)."""
    p = cached('27b', W.qwen35_27b_prefill)
    y = gdn.gdn_conv1d_silu(p.x.to(cuda_device), p.conv_w.to(cuda_device))
    torch.cuda.synchronize()
    for t in [0, 1, 2, 3, 4095, 32768, 65535]:
        lo = max(0, t - 3)
        y_ref = oracle.conv1d_silu(p.x[lo:t + 1].float().numpy(), p.conv_w.float().numpy())
        # rows before t are reconstructed from a window starting at lo, so only row t is exact
        if lo == 0:
            ref = y_ref[t]
        else:
            ref = y_ref[-1]
        np.testing.assert_allclose(np64(y[t]), ref, rtol=2.0 ** -8, atol=1e-6)


# --------------------------------------------------------------------- bf16 prefill

def test_prefill_bf16_ragged_9b_shape(cuda_device):
    """9B-shaped heads, T = 300 (several chunks plus a ragged tail), every head compared."""
    p = W.make_prefill(W.QWEN35_9B, 300, seed=31, g_low=-0.5)
    sh = p.shape
    o_ref, f_ref, _ = oracle.layer_prefill(p.x.float().numpy(), p.conv_w.float().numpy(),
                                           p.g.numpy(), p.beta.numpy(), sh.Hk, sh.Hv, sh.dk, sh.dv)
    o, fin, _ = run_layer(p, cuda_device)
    check("test_prefill_bf16_ragged_9b_shape", "o per head", worst_head_o(np64(o), o_ref, None), BF16_TOL)
    check("test_prefill_bf16_ragged_9b_shape", "state per head", worst_head_state(np64(fin), f_ref), BF16_TOL)


def test_prefill_bf16_varlen_with_state(cuda_device):
    """27B-shaped heads, packed sequences of 1, 64, 65, 130, 7 and 0 tokens, nonzero
    initial states and carried conv taps; every sequence and head compared."""
    lengths = [1, 64, 65, 130, 7, 0]
    p = W.make_prefill(W.QWEN35_27B, 0, seed=32, g_low=-0.3, init_std=0.02, lengths=lengths)
    sh = p.shape
    rng = np.random.default_rng(33)
    cs_in = torch.from_numpy(rng.standard_normal((len(lengths), 3, sh.conv_channels),
                                                 dtype=np.float32)).to(torch.bfloat16)
    cu = p.cu_seqlens.numpy()
    o_ref, f_ref, cs_ref = oracle.layer_prefill(p.x.float().numpy(), p.conv_w.float().numpy(),
                                                p.g.numpy(), p.beta.numpy(), sh.Hk, sh.Hv,
                                                sh.dk, sh.dv, cu, p.initial_state.numpy(),
                                                cs_in.float().numpy())
    o, fin, cs = run_layer(p, cuda_device, conv_state_in=cs_in, want_conv_state=True)
    check("test_prefill_bf16_varlen_with_state", "o per head", worst_head_o(np64(o), o_ref, cu), BF16_TOL)
    check("test_prefill_bf16_varlen_with_state", "state per head", worst_head_state(np64(fin), f_ref), BF16_TOL)
    np.testing.assert_array_equal(np64(fin)[5], p.initial_state.numpy()[5])   # empty sequence
    np.testing.assert_array_equal(np64(cs), cs_ref)


def test_prefill_bf16_d128_without_l2norm(cuda_device):
    """bf16 heads of 128 with q and k used as given (qk_l2norm = 0): the shape the
    tensor-core path serves, but with the flag off, against the oracle without the norm.
    Keys are drawn at norm ~1 so the un-normalised delta rule stays bounded."""
    sh = W.LayerShape(2, 4, 128, 128)
    r = W.make_recurrence(sh, 200, seed=48, dtype=torch.float32, init_std=0.02)
    q = (r.q / np.sqrt(sh.dk)).to(torch.bfloat16)
    k = (r.k / np.sqrt(sh.dk)).to(torch.bfloat16)
    v = r.v.to(torch.bfloat16)
    fin = torch.empty((1, sh.Hv, sh.dv, sh.dk), dtype=torch.float32, device=cuda_device)
    o = gdn.gdn_chunk_prefill(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device),
                              r.g.to(cuda_device), r.beta.to(cuda_device), None,
                              r.initial_state.to(cuda_device), fin, 1.0, False)
    torch.cuda.synchronize()
    o_r, fin_r = oracle.recurrence(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                   r.g.numpy(), r.beta.numpy(), initial_state=r.initial_state.numpy(),
                                   l2norm=False)
    check("test_prefill_bf16_d128_without_l2norm", "o per head", worst_head_o(np64(o), o_r, [0, 200]), BF16_TOL)
    check("test_prefill_bf16_d128_without_l2norm", "state per head", worst_head_state(np64(fin), fin_r), BF16_TOL)


def test_prefill_status_after_a_call(cuda_device):
    """The status word of a completed tensor-core prefill reads OK, also through check=True;
    a recurrent-path call that was handed a workspace leaves it cleared."""
    sh = W.LayerShape(2, 4, 128, 128)
    r = W.make_recurrence(sh, 300, seed=54, dtype=torch.bfloat16)
    args = [t.to(cuda_device) for t in (r.q, r.k, r.v, r.g, r.beta)]
    need = gdn.gdn_chunk_prefill_workspace_size(300, 1, sh.Hk, sh.Hv, sh.dk, sh.dv, torch.bfloat16)
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device=cuda_device)   # garbage on entry
    gdn.gdn_chunk_prefill(*args, workspace=ws, check=True)
    gdn.gdn_prefill_status(ws)
    ws.fill_(0xFF)
    gdn.gdn_chunk_prefill(*args, qk_l2norm=False, workspace=ws)   # token-recurrent path
    gdn.gdn_prefill_status(ws)


def test_prefill_final_state_in_place(cuda_device):
    p = W.make_prefill(W.QWEN35_9B, 70, seed=34, init_std=0.02)
    sh = p.shape
    o_ref, f_ref, _ = oracle.layer_prefill(p.x.float().numpy(), p.conv_w.float().numpy(),
                                           p.g.numpy(), p.beta.numpy(), sh.Hk, sh.Hv, sh.dk, sh.dv,
                                           None, p.initial_state.numpy())
    st = p.initial_state.to(cuda_device).clone()
    o = gdn.prefill_layer(p.x.to(cuda_device), p.conv_w.to(cuda_device), p.g.to(cuda_device),
                          p.beta.to(cuda_device), sh.Hk, sh.Hv, sh.dk, initial_state=st,
                          final_state=st)
    torch.cuda.synchronize()
    check("test_prefill_final_state_in_place", "o per head", worst_head_o(np64(o), o_ref, None), BF16_TOL)
    check("test_prefill_final_state_in_place", "state per head", worst_head_state(np64(st), f_ref), BF16_TOL)


def test_prefill_empty_batch_passes_state(cuda_device):
    sh = W.QWEN35_9B
    init = torch.randn(1, sh.Hv, sh.dv, sh.dk, device=cuda_device)
    fin = torch.empty_like(init)
    e = torch.empty((0, sh.Hk, sh.dk), dtype=torch.bfloat16, device=cuda_device)
    ev = torch.empty((0, sh.Hv, sh.dv), dtype=torch.bfloat16, device=cuda_device)
    eg = torch.empty((0, sh.Hv), dtype=torch.float32, device=cuda_device)
    gdn.gdn_chunk_prefill(e, e, ev, eg, eg, initial_state=init, final_state=fin)
    torch.cuda.synchronize()
    assert torch.equal(fin, init)


def test_prefill_9b_full(cuda_device):
    """Qwen3.5-9B-shaped layer, T = 8192, every head against the oracle."""
    p = W.qwen35_9b_prefill()
    sh = p.shape
    o, fin, _ = run_layer(p, cuda_device)
    o_ref, f_ref, _ = oracle.layer_prefill(p.x.float().numpy(), p.conv_w.float().numpy(),
                                           p.g.numpy(), p.beta.numpy(), sh.Hk, sh.Hv, sh.dk, sh.dv)
    check("test_prefill_9b_full", "o per head", worst_head_o(np64(o), o_ref, None), BF16_TOL)
    check("test_prefill_9b_full", "state per head", worst_head_state(np64(fin), f_ref), BF16_TOL)


def test_prefill_27b_64k_sampled_heads(cuda_device):
    """Qwen3.5-27B-shaped layer at T = 65536 (the benchmark workload); value heads 0, 25
    and 47 (key heads 0, 8, 15) against the oracle over the whole sequence."""
    p = cached('27b', W.qwen35_27b_prefill)
    o, fin, _ = run_layer(p, cuda_device)
    heads = [0, 25, 47]
    ref = oracle_layer_heads(p, heads)
    o_np, f_np = np64(o), np64(fin)
    check("test_prefill_27b_64k_sampled_heads", "o per head",
          max(frob_rel(o_np[:, h], ref[(0, h)][0]) for h in heads), BF16_TOL)
    check("test_prefill_27b_64k_sampled_heads", "state per head",
          max(frob_rel(f_np[0, h], ref[(0, h)][1]) for h in heads), BF16_TOL)


def test_prefill_27b_varlen_sampled(cuda_device):
    """32 packed sequences (log-uniform lengths, nonzero initial states): the shortest
    sequence on every head and the longest on two heads."""
    p = W.qwen35_27b_varlen()
    o, fin, _ = run_layer(p, cuda_device)
    cu = p.cu_seqlens.numpy()
    lens = np.diff(cu)
    short, long_ = int(np.argmin(lens)), int(np.argmax(lens))
    o_np, f_np = np64(o), np64(fin)
    checks = [(short, list(range(p.shape.Hv))), (long_, [7, 40])]
    eo, es = 0.0, 0.0
    for n, heads in checks:
        ref = oracle_layer_heads(p, heads, seqs=[n])
        a, b = int(cu[n]), int(cu[n + 1])
        for h in heads:
            o_r, f_r = ref[(n, h)]
            eo = max(eo, frob_rel(o_np[a:b, h], o_r))
            es = max(es, frob_rel(f_np[n, h], f_r))
    check("test_prefill_27b_varlen_sampled", "o per head", eo, BF16_TOL)
    check("test_prefill_27b_varlen_sampled", "state per head", es, BF16_TOL)


# --------------------------------------------------------------------------- decode

def test_decode_fp32_small(cuda_device):
    d = W.make_decode(W.LayerShape(2, 4, 32, 32), B=3, steps=5, seed=41, dtype=torch.float32)
    sh = d.shape
    cs = d.conv_state.to(cuda_device).clone()
    st = d.state.to(cuda_device).clone()
    cs_r, st_r = d.conv_state.numpy().astype(np.float64), d.state.numpy().astype(np.float64)
    w = d.conv_w.to(cuda_device)
    for t in range(5):
        o = gdn.gdn_decode_step(d.xs[t].to(cuda_device), w, cs, d.gs[t].to(cuda_device),
                                d.betas[t].to(cuda_device), st, sh.Hk)
        o_r, st_r, cs_r = oracle.decode_step(d.xs[t].numpy(), d.conv_w.numpy(), cs_r,
                                             d.gs[t].numpy(), d.betas[t].numpy(), st_r, sh.Hk,
                                             sh.Hv, sh.dk, sh.dv)
        torch.cuda.synchronize()
        check("test_decode_fp32_small", "max rel o", max_rel(np64(o), o_r), FP32_TOL)
        check("test_decode_fp32_small", "max rel state", max_rel(np64(st), st_r), FP32_TOL)
        np.testing.assert_array_equal(np64(cs), cs_r)


def test_decode_27b_batch256_100_steps(cuda_device):
    """The 27B decode workload (B = 256, 100 steps, states updated in place); sequences
    0, 131 and 255 against the oracle after every 10th step."""
    d = W.qwen35_27b_decode()
    sh = d.shape
    sample = [0, 131, 255]
    cs = d.conv_state.to(cuda_device).clone()
    st = d.state.to(cuda_device).clone()
    w = d.conv_w.to(cuda_device)
    cs_r = d.conv_state.float().numpy()[sample].astype(np.float64)
    st_r = d.state.numpy()[sample].astype(np.float64)
    for t in range(100):
        o = gdn.gdn_decode_step(d.xs[t].to(cuda_device), w, cs, d.gs[t].to(cuda_device),
                                d.betas[t].to(cuda_device), st, sh.Hk)
        o_r, st_r, cs_r = oracle.decode_step(d.xs[t].float().numpy()[sample],
                                             d.conv_w.float().numpy(), cs_r,
                                             d.gs[t].numpy()[sample], d.betas[t].numpy()[sample],
                                             st_r, sh.Hk, sh.Hv, sh.dk, sh.dv)
        if (t + 1) % 10 == 0:
            torch.cuda.synchronize()
            o_g = np64(o)[sample]
            st_g = np64(st[sample])
            check(f"test_decode_27b_batch256_100_steps (step {t + 1})", "o per head",
                  max(frob_rel(o_g[j, h], o_r[j, h]) for j in range(len(sample)) for h in range(sh.Hv)),
                  BF16_TOL)
            check(f"test_decode_27b_batch256_100_steps (step {t + 1})", "state per head",
                  max(frob_rel(st_g[j, h], st_r[j, h]) for j in range(len(sample)) for h in range(sh.Hv)),
                  BF16_TOL)
            np.testing.assert_array_equal(np64(cs[sample]), cs_r)


def test_decode_matches_prefill_on_gpu(cuda_device):
    """Eight decode steps and a prefill of the same eight tokens from the same states, each
    against the oracle's eight steps (bf16 tolerance)."""
    sh = W.LayerShape(2, 6, 64, 64)
    d = W.make_decode(sh, B=2, steps=8, seed=42)
    cs = d.conv_state.to(cuda_device).clone()
    st = d.state.to(cuda_device).clone()
    w = d.conv_w.to(cuda_device)
    outs = []
    for t in range(8):
        outs.append(gdn.gdn_decode_step(d.xs[t].to(cuda_device), w, cs, d.gs[t].to(cuda_device),
                                        d.betas[t].to(cuda_device), st, sh.Hk))
    x = torch.stack(d.xs, 1).reshape(16, -1).to(cuda_device)
    g = torch.stack(d.gs, 1).reshape(16, -1).to(cuda_device)
    b = torch.stack(d.betas, 1).reshape(16, -1).to(cuda_device)
    cu = torch.tensor([0, 8, 16], dtype=torch.int32, device=cuda_device)
    fin = torch.empty_like(st)
    o_p = gdn.prefill_layer(x, w, g, b, sh.Hk, sh.Hv, sh.dk, cu, d.state.to(cuda_device),
                            d.conv_state.to(cuda_device), fin)
    torch.cuda.synchronize()
    o_d = torch.stack(outs, 1).reshape(16, sh.Hv, sh.dv)
    o_r, st_r, _ = oracle.decode_tokens(torch.stack(d.xs, 1).float().numpy(), d.conv_w.float().numpy(),
                                        d.conv_state.float().numpy(), torch.stack(d.gs, 1).numpy(),
                                        torch.stack(d.betas, 1).numpy(), d.state.numpy(), sh.Hk, sh.Hv,
                                        sh.dk, sh.dv)
    o_r = o_r.reshape(16, sh.Hv, sh.dv)
    for name, o, s in (("8 decode steps", o_d, st), ("prefill of the 8 tokens", o_p, fin)):
        check(f"test_decode_matches_prefill_on_gpu ({name})", "o per head",
              worst_head_o(np64(o), o_r, [0, 8, 16]), BF16_TOL)
        check(f"test_decode_matches_prefill_on_gpu ({name})", "state per head",
              worst_head_state(np64(s), st_r), BF16_TOL)


# ------------------------------------------------------------ multi-token decode

# the token count is a template parameter of the kernel: every count is its own code path
@pytest.mark.parametrize("n_tok", [1, 2, 3, 4, 5, 6, 7, 8])
def test_decode_tokens_fp32_small(cuda_device, n_tok):
    """n_tok tokens per sequence in one call against the oracle (fp32, element by element);
    n_tok < 3 keeps old taps in the new conv state, n_tok >= 3 replaces them all."""
    sh = W.LayerShape(2, 4, 32, 32)
    d = W.make_decode(sh, B=3, steps=n_tok, seed=43 + n_tok, dtype=torch.float32)
    x = torch.stack(d.xs, 1); g = torch.stack(d.gs, 1); b = torch.stack(d.betas, 1)
    cs = d.conv_state.to(cuda_device).clone()
    st = d.state.to(cuda_device).clone()
    o = gdn.gdn_decode_tokens(x.to(cuda_device), d.conv_w.to(cuda_device), cs, g.to(cuda_device),
                              b.to(cuda_device), st, sh.Hk)
    torch.cuda.synchronize()
    o_r, st_r, cs_r = oracle.decode_tokens(x.numpy(), d.conv_w.numpy(), d.conv_state.numpy(),
                                           g.numpy(), b.numpy(), d.state.numpy(), sh.Hk, sh.Hv,
                                           sh.dk, sh.dv)
    assert o.shape == (3, n_tok, sh.Hv, sh.dv)
    check("test_decode_tokens_fp32_small", "max rel o", max_rel(np64(o), o_r), FP32_TOL)
    check("test_decode_tokens_fp32_small", "max rel state", max_rel(np64(st), st_r), FP32_TOL)
    np.testing.assert_array_equal(np64(cs), cs_r)


@pytest.mark.parametrize("n_tok", [1, 2, 3, 4, 5, 6, 7, 8])
def test_decode_tokens_27b_bf16(cuda_device, n_tok):
    """27B-shaped heads, 16 sequences, n_tok tokens each in one call, every head against the
    oracle (bf16 tolerance); the conv taps are copies and must match exactly."""
    d = W.make_decode(W.QWEN35_27B, B=16, steps=n_tok, seed=44)
    sh = d.shape
    x = torch.stack(d.xs, 1); g = torch.stack(d.gs, 1); b = torch.stack(d.betas, 1)
    cs = d.conv_state.to(cuda_device).clone()
    st = d.state.to(cuda_device).clone()
    o = gdn.gdn_decode_tokens(x.to(cuda_device), d.conv_w.to(cuda_device), cs, g.to(cuda_device),
                              b.to(cuda_device), st, sh.Hk)
    torch.cuda.synchronize()
    o_r, st_r, cs_r = oracle.decode_tokens(x.float().numpy(), d.conv_w.float().numpy(),
                                           d.conv_state.float().numpy(), g.numpy(), b.numpy(),
                                           d.state.numpy(), sh.Hk, sh.Hv, sh.dk, sh.dv)
    o_g, st_g = np64(o), np64(st)
    check(f"test_decode_tokens_27b_bf16[{n_tok}]", "o per head",
          max(frob_rel(o_g[j, :, h], o_r[j, :, h]) for j in range(16) for h in range(sh.Hv)), BF16_TOL)
    check(f"test_decode_tokens_27b_bf16[{n_tok}]", "state per head",
          max(frob_rel(st_g[j, h], st_r[j, h]) for j in range(16) for h in range(sh.Hv)), BF16_TOL)
    np.testing.assert_array_equal(np64(cs), cs_r)


def test_decode_tokens_and_single_steps_against_oracle(cuda_device):
    """Four tokens in one call and four gdn_decode_step calls from the same states, each
    against the oracle's four steps (27B-shaped heads, 8 sequences)."""
    d = W.make_decode(W.QWEN35_27B, B=8, steps=4, seed=45)
    sh = d.shape
    w = d.conv_w.to(cuda_device)
    cs1 = d.conv_state.to(cuda_device).clone(); st1 = d.state.to(cuda_device).clone()
    outs = [gdn.gdn_decode_step(d.xs[t].to(cuda_device), w, cs1, d.gs[t].to(cuda_device),
                                d.betas[t].to(cuda_device), st1, sh.Hk) for t in range(4)]
    cs4 = d.conv_state.to(cuda_device).clone(); st4 = d.state.to(cuda_device).clone()
    x = torch.stack(d.xs, 1); g = torch.stack(d.gs, 1); b = torch.stack(d.betas, 1)
    o4 = gdn.gdn_decode_tokens(x.to(cuda_device), w, cs4, g.to(cuda_device), b.to(cuda_device),
                               st4, sh.Hk)
    torch.cuda.synchronize()
    o_r, st_r, cs_r = oracle.decode_tokens(x.float().numpy(), d.conv_w.float().numpy(),
                                           d.conv_state.float().numpy(), g.numpy(), b.numpy(),
                                           d.state.numpy(), sh.Hk, sh.Hv, sh.dk, sh.dv)
    o1 = np64(torch.stack(outs, 1))
    for name, o, st, cs in (("single steps", o1, np64(st1), cs1), ("one 4-token call", np64(o4), np64(st4), cs4)):
        check(f"test_decode_tokens_and_single_steps_against_oracle ({name})", "o per head",
              max(frob_rel(o[j, :, h], o_r[j, :, h]) for j in range(8) for h in range(sh.Hv)), BF16_TOL)
        check(f"test_decode_tokens_and_single_steps_against_oracle ({name})", "state per head",
              max(frob_rel(st[j, h], st_r[j, h]) for j in range(8) for h in range(sh.Hv)), BF16_TOL)
        np.testing.assert_array_equal(np64(cs), cs_r)


# ---------------------------------------------------------------- bf16 states

def test_decode_bf16_state_27b(cuda_device):
    """27B-shaped heads, 16 sequences, 20 single-token steps with the states stored in bf16;
    the oracle rounds its state to bf16 after every step. Checked every 5th step."""
    d = W.make_decode(W.QWEN35_27B, B=16, steps=20, seed=46)
    sh = d.shape
    st_r = oracle.round_bf16(d.state.numpy())
    st = torch.from_numpy(st_r).to(torch.bfloat16).to(cuda_device)
    cs = d.conv_state.to(cuda_device).clone()
    cs_r = d.conv_state.float().numpy().astype(np.float64)
    w = d.conv_w.to(cuda_device)
    for t in range(20):
        o = gdn.gdn_decode_step(d.xs[t].to(cuda_device), w, cs, d.gs[t].to(cuda_device),
                                d.betas[t].to(cuda_device), st, sh.Hk)
        o_r, st_r, cs_r = oracle.decode_step(d.xs[t].float().numpy(), d.conv_w.float().numpy(),
                                             cs_r, d.gs[t].numpy(), d.betas[t].numpy(), st_r,
                                             sh.Hk, sh.Hv, sh.dk, sh.dv, state_dtype="bf16")
        if (t + 1) % 5 == 0:
            torch.cuda.synchronize()
            o_g, st_g = np64(o), np64(st)
            check(f"test_decode_bf16_state_27b (step {t + 1})", "o per head",
                  max(frob_rel(o_g[j, h], o_r[j, h]) for j in range(16) for h in range(sh.Hv)), BF16_TOL)
            check(f"test_decode_bf16_state_27b (step {t + 1})", "state per head",
                  max(frob_rel(st_g[j, h], st_r[j, h]) for j in range(16) for h in range(sh.Hv)), BF16_TOL)
            np.testing.assert_array_equal(np64(cs), cs_r)
    assert st.dtype == torch.bfloat16


@pytest.mark.parametrize("n_tok", [1, 4])
def test_decode_tokens_bf16_state_27b(cuda_device, n_tok):
    """n_tok tokens in one call with a bf16 state (rounded once, after the last token)."""
    d = W.make_decode(W.QWEN35_27B, B=16, steps=n_tok, seed=47)
    sh = d.shape
    x = torch.stack(d.xs, 1); g = torch.stack(d.gs, 1); b = torch.stack(d.betas, 1)
    s0 = oracle.round_bf16(d.state.numpy())
    st = torch.from_numpy(s0).to(torch.bfloat16).to(cuda_device)
    cs = d.conv_state.to(cuda_device).clone()
    o = gdn.gdn_decode_tokens(x.to(cuda_device), d.conv_w.to(cuda_device), cs, g.to(cuda_device),
                              b.to(cuda_device), st, sh.Hk)
    torch.cuda.synchronize()
    o_r, st_r, cs_r = oracle.decode_tokens(x.float().numpy(), d.conv_w.float().numpy(),
                                           d.conv_state.float().numpy(), g.numpy(), b.numpy(), s0,
                                           sh.Hk, sh.Hv, sh.dk, sh.dv, state_dtype="bf16")
    o_g, st_g = np64(o), np64(st)
    check(f"test_decode_tokens_bf16_state_27b[{n_tok}]", "o per head",
          max(frob_rel(o_g[j, :, h], o_r[j, :, h]) for j in range(16) for h in range(sh.Hv)), BF16_TOL)
    check(f"test_decode_tokens_bf16_state_27b[{n_tok}]", "state per head",
          max(frob_rel(st_g[j, h], st_r[j, h]) for j in range(16) for h in range(sh.Hv)), BF16_TOL)
    np.testing.assert_array_equal(np64(cs), cs_r)


# ------------------------------------------------------- states at block boundaries

def _block_state_reference(r, lengths, block, rows, n_rows, l2norm=True):
    """Oracle state after each block of each sequence: the recurrence over that prefix."""
    ref = {}
    cu = np.concatenate([[0], np.cumsum(lengths)])
    for n, L in enumerate(lengths):
        for m in range(1, L // block + 1):
            row = rows[n] + m - 1
            if not 0 <= row < n_rows:
                continue
            a, b = cu[n], cu[n] + m * block
            _, fin = oracle.recurrence(r.q[a:b].float().numpy(), r.k[a:b].float().numpy(),
                                       r.v[a:b].float().numpy(), r.g[a:b].numpy(), r.beta[a:b].numpy(),
                                       initial_state=r.initial_state[n:n + 1].numpy(), l2norm=l2norm)
            ref[row] = fin[0]
    return ref


def _run_with_blocks(r, dev, block, rows, n_rows):
    sh = r.shape
    n = r.cu_seqlens.numel() - 1
    bs = torch.full((n_rows, sh.Hv, sh.dv, sh.dk), float("nan"), dtype=torch.float32, device=dev)
    fin = torch.empty((n, sh.Hv, sh.dv, sh.dk), dtype=torch.float32, device=dev)
    args = (r.q.to(dev), r.k.to(dev), r.v.to(dev), r.g.to(dev), r.beta.to(dev), r.cu_seqlens.to(dev),
            r.initial_state.to(dev))
    o = gdn.gdn_chunk_prefill(*args, fin, 1.0, True, block_tokens=block, block_states=bs,
                              block_rows=torch.tensor(rows, dtype=torch.int32, device=dev))
    fin0 = torch.empty_like(fin)
    o0 = gdn.gdn_chunk_prefill(*args, fin0, 1.0, True)
    torch.cuda.synchronize()
    assert torch.equal(o, o0) and torch.equal(fin, fin0)   # block states change nothing else
    return np64(bs)


def test_prefill_block_states_bf16(cuda_device):
    """Tensor-core path (bf16, heads of 128): block states of four packed sequences, one of
    them shorter than a block and one a multiple of the block, against oracle prefixes."""
    lengths, block = [300, 128, 1000, 64], 128
    r = W.make_recurrence(W.LayerShape(2, 4, 128, 128), 0, seed=49, dtype=torch.bfloat16,
                          init_std=0.02, lengths=lengths)
    rows = [0, 2, 3, 10]
    got = _run_with_blocks(r, cuda_device, block, rows, 10)
    ref = _block_state_reference(r, lengths, block, rows, 10)
    assert sorted(ref) == list(range(10))
    check("test_prefill_block_states_bf16", "state per head",
          max(frob_rel(got[row, h], s_ref[h]) for row, s_ref in ref.items() for h in range(4)), BF16_TOL)


def test_prefill_block_states_fp32_rows_out_of_range(cuda_device):
    """Token-recurrent path (fp32): block states against oracle prefixes; rows past the end
    of block_states are skipped and the buffer's other rows stay untouched."""
    lengths, block = [150, 64, 200], 64
    r = W.make_recurrence(W.LayerShape(2, 2, 16, 16), 0, seed=50, dtype=torch.float32,
                          init_std=0.1, lengths=lengths)
    rows, n_rows = [0, 3, 4], 6        # sequence 2's third boundary would be row 6: skipped;
    got = _run_with_blocks(r, cuda_device, block, rows, n_rows)   # row 2 is never written
    ref = _block_state_reference(r, lengths, block, rows, n_rows)
    assert sorted(ref) == [0, 1, 3, 4, 5]
    check("test_prefill_block_states_fp32_rows_out_of_range", "max rel state",
          max(max_rel(got[row], s_ref) for row, s_ref in ref.items()), FP32_TOL)
    assert np.isnan(got[2]).all()


# ------------------------------------------------------- bf16 states in the prefill

@pytest.mark.parametrize("path", ["chunked_tc", "recurrent"])
def test_prefill_bf16_states(cuda_device, path):
    """Initial, final and block states stored in bf16 (fp32 math): 27B-shaped heads on the
    tensor-core path, and fp32 activations with heads of 32 on the token-recurrent path. The
    oracle starts from the same bf16 initial states and rounds its fp64 final and block states
    to bf16 once, as the kernels do; per-head bf16 gate."""
    dev = cuda_device
    if path == "chunked_tc":
        sh, dt, lengths = W.QWEN35_27B, torch.bfloat16, [300, 129, 64]
    else:
        sh, dt, lengths = W.LayerShape(2, 4, 32, 32), torch.float32, [150, 64, 70]
    r = W.make_recurrence(sh, 0, seed=57, dtype=dt, init_std=0.02, lengths=lengths)
    assert gdn.gdn_chunk_prefill_path(dt, sh.Hk, sh.Hv, sh.dk, sh.dv) == path
    s0 = oracle.round_bf16(r.initial_state.numpy())
    init = torch.from_numpy(s0).to(torch.bfloat16).to(dev)
    n = len(lengths)
    fin = torch.empty((n, sh.Hv, sh.dv, sh.dk), dtype=torch.bfloat16, device=dev)
    bs = torch.full((8, sh.Hv, sh.dv, sh.dk), float("nan"), dtype=torch.bfloat16, device=dev)
    rows = torch.tensor([0, 4, 6], dtype=torch.int32, device=dev)
    o = gdn.gdn_chunk_prefill(r.q.to(dev), r.k.to(dev), r.v.to(dev), r.g.to(dev), r.beta.to(dev),
                              r.cu_seqlens.to(dev), init, fin, block_tokens=64, block_states=bs,
                              block_rows=rows)
    torch.cuda.synchronize()
    cu = r.cu_seqlens.numpy()
    o_r, f_r = oracle.recurrence(r.q.float().numpy(), r.k.float().numpy(), r.v.float().numpy(),
                                 r.g.numpy(), r.beta.numpy(), cu, s0)
    case = f"test_prefill_bf16_states[{path}]"
    tol = BF16_TOL if dt == torch.bfloat16 else FP32_TOL
    if dt == torch.bfloat16:
        check(case, "o per head", worst_head_o(np64(o), o_r, cu), tol)
    else:
        check(case, "max rel o", max_rel(np64(o), o_r), tol)
    check(case, "state per head", worst_head_state(np64(fin), oracle.round_bf16(f_r)), BF16_TOL)
    assert fin.dtype == torch.bfloat16
    # block states: rows 0..3 = sequence 0 after 64, 128, 192, 256 tokens; rows 4, 5 =
    # sequence 1 after 64, 128; row 6 = sequence 2 after 64 (its final state); row 7 unused
    want = {0: (0, 64), 1: (0, 128), 2: (0, 192), 3: (0, 256), 4: (1, 64), 5: (1, 128), 6: (2, 64)}
    got = np64(bs)
    worst = 0.0
    for row, (nq, m) in want.items():
        a = cu[nq]
        _, fr = oracle.recurrence(r.q[a:a + m].float().numpy(), r.k[a:a + m].float().numpy(),
                                  r.v[a:a + m].float().numpy(), r.g[a:a + m].numpy(),
                                  r.beta[a:a + m].numpy(), initial_state=s0[nq:nq + 1])
        worst = max(worst, worst_head_state(got[row:row + 1], oracle.round_bf16(fr)))
    check(case, "block states", worst, BF16_TOL)
    assert np.isnan(got[7]).all()
