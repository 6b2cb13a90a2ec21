"""The seeded input generators that the parity tests and the benchmark share: the same seed
draws the same inputs, different seeds differ, and the draws have the stated distributions
(x ~ N(0, 1), conv w ~ N(0, 0.5), g ~ U[g_low, 0], beta = sigmoid(N(0, 1)), log-uniform
varlen lengths in [512, 32768])."""
import math

import numpy as np
import torch

from gated_deltanet_mixer_causal_b200 import workloads as W


def test_same_seed_same_inputs_other_seed_other_inputs():
    a = W.make_prefill(W.TINY, 256, seed=5, init_std=0.1)
    b = W.make_prefill(W.TINY, 256, seed=5, init_std=0.1)
    c = W.make_prefill(W.TINY, 256, seed=6, init_std=0.1)
    for name in ("x", "conv_w", "g", "beta", "initial_state"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
        assert not torch.equal(getattr(a, name), getattr(c, name)), name
    d1 = W.make_decode(W.TINY, B=4, steps=3, seed=5)
    d2 = W.make_decode(W.TINY, B=4, steps=3, seed=5)
    assert all(torch.equal(u, v) for u, v in zip(d1.xs + d1.gs + d1.betas, d2.xs + d2.gs + d2.betas))
    assert torch.equal(d1.state, d2.state) and torch.equal(d1.conv_state, d2.conv_state)


def test_stated_distributions():
    p = W.make_prefill(W.QWEN35_9B, 2048, seed=1, g_low=-0.5, dtype=torch.float32)
    x, w, g, b = (t.double().numpy() for t in (p.x, p.conv_w, p.g, p.beta))
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    assert abs(w.std() - 0.5) < 0.02
    assert g.min() >= -0.5 and g.max() <= 0.0 and abs(g.mean() + 0.25) < 0.01
    logit = np.log(b / (1 - b))
    assert 0 < b.min() and b.max() < 1 and abs(logit.std() - 1.0) < 0.02
    assert p.x.shape == (2048, W.QWEN35_9B.conv_channels) and W.QWEN35_9B.conv_channels == 8192


def test_varlen_lengths_are_log_uniform_within_bounds():
    p = W.make_prefill(W.TINY, 0, seed=4, varlen_n=400)
    L = np.diff(p.cu_seqlens.numpy())
    assert len(L) == 400 and L.min() >= 512 and L.max() <= 32768 and p.T == L.sum()
    u = (np.log(L) - math.log(512)) / (math.log(32768) - math.log(512))
    assert abs(u.mean() - 0.5) < 0.05 and abs(u.std() - math.sqrt(1 / 12)) < 0.03
