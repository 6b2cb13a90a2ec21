"""Parity metrics and oracle helpers shared by the GPU parity tests.

Tolerances (the mixer's stated gates):
  fp32 inputs: max|x - r| / max|r| <= 1e-4 per tensor;
  bf16 inputs: ||x_h - r_h||_F / ||r_h||_F <= 2e-2 per (sequence, value head), for the
  outputs (over tokens x dv) and for the final states.
"""
import numpy as np
import torch

import oracle

FP32_TOL = 1e-4
BF16_TOL = 2e-2

# (test case, quantity, worst error, tolerance) of every checked comparison; the terminal
# summary prints them so that each parity test's margin is on record.
MARGINS = []


def check(case: str, what: str, err: float, tol: float) -> float:
    """Record a worst error against its tolerance, then assert it is within."""
    MARGINS.append((case, what, float(err), float(tol)))
    assert err <= tol, f"{case}: {what} error {err:.3e} > {tol:.1e}"
    return err


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def max_rel(x, r) -> float:
    x = np.asarray(x, np.float64); r = np.asarray(r, np.float64)
    return float(np.max(np.abs(x - r)) / max(np.max(np.abs(r)), 1e-30))


def frob_rel(x, r) -> float:
    x = np.asarray(x, np.float64); r = np.asarray(r, np.float64)
    return float(np.linalg.norm(x - r) / max(np.linalg.norm(r), 1e-30))


def worst_head_o(o, o_ref, cu) -> float:
    """Worst per-(sequence, head) relative Frobenius error of o [T, Hv, dv]."""
    cu = [0, o.shape[0]] if cu is None else list(np.asarray(cu))
    worst = 0.0
    for n in range(len(cu) - 1):
        a, b = int(cu[n]), int(cu[n + 1])
        if b == a:
            continue
        for h in range(o.shape[1]):
            worst = max(worst, frob_rel(o[a:b, h], o_ref[a:b, h]))
    return worst


def worst_head_state(s, s_ref) -> float:
    worst = 0.0
    for n in range(s.shape[0]):
        for h in range(s.shape[1]):
            worst = max(worst, frob_rel(s[n, h], s_ref[n, h]))
    return worst


def head_channels(Hk, Hv, d, heads):
    """Conv channels of q, k (key head h // G) and v for each listed value head, as one
    [q_0..q_m | k_0..k_m | v_0..v_m] block that the oracle treats as m independent heads."""
    G = Hv // Hk
    qs, ks, vs = [], [], []
    for h in heads:
        hk = h // G
        qs.append(np.arange(hk * d, (hk + 1) * d))
        ks.append(np.arange(Hk * d + hk * d, Hk * d + (hk + 1) * d))
        vs.append(np.arange(2 * Hk * d + h * d, 2 * Hk * d + (h + 1) * d))
    return np.concatenate(qs + ks + vs)


def oracle_layer_heads(p, heads, seqs=None):
    """Oracle outputs for selected value heads (and optionally selected sequences) of a
    packed prefill workload: returns {(n, h): (o [L, d], final [d, d])}."""
    sh = p.shape
    d = sh.dk
    ch = head_channels(sh.Hk, sh.Hv, d, heads)
    cu = None if p.cu_seqlens is None else p.cu_seqlens.numpy()
    bounds = [(0, p.T)] if cu is None else [(int(cu[i]), int(cu[i + 1])) for i in range(len(cu) - 1)]
    seqs = range(len(bounds)) if seqs is None else seqs
    m = len(heads)
    out = {}
    cht = torch.from_numpy(ch)
    w = p.conv_w.float().numpy()[ch]
    for n in seqs:
        a, b = bounds[n]
        xs = p.x[a:b][:, cht].float().numpy()
        init = None
        if p.initial_state is not None:
            init = p.initial_state[n:n + 1, heads].numpy().astype(np.float64)
        o, fin, _ = oracle.layer_prefill(xs, w, p.g[a:b, heads].numpy(), p.beta[a:b, heads].numpy(),
                                         m, m, d, d, None, init)
        for j, h in enumerate(heads):
            out[(n, h)] = (o[:, j], fin[0, j])
    return out
