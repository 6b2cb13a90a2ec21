"""Chunked (WY / UT-transform) form of the gated delta rule, fp64 numpy.

TEST INFRASTRUCTURE. This is not the oracle: it is a second, independent derivation that
the pins compare against the sequential oracle ("chunked == sequential"), and a readable
statement of the algebra the GPU prefill follows. It shares no code with the CUDA path.

The pages give only the per-token update (romaanj.github.io "Inside Qwen3.5", section 5:
S <- alpha S + beta (v - S k) k^T, decay first). Within a chunk of L tokens starting
from state S0, write u_r = beta_r (v_r - alpha_r S_{r-1} k_r), so S_r = alpha_r S_{r-1} +
u_r k_r^T. With G_r = sum_{i<=r} g_i (inclusive, in-chunk) the unrolled state is

    S_r = e^{G_r} S0 + sum_{i<=r} e^{G_r - G_i} u_i k_i^T,

hence (I + A) U = diag(beta) V - diag(beta e^G) K S0^T with
A_ri = beta_r e^{G_r - G_i} (k_r . k_i) for i < r (strictly lower triangular). With
Tm = (I + A)^{-1}:

    W  = Tm diag(beta e^G) K,      U~ = Tm diag(beta) V,      U = U~ - W S0^T
    O  = diag(e^G) Q S0^T + (M o Q K^T) U,     M_ri = e^{G_r - G_i} (i <= r), else 0
    S_L = e^{G_{L-1}} S0 + U^T diag(e^{G_{L-1} - G}) K
"""
from __future__ import annotations

import numpy as np

L2_EPS = 1e-6


def _l2(x, on, eps):
    x = np.asarray(x, np.float64)
    if not on:
        return x
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def chunk_step(Q, K, V, g, beta, S0):
    """One chunk for one (sequence, v-head): Q, K [L, dk]; V [L, dv]; g, beta [L];
    S0 [dv, dk]. Returns (O [L, dv], S_L)."""
    L = Q.shape[0]
    G = np.cumsum(g)
    diff = G[:, None] - G[None, :]
    lower = np.tril(np.ones((L, L), bool))
    strict = np.tril(np.ones((L, L), bool), -1)
    decay = np.where(lower, np.exp(np.where(lower, diff, 0.0)), 0.0)
    A = np.where(strict, beta[:, None] * decay * (K @ K.T), 0.0)
    Tm = np.linalg.inv(np.eye(L) + A)
    W = Tm @ ((beta * np.exp(G))[:, None] * K)
    Ut = Tm @ (beta[:, None] * V)
    U = Ut - W @ S0.T
    O = np.exp(G)[:, None] * (Q @ S0.T) + (decay * (Q @ K.T)) @ U
    S = np.exp(G[-1]) * S0 + U.T @ (np.exp(G[-1] - G)[:, None] * K)
    return O, S


def chunked_recurrence(q, k, v, g, beta, cu_seqlens=None, initial_state=None, chunk=64,
                       scale=1.0, l2norm=True, eps=L2_EPS):
    """Same contract as ``oracle.recurrence``; chunks restart at every sequence start."""
    q = _l2(q, l2norm, eps); k = _l2(k, l2norm, eps)
    v = np.asarray(v, np.float64); g = np.asarray(g, np.float64)
    beta = np.asarray(beta, np.float64)
    T, Hk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    G = Hv // Hk
    cu = np.array([0, T]) if cu_seqlens is None else np.asarray(cu_seqlens)
    n_seq = len(cu) - 1
    o = np.zeros((T, Hv, dv))
    fin = np.zeros((n_seq, Hv, dv, dk))
    for n in range(n_seq):
        bos, eos = int(cu[n]), int(cu[n + 1])
        for h in range(Hv):
            hk = h // G
            S = np.zeros((dv, dk)) if initial_state is None else np.array(initial_state[n, h], np.float64)
            for c0 in range(bos, eos, chunk):
                sl = slice(c0, min(c0 + chunk, eos))
                O, S = chunk_step(q[sl, hk], k[sl, hk], v[sl, h], g[sl, h], beta[sl, h], S)
                o[sl, h] = scale * O
            fin[n, h] = S
    return o, fin
