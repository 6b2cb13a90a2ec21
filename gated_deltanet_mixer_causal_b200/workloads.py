"""Seeded synthetic inputs shaped like the Qwen3.5 Gated DeltaNet layers.

This module draws random numbers and rounds them to the input dtype; it holds none of
the mixer's arithmetic. Both the CUDA path and the fp64 oracle consume exactly the
arrays made here (bf16 or fp32), so the two sides see identical bytes.

Shapes come from the pages: Qwen3.5-27B Gated DeltaNet layers have 16 key heads and 48
value heads of 128 with conv kernel 4 and an fp32 state ("Inside Qwen3.5", config
footnote); Qwen3.5-9B layers have 32 heads of 128 ("hybrid-mamba-transformer-bench",
section 1), 16 of which serve q/k here. Distributions: x ~ N(0, 1) for the pre-conv q|k|v
channels, conv taps ~ N(0, 0.5) (standard deviation), log-decay g ~ U[lo, 0],
beta = sigmoid(N(0, 1)), initial states ~ N(0, 0.02). Numbers are drawn with numpy's
PCG64 generator in a fixed order: lengths (varlen only), x, conv w, g, beta, initial
states (or, for decode, states, conv taps, then per step x, g, beta).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class LayerShape:
    Hk: int
    Hv: int
    dk: int
    dv: int

    @property
    def conv_channels(self) -> int:
        return 2 * self.Hk * self.dk + self.Hv * self.dv


QWEN35_9B = LayerShape(Hk=16, Hv=32, dk=128, dv=128)     # 2048 + 2048 + 4096 channels
QWEN35_27B = LayerShape(Hk=16, Hv=48, dk=128, dv=128)    # 2048 + 2048 + 6144 channels
TINY = LayerShape(Hk=2, Hv=2, dk=16, dv=16)


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def _normal(rng, shape, std=1.0, block_rows=4096) -> np.ndarray:
    """float32 normals drawn in row blocks (bounded host memory for the 64K inputs)."""
    out = np.empty(shape, np.float32)
    flat = out.reshape(shape[0], -1)
    for r0 in range(0, shape[0], block_rows):
        r1 = min(shape[0], r0 + block_rows)
        flat[r0:r1] = rng.standard_normal((r1 - r0, flat.shape[1]), dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out


def _sigmoid(z: np.ndarray) -> np.ndarray:
    return (1.0 / (1.0 + np.exp(-z.astype(np.float64)))).astype(np.float32)


def _as(a: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(dtype)


@dataclasses.dataclass
class PrefillInputs:
    """One packed prefill batch. ``x`` holds the pre-conv q|k|v channels."""
    shape: LayerShape
    x: torch.Tensor                  # [T, Cc]  dtype
    conv_w: torch.Tensor             # [Cc, 4]  dtype
    g: torch.Tensor                  # [T, Hv]  fp32 log-decay
    beta: torch.Tensor               # [T, Hv]  fp32
    cu_seqlens: Optional[torch.Tensor]   # int32 [N+1] or None
    initial_state: Optional[torch.Tensor]  # fp32 [N, Hv, dv, dk] or None
    chunk: int = 64

    @property
    def T(self) -> int:
        return self.x.shape[0]

    @property
    def n_seq(self) -> int:
        return 1 if self.cu_seqlens is None else self.cu_seqlens.numel() - 1


def make_prefill(shape: LayerShape, T: int, seed: int, dtype=torch.bfloat16,
                 g_low: float = -0.5, init_std: Optional[float] = None,
                 lengths: Optional[List[int]] = None, conv_std: float = 0.5,
                 varlen_n: Optional[int] = None) -> PrefillInputs:
    """``varlen_n`` draws that many log-uniform lengths in [512, 32768] first."""
    rng = _rng(seed)
    cu = None
    if varlen_n is not None:
        lengths = _loguniform_lengths(rng, varlen_n, 512, 32768)
    if lengths is not None:
        T = int(sum(lengths))
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32))
    Cc = shape.conv_channels
    x = _normal(rng, (T, Cc))
    w = _normal(rng, (Cc, 4), std=conv_std)
    g = rng.uniform(g_low, 0.0, size=(T, shape.Hv)).astype(np.float32)
    beta = _sigmoid(rng.standard_normal((T, shape.Hv)))
    n_seq = 1 if lengths is None else len(lengths)
    init = None
    if init_std is not None:
        init = _as(_normal(rng, (n_seq, shape.Hv, shape.dv, shape.dk), std=init_std), torch.float32)
    return PrefillInputs(shape, _as(x, dtype), _as(w, dtype), _as(g, torch.float32),
                         _as(beta, torch.float32), cu, init)


@dataclasses.dataclass
class RecurrenceInputs:
    """Post-conv q, k, v fed straight to the chunked prefill (no conv)."""
    shape: LayerShape
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    g: torch.Tensor
    beta: torch.Tensor
    cu_seqlens: Optional[torch.Tensor]
    initial_state: Optional[torch.Tensor]


def make_recurrence(shape: LayerShape, T: int, seed: int, dtype=torch.float32,
                    g_low: float = -0.5, init_std: Optional[float] = None,
                    lengths: Optional[List[int]] = None) -> RecurrenceInputs:
    rng = _rng(seed)
    cu = None
    if lengths is not None:
        T = int(sum(lengths))
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32))
    q = _normal(rng, (T, shape.Hk, shape.dk))
    k = _normal(rng, (T, shape.Hk, shape.dk))
    v = _normal(rng, (T, shape.Hv, shape.dv))
    g = rng.uniform(g_low, 0.0, size=(T, shape.Hv)).astype(np.float32)
    beta = _sigmoid(rng.standard_normal((T, shape.Hv)))
    n_seq = 1 if lengths is None else len(lengths)
    init = None
    if init_std is not None:
        init = _as(_normal(rng, (n_seq, shape.Hv, shape.dv, shape.dk), std=init_std), torch.float32)
    return RecurrenceInputs(shape, _as(q, dtype), _as(k, dtype), _as(v, dtype),
                            _as(g, torch.float32), _as(beta, torch.float32), cu, init)


# The method's defining edge cases, as inputs (see make_edge_recurrence).
EDGE_CASES = ("beta0", "g0_beta1", "orthonormal", "repeated_key", "collinear", "strong_decay")


def make_edge_recurrence(kind: str, shape: LayerShape, T: int, seed: int, dtype=torch.bfloat16,
                         init_std: float = 0.02, lengths: Optional[List[int]] = None) -> RecurrenceInputs:
    """Inputs for the edge cases of the gated delta rule. q, k, v ~ N(0, 1) and
    S0 ~ N(0, init_std) are drawn first (in that order, then g and beta as below):

    beta0        beta = 0 (pure decay); g ~ U[-0.02, 0]
    g0_beta1     g = 0 (alpha = 1), beta = 1
    orthonormal  g = 0, beta = 1, S0 = 0; the key of token t is column (t mod dk) of a random
                 orthogonal matrix (QR of an N(0, 1) matrix, one per key head), so keys are
                 mutually orthogonal and each repeats every dk tokens
    repeated_key g ~ U[-0.3, 0], beta = sigmoid(N(0, 1)); tokens 64..127 share one key and
                 have beta = 1 (a whole chunk rewriting the same association)
    collinear    k_t = k0 + 0.05 n_t with n_t ~ N(0, 1) (one k0 per key head);
                 beta ~ U[0.9, 1], g ~ U[-0.1, 0]
    strong_decay g ~ U[-8, 0], beta = sigmoid(N(0, 1))
    """
    assert kind in EDGE_CASES, kind
    rng = _rng(seed)
    cu = None
    if lengths is not None:
        T = int(sum(lengths))
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32))
    Hk, Hv, dk, dv = shape.Hk, shape.Hv, shape.dk, shape.dv
    q = _normal(rng, (T, Hk, dk))
    k = _normal(rng, (T, Hk, dk))
    v = _normal(rng, (T, Hv, dv))
    n_seq = 1 if lengths is None else len(lengths)
    init = _normal(rng, (n_seq, Hv, dv, dk), std=init_std)
    if kind == "beta0":
        g = rng.uniform(-0.02, 0.0, size=(T, Hv)).astype(np.float32)
        beta = np.zeros((T, Hv), np.float32)
    elif kind == "g0_beta1":
        g = np.zeros((T, Hv), np.float32)
        beta = np.ones((T, Hv), np.float32)
    elif kind == "orthonormal":
        g = np.zeros((T, Hv), np.float32)
        beta = np.ones((T, Hv), np.float32)
        init[:] = 0.0
        for j in range(Hk):
            basis, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
            k[:, j] = basis[:, np.arange(T) % dk].T.astype(np.float32)
    elif kind == "repeated_key":
        g = rng.uniform(-0.3, 0.0, size=(T, Hv)).astype(np.float32)
        beta = _sigmoid(rng.standard_normal((T, Hv)))
        a, b = min(64, T), min(128, T)
        k[a:b] = k[a]
        beta[a:b] = 1.0
    elif kind == "collinear":
        k0 = rng.standard_normal((1, Hk, dk)).astype(np.float32)
        k = k0 + np.float32(0.05) * _normal(rng, (T, Hk, dk))
        beta = rng.uniform(0.9, 1.0, size=(T, Hv)).astype(np.float32)
        g = rng.uniform(-0.1, 0.0, size=(T, Hv)).astype(np.float32)
    else:   # strong_decay
        g = rng.uniform(-8.0, 0.0, size=(T, Hv)).astype(np.float32)
        beta = _sigmoid(rng.standard_normal((T, Hv)))
    return RecurrenceInputs(shape, _as(q, dtype), _as(k, dtype), _as(v, dtype),
                            _as(g, torch.float32), _as(beta, torch.float32), cu,
                            _as(init, torch.float32))


@dataclasses.dataclass
class DecodeInputs:
    shape: LayerShape
    conv_w: torch.Tensor         # [Cc, 4]
    conv_state: torch.Tensor     # [B, 3, Cc]
    state: torch.Tensor          # [B, Hv, dv, dk] fp32
    xs: List[torch.Tensor]       # per step [B, Cc]
    gs: List[torch.Tensor]       # per step [B, Hv]
    betas: List[torch.Tensor]    # per step [B, Hv]


def make_decode(shape: LayerShape, B: int, steps: int, seed: int, dtype=torch.bfloat16,
                g_low: float = -0.3, state_std: float = 0.02) -> DecodeInputs:
    rng = _rng(seed)
    Cc = shape.conv_channels
    state = _normal(rng, (B, shape.Hv, shape.dv, shape.dk), std=state_std)
    conv_state = _normal(rng, (B, 3, Cc))
    w = _normal(rng, (Cc, 4), std=0.5)
    xs, gs, bs = [], [], []
    for _ in range(steps):
        xs.append(_as(_normal(rng, (B, Cc)), dtype))
        gs.append(_as(rng.uniform(g_low, 0.0, size=(B, shape.Hv)).astype(np.float32), torch.float32))
        bs.append(_as(_sigmoid(rng.standard_normal((B, shape.Hv))), torch.float32))
    return DecodeInputs(shape, _as(w, dtype), _as(conv_state, dtype), _as(state, torch.float32),
                        xs, gs, bs)


def _loguniform_lengths(rng, n_seq: int, lo: int, hi: int) -> List[int]:
    """Log-uniform lengths: round(exp(U[ln lo, ln hi]))."""
    u = rng.uniform(math.log(lo), math.log(hi), size=n_seq)
    return [int(round(math.exp(a))) for a in u]


# The five workloads of the mixer, by name. Seeds: tiny 0, 9B 1, 27B 2, decode 3, varlen 4.
def tiny_recurrence() -> RecurrenceInputs:
    """T=64, 2 k-heads = 2 v-heads, d=16, fp32, g ~ U[-0.5, 0], zero initial state."""
    return make_recurrence(TINY, 64, seed=0, dtype=torch.float32, g_low=-0.5)


def tiny_layer() -> PrefillInputs:
    """The same tiny shape as a whole layer (conv w ~ N(0, 0.5)), fp32."""
    p = make_prefill(TINY, 64, seed=0, dtype=torch.float32, g_low=-0.5)
    p.chunk = 16
    return p


def qwen35_9b_prefill(T: int = 8192) -> PrefillInputs:
    return make_prefill(QWEN35_9B, T, seed=1, g_low=-0.5)


def qwen35_27b_prefill(T: int = 65536) -> PrefillInputs:
    return make_prefill(QWEN35_27B, T, seed=2, g_low=-0.3)


def qwen35_27b_decode(B: int = 256, steps: int = 100) -> DecodeInputs:
    return make_decode(QWEN35_27B, B, steps, seed=3, g_low=-0.3)


def qwen35_27b_varlen(n_seq: int = 32) -> PrefillInputs:
    """32 sequences, log-uniform lengths in [512, 32768], nonzero initial states."""
    return make_prefill(QWEN35_27B, 0, seed=4, g_low=-0.3, init_std=0.02, varlen_n=n_seq)
