"""fp64 CPU oracle for the Gated DeltaNet token mixer (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this package. It shares no code with the CUDA library: the arithmetic lives in
``gdn_oracle.c`` (plain C, fp64, sequential in token order) and this module only
marshals numpy arrays into it. ``chunked.py`` holds a second, independent fp64
derivation (the chunked WY/UT form) that the pins compare against the sequential one.

Sources for what is computed: "Inside Qwen3.5: a hybrid linear + full attention LLM"
(romaanj.github.io/study/models/hybrid-attention), section 2 (o = S q, S = sum v k^T),
section 4-5 (the gated delta rule, the width-4 causal conv and the q/k L2 norm as
stabilisers, alpha/beta per token and per head) and the config footnote (16 K / 48 V
heads x 128, conv kernel 4, fp32 state); "Hybrid Mamba-Transformer MoE"
(sotaaz.com), section "Gated DeltaNet" (the ungated DeltaNet update).

Decode entry points are prefills: ``decode_step`` of B sequences of one token,
``decode_tokens`` of B sequences of n tokens, from the carried conv taps and states. A state
stored in bf16 between calls (a serving option; the pages' model keeps fp32 states) is
modelled by rounding the fp64 result with ``round_bf16`` once per call.

Every function here is pinned by tests in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
# A test may point this at a deliberately broken build of the same source (mutation
# tests that check the pins catch planted mistakes).
_LIB_PATH = os.environ.get("GDN_ORACLE_LIB") or os.path.join(_HERE, "liboracle.so")
_lib = None

L2_EPS = 1e-6


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle.so`` (gcc, -O2, no fast-math)."""
    if os.environ.get("GDN_ORACLE_LIB"):
        return _LIB_PATH
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
             "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        lib.gdn_oracle_conv1d_silu.argtypes = [P, P, i64, i32, P, P, i32, P, P]
        lib.gdn_oracle_conv1d_silu.restype = ctypes.c_int
        lib.gdn_oracle_recurrence.argtypes = [P, P, P, P, P, P, i64, i32, i32, i32, i32,
                                              P, i32, P, P, f64, i32, f64, i32]
        lib.gdn_oracle_recurrence.restype = ctypes.c_int
        lib.gdn_oracle_layer_state_bytes.argtypes = [i32, i32, i32, i32, i32, i32, i32]
        lib.gdn_oracle_layer_state_bytes.restype = i64
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _cu(cu_seqlens, T):
    if cu_seqlens is None:
        return None, 1
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    assert cu.ndim == 1 and cu[0] == 0 and cu[-1] == T and np.all(np.diff(cu) >= 0)
    return cu, cu.shape[0] - 1


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def conv1d_silu(x, w, cu_seqlens=None, conv_state_in=None, return_state=False):
    """Width-4 depthwise causal conv + SiLU over ``x`` [T, Cc] with taps ``w`` [Cc, 4].

    ``w[c, 3]`` multiplies the current token, ``w[c, 0]`` the token three back. Each
    sequence (``cu_seqlens``) starts from ``conv_state_in[n]`` ([3, Cc], oldest first) or
    from zeros. Returns y (and the per-sequence last three inputs when asked).
    """
    x = _f64(x); w = _f64(w)
    T, Cc = x.shape
    assert w.shape == (Cc, 4)
    cu, n_seq = _cu(cu_seqlens, T)
    sin = None if conv_state_in is None else _f64(conv_state_in)
    if sin is not None:
        assert sin.shape == (n_seq, 3, Cc)
    y = np.empty((T, Cc), np.float64)
    sout = np.empty((n_seq, 3, Cc), np.float64) if return_state else None
    rc = _load().gdn_oracle_conv1d_silu(_ptr(x), _ptr(y), T, Cc, _ptr(w), _ptr(cu), n_seq,
                                        _ptr(sin), _ptr(sout))
    assert rc == 0
    return (y, sout) if return_state else y


def recurrence(q, k, v, g, beta, cu_seqlens=None, initial_state=None, scale=1.0,
               l2norm=True, eps=L2_EPS, n_threads=None):
    """Sequential gated delta rule, token by token, in fp64.

    q, k [T, Hk, dk]; v [T, Hv, dv]; g (log-decay), beta [T, Hv];
    initial_state [N, Hv, dv, dk] or None (zeros). Returns (o [T, Hv, dv], final_state).
    """
    q = _f64(q); k = _f64(k); v = _f64(v); g = _f64(g); beta = _f64(beta)
    T, Hk, dk = q.shape
    _, Hv, dv = v.shape
    assert k.shape == q.shape and v.shape[0] == T and g.shape == (T, Hv) and beta.shape == (T, Hv)
    cu, n_seq = _cu(cu_seqlens, T)
    init = None if initial_state is None else _f64(initial_state)
    if init is not None:
        assert init.shape == (n_seq, Hv, dv, dk)
    o = np.zeros((T, Hv, dv), np.float64)
    fin = np.zeros((n_seq, Hv, dv, dk), np.float64)
    rc = _load().gdn_oracle_recurrence(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(o), T, Hk, Hv, dk, dv,
        _ptr(cu), n_seq, _ptr(init), _ptr(fin), float(scale), int(bool(l2norm)), float(eps),
        int(n_threads or default_threads()))
    assert rc == 0
    return o, fin


def split_qkv(y, Hk, Hv, dk, dv):
    """Channel order of the conv output: [q: Hk*dk | k: Hk*dk | v: Hv*dv]."""
    T = y.shape[0]
    q = y[:, : Hk * dk].reshape(T, Hk, dk)
    k = y[:, Hk * dk: 2 * Hk * dk].reshape(T, Hk, dk)
    v = y[:, 2 * Hk * dk:].reshape(T, Hv, dv)
    return q, k, v


def layer_prefill(x, conv_w, g, beta, Hk, Hv, dk, dv, cu_seqlens=None, initial_state=None,
                  conv_state_in=None, scale=1.0, n_threads=None):
    """The whole mixer core over a packed batch: conv + SiLU, q/k L2, recurrence.

    Returns (o, final_state, conv_state_out).
    """
    y, conv_out = conv1d_silu(x, conv_w, cu_seqlens, conv_state_in, return_state=True)
    q, k, v = split_qkv(y, Hk, Hv, dk, dv)
    o, fin = recurrence(q, k, v, g, beta, cu_seqlens, initial_state, scale, True,
                        n_threads=n_threads)
    return o, fin, conv_out


def round_bf16(a):
    """Round to the nearest bfloat16 value (ties to even), returned as float64: the storage
    of a bf16 state between decode calls."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).to(torch.bfloat16).to(
        torch.float64).numpy()


def decode_step(x, conv_w, conv_state, g, beta, state, Hk, Hv, dk, dv, scale=1.0,
                n_threads=None, state_dtype="f32"):
    """One token for each of B sequences: a decode step is the prefill of B sequences
    of length one that start from the carried conv taps and recurrent states.

    x [B, Cc]; conv_state [B, 3, Cc]; g, beta [B, Hv]; state [B, Hv, dv, dk].
    state_dtype "bf16": the state is stored in bf16, so the new state is rounded to bf16.
    Returns (o [B, Hv, dv], new_state, new_conv_state); inputs are not modified.
    """
    B = np.asarray(x).shape[0]
    cu = np.arange(B + 1, dtype=np.int32)
    o, S, cs = layer_prefill(x, conv_w, g, beta, Hk, Hv, dk, dv, cu, state, conv_state, scale,
                             n_threads)
    return o, (round_bf16(S) if state_dtype == "bf16" else S), cs


def decode_tokens(x, conv_w, conv_state, g, beta, state, Hk, Hv, dk, dv, scale=1.0,
                  n_threads=None, state_dtype="f32"):
    """n consecutive tokens for each of B sequences: the prefill of B sequences of n tokens
    that start from the carried conv taps and recurrent states.

    x [B, n, Cc]; conv_state [B, 3, Cc]; g, beta [B, n, Hv]; state [B, Hv, dv, dk].
    state_dtype "bf16": the state is stored in bf16, rounded once after the n tokens.
    Returns (o [B, n, Hv, dv], new_state, new_conv_state); inputs are not modified.
    """
    x = np.asarray(x)
    B, n, Cc = x.shape
    cu = np.arange(0, (B + 1) * n, n, dtype=np.int32)
    o, S, cs = layer_prefill(x.reshape(B * n, Cc), conv_w, np.asarray(g).reshape(B * n, Hv),
                             np.asarray(beta).reshape(B * n, Hv), Hk, Hv, dk, dv, cu, state,
                             conv_state, scale, n_threads)
    return o.reshape(B, n, Hv, dv), (round_bf16(S) if state_dtype == "bf16" else S), cs


def layer_state_bytes(Hv, dk, dv, state_bytes, conv_channels, conv_taps, conv_bytes) -> int:
    """Per-layer constant footprint of one sequence: Hv dv x dk matrices plus the conv
    buffer (channels x taps elements)."""
    return int(_load().gdn_oracle_layer_state_bytes(Hv, dk, dv, state_bytes, conv_channels,
                                                    conv_taps, conv_bytes))
