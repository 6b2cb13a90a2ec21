"""ctypes binding of libgdn.so (declared in include/gdn.h): argument marshalling only.

Each function has the C entry point's name, takes torch tensors on a CUDA device,
checks shapes/dtypes/strides, passes raw pointers and the current torch stream, and
raises ``GDNError`` on a non-OK status. Every step of the computation runs in the CUDA
library; there is no CPU or PyTorch fallback. If the library is missing, the first call
raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn.so")

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_WORKSPACE, GDN_ERR_CUDA, GDN_ERR_TIMEOUT = range(6)
GDN_F32, GDN_BF16 = 0, 1

# name -> (restype, argtypes); mirrors include/gdn.h
_P, _I32, _I64, _F32, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "gdn_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "gdn_last_error": (ctypes.c_char_p, []),
    "gdn_version": (ctypes.c_char_p, []),
    "gdn_conv1d_silu": (ctypes.c_int, [_P, _P, ctypes.c_int, _P, _P, _I32, _I64, _I32, _P, _P, _P]),
    "gdn_chunk_prefill_workspace_size": (_SZ, [_I64, _I32, _I32, _I32, _I32, _I32, ctypes.c_int]),
    "gdn_chunk_prefill": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.c_int, _I64, _I32, _I32,
                                          _I32, _I32, _I64, _I64, _P, _I32, _P, _P, _F32, _I32,
                                          _P, _SZ, _P]),
    "gdn_chunk_prefill_ex": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.c_int, _I64, _I32, _I32,
                                             _I32, _I32, _I64, _I64, _P, _I32, _P, _P, ctypes.c_int,
                                             _F32, _I32, _I32, _P, _P, _I64, _P, _SZ, _P]),
    "gdn_prefill_status": (ctypes.c_int, [_P, _P]),
    "gdn_prefill_noalloc_status": (ctypes.c_int, [_P]),
    "gdn_decode_step": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, ctypes.c_int, _I32, _I32,
                                        _I32, _I32, _I32, _F32, _P]),
    "gdn_decode_tokens": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, ctypes.c_int, _I32, _I32, _I32,
                                         _I32, _I32, _I32, _F32, _P]),
    "gdn_decode_step_ex": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.c_int, _P, ctypes.c_int,
                                          _I32, _I32, _I32, _I32, _I32, _F32, _P]),
    "gdn_decode_tokens_ex": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.c_int, _P, ctypes.c_int,
                                            _I32, _I32, _I32, _I32, _I32, _I32, _F32, _P]),
    "gdn_chunk_prefill_path": (_I32, [ctypes.c_int, _I32, _I32, _I32, _I32, _I32]),
    "gdn_chunk_prefill_launches": (_I32, [_I64, _I32, _I32, _I32, _I32, _I32, ctypes.c_int, _I32, _I32]),
    "gdn_chunk_prefill_noalloc": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.c_int, _I64, _I32,
                                                  _I32, _I32, _I32, _I64, _I64, _P, _I32, _P, _P,
                                                  _F32, _I32, _P]),
}

_lib = None


class GDNError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}: {detail}")


def lib() -> ctypes.CDLL:
    """Load libgdn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libgdn.so is not built ({LIB_PATH}); run "
                               "`python -m gated_deltanet_mixer_causal_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().gdn_status_string(status).decode()


def _check(status: int, where: str):
    if status != GDN_OK:
        raise GDNError(status, where, lib().gdn_last_error().decode())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t: Optional[torch.Tensor], name: str, shape=None, dtype=None, device=None, dense=True):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if dense and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def gdn_conv1d_silu(x: torch.Tensor, w: torch.Tensor, cu_seqlens: Optional[torch.Tensor] = None,
                    conv_state_in: Optional[torch.Tensor] = None,
                    conv_state_out: Optional[torch.Tensor] = None,
                    y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Width-4 causal conv + SiLU: x [T, Cc] -> y [T, Cc] (see include/gdn.h)."""
    T, Cc = x.shape
    dev = x.device
    n_seq = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    _need(x, "x", device=dev)
    _need(w, "w", (Cc, 4), x.dtype, dev)
    _need(cu_seqlens, "cu_seqlens", dtype=torch.int32, device=dev)
    _need(conv_state_in, "conv_state_in", (n_seq, 3, Cc), x.dtype, dev)
    _need(conv_state_out, "conv_state_out", (n_seq, 3, Cc), x.dtype, dev)
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", (T, Cc), x.dtype, dev)
    _check(lib().gdn_conv1d_silu(_ptr(x), _ptr(y), _dtype_code(x), _ptr(w), _ptr(cu_seqlens),
                                 n_seq, T, Cc, _ptr(conv_state_in), _ptr(conv_state_out),
                                 _stream(dev)), "gdn_conv1d_silu")
    return y


def gdn_chunk_prefill_workspace_size(T: int, n_seq: int, Hk: int, Hv: int, dk: int, dv: int,
                                     dtype: torch.dtype) -> int:
    code = GDN_BF16 if dtype == torch.bfloat16 else GDN_F32
    n = lib().gdn_chunk_prefill_workspace_size(T, n_seq, Hk, Hv, dk, dv, code)
    if n == ctypes.c_size_t(-1).value:
        raise GDNError(GDN_ERR_UNSUPPORTED, "gdn_chunk_prefill_workspace_size", "unsupported shape")
    return int(n)


PATH_NAMES = {0: "recurrent", 1: "chunked_tc"}


def gdn_chunk_prefill_path(dtype: torch.dtype, Hk: int, Hv: int, dk: int, dv: int,
                           qk_l2norm: bool = True) -> str:
    """Which kernels gdn_chunk_prefill runs for these arguments: "chunked_tc" (the chunked
    form on tcgen05 tensor cores) or "recurrent" (the token-by-token fp32 kernel)."""
    code = GDN_BF16 if dtype == torch.bfloat16 else GDN_F32
    p = lib().gdn_chunk_prefill_path(code, Hk, Hv, dk, dv, int(bool(qk_l2norm)))
    if p < 0:
        raise GDNError(GDN_ERR_UNSUPPORTED, "gdn_chunk_prefill_path", "unsupported shape")
    return PATH_NAMES[p]


def gdn_chunk_prefill_launches(T: int, n_seq: int, Hk: int, Hv: int, dk: int, dv: int,
                               dtype: torch.dtype, num_sms: int, qk_l2norm: bool = True) -> int:
    """How many of this library's kernels one gdn_chunk_prefill call with these sizes enqueues
    on a GPU of num_sms SMs (host-only, no GPU needed)."""
    code = GDN_BF16 if dtype == torch.bfloat16 else GDN_F32
    n = lib().gdn_chunk_prefill_launches(T, n_seq, Hk, Hv, dk, dv, code, int(bool(qk_l2norm)), num_sms)
    if n < 0:
        raise GDNError(GDN_ERR_UNSUPPORTED, "gdn_chunk_prefill_launches", "unsupported arguments")
    return int(n)


def _row_view(t: torch.Tensor, name: str):
    """[T, H, d] with unit inner stride and dense heads; returns the token stride."""
    if t.dim() != 3 or t.stride(2) != 1 or t.stride(1) != t.shape[2]:
        raise ValueError(f"{name} must be [T, H, d] with dense heads (strides (*, d, 1)), "
                         f"got strides {t.stride()}")
    return t.stride(0)


def gdn_chunk_prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                      beta: torch.Tensor, cu_seqlens: Optional[torch.Tensor] = None,
                      initial_state: Optional[torch.Tensor] = None,
                      final_state: Optional[torch.Tensor] = None, scale: float = 1.0,
                      qk_l2norm: bool = True, o: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None, block_tokens: int = 0,
                      block_states: Optional[torch.Tensor] = None,
                      block_rows: Optional[torch.Tensor] = None, check: bool = False) -> torch.Tensor:
    """Gated delta rule over packed sequences (see include/gdn.h). Returns o [T, Hv, dv].

    q, k: [T, Hk, dk] and v: [T, Hv, dv] may be token-strided views (e.g. of the conv
    output). ``final_state`` ([N, Hv, dv, dk]) is written when given. States are fp32, or
    bf16 storage (fp32 math): the dtype of ``initial_state`` / ``final_state`` /
    ``block_states``, which must agree. With ``block_tokens`` > 0 (a multiple of 64) the
    state after every block_tokens tokens of sequence n goes to ``block_states``
    ([R, Hv, dv, dk]) rows block_rows[n], +1, ...
    ``check``: wait for the call and raise GDNError if a bounded device-side wait gave up.
    """
    T, Hk, dk = q.shape
    _, Hv, dv = v.shape
    dev = q.device
    n_seq = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    qs = _row_view(q, "q"); ks = _row_view(k, "k"); vs = _row_view(v, "v")
    if k.shape != q.shape or ks != qs:
        raise ValueError("k must match q in shape and token stride")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, dtype=q.dtype, device=dev, dense=False)
    _need(g, "g", (T, Hv), torch.float32, dev)
    _need(beta, "beta", (T, Hv), torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", dtype=torch.int32, device=dev)
    st_dtype = next((t.dtype for t in (initial_state, final_state, block_states if block_tokens else None)
                     if t is not None), torch.float32)
    if st_dtype not in (torch.float32, torch.bfloat16):
        raise ValueError(f"states must be fp32 or bf16, got {st_dtype}")
    _need(initial_state, "initial_state", (n_seq, Hv, dv, dk), st_dtype, dev)
    _need(final_state, "final_state", (n_seq, Hv, dv, dk), st_dtype, dev)
    if o is None:
        o = torch.empty((T, Hv, dv), dtype=q.dtype, device=dev)
    _need(o, "o", (T, Hv, dv), q.dtype, dev)
    need = gdn_chunk_prefill_workspace_size(T, n_seq, Hk, Hv, dk, dv, q.dtype)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    n_rows = 0
    if block_tokens:
        if block_states is None or block_rows is None:
            raise ValueError("block_tokens needs block_states and block_rows")
        _need(block_states, "block_states", dtype=st_dtype, device=dev)
        if tuple(block_states.shape[1:]) != (Hv, dv, dk):
            raise ValueError(f"block_states has shape {tuple(block_states.shape)}, expected [R, {Hv}, {dv}, {dk}]")
        _need(block_rows, "block_rows", (n_seq,), torch.int32, dev)
        n_rows = block_states.shape[0]
    _check(lib().gdn_chunk_prefill_ex(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(o), _dtype_code(q), T, Hk, Hv, dk, dv,
        qs, vs, _ptr(cu_seqlens), n_seq, _ptr(initial_state), _ptr(final_state),
        GDN_BF16 if st_dtype == torch.bfloat16 else GDN_F32, float(scale),
        int(bool(qk_l2norm)), int(block_tokens), _ptr(block_states if block_tokens else None),
        _ptr(block_rows if block_tokens else None), n_rows, _ptr(workspace), ws_bytes,
        _stream(dev)), "gdn_chunk_prefill")
    if check and workspace is not None:
        gdn_prefill_status(workspace)
    return o


def gdn_prefill_status(workspace: torch.Tensor) -> None:
    """Wait for the last prefill that used ``workspace`` and raise GDNError(GDN_ERR_TIMEOUT)
    if one of its bounded device-side waits gave up (its outputs are then invalid)."""
    _check(lib().gdn_prefill_status(_ptr(workspace), _stream(workspace.device)), "gdn_prefill_status")


def gdn_prefill_noalloc_status(device: Optional[torch.device] = None) -> None:
    """gdn_prefill_status for gdn_chunk_prefill_noalloc's static scratch on ``device``."""
    dev = device or torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        _check(lib().gdn_prefill_noalloc_status(_stream(dev)), "gdn_prefill_noalloc_status")


def gdn_chunk_prefill_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                              g: torch.Tensor, beta: torch.Tensor,
                              cu_seqlens: Optional[torch.Tensor] = None,
                              initial_state: Optional[torch.Tensor] = None,
                              final_state: Optional[torch.Tensor] = None, scale: float = 1.0,
                              qk_l2norm: bool = True, o: Optional[torch.Tensor] = None) -> torch.Tensor:
    """gdn_chunk_prefill with the library's static scratch instead of a workspace, for
    callers that cannot allocate device memory (see include/gdn.h for the size limit and
    the rule that overlapping calls race). Pass ``o`` to keep this call allocation-free
    on the Python side as well."""
    T, Hk, dk = q.shape
    _, Hv, dv = v.shape
    dev = q.device
    n_seq = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    qs = _row_view(q, "q"); ks = _row_view(k, "k"); vs = _row_view(v, "v")
    if k.shape != q.shape or ks != qs:
        raise ValueError("k must match q in shape and token stride")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, dtype=q.dtype, device=dev, dense=False)
    _need(g, "g", (T, Hv), torch.float32, dev)
    _need(beta, "beta", (T, Hv), torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", dtype=torch.int32, device=dev)
    _need(initial_state, "initial_state", (n_seq, Hv, dv, dk), torch.float32, dev)
    _need(final_state, "final_state", (n_seq, Hv, dv, dk), torch.float32, dev)
    if o is None:
        o = torch.empty((T, Hv, dv), dtype=q.dtype, device=dev)
    _need(o, "o", (T, Hv, dv), q.dtype, dev)
    # the scratch array is per device: make the tensors' device current for the call
    with torch.cuda.device(dev):
        _check(lib().gdn_chunk_prefill_noalloc(
            _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(o), _dtype_code(q), T, Hk, Hv,
            dk, dv, qs, vs, _ptr(cu_seqlens), n_seq, _ptr(initial_state), _ptr(final_state),
            float(scale), int(bool(qk_l2norm)), _stream(dev)), "gdn_chunk_prefill_noalloc")
    return o


def gdn_decode_step(x: torch.Tensor, conv_w: torch.Tensor, conv_state: torch.Tensor,
                    g: torch.Tensor, beta: torch.Tensor, state: torch.Tensor, Hk: int,
                    o: Optional[torch.Tensor] = None, scale: float = 1.0) -> torch.Tensor:
    """One decode token per sequence; conv_state and state are updated in place. The state
    is fp32, or bf16 (stored in bf16, updated in fp32)."""
    B, Cc = x.shape
    _, Hv, dv, dk = state.shape
    dev = x.device
    if Cc != 2 * Hk * dk + Hv * dv:
        raise ValueError(f"x has {Cc} channels, expected 2*Hk*dk + Hv*dv = {2 * Hk * dk + Hv * dv}")
    _need(x, "x", device=dev)
    _need(conv_w, "conv_w", (Cc, 4), x.dtype, dev)
    _need(conv_state, "conv_state", (B, 3, Cc), x.dtype, dev)
    _need(g, "g", (B, Hv), torch.float32, dev)
    _need(beta, "beta", (B, Hv), torch.float32, dev)
    _need(state, "state", (B, Hv, dv, dk), None, dev)
    if o is None:
        o = torch.empty((B, Hv, dv), dtype=x.dtype, device=dev)
    _need(o, "o", (B, Hv, dv), x.dtype, dev)
    _check(lib().gdn_decode_step_ex(_ptr(x), _ptr(conv_w), _ptr(conv_state), _ptr(g), _ptr(beta),
                                    _ptr(state), _dtype_code(state), _ptr(o), _dtype_code(x), B,
                                    Hk, Hv, dk, dv, float(scale), _stream(dev)), "gdn_decode_step")
    return o


def gdn_decode_tokens(x: torch.Tensor, conv_w: torch.Tensor, conv_state: torch.Tensor,
                      g: torch.Tensor, beta: torch.Tensor, state: torch.Tensor, Hk: int,
                      o: Optional[torch.Tensor] = None, scale: float = 1.0) -> torch.Tensor:
    """n_tok (1..8) consecutive tokens per sequence, x [B, n_tok, Cc]; conv_state and state
    (fp32, or bf16 storage) are updated in place. Returns o [B, n_tok, Hv, dv]."""
    B, n_tok, Cc = x.shape
    _, Hv, dv, dk = state.shape
    dev = x.device
    if Cc != 2 * Hk * dk + Hv * dv:
        raise ValueError(f"x has {Cc} channels, expected 2*Hk*dk + Hv*dv = {2 * Hk * dk + Hv * dv}")
    _need(x, "x", device=dev)
    _need(conv_w, "conv_w", (Cc, 4), x.dtype, dev)
    _need(conv_state, "conv_state", (B, 3, Cc), x.dtype, dev)
    _need(g, "g", (B, n_tok, Hv), torch.float32, dev)
    _need(beta, "beta", (B, n_tok, Hv), torch.float32, dev)
    _need(state, "state", (B, Hv, dv, dk), None, dev)
    if o is None:
        o = torch.empty((B, n_tok, Hv, dv), dtype=x.dtype, device=dev)
    _need(o, "o", (B, n_tok, Hv, dv), x.dtype, dev)
    _check(lib().gdn_decode_tokens_ex(_ptr(x), _ptr(conv_w), _ptr(conv_state), _ptr(g), _ptr(beta),
                                      _ptr(state), _dtype_code(state), _ptr(o), _dtype_code(x), B,
                                      n_tok, Hk, Hv, dk, dv, float(scale), _stream(dev)),
           "gdn_decode_tokens")
    return o
