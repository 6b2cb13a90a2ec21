"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
function include/gdn.h declares, and rejects invalid arguments before launching.

Invalid calls return before any CUDA call, so fake device addresses are safe here.
"""
import ctypes
import os
import re

import pytest

import gated_deltanet_mixer_causal_b200 as gdn
from gated_deltanet_mixer_causal_b200 import _lib
from gated_deltanet_mixer_causal_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")

FAKE = 0x7f0000000000        # 16-byte aligned, never dereferenced (validation fails first)


@pytest.fixture(scope="module")
def L():
    build()
    return _lib.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\*\s]+?\b(gdn_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["gdn_conv1d_silu", "gdn_chunk_prefill", "gdn_chunk_prefill_workspace_size",
              "gdn_decode_step", "gdn_status_string", "gdn_last_error", "gdn_version"]:
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), f"{name} declared in gdn.h but not exported"
        assert name in _lib.SIGNATURES, f"{name} has no Python binding"


def test_status_strings(L):
    for code, name in enumerate(["GDN_OK", "GDN_ERR_INVALID_ARG", "GDN_ERR_UNSUPPORTED",
                                 "GDN_ERR_WORKSPACE", "GDN_ERR_CUDA", "GDN_ERR_TIMEOUT"]):
        assert L.gdn_status_string(code).decode() == name
    assert L.gdn_version().decode().count(".") == 2


def _conv(L, **kw):
    a = dict(x=FAKE, y=FAKE + (1 << 30), dt=1, w=FAKE + (2 << 30), cu=None, n=1, T=64, Cc=64,
             sin=None, sout=None)
    a.update(kw)
    return L.gdn_conv1d_silu(a["x"], a["y"], a["dt"], a["w"], a["cu"], a["n"], a["T"], a["Cc"],
                             a["sin"], a["sout"], None)


def test_conv_validation(L):
    assert _conv(L, T=-1) == _lib.GDN_ERR_INVALID_ARG
    assert _conv(L, Cc=12) == _lib.GDN_ERR_INVALID_ARG
    assert _conv(L, dt=7) == _lib.GDN_ERR_UNSUPPORTED
    assert _conv(L, x=None) == _lib.GDN_ERR_INVALID_ARG
    assert _conv(L, y=FAKE + 8) == _lib.GDN_ERR_INVALID_ARG             # misaligned
    assert _conv(L, y=FAKE + 64) == _lib.GDN_ERR_INVALID_ARG            # overlaps x
    assert "overlaps" in L.gdn_last_error().decode()
    assert _conv(L, sin=FAKE + (3 << 30), sout=FAKE + (3 << 30) + 16) == _lib.GDN_ERR_INVALID_ARG
    assert _conv(L, cu=FAKE + (4 << 30), n=0) == _lib.GDN_ERR_INVALID_ARG


def _prefill(L, **kw):
    a = dict(q=FAKE, k=FAKE + (1 << 30), v=FAKE + (2 << 30), g=FAKE + (3 << 30),
             b=FAKE + (4 << 30), o=FAKE + (5 << 30), dt=1, T=100, Hk=2, Hv=4, dk=64, dv=64,
             qks=0, vs=0, cu=None, n=1, init=None, fin=None, ws=None, wsb=0)
    a.update(kw)
    return L.gdn_chunk_prefill(a["q"], a["k"], a["v"], a["g"], a["b"], a["o"], a["dt"], a["T"],
                               a["Hk"], a["Hv"], a["dk"], a["dv"], a["qks"], a["vs"], a["cu"],
                               a["n"], a["init"], a["fin"], 1.0, 1, a["ws"], a["wsb"], None)


def test_prefill_validation(L):
    assert _prefill(L, dk=48, dv=48) == _lib.GDN_ERR_UNSUPPORTED
    assert _prefill(L, dk=64, dv=128) == _lib.GDN_ERR_UNSUPPORTED
    assert _prefill(L, Hv=3) == _lib.GDN_ERR_UNSUPPORTED
    assert _prefill(L, Hk=0) == _lib.GDN_ERR_INVALID_ARG
    assert _prefill(L, T=-5) == _lib.GDN_ERR_INVALID_ARG
    assert _prefill(L, qks=100) == _lib.GDN_ERR_INVALID_ARG           # shorter than a row
    assert _prefill(L, qks=132) == _lib.GDN_ERR_INVALID_ARG           # not a multiple of 8
    assert _prefill(L, g=None) == _lib.GDN_ERR_INVALID_ARG
    assert _prefill(L, o=FAKE + 4) == _lib.GDN_ERR_INVALID_ARG        # misaligned
    assert _prefill(L, o=FAKE + (2 << 30) + 512) == _lib.GDN_ERR_INVALID_ARG   # o overlaps v
    st = FAKE + (6 << 30)
    assert _prefill(L, init=st, fin=st + 4096) == _lib.GDN_ERR_INVALID_ARG    # partial overlap
    need = L.gdn_chunk_prefill_workspace_size(100, 1, 2, 4, 64, 64, 1)
    if need > 0:
        assert _prefill(L, wsb=need - 1, ws=FAKE + (7 << 30)) == _lib.GDN_ERR_WORKSPACE
    assert L.gdn_chunk_prefill_workspace_size(100, 1, 2, 3, 64, 64, 1) == ctypes.c_size_t(-1).value
    # the bf16 tensor-core path (d = 128) needs workspace; short workspace is refused
    need = L.gdn_chunk_prefill_workspace_size(100, 1, 2, 4, 128, 128, 1)
    assert need > 0
    assert L.gdn_chunk_prefill_workspace_size(100, 1, 2, 4, 128, 128, 0) == 0   # fp32: none
    ws = FAKE + (7 << 30)
    assert _prefill(L, dk=128, dv=128, ws=ws, wsb=need - 1) == _lib.GDN_ERR_WORKSPACE
    assert _prefill(L, dk=128, dv=128, ws=None, wsb=need) == _lib.GDN_ERR_WORKSPACE
    assert _prefill(L, dk=128, dv=128, ws=ws + 16, wsb=need) == _lib.GDN_ERR_INVALID_ARG  # not 256-aligned


def _decode(L, **kw):
    a = dict(x=FAKE, w=FAKE + (1 << 30), cs=FAKE + (2 << 30), g=FAKE + (3 << 30),
             b=FAKE + (4 << 30), st=FAKE + (5 << 30), o=FAKE + (6 << 30), dt=1, B=8, Hk=2, Hv=4,
             dk=32, dv=32)
    a.update(kw)
    return L.gdn_decode_step(a["x"], a["w"], a["cs"], a["g"], a["b"], a["st"], a["o"], a["dt"],
                             a["B"], a["Hk"], a["Hv"], a["dk"], a["dv"], 1.0, None)


def test_decode_validation(L):
    assert _decode(L, B=-1) == _lib.GDN_ERR_INVALID_ARG
    assert _decode(L, B=0) == _lib.GDN_OK                       # no-op, nothing launched
    assert _decode(L, dk=24, dv=24) == _lib.GDN_ERR_UNSUPPORTED
    assert _decode(L, Hv=5) == _lib.GDN_ERR_UNSUPPORTED
    assert _decode(L, st=None) == _lib.GDN_ERR_INVALID_ARG
    assert _decode(L, o=FAKE + (5 << 30) + 128) == _lib.GDN_ERR_INVALID_ARG   # o inside state
    assert _decode(L, cs=FAKE + 16) == _lib.GDN_ERR_INVALID_ARG               # conv_state over x


def _decode_tokens(L, **kw):
    a = dict(x=FAKE, w=FAKE + (1 << 30), cs=FAKE + (2 << 30), g=FAKE + (3 << 30),
             b=FAKE + (4 << 30), st=FAKE + (5 << 30), o=FAKE + (6 << 30), dt=1, B=8, n=4, Hk=2,
             Hv=4, dk=32, dv=32)
    a.update(kw)
    return L.gdn_decode_tokens(a["x"], a["w"], a["cs"], a["g"], a["b"], a["st"], a["o"], a["dt"],
                               a["B"], a["n"], a["Hk"], a["Hv"], a["dk"], a["dv"], 1.0, None)


def test_decode_tokens_validation(L):
    assert _decode_tokens(L, n=0) == _lib.GDN_ERR_INVALID_ARG
    assert _decode_tokens(L, n=9) == _lib.GDN_ERR_INVALID_ARG
    assert _decode_tokens(L, B=-1) == _lib.GDN_ERR_INVALID_ARG
    assert _decode_tokens(L, B=0) == _lib.GDN_OK                       # no-op, nothing launched
    assert _decode_tokens(L, dk=24, dv=24) == _lib.GDN_ERR_UNSUPPORTED
    assert _decode_tokens(L, Hv=5) == _lib.GDN_ERR_UNSUPPORTED
    # 8 tokens of 32 value heads of 128 per key head need more than one CTA's shared memory
    assert _decode_tokens(L, n=8, Hk=1, Hv=32, dk=128, dv=128) == _lib.GDN_ERR_UNSUPPORTED
    assert _decode_tokens(L, st=None) == _lib.GDN_ERR_INVALID_ARG
    # x holds B * n tokens: a conv_state placed inside it overlaps
    assert _decode_tokens(L, cs=FAKE + 8 * 3 * 256 * 2) == _lib.GDN_ERR_INVALID_ARG
    assert _decode_tokens(L, o=FAKE + (5 << 30) + 128) == _lib.GDN_ERR_INVALID_ARG   # o inside state


def test_decode_state_dtype_validation(L):
    def step(state_dt, **kw):
        a = dict(x=FAKE, w=FAKE + (1 << 30), cs=FAKE + (2 << 30), g=FAKE + (3 << 30),
                 b=FAKE + (4 << 30), st=FAKE + (5 << 30), o=FAKE + (6 << 30), B=8)
        a.update(kw)
        return L.gdn_decode_step_ex(a["x"], a["w"], a["cs"], a["g"], a["b"], a["st"], state_dt,
                                    a["o"], 1, a["B"], 2, 4, 32, 32, 1.0, None)
    assert step(7) == _lib.GDN_ERR_UNSUPPORTED
    assert step(1, B=0) == _lib.GDN_OK
    # a bf16 state of 8 x 4 x 32 x 32 is 64 KB: o placed 40 KB in overlaps only as bf16 ... and
    # as fp32 (128 KB); 72 KB in overlaps the fp32 state but not the bf16 one
    assert step(1, o=FAKE + (5 << 30) + 40 * 1024) == _lib.GDN_ERR_INVALID_ARG
    assert step(0, o=FAKE + (5 << 30) + 72 * 1024) == _lib.GDN_ERR_INVALID_ARG
    assert L.gdn_decode_tokens_ex(FAKE, FAKE + (1 << 30), FAKE + (2 << 30), FAKE + (3 << 30),
                                  FAKE + (4 << 30), FAKE + (5 << 30), 9, FAKE + (6 << 30), 1, 8, 4,
                                  2, 4, 32, 32, 1.0, None) == _lib.GDN_ERR_UNSUPPORTED


def test_prefill_block_state_validation(L):
    def call(bt, bs, br, nr, **kw):
        a = dict(q=FAKE, k=FAKE + 256, v=FAKE + (1 << 30), g=FAKE + (2 << 30), b=FAKE + (3 << 30),
                 o=FAKE + (4 << 30), fin=FAKE + (5 << 30))
        a.update(kw)
        return L.gdn_chunk_prefill_ex(a["q"], a["k"], a["v"], a["g"], a["b"], a["o"], 0, 128, 2,
                                      4, 32, 32, 128, 128, None, 1, None, a["fin"],
                                      kw.get("state_dt", _lib.GDN_F32), 1.0, 1, bt, bs, br, nr,
                                      None, 0, None)
    rows = FAKE + (7 << 30)
    assert call(-64, FAKE + (6 << 30), rows, 4) == _lib.GDN_ERR_INVALID_ARG
    assert call(96, FAKE + (6 << 30), rows, 4) == _lib.GDN_ERR_INVALID_ARG      # not a multiple of 64
    assert call(64, None, rows, 4) == _lib.GDN_ERR_INVALID_ARG
    assert call(64, FAKE + (6 << 30), None, 4) == _lib.GDN_ERR_INVALID_ARG
    assert call(64, FAKE + (6 << 30), rows, 0) == _lib.GDN_ERR_INVALID_ARG
    assert call(64, FAKE + (6 << 30) + 8, rows, 4) == _lib.GDN_ERR_INVALID_ARG  # misaligned
    assert call(64, FAKE + (5 << 30) + 4096, rows, 4) == _lib.GDN_ERR_INVALID_ARG  # inside final_state
    # the state dtype: unknown codes are unsupported; with bf16 states the buffers are half
    # the size, so a block buffer starting 64 KB after a bf16 final state no longer overlaps it
    assert call(64, FAKE + (6 << 30), rows, 4, state_dt=7) == _lib.GDN_ERR_UNSUPPORTED
    fin_f32_bytes = 1 * 4 * 32 * 32 * 4
    assert call(64, FAKE + (5 << 30) + fin_f32_bytes // 2, rows, 4, state_dt=_lib.GDN_F32) == \
        _lib.GDN_ERR_INVALID_ARG


def test_workspace_holds_the_piece_state_for_long_single_sequences(L):
    """One sequence of 512 chunks or more (32,768 tokens) is prefilled in pieces, and the
    workspace then also holds the fp32 state passed between them (Hv x d x d x 4 bytes); a
    shorter sequence, or the same tokens as two sequences, has no such region."""
    Hk, Hv, d = 16, 48, 128
    size = lambda T, n: L.gdn_chunk_prefill_workspace_size(T, n, Hk, Hv, d, d, _lib.GDN_BF16)
    per_slot = size(32767 - 64, 1) - size(32767 - 128, 1)     # one more chunk slot, no state
    state = Hv * d * d * 4
    assert size(32768, 1) - size(32767, 1) >= state
    assert size(32768, 1) - size(32767, 1) < state + per_slot + 1024
    assert size(32768, 2) - size(32767, 2) < per_slot + 1024    # two sequences: no piece state


def test_prefill_beyond_32bit_coordinates_is_refused(L):
    """bf16 heads of 128: the tensor-core path's rows are int32 TMA coordinates, so a batch
    whose chunk rows pass 2^31 is unsupported (and says so before any launch); the same size
    with the norm off takes the token-recurrent path, which needs no workspace."""
    T, Hk, Hv, d = 30_000_000, 16, 48, 128
    assert L.gdn_chunk_prefill_workspace_size(T, 1, Hk, Hv, d, d, _lib.GDN_BF16) == 2 ** 64 - 1
    assert L.gdn_chunk_prefill_workspace_size(1_000_000, 1, Hk, Hv, d, d, _lib.GDN_BF16) < 2 ** 40
    # q, k, v as views of one conv output (hundreds of GB at this T); g, beta, o far apart
    st = L.gdn_chunk_prefill(FAKE, FAKE, FAKE, FAKE + (1 << 40), FAKE + (1 << 40) + (1 << 34),
                             FAKE + (1 << 41), _lib.GDN_BF16, T, Hk, Hv, d, d, 2 * Hk * d + Hv * d,
                             2 * Hk * d + Hv * d, None, 1, None, None, 1.0, 1, None, 0, None)
    assert st == _lib.GDN_ERR_UNSUPPORTED and "split the batch" in L.gdn_last_error().decode()


def test_prefill_status_needs_a_workspace(L):
    assert L.gdn_prefill_status(None, None) == _lib.GDN_ERR_INVALID_ARG


def test_python_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(8, 64, dtype=torch.bfloat16)
    w = torch.zeros(64, 4, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        gdn.gdn_conv1d_silu(x, w)


def test_prefill_path_query(L):
    """The path each shape takes is visible before the call: the tensor-core chunked form
    for bf16 heads of 128 with the L2 norm, the token-recurrent kernel otherwise."""
    B, F = _lib.GDN_BF16, _lib.GDN_F32
    assert L.gdn_chunk_prefill_path(B, 16, 48, 128, 128, 1) == 1
    assert L.gdn_chunk_prefill_path(B, 16, 48, 128, 128, 0) == 0
    assert L.gdn_chunk_prefill_path(F, 2, 2, 16, 16, 1) == 0
    assert L.gdn_chunk_prefill_path(B, 2, 4, 64, 64, 1) == 0
    assert L.gdn_chunk_prefill_path(B, 1, 16, 128, 128, 1) == 0      # 16 value heads per key head
    assert L.gdn_chunk_prefill_path(B, 3, 4, 128, 128, 1) == -1      # Hv % Hk != 0
    assert L.gdn_chunk_prefill_path(B, 2, 4, 96, 96, 1) == -1        # head size not built


def test_noalloc_refusal_follows_the_path(L):
    """The no-allocation prefill refuses a size only when the path it takes needs more
    scratch than its static array: with the L2 norm on (tensor-core path) the call returns
    GDN_ERR_WORKSPACE before any CUDA call; with it off (token-recurrent path, no scratch) it
    is not refused and goes on to the device (which a machine without a GPU reports as a
    CUDA error)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("passes fake device addresses; the second call would launch on a GPU")
    T, Hk, Hv, d = 3000, 16, 48, 128
    args = (FAKE, FAKE + (1 << 34), FAKE + (2 << 34), FAKE + (3 << 34), FAKE + (4 << 34),
            FAKE + (5 << 34), _lib.GDN_BF16, T, Hk, Hv, d, d, 0, 0, None, 1, None, None, 1.0)
    st = L.gdn_chunk_prefill_noalloc(*args, 1, None)
    assert st == _lib.GDN_ERR_WORKSPACE
    assert "nothing was launched" in L.gdn_last_error().decode()
    st = L.gdn_chunk_prefill_noalloc(*args, 0, None)
    assert st == _lib.GDN_ERR_CUDA
