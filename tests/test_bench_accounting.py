"""The benchmark's algorithmic work counts, the denominators of every roofline fraction it
prints, rebuilt here from an explicit list of what the chunked form and the kernels move.

The FLOP count follows the chunked WY/UT form (one chunk of C tokens from state S0, per
value head; the key-head products are shared by the G value heads of a key head):
KK^T and QK^T per key head, the unit-lower-triangular inverse (I + A)^-1, W = Pk K and
U~ = P V, U = U~ - W S0^T, O = diag(e^G) Q S0^T + (M o QK^T) U, and the state update
S = e^{G_L} S0 + U^T diag(.) K. A GEMM of M x N x K counts 2MNK; the triangular inverse of
an n x n unit-lower matrix counts n^3 / 3 (textbook forward-substitution count, leading
term).
"""
import importlib.util
import os

import pytest
import torch

import gated_deltanet_mixer_causal_b200 as gdn
from gated_deltanet_mixer_causal_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def chunk_gemms(C, d, G):
    """(M, N, K, times) for one chunk and one value head; key-head products weigh 1/G."""
    return [
        (C, C, d, 1 / G),   # K K^T (per key head)
        (C, C, d, 1 / G),   # Q K^T (per key head)
        (C, d, C, 1),       # W  = Pk K
        (C, d, C, 1),       # U~ = P V
        (C, d, d, 1),       # W S0^T
        (C, d, d, 1),       # Q S0^T
        (C, d, C, 1),       # (M o QK^T) U
        (d, d, C, 1),       # U^T diag(.) K  (state update)
    ]


@pytest.mark.parametrize("shape,C", [(W.QWEN35_27B, 64), (W.QWEN35_9B, 64), (W.QWEN35_27B, 32),
                                     (W.TINY, 16)])
def test_prefill_flops_match_gemm_list(bench, shape, C):
    G = shape.Hv // shape.Hk
    per_chunk = sum(2 * m * n * k * w for m, n, k, w in chunk_gemms(C, shape.dk, G)) + C ** 3 / 3
    expect = shape.Hv * per_chunk / C
    assert bench.prefill_flops_per_token(shape, C) == pytest.approx(expect, rel=1e-12)


# which kernel applies each product of chunk_gemms (same order); the triangular inverse is
# the intra-chunk kernel's
KERNEL_OF = ["chunk_intra", "chunk_intra", "chunk_intra", "chunk_intra",
             "chunk_chain", "chunk_chain", "chunk_chain", "chunk_chain"]


@pytest.mark.parametrize("shape,C", [(W.QWEN35_27B, 64), (W.QWEN35_9B, 64), (W.TINY, 16)])
def test_prefill_kernel_split_matches_gemm_list(bench, shape, C):
    """The per-kernel FLOP attribution: each kernel's GEMMs from the list above, and the two
    kernels together account for the whole call."""
    G = shape.Hv // shape.Hk
    for kernel in ("chunk_intra", "chunk_chain"):
        per_chunk = sum(2 * m * n * k * w for (m, n, k, w), kk in zip(chunk_gemms(C, shape.dk, G), KERNEL_OF)
                        if kk == kernel)
        if kernel == "chunk_intra":
            per_chunk += C ** 3 / 3
        assert bench.prefill_kernel_flops_per_token(kernel, shape, C) == pytest.approx(
            shape.Hv * per_chunk / C, rel=1e-12)
    split = bench.prefill_kernel_split(65536, 3.1, 1590.0)
    kernels = [v for k, v in split.items() if k != "overlap"]
    assert sum(v["flops"] for v in kernels) == pytest.approx(
        bench.prefill_flops_per_token() * 65536, rel=1e-12)
    assert split["overlap"]["device_ms_sum"] == pytest.approx(sum(v["device_ms"] for v in kernels))


def test_prefill_roofline_time_27b_64k(bench):
    """7.67 MFLOP per token for the 27B layer; at 1,391.6 TFLOP/s (sustained bf16) the
    65,536-token prefill cannot take less than 0.361 ms."""
    f = bench.prefill_flops_per_token(W.QWEN35_27B)
    assert f == pytest.approx(7.67e6, rel=2e-3)
    assert f * 65536 / 1391.6e12 * 1e3 == pytest.approx(0.361, abs=1e-3)


def test_conv_bytes(bench):
    """x read and y written once, plus the weights (4 taps per channel) read once, all bf16."""
    sh = W.QWEN35_27B
    assert sh.conv_channels == 2 * 16 * 128 + 48 * 128
    T = 8192
    assert bench.conv_bytes(T, sh) == T * sh.conv_channels * 2 + T * sh.conv_channels * 2 \
        + 4 * sh.conv_channels * 2


@pytest.mark.parametrize("state_bytes", [4, 2])
def test_decode_bytes(bench, state_bytes):
    """One decode step over B sequences: every state read and written once, conv taps (3 per
    channel, bf16) read and written, one token of x in and o out, g and beta (fp32), the
    bf16 weights (4 taps per channel)."""
    sh, B = W.QWEN35_27B, 256
    Cc = sh.conv_channels
    states = B * sh.Hv * sh.dv * sh.dk * state_bytes
    taps = B * 3 * Cc * 2
    expect = 2 * states + 2 * taps + B * Cc * 2 + B * sh.Hv * sh.dv * 2 + B * sh.Hv * 4 * 2 + Cc * 4 * 2
    assert bench.decode_bytes(B, sh, state_bytes=state_bytes) == expect
    if state_bytes == 4:
        # 48 heads x 128 x 128 fp32 = 3 MiB of state per sequence; the 256 states read and
        # written are about 97.6 % of the step's bytes (the conv taps most of the rest)
        assert states == 256 * 3 * 2 ** 20
        assert 0.97 < 2 * states / expect < 0.98


def test_decode_tokens_bytes_reduce_to_one_step(bench):
    """A one-token multi-token call moves exactly what a decode step moves, and every further
    token adds only its x, o, g and beta."""
    sh, B = W.QWEN35_27B, 256
    one = bench.decode_tokens_bytes(B, 1, sh)
    assert one == bench.decode_bytes(B, sh)
    per_token = B * sh.conv_channels * 2 + B * sh.Hv * sh.dv * 2 + 2 * B * sh.Hv * 4
    for n in (2, 4, 8):
        assert bench.decode_tokens_bytes(B, n, sh) - one == (n - 1) * per_token


def test_prefill_launch_count(bench):
    """The plan kernel, then one intra-chunk and one chain launch; a single sequence of 512
    chunks or more runs in eight pieces: one chain launch per piece, one intra-chunk launch for
    the chunks done up front (544 of 1024 for the 27B layer at 65,536 tokens, 272 of 512 at
    32,768) and one for the rest of each later piece. One pass below 32,768 tokens, for several
    sequences, or when the chains would leave fewer than 16 SMs."""
    sh = W.QWEN35_27B
    assert bench.gdn_prefill_launches(65536, 1, sh) == 1 + 1 + 4 + 8
    assert bench.gdn_prefill_launches(32768, 1, sh) == 1 + 1 + 4 + 8
    assert bench.gdn_prefill_launches(33000, 1, sh) == 1 + 1 + 4 + 8   # 516 chunks, pieces of 65
    assert bench.gdn_prefill_launches(16384, 1, sh) == 3
    assert bench.gdn_prefill_launches(65536, 2, sh) == 3
    assert bench.gdn_prefill_launches(65536, 1, W.LayerShape(16, 80, 128, 128)) == 3
    # the 9B layer (Hv 32): its chains leave 84 SMs, enough for the intra-chunk work of every
    # piece after the first to keep up with them
    assert bench.gdn_prefill_launches(65536, 1, W.QWEN35_9B) == 1 + 1 + 7 + 8
    assert bench.gdn_prefill_launches(0, 1, sh) == 2
    assert gdn.gdn_chunk_prefill_launches(4096, 1, 2, 2, 16, 16, torch.float32, 148) == 1
    assert gdn.gdn_chunk_prefill_launches(65536, 1, 16, 48, 128, 128, torch.bfloat16, 148, qk_l2norm=False) == 1
