"""Pins for the fp64 oracle: checks against facts that the pages and mathematics fix,
not against the oracle itself.

Each test names the mistake it is there to catch. Sources: "Inside Qwen3.5: a hybrid
linear + full attention LLM" (romaanj.github.io), sections 2, 5, 6; "Hybrid
Mamba-Transformer MoE" (sotaaz.com), section "Gated DeltaNet"; "Hybrid Mamba-Transformer
bench" (sotaaz.com), section 1.
"""
import json
import os

import numpy as np
import pytest
from scipy.special import expit

import oracle
from oracle.chunked import chunked_recurrence

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "cache_arithmetic.json")


def rng(seed):
    return np.random.default_rng(seed)


def unit_rows(a):
    return a / np.linalg.norm(a, axis=-1, keepdims=True)


# ----------------------------------------------------------------------------- conv

def test_conv_current_tap_only_is_silu(oracle_mod):
    """w = [0,0,0,1] leaves SiLU(x) (catches a reversed tap order or missing SiLU)."""
    r = rng(1)
    x = r.standard_normal((23, 7))
    w = np.tile([0.0, 0.0, 0.0, 1.0], (7, 1))
    y = oracle.conv1d_silu(x, w)
    np.testing.assert_allclose(y, x * expit(x), rtol=1e-15, atol=1e-15)


def test_conv_oldest_tap_shifts_by_three(oracle_mod):
    """w = [1,0,0,0] reads the token three back, zero before the start."""
    r = rng(2)
    x = r.standard_normal((10, 3))
    w = np.tile([1.0, 0.0, 0.0, 0.0], (3, 1))
    y = oracle.conv1d_silu(x, w)
    shifted = np.vstack([np.zeros((3, 3)), x[:-3]])
    np.testing.assert_allclose(y, shifted * expit(shifted), rtol=1e-15, atol=1e-15)


def test_conv_equals_numpy_convolve_varlen_with_state(oracle_mod):
    """Per channel, the causal conv is np.convolve with reversed taps; each packed
    sequence restarts from its own carried taps (catches a missing reset at cu_seqlens,
    a tap-order error, or a wrong state index)."""
    r = rng(3)
    Cc = 5
    lengths = [1, 2, 7, 4]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    T = int(cu[-1])
    x = r.standard_normal((T, Cc))
    w = r.standard_normal((Cc, 4))
    s_in = r.standard_normal((len(lengths), 3, Cc))
    y, s_out = oracle.conv1d_silu(x, w, cu, s_in, return_state=True)
    for n, L in enumerate(lengths):
        seg = x[cu[n]:cu[n + 1]]
        ext = np.vstack([s_in[n], seg])          # [3 + L, Cc], oldest first
        for c in range(Cc):
            z = np.convolve(ext[:, c], w[c][::-1])[3:3 + L]
            np.testing.assert_allclose(y[cu[n]:cu[n + 1], c], z * expit(z), rtol=1e-13, atol=1e-14)
        np.testing.assert_array_equal(s_out[n], ext[-3:])


def test_conv_state_absent_means_zero_padding(oracle_mod):
    r = rng(4)
    x = r.standard_normal((6, 4)); w = r.standard_normal((4, 4))
    cu = np.array([0, 6], np.int32)
    a = oracle.conv1d_silu(x, w, cu, np.zeros((1, 3, 4)))
    b = oracle.conv1d_silu(x, w, None, None)
    np.testing.assert_array_equal(a, b)


# ------------------------------------------------------------------- recurrence pins

def _random_case(r, T, Hk, Hv, d, init=True):
    q = r.standard_normal((T, Hk, d)); k = r.standard_normal((T, Hk, d))
    v = r.standard_normal((T, Hv, d))
    g = r.uniform(-0.5, 0.0, (T, Hv)); beta = expit(r.standard_normal((T, Hv)))
    S0 = r.standard_normal((1, Hv, d, d)) * 0.3 if init else None
    return q, k, v, g, beta, S0


def test_beta_zero_is_pure_decay(oracle_mod):
    """beta = 0: S_T = e^{sum g} S0 and o_t = e^{G_t} S0 q_t with a non-symmetric S0
    (catches S vs S^T, a decay applied to the wrong side, or a wrong cumulative index)."""
    r = rng(5)
    T, H, d = 9, 2, 4
    q, k, v, g, _, S0 = _random_case(r, T, H, H, d)
    beta = np.zeros((T, H))
    o, fin = oracle.recurrence(q, k, v, g, beta, initial_state=S0, l2norm=False)
    G = np.cumsum(g, axis=0)
    for h in range(H):
        for t in range(T):
            np.testing.assert_allclose(o[t, h], np.exp(G[t, h]) * S0[0, h] @ q[t, h], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(fin[0, h], np.exp(G[-1, h]) * S0[0, h], rtol=1e-13)


def test_orthonormal_keys_write_exactly_and_equal_linear_attention(oracle_mod):
    """alpha = 1, beta = 1, distinct orthonormal keys, zero init: every write stores v
    exactly (S k_i = v_i) and the output is causal linear attention
    o_t = sum_{i<=t} (k_i . q_t) v_i, the masked dense product (catches reading o before
    the write, a dropped beta, or a wrong sign in the error term)."""
    r = rng(6)
    d, T = 8, 6
    Qm, _ = np.linalg.qr(r.standard_normal((d, d)))
    keys = Qm[:T]                                   # orthonormal rows
    q = r.standard_normal((T, 1, d)); k = keys[:, None, :]
    v = r.standard_normal((T, 1, d))
    g = np.zeros((T, 1)); beta = np.ones((T, 1))
    o, fin = oracle.recurrence(q, k, v, g, beta, l2norm=False)
    lin = np.tril(q[:, 0] @ keys.T) @ v[:, 0]       # [T, d]
    np.testing.assert_allclose(o[:, 0], lin, rtol=1e-12, atol=1e-12)
    for i in range(T):
        np.testing.assert_allclose(fin[0, 0] @ keys[i], v[i, 0], rtol=1e-12, atol=1e-12)


def test_same_key_twice_replaces_the_value(oracle_mod):
    """A new value for an old key replaces the stale association (section 5 of the
    Qwen3.5 page): alpha = beta = 1, write (k, v1) then (k, v2), read S k = v2."""
    r = rng(7)
    d = 5
    kvec = unit_rows(r.standard_normal(d))
    k = np.stack([kvec, kvec])[:, None, :]
    v = r.standard_normal((2, 1, d))
    q = k.copy()
    o, fin = oracle.recurrence(q, k, v, np.zeros((2, 1)), np.ones((2, 1)), l2norm=False)
    np.testing.assert_allclose(fin[0, 0] @ kvec, v[1, 0], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(o[1, 0], v[1, 0], rtol=1e-13, atol=1e-13)


def _product_form(q, k, v, g, beta, S0):
    """S_t = S0 prod_{s<=t} A_s + sum_{i<=t} beta_i v_i k_i^T prod_{i<s<=t} A_s with
    A_s = alpha_s (I - beta_s k_s k_s^T), expanded by explicit products."""
    T, d = k.shape
    A = [np.exp(g[s]) * (np.eye(d) - beta[s] * np.outer(k[s], k[s])) for s in range(T)]
    outs, S_t = [], None
    for t in range(T):
        P = np.eye(d)
        for s in range(t + 1):
            P = P @ A[s]
        S_t = S0 @ P
        for i in range(t + 1):
            Pi = np.eye(d)
            for s in range(i + 1, t + 1):
                Pi = Pi @ A[s]
            S_t = S_t + beta[i] * np.outer(v[i], k[i]) @ Pi
        outs.append(S_t @ q[t])
    return np.array(outs), S_t


@pytest.mark.parametrize("d,T", [(2, 8), (3, 5), (2, 1)])
def test_brute_force_product_expansion(oracle_mod, d, T):
    """Tiny cases against the closed product form S_t = alpha_t S_{t-1}(I - beta_t k k^T)
    + beta_t v k^T (catches an undecayed state in the error term, a sign or an index
    slip), with grouped heads (Hv = 2 Hk) to pin the k-head map h // G."""
    r = rng(8 + d + T)
    q, k, v, g, beta, S0 = _random_case(r, T, 1, 2, d)
    o, fin = oracle.recurrence(q, k, v, g, beta, initial_state=S0, l2norm=True)
    qn = q[:, 0] / np.sqrt(np.sum(q[:, 0] ** 2, -1, keepdims=True) + 1e-6)
    kn = k[:, 0] / np.sqrt(np.sum(k[:, 0] ** 2, -1, keepdims=True) + 1e-6)
    for h in range(2):
        ob, Sb = _product_form(qn, kn, v[:, h], g[:, h], beta[:, h], S0[0, h])
        np.testing.assert_allclose(o[:, h], ob, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(fin[0, h], Sb, rtol=1e-11, atol=1e-12)


def test_alpha_one_is_the_deltanet_update(oracle_mod):
    """g = 0 reduces to S_t = S_{t-1} - beta (S_{t-1} k) k^T + beta v k^T (the ungated
    DeltaNet of the sotaaz page), checked through the product expansion with alpha=1."""
    r = rng(9)
    q, k, v, _, beta, S0 = _random_case(r, 6, 1, 1, 3)
    g = np.zeros((6, 1))
    o, fin = oracle.recurrence(q, k, v, g, beta, initial_state=S0, l2norm=False)
    ob, Sb = _product_form(q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0], S0[0, 0])
    np.testing.assert_allclose(o[:, 0], ob, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(fin[0, 0], Sb, rtol=1e-12, atol=1e-12)


def test_l2_norm_and_eps_placement(oracle_mod):
    """One token, alpha = beta = 1, q = k unnormalised: o = v |k|^2 / (|k|^2 + eps)
    (pins the L2 normalisation of both q and k and eps inside the square root)."""
    r = rng(10)
    d = 6
    kv = r.standard_normal(d) * 0.01           # small norm so eps shows
    k = kv[None, None, :]; q = k.copy()
    v = r.standard_normal((1, 1, d))
    o, _ = oracle.recurrence(q, k, v, np.zeros((1, 1)), np.ones((1, 1)), l2norm=True, eps=1e-6)
    n2 = np.sum(kv ** 2)
    np.testing.assert_allclose(o[0, 0], v[0, 0] * n2 / (n2 + 1e-6), rtol=1e-13)


def test_scale_multiplies_output_only(oracle_mod):
    r = rng(11)
    args = _random_case(r, 7, 1, 2, 4)
    o1, f1 = oracle.recurrence(*args[:5], initial_state=args[5])
    o2, f2 = oracle.recurrence(*args[:5], initial_state=args[5], scale=0.25)
    np.testing.assert_allclose(o2, 0.25 * o1, rtol=1e-15)
    np.testing.assert_array_equal(f1, f2)


@pytest.mark.parametrize("chunk", [1, 4, 16, 64])
def test_chunked_form_equals_sequential(oracle_mod, chunk):
    """The chunked WY/UT derivation equals the token-by-token recurrence in fp64, with
    grouped heads, initial states and ragged packed sequences (chunk 64 > every length
    covers C = T)."""
    r = rng(12)
    lengths = [5, 17, 1, 30]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    T = int(cu[-1])
    q = r.standard_normal((T, 2, 8)); k = r.standard_normal((T, 2, 8))
    v = r.standard_normal((T, 4, 8))
    g = r.uniform(-0.5, 0, (T, 4)); beta = expit(r.standard_normal((T, 4)))
    S0 = r.standard_normal((4, 4, 8, 8)) * 0.1
    o, fin = oracle.recurrence(q, k, v, g, beta, cu, S0)
    oc, fc = chunked_recurrence(q, k, v, g, beta, cu, S0, chunk=chunk)
    assert np.max(np.abs(oc - o)) <= 1e-12 * max(1.0, np.max(np.abs(o)))
    assert np.max(np.abs(fc - fin)) <= 1e-12 * max(1.0, np.max(np.abs(fin)))


def test_state_stays_bounded(oracle_mod):
    """|k| <= 1, beta in [0,1], alpha <= 1 give |S_t|_2 <= alpha_t |S_{t-1}|_2 + beta_t |v_t|
    (the bound the L2 norm buys, section 5); each token is run as its own call, which
    also exercises resuming from a carried state."""
    r = rng(13)
    T, d = 40, 6
    q, k, v, g, beta, S0 = _random_case(r, T, 1, 1, d)
    S = S0
    for t in range(T):
        _, S_new = oracle.recurrence(q[t:t + 1], k[t:t + 1], v[t:t + 1], g[t:t + 1],
                                     beta[t:t + 1], initial_state=S)
        lhs = np.linalg.norm(S_new[0, 0], 2)
        rhs = np.exp(g[t, 0]) * np.linalg.norm(S[0, 0], 2) + beta[t, 0] * np.linalg.norm(v[t, 0])
        assert lhs <= rhs * (1 + 1e-12)
        S = S_new


def test_packing_equals_separate_runs(oracle_mod):
    r = rng(14)
    lengths = [3, 9, 4]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    T = int(cu[-1]); Hk, Hv, d = 1, 3, 4
    x = r.standard_normal((T, 2 * Hk * d + Hv * d)); w = r.standard_normal((x.shape[1], 4))
    g = r.uniform(-0.5, 0, (T, Hv)); beta = expit(r.standard_normal((T, Hv)))
    S0 = r.standard_normal((3, Hv, d, d)) * 0.1
    cs0 = r.standard_normal((3, 3, x.shape[1]))
    o, fin, cs = oracle.layer_prefill(x, w, g, beta, Hk, Hv, d, d, cu, S0, cs0)
    for n in range(3):
        sl = slice(cu[n], cu[n + 1])
        on, fn, csn = oracle.layer_prefill(x[sl], w, g[sl], beta[sl], Hk, Hv, d, d,
                                           np.array([0, lengths[n]], np.int32), S0[n:n + 1], cs0[n:n + 1])
        np.testing.assert_array_equal(o[sl], on)
        np.testing.assert_array_equal(fin[n], fn[0])
        np.testing.assert_array_equal(cs[n], csn[0])


def test_split_and_resume_equals_one_run(oracle_mod):
    """prefill(x[0:T]) == prefill(x[T1:T]) started from prefill(x[0:T1])'s final state and
    conv taps (the state is the checkpoint)."""
    r = rng(15)
    T, T1, Hk, Hv, d = 13, 5, 2, 2, 4
    Cc = 2 * Hk * d + Hv * d
    x = r.standard_normal((T, Cc)); w = r.standard_normal((Cc, 4))
    g = r.uniform(-0.5, 0, (T, Hv)); beta = expit(r.standard_normal((T, Hv)))
    o, fin, cs = oracle.layer_prefill(x, w, g, beta, Hk, Hv, d, d)
    oa, fa, ca = oracle.layer_prefill(x[:T1], w, g[:T1], beta[:T1], Hk, Hv, d, d)
    ob, fb, cb = oracle.layer_prefill(x[T1:], w, g[T1:], beta[T1:], Hk, Hv, d, d,
                                      np.array([0, T - T1], np.int32), fa, ca)
    np.testing.assert_allclose(np.concatenate([oa, ob]), o, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(fb, fin, rtol=1e-13, atol=1e-14)
    np.testing.assert_array_equal(cb, cs)


def test_decode_steps_equal_prefill(oracle_mod):
    """Ten single-token decode steps over a batch equal one prefill of those ten tokens
    per sequence from the same states (the conv taps shift one place per step)."""
    r = rng(16)
    B, steps, Hk, Hv, d = 3, 10, 1, 2, 4
    Cc = 2 * Hk * d + Hv * d
    w = r.standard_normal((Cc, 4))
    S = r.standard_normal((B, Hv, d, d)) * 0.1
    cs = r.standard_normal((B, 3, Cc))
    xs = r.standard_normal((steps, B, Cc)); gs = r.uniform(-0.3, 0, (steps, B, Hv))
    bs = expit(r.standard_normal((steps, B, Hv)))
    S_d, cs_d, outs = S.copy(), cs.copy(), []
    for t in range(steps):
        o, S_d, cs_d = oracle.decode_step(xs[t], w, cs_d, gs[t], bs[t], S_d, Hk, Hv, d, d)
        outs.append(o)
    outs = np.stack(outs)                           # [steps, B, Hv, d]
    cu = np.arange(0, (B + 1) * steps, steps, dtype=np.int32)
    xp = xs.transpose(1, 0, 2).reshape(B * steps, Cc)
    o_p, S_p, cs_p = oracle.layer_prefill(xp, w, gs.transpose(1, 0, 2).reshape(-1, Hv),
                                          bs.transpose(1, 0, 2).reshape(-1, Hv), Hk, Hv, d, d,
                                          cu, S, cs)
    np.testing.assert_allclose(outs.transpose(1, 0, 2, 3).reshape(B * steps, Hv, d), o_p, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(S_d, S_p, rtol=1e-13, atol=1e-14)
    np.testing.assert_array_equal(cs_d, cs_p)
    np.testing.assert_array_equal(cs_d, xs[-3:].transpose(1, 0, 2))


def test_decode_tokens_equal_single_steps(oracle_mod):
    """A multi-token decode call equals its tokens taken one decode step at a time, with
    o[b, t] the output of sequence b's t-th token."""
    r = rng(18)
    B, n, Hk, Hv, d = 3, 5, 1, 2, 4
    Cc = 2 * Hk * d + Hv * d
    w = r.standard_normal((Cc, 4))
    S = r.standard_normal((B, Hv, d, d)) * 0.1
    cs = r.standard_normal((B, 3, Cc))
    xs = r.standard_normal((B, n, Cc)); gs = r.uniform(-0.3, 0, (B, n, Hv))
    bs = expit(r.standard_normal((B, n, Hv)))
    o_m, S_m, cs_m = oracle.decode_tokens(xs, w, cs, gs, bs, S, Hk, Hv, d, d)
    S_d, cs_d = S.copy(), cs.copy()
    for t in range(n):
        o, S_d, cs_d = oracle.decode_step(xs[:, t], w, cs_d, gs[:, t], bs[:, t], S_d, Hk, Hv, d, d)
        np.testing.assert_allclose(o_m[:, t], o, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(S_m, S_d, rtol=1e-13, atol=1e-14)
    np.testing.assert_array_equal(cs_m, cs_d)
    np.testing.assert_array_equal(cs_m, xs[:, -3:])


def test_bf16_state_rounding(oracle_mod):
    """bf16 keeps 8 significant bits: exact halfway cases go to the even neighbour, bf16
    values are fixed points, and every value moves by at most half a unit in the last place."""
    u = 2.0 ** -7                                      # ulp of bf16 in [1, 2)
    cases = {1.0 + u / 2: 1.0, 1.0 + 1.5 * u: 1.0 + 2 * u, 1.0 + 0.49 * u: 1.0,
             -(1.0 + 2.5 * u): -(1.0 + 2 * u),
             3.0 * 2.0 ** -133: 3.0 * 2.0 ** -133,     # subnormal: a multiple of 2^-133
             3.0 * 2.0 ** -140: 0.0}                   # below half the smallest subnormal
    for v, want in cases.items():
        assert oracle.round_bf16(np.array([v]))[0] == want, v
    r = rng(19).standard_normal(10000) * 10.0 ** rng(20).uniform(-6, 6, 10000)
    b = oracle.round_bf16(r)
    np.testing.assert_array_equal(oracle.round_bf16(b), b)
    ulp = 2.0 ** (np.floor(np.log2(np.abs(r))) - 7)
    assert np.all(np.abs(b - r) <= ulp / 2)


def test_empty_sequence_passes_state_through(oracle_mod):
    r = rng(17)
    q, k, v, g, beta, S0 = _random_case(r, 4, 1, 1, 3)
    cu = np.array([0, 0, 4], np.int32)
    S0 = np.concatenate([S0, S0 * 2])
    o, fin = oracle.recurrence(q, k, v, g, beta, cu, S0)
    np.testing.assert_array_equal(fin[0], S0[0])


# ----------------------------------------------------------------------- byte counts

def _golden():
    with open(GOLDEN) as f:
        return {e["name"]: e for e in json.load(f)["entries"]}


def test_page_cache_arithmetic(oracle_mod):
    E = _golden()
    e = E["qwen35_27b_layer_constant_state"]
    per_layer = oracle.layer_state_bytes(e["Hv"], e["dk"], e["dv"], e["state_bytes"],
                                         e["conv_channels"], e["conv_taps"], e["conv_bytes"])
    assert per_layer == e["expected_bytes"]

    b = E["qwen35_27b_break_even_tokens"]
    kv = b["kv_heads"] * b["kv_head_dim"] * 2 * b["kv_bytes"]
    assert kv == b["expected_kv_bytes_per_token"]
    assert round(per_layer / kv) == b["expected_tokens"]

    m = E["qwen35_27b_48_layers_state_MB"]
    assert round(m["layers"] * per_layer / 2 ** 20) == m["expected_MiB_rounded"]

    c = E["qwen35_27b_native_context_cache"]
    hybrid = c["full_layers"] * kv * c["context"] + c["linear_layers"] * per_layer
    assert round(hybrid / 2 ** 30, 1) == c["expected_hybrid_GiB_1dp"]
    assert c["all_full_layers"] * kv * c["context"] / 2 ** 30 == c["expected_all_full_GiB"]

    s = E["qwen35_9b_recurrent_state_bf16_reading"]
    mats = s["layers"] * oracle.layer_state_bytes(s["Hv"], s["dk"], s["dv"], s["state_bytes"], 0, 0, 0)
    assert mats == s["expected_bytes_matrices"]
    assert round(mats / 1e6) == s["expected_MB_rounded"]

    t = E["qwen3_8b_kv_cache"]
    per_tok = t["layers"] * t["kv_heads"] * t["head_dim"] * 2 * t["kv_bytes"]
    assert per_tok == t["expected_bytes_per_token"]
    assert round(per_tok * t["tokens"] / 2 ** 30, 2) == t["expected_GiB_2dp"]


def test_measured_hybrid_cache_fits_fp32_state_not_bf16(oracle_mod):
    """The 9B hybrid's measured 1.94 GB at 61,839 tokens is reproduced with fp32
    recurrent state and not with bf16 state: the reading that the state is fp32."""
    e = _golden()["qwen35_9b_measured_cache_implies_fp32_state"]
    kv = e["attn_layers"] * e["kv_heads"] * e["head_dim"] * 2 * e["kv_bytes"] * e["tokens"]

    def total(state_bytes):
        per = oracle.layer_state_bytes(e["Hv"], e["dk"], e["dv"], state_bytes,
                                       e["conv_channels"], e["conv_taps"], e["conv_bytes"])
        return (kv + e["gdn_layers"] * per) / 2 ** 30

    assert round(total(4), 2) == e["expected_GiB_2dp"]
    assert round(total(2), 2) != e["expected_GiB_2dp"]
