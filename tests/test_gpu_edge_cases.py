"""GPU parity on the gated delta rule's defining edge cases, through the tensor-core path.

Each case drives gdn_chunk_prefill (bf16, heads of 128, three value heads per key head,
several chunks and a ragged tail) against the fp64 oracle element by element at the bf16
per-head gate, and where the case has a closed form, checks that too:

  beta = 0        pure decay: S_T = e^{sum g} S_0 ("Inside Qwen3.5", section 5: alpha forgets)
  g = 0, beta = 1 no forgetting, full-strength writes over 1,100 tokens (the state at its
                  largest)
  orthonormal     alpha = beta = 1 with mutually orthogonal keys: after its last write each key
                  reads back exactly the value last written with it (S k = v)
  repeated key    one key rewritten through a whole chunk at beta = 1: the new value replaces
                  the stale association (section 5), and the chunk's (I + A) is the all-ones
                  lower triangle
  collinear       near-collinear keys at beta in [0.9, 1]: the worst conditioning of the
                  triangular solve
  strong decay    g ~ U[-8, 0]: the in-chunk cumulative decay leaves the fp32 range of e^{G}
"""
import numpy as np
import pytest
import torch

import gated_deltanet_mixer_causal_b200 as gdn
from gated_deltanet_mixer_causal_b200 import workloads as W
import oracle
from parity import BF16_TOL, check, frob_rel, np64, worst_head_o, worst_head_state

pytestmark = pytest.mark.gpu

SHAPE = W.LayerShape(2, 6, 128, 128)
CASES = {   # kind: (lengths, seed)
    "beta0": ([300], 71),
    "g0_beta1": ([1100], 72),
    "orthonormal": ([300], 73),
    "repeated_key": ([300], 74),
    "collinear": ([700, 333], 75),
    "strong_decay": ([500, 129], 76),
}


def _run(r, dev):
    sh = r.shape
    n = 1 if r.cu_seqlens is None else r.cu_seqlens.numel() - 1
    fin = torch.empty((n, sh.Hv, sh.dv, sh.dk), dtype=torch.float32, device=dev)
    cu = None if r.cu_seqlens is None else r.cu_seqlens.to(dev)
    o = gdn.gdn_chunk_prefill(r.q.to(dev), r.k.to(dev), r.v.to(dev), r.g.to(dev),
                              r.beta.to(dev), cu, r.initial_state.to(dev), fin, check=True)
    torch.cuda.synchronize()
    return np64(o), np64(fin)


@pytest.mark.parametrize("kind", W.EDGE_CASES)
def test_prefill_edge_case_against_oracle(cuda_device, kind):
    lengths, seed = CASES[kind]
    r = W.make_edge_recurrence(kind, SHAPE, 0, seed=seed, lengths=lengths)
    sh = r.shape
    assert gdn.gdn_chunk_prefill_path(torch.bfloat16, sh.Hk, sh.Hv, sh.dk, sh.dv) == "chunked_tc"
    o, fin = _run(r, cuda_device)
    cu = r.cu_seqlens.numpy()
    o_r, f_r = oracle.recurrence(r.q.float().numpy(), r.k.float().numpy(), r.v.float().numpy(),
                                 r.g.numpy(), r.beta.numpy(), cu, r.initial_state.numpy())
    check(f"edge {kind}", "o per head", worst_head_o(o, o_r, cu), BF16_TOL)
    check(f"edge {kind}", "state per head", worst_head_state(fin, f_r), BF16_TOL)
    assert np.isfinite(o).all() and np.isfinite(fin).all()


def test_beta0_is_pure_decay(cuda_device):
    """beta = 0: the final state is the initial state decayed by e^{sum g} (closed form)."""
    r = W.make_edge_recurrence("beta0", SHAPE, 0, seed=77, lengths=[300])
    _, fin = _run(r, cuda_device)
    decay = np.exp(r.g.double().numpy().sum(0))                      # [Hv]
    ref = r.initial_state.double().numpy()[0] * decay[:, None, None]
    check("edge beta0 closed form", "state per head", worst_head_state(fin, ref[None]), BF16_TOL)


def test_orthonormal_keys_read_back_their_last_value(cuda_device):
    """alpha = beta = 1, orthonormal keys from a zero state: S k_j equals the value last
    written with key j (the keys are the bf16-rounded orthonormal columns, normalised)."""
    r = W.make_edge_recurrence("orthonormal", SHAPE, 0, seed=78, lengths=[300])
    sh = r.shape
    _, fin = _run(r, cuda_device)
    G = sh.Hv // sh.Hk
    k = r.k.double().numpy()
    k = k / np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.v.double().numpy()
    T = k.shape[0]
    worst = 0.0
    for h in range(sh.Hv):
        last = {t % sh.dk: t for t in range(T)}      # token of each key's last write
        ts = np.array(sorted(last.values()))
        got = fin[0, h] @ k[ts, h // G].T            # [dv, n]
        worst = max(worst, np.linalg.norm(got - v[ts, h].T) / np.linalg.norm(fin[0, h]))
    # the bf16-rounded keys are orthogonal only to ~1e-3, so S k_j carries that much of the
    # other keys' values; the residual is measured against |S|_F as the state gate is
    check("edge orthonormal S k = v", "per head / |S|", worst, BF16_TOL)


def test_repeated_key_replaces_the_association(cuda_device):
    """A key written again and again at beta = 1 with alpha = 1 for the chunk: the state
    after the chunk maps that key to the chunk's last value, up to the decay of the tokens
    after it (here checked on a sequence that ends with that chunk, with g = 0 in it)."""
    r = W.make_edge_recurrence("repeated_key", SHAPE, 0, seed=79, lengths=[128])
    r.g[64:128] = 0.0
    sh = r.shape
    _, fin = _run(r, cuda_device)
    G = sh.Hv // sh.Hk
    k = r.k.double().numpy()[127]
    k = k / np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.v.double().numpy()[127]
    # |(S - S_exact) k| <= |S - S_exact|_F, so the per-head state gate bounds this residual
    # by BF16_TOL |S|_F (the state norm, not |v|, is the scale the gate is stated in)
    worst = max(np.linalg.norm(fin[0, h] @ k[h // G] - v[h]) / np.linalg.norm(fin[0, h])
                for h in range(sh.Hv))
    check("edge repeated key S k = v_last", "per head / |S|", worst, BF16_TOL)
