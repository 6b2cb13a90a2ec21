"""Context-parallel prefill of one sequence split across ranks: the exchange and the fold
run as gloo ranks on the CPU with the oracle as the per-segment prefill (exact in fp64); on
one GPU the same pieces run with the library's prefill, segment by segment, and are compared
with the oracle."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))

from gated_deltanet_mixer_causal_b200 import context_parallel as cp  # noqa: E402
from gated_deltanet_mixer_causal_b200 import workloads as W  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_prefill(q, k, v, g, beta, initial_state):
    import oracle
    o, fin = oracle.recurrence(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                               g.double().numpy(), beta.double().numpy(),
                               initial_state=initial_state.double().numpy(), l2norm=True)
    return torch.from_numpy(o), torch.from_numpy(fin)


def _sequence(T, seed):
    return W.make_recurrence(W.LayerShape(2, 4, 8, 8), T, seed=seed, dtype=torch.float32,
                             init_std=0.1)


def _worker(rank, world, port, lengths, seed, with_state, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r = _sequence(sum(lengths), seed)
        a = sum(lengths[:rank]); b = a + lengths[rank]
        o, fin = cp.cp_prefill(r.q[a:b], r.k[a:b], r.v[a:b], r.g[a:b], r.beta[a:b],
                               initial_state=r.initial_state if with_state else None,
                               prefill=_oracle_prefill)
        out[rank] = (o.numpy(), fin.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("lengths,with_state", [([40, 57], True), ([33, 1, 70], True),
                                               ([64, 20], False), ([20, 30, 10, 40], True)])
def test_cp_prefill_gloo_equals_one_run(oracle_mod, lengths, with_state):
    world, seed = len(lengths), 51 + len(lengths)
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), lengths, seed, with_state, out), nprocs=world,
             join=True)
    r = _sequence(sum(lengths), seed)
    s0 = r.initial_state if with_state else torch.zeros_like(r.initial_state)
    o_ref, fin_ref = _oracle_prefill(r.q, r.k, r.v, r.g, r.beta, s0)
    o = np.concatenate([out[i][0] for i in range(world)])
    np.testing.assert_allclose(o, o_ref.numpy(), rtol=1e-10, atol=1e-12)
    for i in range(world):
        np.testing.assert_allclose(out[i][1], fin_ref.numpy(), rtol=1e-10, atol=1e-12)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_cp_pieces_on_gpu_against_oracle(cuda_device, dtype):
    """Two segments on one GPU with the library's prefill: each segment's transition P (the
    v = 0 run from the identity) and zero-start state S_loc, the fold, and the second pass,
    against the fp64 oracle run over the whole sequence (and over each segment for P and
    S_loc). fp32 (token-recurrent path) at 1e-4; bf16 heads of 128 (tensor-core path) at the
    bf16 per-head gate."""
    import oracle
    from parity import BF16_TOL, FP32_TOL, check, frob_rel, max_rel, np64
    r = W.make_recurrence(W.LayerShape(2, 4, 128, 128), 700, seed=53, dtype=dtype, init_std=0.02)
    dev = cuda_device
    q, k, v, g, b = (t.to(dev) for t in (r.q, r.k, r.v, r.g, r.beta))
    s0 = r.initial_state.to(dev)
    prefill = cp._library_prefill(1.0, True)
    cuts = [(0, 300), (300, 700)]
    sums = [cp.segment_summary(q[a:e], k[a:e], v[a:e], g[a:e], b[a:e], prefill) for a, e in cuts]
    states = cp.fold(sums, s0)
    o_cp = torch.cat([prefill(q[a:e], k[a:e], v[a:e], g[a:e], b[a:e], states[i].contiguous())[0]
                      for i, (a, e) in enumerate(cuts)])
    torch.cuda.synchronize()
    qn, kn, vn = (t.double().numpy() for t in (r.q, r.k, r.v))
    gn, bn = r.g.double().numpy(), r.beta.double().numpy()
    o_ref, fin_ref = oracle.recurrence(qn, kn, vn, gn, bn, initial_state=r.initial_state.numpy())
    case = f"test_cp_pieces_on_gpu_against_oracle[{'f32' if dtype == torch.float32 else 'bf16'}]"
    eye = np.broadcast_to(np.eye(128), (1, 4, 128, 128))
    for i, (a, e) in enumerate(cuts):
        _, p_ref = oracle.recurrence(qn[a:e], kn[a:e], np.zeros_like(vn[a:e]), gn[a:e], bn[a:e],
                                     initial_state=eye)
        _, l_ref = oracle.recurrence(qn[a:e], kn[a:e], vn[a:e], gn[a:e], bn[a:e])
        s_loc, P = np64(sums[i][0]), np64(sums[i][1])
        if dtype == torch.float32:
            check(case, f"P seg {i}", max_rel(P, p_ref), FP32_TOL)
            check(case, f"S_loc seg {i}", max_rel(s_loc, l_ref), FP32_TOL)
        else:
            check(case, f"P seg {i}", max(frob_rel(P[0, h], p_ref[0, h]) for h in range(4)), BF16_TOL)
            check(case, f"S_loc seg {i}", max(frob_rel(s_loc[0, h], l_ref[0, h]) for h in range(4)),
                  BF16_TOL)
    o, fin = np64(o_cp), np64(states[-1])
    if dtype == torch.float32:
        check(case, "max rel o", max_rel(o, o_ref), FP32_TOL)
        check(case, "max rel state", max_rel(fin, fin_ref), FP32_TOL)
    else:
        check(case, "o per head", max(frob_rel(o[:, h], o_ref[:, h]) for h in range(4)), BF16_TOL)
        check(case, "state per head", max(frob_rel(fin[0, h], fin_ref[0, h]) for h in range(4)),
              BF16_TOL)
