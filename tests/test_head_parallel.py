"""Head-group split of the mixer (key heads with their value heads and the matching conv
channels per rank): gloo ranks on the CPU with the oracle as each rank's layer prefill and
decode step, reassembled and compared with one whole-layer oracle run; on one GPU the
library runs each rank's slice in turn and is compared with the oracle."""
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

from gated_deltanet_mixer_causal_b200 import head_parallel as hp  # noqa: E402
from gated_deltanet_mixer_causal_b200 import workloads as W  # noqa: E402

SHAPE = W.LayerShape(4, 12, 8, 8)        # 4 key heads, 3 value heads each, heads of 8


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_layer(x, w, g, b, hk, hv, d, cu, init):
    import oracle
    o, fin, _ = oracle.layer_prefill(x.double().numpy(), w.double().numpy(), g.double().numpy(),
                                     b.double().numpy(), hk, hv, d, d,
                                     None if cu is None else cu.numpy(),
                                     None if init is None else init.double().numpy())
    return torch.from_numpy(o), torch.from_numpy(fin)


def _batch():
    return W.make_prefill(SHAPE, 0, seed=81, dtype=torch.float32, init_std=0.1,
                          lengths=[37, 64, 5])


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        p = _batch()
        sh = p.shape
        o, fin = hp.head_parallel_prefill(p.x, p.conv_w, p.g, p.beta, sh.Hk, sh.Hv, sh.dk, rank,
                                          world, p.cu_seqlens, p.initial_state,
                                          prefill=_oracle_layer)
        o_all = hp.gather_heads(o, 1)
        fin_all = hp.gather_heads(fin, 1)
        # one decode step on the same split: the rank's conv taps and states, its slice of x
        import oracle
        d = W.make_decode(sh, B=3, steps=1, seed=82, dtype=torch.float32)
        xs, ws, cs, gs, bs, st = hp.shard_decode_inputs(d.xs[0], d.conv_w, d.conv_state, d.gs[0],
                                                        d.betas[0], d.state, sh.Hk, sh.Hv, sh.dk,
                                                        rank, world)
        hk0, hk1, hv0, hv1 = hp.head_range(sh.Hk, sh.Hv, rank, world)
        od, sd, _ = oracle.decode_step(xs.numpy(), ws.numpy(), cs.numpy(), gs.numpy(), bs.numpy(),
                                       st.numpy(), hk1 - hk0, hv1 - hv0, sh.dk, sh.dv)
        od_all = hp.gather_heads(torch.from_numpy(od), 1)
        sd_all = hp.gather_heads(torch.from_numpy(sd), 1)
        out[rank] = (o_all.numpy(), fin_all.numpy(), od_all.numpy(), sd_all.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_head_split_gloo_equals_whole_layer(oracle_mod, world):
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    p = _batch()
    sh = p.shape
    o_ref, fin_ref = _oracle_layer(p.x, p.conv_w, p.g, p.beta, sh.Hk, sh.Hv, sh.dk, p.cu_seqlens,
                                   p.initial_state)
    import oracle
    d = W.make_decode(sh, B=3, steps=1, seed=82, dtype=torch.float32)
    od_ref, sd_ref, _ = oracle.decode_step(d.xs[0].numpy(), d.conv_w.numpy(), d.conv_state.numpy(),
                                           d.gs[0].numpy(), d.betas[0].numpy(), d.state.numpy(),
                                           sh.Hk, sh.Hv, sh.dk, sh.dv)
    for r in range(world):
        o, fin, od, sd = out[r]
        np.testing.assert_allclose(o, o_ref.numpy(), rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(fin, fin_ref.numpy(), rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(od, od_ref, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(sd, sd_ref, rtol=1e-12, atol=1e-14)


def test_head_range_and_channels():
    assert hp.head_range(16, 48, 1, 4) == (4, 8, 12, 24)
    ch = hp.channel_index(16, 48, 128, 1, 4)
    assert ch.numel() == (2 * 4 + 12) * 128
    assert ch[0] == 4 * 128 and ch[4 * 128] == 16 * 128 + 4 * 128
    assert ch[8 * 128] == 2 * 16 * 128 + 12 * 128
    # the ranks' channels partition the layer's channels
    allc = torch.cat([hp.channel_index(16, 48, 128, r, 4) for r in range(4)])
    assert torch.equal(allc.sort().values, torch.arange(2 * 16 * 128 + 48 * 128))
    with pytest.raises(ValueError):
        hp.head_range(16, 48, 0, 3)


@pytest.mark.gpu
def test_head_split_on_gpu_against_oracle(cuda_device):
    """27B-shaped layer (16 key / 48 value heads of 128) split over 4 head groups: each group
    runs the library's conv + chunked prefill on its slice (one after another on one GPU) and
    its value heads are compared with the whole-layer oracle."""
    from parity import BF16_TOL, check, frob_rel, np64
    import oracle
    p = W.make_prefill(W.QWEN35_27B, 0, seed=83, g_low=-0.3, init_std=0.02, lengths=[200, 77])
    sh = p.shape
    dev = cuda_device
    x, w, g, b = (t.to(dev) for t in (p.x, p.conv_w, p.g, p.beta))
    cu, s0 = p.cu_seqlens.to(dev), p.initial_state.to(dev)
    o_ref, f_ref, _ = oracle.layer_prefill(p.x.float().numpy(), p.conv_w.float().numpy(),
                                           p.g.numpy(), p.beta.numpy(), sh.Hk, sh.Hv, sh.dk, sh.dv,
                                           p.cu_seqlens.numpy(), p.initial_state.numpy())
    world, eo, es = 4, 0.0, 0.0
    cun = p.cu_seqlens.numpy()
    for r in range(world):
        o, fin = hp.head_parallel_prefill(x, w, g, b, sh.Hk, sh.Hv, sh.dk, r, world, cu, s0)
        torch.cuda.synchronize()
        _, _, hv0, hv1 = hp.head_range(sh.Hk, sh.Hv, r, world)
        o, fin = np64(o), np64(fin)
        for j, h in enumerate(range(hv0, hv1)):
            for n in range(2):
                a, e = cun[n], cun[n + 1]
                eo = max(eo, frob_rel(o[a:e, j], o_ref[a:e, h]))
                es = max(es, frob_rel(fin[n, j], f_ref[n, h]))
    check("test_head_split_on_gpu_against_oracle", "o per head", eo, BF16_TOL)
    check("test_head_split_on_gpu_against_oracle", "state per head", es, BF16_TOL)
