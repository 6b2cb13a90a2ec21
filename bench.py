#!/usr/bin/env python
"""Benchmark of the Gated DeltaNet mixer hot path on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
  prefill: gdn_conv1d_silu + gdn_chunk_prefill over a Qwen3.5-27B-shaped layer
           (16 key heads, 48 value heads of 128, conv over 10240 channels) at T = 65536,
           returning the final 48 x 128 x 128 fp32 state;
  decode : gdn_decode_step for 256 sequences x 1 token, 27B-shaped fp32 states
           (256 x 48 x 128 x 128, 805 MB) and 3-tap conv states updated in place.

value  = prefill tokens/s for the layer (device time of the prefill phase, events on the
         launching stream); the decode phase is reported in "decode" as state GB/s.
Inputs (1.34 GB x, 805 MB state) exceed the 126 MB L2, so no flush is needed.

``--impl reference`` times the fp64 CPU oracle on the host cores instead (bounded sample).
Run with torchrun for N > 1: every rank runs its own independent 64K sequence and decode
batch (no data-path collective; weak scaling); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_deltanet_mixer_causal_b200 import workloads as W  # noqa: E402

METRIC = "GDN prefill tokens/s/layer @64K + decode state GB/s, % of roofline"
UNIT = "tokens/s/layer"
SHAPE = W.QWEN35_27B
T_PREFILL = 65536
B_DECODE = 256

# algorithmic work (chunked form counted at C = 64; see the design notes)
def prefill_flops_per_token(sh=SHAPE, C=64):
    d, G = sh.dk, sh.Hv // sh.Hk
    return sh.Hv * (6 * d * d + 6 * C * d + C * C / 3 + 4 * C * d / G)


def prefill_bytes_per_token(sh=SHAPE):
    # q|k|v in (post-conv y for the chunked call, pre-conv x for the layer), o out, g, beta
    return sh.conv_channels * 2 + sh.Hv * sh.dv * 2 + 2 * sh.Hv * 4


def conv_bytes(T, sh=SHAPE):
    return 2 * T * sh.conv_channels * 2 + sh.conv_channels * 4 * 2


def decode_bytes(B, sh=SHAPE, state_bytes=4):
    Cc = sh.conv_channels
    state = B * sh.Hv * sh.dv * sh.dk * state_bytes
    return (2 * state + B * Cc * 2 + 2 * B * 3 * Cc * 2 + B * sh.Hv * sh.dv * 2
            + 2 * B * sh.Hv * 4 + Cc * 4 * 2)


def decode_tokens_bytes(B, n_tok, sh=SHAPE):
    """A multi-token call: each state read and written once, n_tok tokens of x, g, beta, o."""
    Cc = sh.conv_channels
    state = B * sh.Hv * sh.dv * sh.dk * 4
    return (2 * state + n_tok * B * Cc * 2 + 2 * B * 3 * Cc * 2 + n_tok * B * sh.Hv * sh.dv * 2
            + n_tok * 2 * B * sh.Hv * 4 + Cc * 4 * 2)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained", p["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        """Samples go to $GDN_CLOCKS_DIR/clocks_gpu<i>.csv when that is set (to keep them),
        else to a temporary file."""
        import tempfile
        self.gpu = gpu_index
        self.proc = None
        keep = os.environ.get("GDN_CLOCKS_DIR")
        self.path = (os.path.join(keep, f"clocks_gpu{gpu_index}.csv") if keep else
                     os.path.join(tempfile.gettempdir(), f"gdn_clocks_gpu{gpu_index}_{os.getpid()}.csv"))

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1])); smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------------- CPU oracle leg

def cpu_oracle_prefill(p: W.PrefillInputs, target_s: float = 12.0, max_tokens: int = 4096,
                       threads: int = 0):
    """Time the fp64 oracle on the first tokens of the same 64K sequence (all 48 heads,
    conv included), sized to about ``target_s`` seconds, on ``threads`` host threads (0: all
    cores). Returns (tok/s, threads, sample)."""
    import oracle
    sh = p.shape
    threads = threads or oracle.default_threads()

    def run(n):
        x = p.x[:n].float().numpy(); w = p.conv_w.float().numpy()
        t0 = time.perf_counter()
        oracle.layer_prefill(x, w, p.g[:n].numpy(), p.beta[:n].numpy(), sh.Hk, sh.Hv, sh.dk,
                             sh.dv, n_threads=threads)
        return time.perf_counter() - t0

    n0 = 64
    t_cal = run(n0)
    n = int(min(max_tokens, max(n0, n0 * target_s / max(t_cal, 1e-6))))
    dt = run(n)
    return n / dt, threads, f"first {n} tokens of the 65536-token 27B-shaped sequence, all 48 heads, conv included"


# ------------------------------------------------------------ per-workload report

def _median_ms(fn, stream, warmup=5, reps=20):
    """Median device time of fn() over reps runs after warmup runs (CUDA events)."""
    for _ in range(warmup):
        fn()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    ts = []
    for i in range(reps):
        ev[i].record(stream)
        fn()
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    ts = [ev[i].elapsed_time(ev[i + 1]) for i in range(reps)]
    return statistics.median(ts)


def _roof(ms, flops, nbytes, tc_tflops, hbm_gbs):
    t_tc = flops / (tc_tflops * 1e12) * 1e3 if flops else 0.0
    t_hbm = nbytes / (hbm_gbs * 1e9) * 1e3
    t_roof = max(t_tc, t_hbm)
    return {"t_roof_ms": t_roof, "roofline_frac": t_roof / ms, "bound": "tensor" if t_tc > t_hbm else "hbm",
            "tflops": flops / (ms / 1e3) / 1e12 if flops else None, "gbs": nbytes / (ms / 1e3) / 1e9}


def measure_configs(gdn, dev, stream, hbm_gbs, tc_peak):
    """Every benchmark workload, timed as CUDA-event medians of 20 runs after 5 warm-ups:
    the layer (conv + prefill) for the prefill workloads, the 100-step block for decode.
    Roofline fraction = t_roof / t_measured with t_roof = max(flops / burst bf16 peak,
    bytes / HBM copy peak) -- the burst peak, since each timed run is milliseconds long and
    runs at the unthrottled clock; flops in the chunked-form count, bytes = pre-conv x in,
    o out, g and beta in (plus initial and final states where given)."""
    out = []

    def layer(p: W.PrefillInputs, name: str, note: str = ""):
        sh = p.shape
        x = p.x.to(dev); w = p.conv_w.to(dev); g = p.g.to(dev); b = p.beta.to(dev)
        cu = p.cu_seqlens.to(dev) if p.cu_seqlens is not None else None
        s0 = p.initial_state.to(dev) if p.initial_state is not None else None
        n = p.n_seq
        fin = torch.empty((n, sh.Hv, sh.dv, sh.dk), dtype=torch.float32, device=dev)
        y = torch.empty_like(x)
        o = torch.empty((p.T, sh.Hv, sh.dv), dtype=x.dtype, device=dev)
        ws_n = gdn.gdn_chunk_prefill_workspace_size(p.T, n, sh.Hk, sh.Hv, sh.dk, sh.dv, x.dtype)
        ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device=dev)
        fn = lambda: gdn.prefill_layer(x, w, g, b, sh.Hk, sh.Hv, sh.dk, cu_seqlens=cu, initial_state=s0,
                                       final_state=fin, y=y, o=o, workspace=ws)
        ms = _median_ms(fn, stream)
        T = p.T
        rec = {"workload": name, "tokens": T, "sequences": n, "ms": ms, "tokens_per_s": T / (ms / 1e3),
               "dtype": "f32" if x.dtype == torch.float32 else "bf16"}
        if x.dtype == torch.bfloat16:
            nbytes = prefill_bytes_per_token(sh) * T + (2 if s0 is not None else 1) * fin.numel() * 4
            rec.update(_roof(ms, prefill_flops_per_token(sh) * T, nbytes, tc_peak, hbm_gbs))
        if note:
            rec["note"] = note
        out.append(rec)
        del x, w, g, b, y, o, ws, fin

    layer(W.tiny_layer(), "tiny fp32 layer: T=64, Hk=Hv=2, d=16",
          "correctness gate; fp32 token-recurrent path; time only")
    layer(W.qwen35_9b_prefill(8192), "Qwen3.5-9B-shaped layer prefill: T=8192, Hk 16, Hv 32, d 128")
    layer(W.qwen35_27b_prefill(65536), "Qwen3.5-27B-shaped layer prefill: T=65536, Hk 16, Hv 48, d 128")
    layer(W.qwen35_27b_varlen(32), "Qwen3.5-27B-shaped varlen prefill: 32 sequences (log-uniform 512..32768), nonzero initial states")

    dcd = W.qwen35_27b_decode(256, 100)
    sh = dcd.shape
    xs = [t.to(dev) for t in dcd.xs]; gs = [t.to(dev) for t in dcd.gs]; bs = [t.to(dev) for t in dcd.betas]
    cs = dcd.conv_state.to(dev); st = dcd.state.to(dev); cw = dcd.conv_w.to(dev)
    do = torch.empty((256, sh.Hv, sh.dv), dtype=xs[0].dtype, device=dev)

    def block():
        for t in range(100):
            gdn.gdn_decode_step(xs[t], cw, cs, gs[t], bs[t], st, sh.Hk, do)
    ms = _median_ms(block, stream, warmup=2, reps=20) / 100
    rec = {"workload": "Qwen3.5-27B-shaped decode: B=256 x 1 token, 100-step block (per step)",
           "tokens": 256, "sequences": 256, "ms": ms, "tokens_per_s": 256 / (ms / 1e3), "dtype": "bf16"}
    rec.update(_roof(ms, 0, decode_bytes(256, sh), tc_peak, hbm_gbs))
    out.append(rec)

    # the same 100-step block with the states stored in bf16
    st16 = st.to(torch.bfloat16)

    def block16():
        for t in range(100):
            gdn.gdn_decode_step(xs[t], cw, cs, gs[t], bs[t], st16, sh.Hk, do)
    ms = _median_ms(block16, stream, warmup=2, reps=20) / 100
    rec = {"workload": "Qwen3.5-27B-shaped decode, bf16 states: B=256 x 1 token, 100-step block (per step)",
           "tokens": 256, "sequences": 256, "ms": ms, "tokens_per_s": 256 / (ms / 1e3), "dtype": "bf16"}
    rec.update(_roof(ms, 0, decode_bytes(256, sh, state_bytes=2), tc_peak, hbm_gbs))
    out.append(rec)
    del st16

    # multi-token decode / verify: 4 tokens per sequence per call (25 calls = 100 tokens)
    n_tok = 4
    xt = [torch.stack(xs[i:i + n_tok], 1) for i in range(0, 100, n_tok)]
    gt = [torch.stack(gs[i:i + n_tok], 1) for i in range(0, 100, n_tok)]
    bt = [torch.stack(bs[i:i + n_tok], 1) for i in range(0, 100, n_tok)]
    ot = torch.empty((256, n_tok, sh.Hv, sh.dv), dtype=xs[0].dtype, device=dev)

    def block4():
        for i in range(len(xt)):
            gdn.gdn_decode_tokens(xt[i], cw, cs, gt[i], bt[i], st, sh.Hk, ot)
    ms = _median_ms(block4, stream, warmup=2, reps=20) / len(xt)
    rec = {"workload": "Qwen3.5-27B-shaped multi-token decode: B=256 x 4 tokens per call (per call)",
           "tokens": 256 * n_tok, "sequences": 256, "ms": ms, "tokens_per_s": 256 * n_tok / (ms / 1e3),
           "dtype": "bf16"}
    rec.update(_roof(ms, 0, decode_tokens_bytes(256, n_tok, sh), tc_peak, hbm_gbs))
    out.append(rec)
    return out


# --------------------------------------------------------------------------- main

def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="gdn", choices=["gdn", "reference"])
    ap.add_argument("--T", type=int, default=T_PREFILL)
    ap.add_argument("--decode-batch", type=int, default=B_DECODE)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload report (run after the timed region, N = 1 only)")
    return ap.parse_args()


def dist_setup(n_gpus):
    """One process per GPU (torchrun's RANK / WORLD_SIZE / LOCAL_RANK); NCCL on GPUs, gloo
    where there is no GPU (the CPU-only reference arm and the multi-process tests)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        timeout = datetime.timedelta(seconds=120)
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=timeout)
    return rank, world, local


def max_over_ranks(v: float, world: int, dev) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def run_reference(args, rank, world):
    if rank != 0:
        return
    p = W.qwen35_27b_prefill(args.T)
    vals, threads, sample = [], 0, ""
    for i in range(args.warmup + args.steps):
        v, threads, sample = cpu_oracle_prefill(p, target_s=3.0, max_tokens=1024)
        if i >= args.warmup:
            vals.append(v)
    value = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, 27B-shaped)",
            "config": {"workload": f"Qwen3.5-27B-shaped GDN layer prefill, T={args.T} (oracle sample)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank, world, local = dist_setup(args.gpus)
    if args.impl == "reference":
        run_reference(args, rank, world)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    import gated_deltanet_mixer_causal_b200 as gdn
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    sh = SHAPE
    hbm_gbs, tc_tflops, tc_sust, peak_src = measured_peaks()

    # ---- inputs, resident in HBM before timing (each rank: its own seed offset)
    p = W.make_prefill(sh, args.T, seed=2 + 1000 * rank, g_low=-0.3)
    dcd = W.make_decode(sh, args.decode_batch, 1, seed=3 + 1000 * rank, g_low=-0.3)
    x = p.x.to(dev); w = p.conv_w.to(dev); g = p.g.to(dev); beta = p.beta.to(dev)
    T, Cc = x.shape
    y = torch.empty_like(x)
    o = torch.empty((T, sh.Hv, sh.dv), dtype=x.dtype, device=dev)
    fin = torch.empty((1, sh.Hv, sh.dv, sh.dk), dtype=torch.float32, device=dev)
    ws_n = gdn.gdn_chunk_prefill_workspace_size(T, 1, sh.Hk, sh.Hv, sh.dk, sh.dv, x.dtype)
    ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device=dev)
    dx = dcd.xs[0].to(dev); dg = dcd.gs[0].to(dev); db = dcd.betas[0].to(dev)
    dcs = dcd.conv_state.to(dev); dst = dcd.state.to(dev); dw = dcd.conv_w.to(dev)
    do = torch.empty((args.decode_batch, sh.Hv, sh.dv), dtype=x.dtype, device=dev)
    q, k, v = gdn.qkv_views(y, sh.Hk, sh.Hv, sh.dk)
    stream = torch.cuda.current_stream(dev)

    def step(ev):
        ev[0].record(stream)
        gdn.gdn_conv1d_silu(x, w, None, None, None, y)
        ev[1].record(stream)
        gdn.gdn_chunk_prefill(q, k, v, g, beta, None, None, fin, 1.0, True, o, ws)
        ev[2].record(stream)
        gdn.gdn_decode_step(dx, dw, dcs, dg, db, dst, sh.Hk, do)
        ev[3].record(stream)

    # launches of this library's kernels per step: conv 1, prefill (per path), decode 1
    launches_per_step = 1 + gdn_prefill_launches(T, 1, sh, torch.cuda.get_device_properties(dev).multi_processor_count) + 1

    for _ in range(args.warmup):
        step([torch.cuda.Event(enable_timing=True) for _ in range(4)])
    torch.cuda.synchronize(dev)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True); t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    clk = clocks.stop()

    total_ms = t_start.elapsed_time(t_end)
    conv_ms = [e[0].elapsed_time(e[1]) for e in evs]
    pre_ms = [e[1].elapsed_time(e[2]) for e in evs]
    dec_ms = [e[2].elapsed_time(e[3]) for e in evs]
    total_ms = max_over_ranks(total_ms, world, dev)
    layer_ms = max_over_ranks(sum(c + p_ for c, p_ in zip(conv_ms, pre_ms)), world, dev)
    dec_sum = max_over_ranks(sum(dec_ms), world, dev)

    value = world * T * args.steps / (layer_ms / 1e3)
    conv_avg, pre_avg, dec_avg = (statistics.mean(conv_ms), statistics.mean(pre_ms),
                                  statistics.mean(dec_ms))
    dec_gbs = decode_bytes(args.decode_batch) / (dec_avg / 1e3) / 1e9
    conv_gbs = conv_bytes(T) / (conv_avg / 1e3) / 1e9
    pre_tflops = prefill_flops_per_token() * T / (pre_avg / 1e3) / 1e12

    # dominant kernel: the prefill call (the chunked gated delta rule)
    kernels = {"prefill": pre_avg, "conv": conv_avg, "decode": dec_avg}
    dominant = max(kernels, key=kernels.get)
    if dominant == "prefill":
        roof = {"kernel": "gdn_chunk_prefill", "bound": "tensor", "achieved": pre_tflops,
                "peak": tc_tflops, "unit": "TFLOP/s", "frac": pre_tflops / tc_tflops,
                "peak_kind": f"bf16 dense burst ({peak_src}): the call runs for milliseconds at the "
                             f"unthrottled clock (see clocks)",
                "frac_of_sustained_peak": pre_tflops / tc_sust,
                "algorithmic_per_launch": prefill_flops_per_token() * T,
                "traffic": traffic("prefill", T),
                "kernels": prefill_kernel_split(T, pre_avg, tc_tflops)}
    elif dominant == "decode":
        roof = {"kernel": "gdn_decode_step", "bound": "hbm", "achieved": dec_gbs, "peak": hbm_gbs,
                "unit": "GB/s", "frac": dec_gbs / hbm_gbs, "peak_kind": f"HBM copy ({peak_src})",
                "algorithmic_per_launch": decode_bytes(args.decode_batch),
                "traffic": traffic("decode", args.decode_batch)}
    else:
        roof = {"kernel": "gdn_conv1d_silu", "bound": "hbm", "achieved": conv_gbs, "peak": hbm_gbs,
                "unit": "GB/s", "frac": conv_gbs / hbm_gbs, "peak_kind": f"HBM copy ({peak_src})",
                "algorithmic_per_launch": conv_bytes(T), "traffic": traffic("conv", T)}

    # ---- end to end: host buffers in pinned memory, copies inside the timed region
    e2e = None
    if args.e2e_steps > 0:
        hx = p.x.pin_memory(); hg = p.g.pin_memory(); hb = p.beta.pin_memory()
        ho = torch.empty((T, sh.Hv, sh.dv), dtype=x.dtype).pin_memory()
        hfin = torch.empty_like(fin, device="cpu").pin_memory()
        hdx = dcd.xs[0].pin_memory(); hdg = dcd.gs[0].pin_memory(); hdb = dcd.betas[0].pin_memory()
        hdo = torch.empty_like(do, device="cpu").pin_memory()

        # the steps are pipelined as a serving loop runs them: step i's inputs go up on one copy
        # stream while step i-1 computes on the compute stream and step i-2's outputs come down
        # on another copy stream (PCIe carries both directions at once), with two sets of device
        # buffers taken in turn; every step's copies are inside the timed region
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        xb, gb, bb = [x, torch.empty_like(x)], [g, torch.empty_like(g)], [beta, torch.empty_like(beta)]
        ob, fb = [o, torch.empty_like(o)], [fin, torch.empty_like(fin)]
        ev_up = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_down = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(i):
            k = i % 2
            up.wait_event(ev_comp[k])      # step i-2 no longer reads buffer set k
            with torch.cuda.stream(up):
                xb[k].copy_(hx, non_blocking=True); gb[k].copy_(hg, non_blocking=True)
                bb[k].copy_(hb, non_blocking=True)
            ev_up[k].record(up)
            stream.wait_event(ev_up[k])
            stream.wait_event(ev_down[k])  # step i-2's outputs have left buffer set k
            gdn.prefill_layer(xb[k], w, gb[k], bb[k], sh.Hk, sh.Hv, sh.dk, final_state=fb[k], y=y,
                              o=ob[k], workspace=ws)
            dx.copy_(hdx, non_blocking=True); dg.copy_(hdg, non_blocking=True)
            db.copy_(hdb, non_blocking=True)
            gdn.gdn_decode_step(dx, dw, dcs, dg, db, dst, sh.Hk, do)
            hdo.copy_(do, non_blocking=True)
            ev_comp[k].record(stream)
            down.wait_event(ev_comp[k])
            with torch.cuda.stream(down):
                ho.copy_(ob[k], non_blocking=True); hfin.copy_(fb[k], non_blocking=True)
            ev_down[k].record(down)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        barrier(world)
        a = torch.cuda.Event(enable_timing=True); b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        up.wait_event(a)
        for i in range(args.e2e_steps):
            e2e_step(i)
        stream.wait_event(ev_down[(args.e2e_steps - 1) % 2])
        b.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(a.elapsed_time(b), world, dev)
        h2d = hx.numel() * 2 + hg.numel() * 4 + hb.numel() * 4 + hdx.numel() * 2 + hdg.numel() * 4 + hdb.numel() * 4
        d2h = ho.numel() * 2 + hfin.numel() * 4 + hdo.numel() * 2
        e2e = {"value": world * T * args.e2e_steps / (e2e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "note": "prefill tokens/s with each step's x, g, beta copied in from pinned host "
                       "memory and its o + final state copied out, decode step included; steps "
                       "pipelined (inputs of step i up while step i-1 computes and step i-2's "
                       "outputs come down), two device buffer sets in turn"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v_cpu, threads, sample = cpu_oracle_prefill(p)
        v_one, _, sample_one = cpu_oracle_prefill(p, target_s=4.0, max_tokens=1024, threads=1)
        cpu = {"value": v_cpu, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample,
               "value_1_thread": v_one, "sample_1_thread": sample_one}

    configs = None
    if rank == 0 and world == 1 and not args.no_configs:
        del x, y, o, ws, dst, dx, dg, db, dcs, do
        torch.cuda.empty_cache()
        configs = measure_configs(gdn, dev, stream, hbm_gbs, tc_tflops)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; x~N(0,1), conv w~N(0,0.5), g~U[-0.3,0], beta=sigmoid(N(0,1)), decode state~N(0,0.02))",
            "config": {"workload": f"Qwen3.5-27B-shaped GDN layer: prefill T={T} (Hk 16, Hv 48, d 128, "
                                   f"conv 10240 ch) + decode step B={args.decode_batch}",
                       "global_batch": world, "seq_len": T, "parallelism": f"dp{world}",
                       "l2": "inputs larger than L2 (126 MB); no flush"},
            "prefill": {"tokens_per_s": value, "conv_ms": conv_avg, "chunk_prefill_ms": pre_avg,
                        "chunk_prefill_ms_steps": [round(t, 4) for t in pre_ms],
                        "chunk_prefill_tflops": pre_tflops,
                        "flops_per_token": prefill_flops_per_token(),
                        "layer_ms": (conv_avg + pre_avg),
                        "conv_gbs": conv_gbs, "conv_frac_hbm": conv_gbs / hbm_gbs},
            "decode": {"value": dec_gbs, "unit": "GB/s", "us_per_step": dec_avg * 1e3,
                       "frac_hbm": dec_gbs / hbm_gbs, "bytes_per_step": decode_bytes(args.decode_batch),
                       "tokens_per_s": world * args.decode_batch / (dec_avg / 1e3)},
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk,
            "configs": configs,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def gdn_prefill_launches(T: int, n_seq: int = 1, sh=SHAPE, num_sms: int = 148) -> int:
    """Kernels one gdn_chunk_prefill call enqueues on the benchmark's path (bf16, d = 128), as
    the library's own schedule counts them: the chunk plan, then the intra-chunk and chain
    kernels once each, or, for a single sequence of 512 chunks or more run in pieces, one chain
    launch per piece and the intra-chunk launches of its schedule."""
    import gated_deltanet_mixer_causal_b200 as gdn
    return gdn.gdn_chunk_prefill_launches(T, n_seq, sh.Hk, sh.Hv, sh.dk, sh.dv, torch.bfloat16, num_sms)


# DRAM traffic (bytes, dram__bytes_read.sum + dram__bytes_write.sum) from one ncu capture
# of each kernel on the small case (T = 8192, decode batch 64), per unit processed (token
# for the prefill kernels and the conv, sequence for the decode step), scaled to the
# benchmark's launch; None when the kernel changed since the capture. The prefill figure is
# the intra-chunk kernel's 468.19 MB plus the chain kernel's 509.36 MB.
TRAFFIC_PER_UNIT = {"prefill": (468.19e6 + 509.36e6) / 8192, "conv": 291.25e6 / 8192,
                    "decode": 357.64e6 / 64}

# The chunked prefill's two kernels: their share of its FLOPs (from the chunked form: the
# intra-chunk kernel forms K K^T and Q K^T per key head, solves the triangular system and
# builds U~ = P V, W = Pk K and Mqk; the chain applies [-W; Q] S0^T, K^T U' and Mqk U), the
# device time each takes alone for a 65536-token call's work (its ncu capture at T = 8192,
# one launch on the whole GPU, scaled by tokens: 168.54 us -> 1348.4 us of intra-chunk work,
# 265.18 us -> 2121.5 us of chain; in the call the two run side by side, so the call takes
# less than their sum), and their DRAM traffic per token from the same captures.
PREFILL_KERNELS = {
    "chunk_intra": {"busy_us_64k": 1348.4, "traffic_per_token": 468.19e6 / 8192},
    "chunk_chain": {"busy_us_64k": 2121.5, "traffic_per_token": 509.36e6 / 8192},
}


def prefill_kernel_flops_per_token(kernel: str, sh=SHAPE, C=64):
    d, G = sh.dk, sh.Hv // sh.Hk
    if kernel == "chunk_chain":
        return sh.Hv * (6 * d * d + 2 * C * d)
    return sh.Hv * (4 * C * d / G + C * C / 3 + 4 * C * d)


def prefill_kernel_split(T: int, prefill_ms: float, peak_tflops: float) -> dict:
    """Per-kernel FLOPs and traffic of one prefill launch, each kernel's rate over its own
    device time (the launch list's, scaled by tokens), and how much of the call the two
    kernels' times overlap."""
    out = {}
    busy = 0.0
    for k, v in PREFILL_KERNELS.items():
        flops = prefill_kernel_flops_per_token(k) * T
        ms = v["busy_us_64k"] / 1e3 * T / 65536
        busy += ms
        out[k] = {"flops": flops, "device_ms": ms, "tflops": flops / (ms / 1e3) / 1e12,
                  "frac": flops / (ms / 1e3) / 1e12 / peak_tflops,
                  "traffic": v["traffic_per_token"] * T}
    out["overlap"] = {"device_ms_sum": busy, "call_ms": prefill_ms,
                      "note": "each kernel's device time alone for the call's work; in the call "
                              "the intra-chunk work of later pieces runs beside the chain "
                              "pieces, so the call is shorter than the sum"}
    return out


def traffic(kernel: str, units: int):
    per = TRAFFIC_PER_UNIT.get(kernel)
    return None if per is None else per * units

if __name__ == "__main__":
    main()
