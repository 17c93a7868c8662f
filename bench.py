#!/usr/bin/env python
"""Refined decode benchmark: microseconds per token and achieved HBM bandwidth
of a Llama-3.1-8B-shaped decode step on B200.

Workload (the largest single-GPU configuration): 32 layers, hidden 4096,
intermediate 14336, 32 query / 8 KV heads of 128, vocab 128256 (fp16 LM head);
2-bit weights + 2 nested refinement bits with k = 32 of every 1,024 input
channels refined per projection; 2-bit KV cache + 2 refinement bits over
32,768 cached tokens with the top 512 tokens refined per KV head; weight
refinement rows in pinned host memory, staged with fetch lead and lag of one
layer on two staging streams.  Batch 1.  Weights, caches and inputs are seeded
synthetic data of those shapes (N(0, 0.02) weights, N(0, 1) activations and
keys/values with 4 key outlier channels per head).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One process per GPU (torchrun for N > 1); every rank runs its own replica of
the step (the method is single-GPU; there is no exchange), the time is the max
over ranks, rank 0 prints one JSON line.  `--impl reference` times the CPU
oracle (the fp64 reference implementation) on a bounded sample of the same
workload.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "refined decode µs/token and achieved HBM GB/s (fraction of ~8 TB/s), 1×B200"
UNIT = "us/token"
T_CTX = 32768
BATCH = 1
SEED = 4
WORKLOAD = ("Llama-3.1-8B-shaped decode step: 32 layers, hidden 4096, inter 14336, 32/8 heads x 128, "
            "vocab 128256 fp16 LM head; 2-bit weights + 2 refinement bits, k=32 per 1024 channels; "
            "2-bit KV + 2 refinement bits, T=32768 cached tokens, top-512 refined per KV head; "
            "weight refinement rows in pinned host memory staged with fetch lead/lag 1")


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region


class ClockSampler:
    def __init__(self, index: int):
        self.index, self.rows, self.proc = index, [], None

    def __enter__(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 8:
                self.rows.append(parts)

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[0]) for r in self.rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in self.rows for n, v in zip(names, r[4:8]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


# ---------------------------------------------------------------------------
# the GPU arm


def build_decoder(batch, t, device):
    import torch

    from bit_decode_selective_b200 import inputs
    from bit_decode_selective_b200.decoder import Decoder, DecoderConfig

    cfg = DecoderConfig()
    dec = Decoder(cfg, batch, t, device=device)
    for l in range(cfg.n_layers):
        ws = {}
        for i, (name, n, k) in enumerate(cfg.shapes()):
            ws[name] = inputs.torch_normal((n, k), 0.02, SEED * 100000 + l * 10 + i, device=device)
        kk = inputs.torch_normal((batch, cfg.h_kv, t, cfg.d), 1.0, SEED * 100000 + l * 10 + 5,
                                 device=device, dtype=torch.float16)
        vv = inputs.torch_normal((batch, cfg.h_kv, t, cfg.d), 1.0, SEED * 100000 + l * 10 + 6,
                                 device=device, dtype=torch.float16)
        # 4 outlier key channels per KV head, as in the KV workloads
        g = torch.Generator(device="cpu").manual_seed(SEED * 100000 + l * 10 + 7)
        for h in range(cfg.h_kv):
            ch = torch.randperm(cfg.d, generator=g)[:4].to(device)
            kk[:, h, :, ch] *= 10
        dec.load_layer(ws, kk, vv)
        del ws, kk, vv
    lm = inputs.torch_normal((cfg.vocab, cfg.hidden), 0.02, SEED * 100000 + 99, device=device,
                             dtype=torch.float16)
    dec.set_lm_head(lm)
    hidden = inputs.torch_normal((batch, cfg.hidden), 1.0, SEED * 100000 + 98, device=device,
                                 dtype=torch.float16)
    return dec, hidden


def count_kernels(graph) -> int | None:
    try:
        from cuda.bindings import runtime as rt
    except Exception:
        try:
            from cuda import cudart as rt
        except Exception:
            return None
    try:
        raw = graph.raw_cuda_graph()
        if isinstance(raw, int):
            raw = rt.cudaGraph_t(init_value=raw)
        err, nodes, n = rt.cudaGraphGetNodes(raw, 0)
        err, nodes, n = rt.cudaGraphGetNodes(raw, n)
        kern = 0
        for nd in nodes:
            err, ty = rt.cudaGraphNodeGetType(nd)
            if ty == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                kern += 1
        return kern
    except Exception:
        return None


# DRAM bytes (read + write) of one refined GEMV launch in an ncu capture
# (`bench.py --case gemv`: the 28,672 x 4,096 launch, 2 + 2 bits, k = 32 per
# 1,024) over that launch's algorithmic bytes; traffic grows in proportion to
# the codes a launch streams, so a launch's traffic is its bytes times this.
GEMV_TRAFFIC_PER_BYTE = 34028288 / 34071040


def gemv_roofline(dec, steps, warmup, hbm_peak):
    """Average duration of the refined GEMV launches of the step, timed with
    CUDA events around a CUDA graph of all of them (the 4 projections of every
    layer, with their lead selections and staged rows) on the launching stream."""
    import torch

    from bit_decode_selective_b200 import abi, bytemodel
    from bit_decode_selective_b200.ops import _p

    cfg = dec.cfg
    xs = {"qkv": dec.x_attn[0], "o": dec.x_o[0], "gate_up": dec.x_mlp[0], "down": dec.x_down[0]}
    ys = {"qkv": dec.qkv_out, "o": dec.o_out, "gate_up": dec.gu_out, "down": dec.down_out}
    # selections and staged rows as the step leaves them (slot 0)
    calls, nbytes = [], 0
    for l in range(cfg.n_layers):
        for name, n, k in cfg.shapes():
            qw = dec.layers[l][name]
            rows = dec.slots[name][0] if dec.slots is not None else None
            calls.append((qw, xs[name], ys[name], dec.sel[name][0], rows))
            nbytes += bytemodel.gemv_bytes(n, k, cfg.w_bits, cfg.w_refine, cfg.group, cfg.kch, cfg.chunk, dec.B)

    def run():
        s = torch.cuda.current_stream()  # the capture stream inside torch.cuda.graph
        for qw, x, y, sel, rows in calls:
            abi.check(abi.sf_gemv_refined(ctypes.byref(qw.desc), _p(x), dec.B, cfg.chunk, cfg.kch, _p(sel), None,
                                          _p(rows), _p(y), _p(dec.gemv_ws), dec.gemv_ws.numel(),
                                          ctypes.c_void_p(s.cuda_stream)),
                      "sf_gemv_refined")

    run()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    sec = e0.elapsed_time(e1) / 1e3 / steps
    launches = len(calls)
    per_launch_s = sec / launches
    per_launch_bytes = nbytes / launches
    achieved = per_launch_bytes / per_launch_s / 1e9
    return {"kernel": "gemv_kernel (refined GEMV, 4 per layer)", "bound": "hbm", "achieved": achieved,
            "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
            "bytes_per_launch": per_launch_bytes, "us_per_launch": per_launch_s * 1e6,
            "launches_per_step": launches}


def max_over_ranks(values, world, device):
    """Each of `values` (per-rank times) maximised over the ranks: the job is
    as slow as its slowest replica.  world 1: unchanged."""
    if world <= 1:
        return [float(v) for v in values]
    import torch

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t]


def job_us_per_token(ms_per_step, world):
    """Microseconds per token over the tokens of all replicas: every rank
    decodes BATCH tokens per step."""
    return ms_per_step * 1e3 / (BATCH * world)


def base_only_ms(dec, hidden, s, steps, warmup):
    """ms per step of the same decoder with channel refinement switched off
    (kch = 0), captured as its own graph on stream s."""
    import torch

    kch = dec.cfg.kch
    dec.cfg.kch = 0
    try:
        with torch.cuda.stream(s):
            dec.step(hidden)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                dec.step(hidden)
            for _ in range(warmup):
                g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            for _ in range(steps):
                g.replay()
            e1.record(s)
            torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) / steps
    finally:
        dec.cfg.kch = kch


def run_ours(args, rank, world, local_rank):
    import torch

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    from bit_decode_selective_b200 import abi, bytemodel

    abi.lib()
    hbm_peak, peak_kind = peaks()
    dec, hidden = build_decoder(BATCH, T_CTX, device)
    cfg = dec.cfg
    s = torch.cuda.Stream(device=device)
    with torch.cuda.stream(s):
        dec.step(hidden)  # warm the library (attributes, first launches)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(g, stream=s):
            dec.step(hidden)
        n_kernels = count_kernels(g)
        g.instantiate()
        for _ in range(args.warmup):
            g.replay()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(local_rank) as clocks:
            e0.record(s)
            for _ in range(args.steps):
                g.replay()
            e1.record(s)
            torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        ms = e0.elapsed_time(e1) / args.steps
        # end to end: pinned host input -> device, step, logits -> pinned host
        h_host = torch.empty_like(hidden, device="cpu").pin_memory()
        h_host.copy_(hidden.cpu())
        out_host = torch.empty(dec.logits.shape, dtype=torch.float32).pin_memory()
        h_dev = hidden
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(s)
        for _ in range(args.steps):
            h_dev.copy_(h_host, non_blocking=True)
            g.replay()
            out_host.copy_(dec.logits, non_blocking=True)
        f1.record(s)
        torch.cuda.synchronize()
        ms_e2e = f0.elapsed_time(f1) / args.steps
        roof = gemv_roofline(dec, max(3, args.steps // 5), max(3, args.warmup), hbm_peak)
        ms_base = base_only_ms(dec, hidden, s, max(3, args.steps // 2), args.warmup)
    roof["peak_kind"] = peak_kind
    ms, ms_e2e, ms_base = max_over_ranks([ms, ms_e2e, ms_base], world, device)
    step_bytes = decode_step_bytes(cfg, BATCH, T_CTX)
    res = {
        "metric": METRIC, "value": job_us_per_token(ms, world), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "batch": BATCH, "context_tokens": T_CTX, "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (the step reads ~3.9 GB)"},
        "hbm": {"algorithmic_bytes_per_step": step_bytes, "achieved_gbs": step_bytes / (ms / 1e3) / 1e9,
                "frac_of_measured_copy": step_bytes / (ms / 1e3) / 1e9 / hbm_peak,
                "frac_of_8tbs": step_bytes / (ms / 1e3) / 1e9 / 8000.0,
                "pcie_bytes_per_step": staged_bytes(cfg, BATCH)},
        "roofline": {**roof, "traffic": roof["bytes_per_launch"] * GEMV_TRAFFIC_PER_BYTE},
        "e2e": {"value": job_us_per_token(ms_e2e, world), "unit": UNIT,
                "h2d_bytes_per_step": hidden.numel() * 2, "d2h_bytes_per_step": dec.logits.numel() * 4},
        "gpu_launches": (n_kernels * args.steps) if n_kernels else None,
        "base_only": {"ms_per_step": ms_base, "refined_over_base_throughput": ms_base / ms,
                      "what": "the same step with no channel refinement (kch = 0: no selection, staging or "
                              "correction of the weights; the KV path unchanged), its own graph"},
        "clocks": clocks.summary(),
    }
    if rank == 0:
        res["cpu_baseline"] = cpu_baseline()
    return res


def decode_step_bytes(cfg, batch, t):
    from bit_decode_selective_b200 import bytemodel

    tot = 0
    for name, n, k in cfg.shapes():
        tot += bytemodel.gemv_bytes(n, k, cfg.w_bits, cfg.w_refine, cfg.group, cfg.kch, cfg.chunk, batch)
    tot += bytemodel.kv_attention_bytes(t + 1, cfg.h_kv, cfg.h_q, cfg.d, cfg.kv_bits, cfg.kv_refine, 32,
                                        cfg.k_tok, batch)
    tot *= cfg.n_layers
    tot += cfg.vocab * cfg.hidden * 2 + batch * (cfg.hidden * 2 + cfg.vocab * 4)
    return tot


def staged_bytes(cfg, batch):
    tot = 0
    for name, n, k in cfg.shapes():
        tot += batch * (k // cfg.chunk) * cfg.kch * n * cfg.w_refine // 8
    return tot * cfg.n_layers if cfg.host_refine else 0


# ---------------------------------------------------------------------------
# the CPU oracle (baseline and reference arm)


def oracle_sample():
    """One full-size decoder layer of the step in the fp64 oracle plus the LM
    head; returns (seconds for the layer, seconds for the LM head, cores)."""
    import oracle
    from oracle.decoder import OracleDecoder
    from bit_decode_selective_b200 import inputs

    cores = oracle.set_threads(0)
    h16, lm = inputs.decoder_io(SEED, 1)
    W = inputs.decoder_layer_weights(SEED, 0)
    Q = {n: oracle.quant_weights(w, 2, 2, 128) for n, w in W.items()}
    del W
    k, v = inputs.decoder_layer_kv(SEED, 0, T_CTX)
    dec = OracleDecoder(h16, k_tok=512, lead=1, lag=1)
    t0 = time.perf_counter()
    dec.layer(Q, k, v, T_CTX)
    t1 = time.perf_counter()
    dec.finish(lm)
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1, cores


def cpu_baseline():
    t_layer, t_head, cores = oracle_sample()
    us = (32 * t_layer + t_head) * 1e6
    return {"value": us, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"layer 0 of 32 at full size (T={T_CTX}, {t_layer:.2f} s) and the LM head "
                      f"({t_head:.2f} s), fp64 oracle with OpenMP on {cores} threads; layer time x32 + head"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    per = []
    cores = None
    for i in range(args.warmup + args.steps):
        t_layer, t_head, cores = oracle_sample()
        if i >= args.warmup:
            per.append(32 * t_layer + t_head)
    sec = statistics.mean(per)
    us = sec * 1e6
    return {"impl": "reference", "metric": METRIC, "value": us, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "batch": BATCH, "context_tokens": T_CTX},
            "cpu_baseline": {"value": us, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": "each step: one full-size layer (x32) + the LM head in the fp64 oracle"},
            "e2e": {"value": us, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_case(name):
    """A few launches of one hot kernel on a small case, for profiler captures
    (no timing): `gemv` = the gate/up-shaped refined GEMV (28,672 x 4,096,
    2 + 2 bits, k = 32 per 1,024), base then refined with a given selection,
    three times; `kv` = score-select-attend over 8 KV heads x 32,768 tokens,
    top-512, three times."""
    import torch

    from bit_decode_selective_b200 import inputs
    from bit_decode_selective_b200.ops import KVCache, QuantWeights, select_channels

    if name == "gemv":
        w = inputs.torch_normal((28672, 4096), 0.02, 1)
        qw = QuantWeights.pack(w, 2, 2, 128)
        del w
        x = inputs.torch_normal((1, 4096), 1.0, 2, dtype=torch.float16)
        y = torch.empty(1, 28672, device="cuda")
        sel = select_channels(x, 1024, 32)
        for _ in range(3):
            qw.gemv(x, 1024, 0, y=y)
            qw.gemv(x, 1024, 32, y=y, sel_in=sel)
    else:
        t = 32768
        k = inputs.torch_normal((1, 8, t, 128), 1.0, 3, dtype=torch.float16)
        v = inputs.torch_normal((1, 8, t, 128), 1.0, 4, dtype=torch.float16)
        c = KVCache(1, 8, t, 2, 2)
        c.pack_tokens(k, v, 0)
        del k, v
        q = inputs.torch_normal((1, 32, 128), 1.0, 5, dtype=torch.float16)
        out = torch.empty(1, 32, 128, device="cuda")
        sel = torch.empty(1, 8, 512, dtype=torch.int32, device="cuda")
        for _ in range(3):
            c.attend_selective(q, t, 512, sel=sel, out=out)
    torch.cuda.synchronize()
    print(json.dumps({"case": name, "ok": True}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--case", choices=["gemv", "kv"], default=None,
                    help="run a few launches of one kernel for a profiler capture instead")
    args = ap.parse_args()
    if args.case:
        run_case(args.case)
        return
    args.warmup = max(args.warmup, 3)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if world > 1:
        import datetime

        import torch

        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    res = run_ours(args, rank, world, local_rank)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch

        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
