#!/usr/bin/env python
"""Throughput of the GPT-2 pretraining step on B200 (tokens/s and MFU).

One step = forward + next-token cross-entropy + backward + AdamW over one
micro-batch of synthetic Zipf(1.1) token ids (stand-in for FineWeb-Edu, which
is not available offline), the workload of "Criei GPT-2 do zero com uma RTX
4090" (section "Configuração do treinamento": GPT-2 small, micro-batch
16 x 1024, vocabulary 50304).  MFU follows "Pré-treinar um LLM" (compute
section): (6 N + 12 L T d) FLOPs per token over the dense bf16 peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 124m|350m|1.5b|lc4096]
    python bench.py --impl reference ...   (the CPU oracle, timed on host cores)

Prints one JSON line (rank 0).  With N > 1 (torchrun) every rank trains its
own micro-batch and gradients are averaged with an NCCL all-reduce before
AdamW (data parallel, weak scaling).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "train tokens/s, GPT-2 124M T=1024 bf16 on 1 B200; MFU (6N+attn FLOPs)"
HBM_KERNELS = ("ln_fwd", "ln_bwd", "colsum", "adamw")
# linear layers of a decoder block with their fused epilogues (gpt2_op_linear_bf16)
LINEAR_KERNELS = ("qkv", "attn_proj", "fc", "mlp_proj")
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

CONFIGS = {
    # name: (n_layer, d, heads, T, vocab_real, vocab_padded, micro_batch)
    "124m": (12, 768, 12, 1024, 50257, 50304, 16),
    "350m": (24, 1024, 16, 1024, 50257, 50304, 16),
    "1.5b": (48, 1600, 25, 1024, 50257, 50304, 8),
    "lc4096": (12, 768, 12, 4096, 50257, 50304, 4),
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def workload_name(name, c):
    L, d, H, T, Vr, V, B = c
    return f"GPT-2 {name} (L{L} d{d} H{H}) T={T} micro-batch {B}, vocab {V}, Zipf(1.1) ids"


# ------------------------------------------------------------ clock sampler --

class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_uuid):
        self.gpu = gpu_uuid
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 7:
                continue
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
            except ValueError:
                continue
            for nm, val in zip(names, f[3:7]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- our arm --

def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    import decoder_only_transformer_step_b200 as gp
    from decoder_only_transformer_step_b200 import inputs, flops
    from decoder_only_transformer_step_b200 import dp

    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    L, d, H, T, Vr, V, B = CONFIGS[args.config]
    mc = gp.ModelConfig(L, d, H, T, Vr, V, B, 0)
    model = gp.GPT2(mc)
    model.init_params(seed=0)
    M = B * T

    # synthetic inputs, uploaded before timing; a small pool cycled over steps
    pool = []
    for s in range(min(4, args.steps + args.warmup)):
        tok, tgt = inputs.zipf_tokens(B, T, n_ids=Vr, seed=1000 + s + 7919 * rank)
        pool.append((torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda()))
    stream = torch.cuda.current_stream()

    # data parallel (N > 1): the gradient exchange per bucket (a decoder block,
    # the final LayerNorm, the embeddings) on a side stream, each bucket's
    # collective started by the event the backward records when the bucket's
    # gradients are final, overlapped with the rest of the backward; all-reduce
    # and the full AdamW, or with --zero1 reduce-scatter, the update of this
    # rank's part of every bucket and an all-gather of the weights
    exchange = None
    if world > 1:
        buckets = dp.gradient_buckets(gp.gpt2_tensors(mc.c()), L)
        events = [torch.cuda.Event() for _ in buckets]
        for ev in events:
            ev.record()
        exchange = dp.BucketedExchange(buckets, zero1=args.zero1, events=events, stream=torch.cuda.Stream())

    def backward(grad_scale, accumulate, last):
        # the exchange runs with the last micro-batch's backward only
        if exchange is None or not last:
            model.backward(grad_scale, accumulate)
            return
        model.backward_bucketed(exchange.events, grad_scale, accumulate)
        for b in dp.completion_order(L):
            exchange.bucket_ready(model.grad, b)
        exchange.finish()

    def optimizer_step(step_no):
        if exchange is None:
            model.adamw_step(step_no)
            return
        exchange.optimizer_step(model.master, lambda off, cnt: model.adamw_step_range(step_no, off, cnt),
                                model.refresh_shadow)

    # one GPU: forward + loss + backward replayed as one CUDA graph per step
    # (gpt2_graph_capture / gpt2_graph_step: the same kernels without the gaps
    # between ~300 separate launches); the ids are copied into the graph's
    # input buffers each step and AdamW runs after it with the step's number.
    # Several GPUs: the eager backward, which records the per-bucket events the
    # overlapped exchange waits on.
    use_graph = world == 1 and not args.eager

    def step(i):
        tok, tgt = pool[i % len(pool)]
        if use_graph:
            model.graph_step(tok, tgt)
        else:
            model.forward_loss(tok, tgt)
            backward(1.0, 0, True)
        optimizer_step(i + 1)

    if use_graph:
        # one eager step sets every kernel up, then the capture
        tok, tgt = pool[0]
        model.forward_loss(tok, tgt)
        model.backward(1.0, 0)
        torch.cuda.synchronize()
        model.graph_capture(B)
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if model.status() != 0:
        raise RuntimeError("device status after warm-up: %d" % model.status())

    uuid = "GPU-" + str(torch.cuda.get_device_properties(local_rank).uuid)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = gp.gpt2_kernel_launches()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(uuid) as clocks:
        e0.record(stream)
        for i in range(args.steps):
            step(args.warmup + i)
        e1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    launches = gp.gpt2_kernel_launches() - launches0
    ms = e0.elapsed_time(e1)
    status = model.status()
    loss = float(model.loss.item())
    if world > 1:
        t = torch.tensor([ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    ms_step = ms / args.steps
    tokens_per_s = world * M * args.steps / (ms / 1e3)

    # end to end through the public API with host buffers (copies inside)
    tok_h = [torch.from_numpy(inputs.zipf_tokens(B, T, n_ids=Vr, seed=5000 + s + 7919 * rank)[0]).pin_memory()
             for s in range(2)]
    tgt_h = [torch.from_numpy(inputs.zipf_tokens(B, T, n_ids=Vr, seed=5000 + s + 7919 * rank)[1]).pin_memory()
             for s in range(2)]
    loss_h = torch.zeros(1).pin_memory()
    e_steps = max(3, args.steps // 2)

    def e2e_step(i):
        if world == 1:
            model.step_host(tok_h[i % 2], tgt_h[i % 2], loss_h, args.warmup + args.steps + i + 1)
        else:
            tok = tok_h[i % 2].cuda(non_blocking=True)
            tgt = tgt_h[i % 2].cuda(non_blocking=True)
            model.forward_loss(tok, tgt)
            backward(1.0, 0, True)
            optimizer_step(args.warmup + args.steps + i + 1)
            loss_h.copy_(model.loss)
            torch.cuda.synchronize()

    e2e_step(0)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i in range(e_steps):
        e2e_step(i + 1)
    torch.cuda.synchronize()
    e2e_s = time.perf_counter() - t0
    if world > 1:
        t = torch.tensor([e2e_s], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_s = float(t.item())
    e2e_tps = world * M * e_steps / e2e_s

    # the pages' optimizer step: the same micro-batch with 32-fold gradient
    # accumulation (grad_scale 1/k, accumulate after the first), then AdamW
    accum = None
    if args.accum > 1:
        k = args.accum

        if use_graph:
            # the accumulating micro-step as the graph: gradients zeroed once per
            # optimizer step, then k micro-steps that add into them
            model.graph_capture(B, grad_scale=1.0 / k, accumulate=1)

        def accum_step(i):
            if use_graph:
                model.zero_grad()
            for j in range(k):
                tok, tgt = pool[(i * k + j) % len(pool)]
                if use_graph:
                    model.graph_step(tok, tgt)
                else:
                    model.forward_loss(tok, tgt)
                    backward(1.0 / k, 1 if j else 0, j == k - 1)
            optimizer_step(args.warmup + args.steps + e_steps + 2 + i)

        a_steps = 2
        accum_step(0)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for i in range(a_steps):
            accum_step(1 + i)
        a1.record(stream)
        torch.cuda.synchronize()
        a_ms = a0.elapsed_time(a1)
        if world > 1:
            t = torch.tensor([a_ms], device="cuda")
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            a_ms = float(t.item())
        accum = {"accumulation": k, "value": round(world * M * k * a_steps / (a_ms / 1e3), 1), "unit": "tokens/s",
                 "ms_per_optimizer_step": round(a_ms / a_steps, 2),
                 "tokens_per_optimizer_step": world * M * k}

    # dominant kernel: the tied LM-head GEMM [M x V x d], timed alone
    roof = lm_head_roofline(gp, model, M, V, d, stream)
    dec = decode_bench(gp, model, L, d, H, T, Vr, V, args.decode_steps) if rank == 0 and args.decode_steps > 0 \
        else None

    peaks, peak_kind = load_peaks()
    fpt = flops.train_flops_per_token(L, d, V, T, T)
    result = {
        "metric": METRIC,
        "value": round(tokens_per_s, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic Zipf(1.1) token ids over [0, 50257), random-init GPT-2 weights",
        "config": {"workload": workload_name(args.config, CONFIGS[args.config]), "batch_per_gpu": B,
                   "seq_len": T, "parallelism": f"dp{world}" + ("-zero1" if world > 1 and args.zero1 else ""),
                   "l2": "inputs larger than L2: the step's working set (>5 GB) exceeds the 126 MB L2",
                   "launch": "one CUDA graph per step (forward, loss, backward) + AdamW" if use_graph
                   else "eager launches"},
        "mfu": round(flops.mfu(tokens_per_s / world, fpt, peaks["bf16_tflops"] * 1e12), 4),
        "mfu_vs_sustained": round(flops.mfu(tokens_per_s / world, fpt, peaks["bf16_tflops_sustained"] * 1e12), 4),
        "mfu_vs_datasheet": round(flops.mfu(tokens_per_s / world, fpt, 2250e12), 4),
        "flops_per_token": fpt,
        "flops_per_token_matmul": flops.matmul_flops_per_token(L, d, V, T),
        "max_memory_gb": round(torch.cuda.max_memory_allocated() / 1e9, 2),
        "peak_source": peak_kind,
        "final_loss": round(loss, 4),
        "device_status": status,
        "gpu_launches": int(launches),
        "e2e": {"value": round(e2e_tps, 1), "unit": "tokens/s", "h2d_bytes_per_step": 2 * M * 4,
                "d2h_bytes_per_step": 4},
        "roofline": roof,
        "clocks": clocks.summary(),
    }
    if accum:
        result["accum"] = accum
    if dec:
        result["decode"] = dec
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(args.config)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def decode_bench(gp, model, L, d, H, T, Vr, V, steps, batch=8, prompt=128):
    """Greedy incremental decoding with the key/value cache on the same model:
    prefill of `batch` prompts of `prompt` tokens, then one CUDA graph per
    decode step (the step's kernels plus the greedy choice, tokens and
    positions on the device), `steps` replays timed with CUDA events after 3
    warm-up replays.  Algorithmic HBM bytes per step: every bf16 weight once
    (the tied LM head reads all of wte), each row's cached K and V of the
    positions it attends to, its new K and V, and the fp32 logits."""
    import torch
    from decoder_only_transformer_step_b200 import inputs
    warm = 3
    steps = min(steps, T - prompt - warm)
    tok = torch.from_numpy(inputs.zipf_tokens(batch, T, n_ids=Vr, seed=777)[0]).cuda()
    plen = torch.full((batch,), prompt, dtype=torch.int32, device="cuda")
    cache = gp.KVCache(model, batch, T)
    cache.prefill(tok, plen)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):   # first launches (kernel attributes) outside the capture
        cache.step()
        cache.greedy_advance()
    torch.cuda.current_stream().wait_stream(side)
    cache.prefill(tok, plen)
    graph = torch.cuda.CUDAGraph()
    l0 = gp.gpt2_kernel_launches()
    with torch.cuda.graph(graph):
        cache.step()
        cache.greedy_advance()
    launches = gp.gpt2_kernel_launches() - l0
    for _ in range(warm):
        graph.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    status = model.status()
    del graph
    weights = L * (12 * d * d + 13 * d) + 2 * d + V * d             # elements read per step
    keys = prompt + warm + (steps - 1) / 2 + 1                       # mean positions attended
    kv = L * 2 * batch * d * (keys + 1)                              # elements read + written
    nbytes = 2 * (weights + kv) + 4 * batch * V
    peaks, _ = load_peaks()
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"workload": f"greedy decode with KV cache, batch {batch}, prompt {prompt}, {steps} new tokens per "
                        "row, one CUDA graph per step", "tokens_per_s": round(batch / (ms / 1e3), 1),
            "ms_per_token_step": round(ms, 4), "gpu_launches_per_step": int(launches),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4), "bytes_per_step": int(nbytes)},
            "device_status": status}


def lm_head_roofline(gp, model, M, V, d, stream):
    import torch
    peaks, kind = load_peaks()
    A = torch.randn(M, d, device="cuda").to(torch.bfloat16)
    wte = model.view(model.shadow, "wte")
    C = torch.empty(M, V, dtype=torch.bfloat16, device="cuda")
    reps = 10
    for _ in range(3):
        gp.gpt2_op_gemm_bf16(A, 0, d, wte, 0, d, C, 0, V, M, V, d, stream=stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        gp.gpt2_op_gemm_bf16(A, 0, d, wte, 0, d, C, 0, V, M, V, d, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    sec = e0.elapsed_time(e1) / 1e3 / reps
    flop = 2.0 * M * V * d
    achieved = flop / sec / 1e12
    peak = peaks["bf16_tflops"]
    del A, C
    return {"kernel": "gemm_tc_kernel<256, pair> (tied LM head, forward: logits = LN_f(x) wte^T)",
            "bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "peak_source": f"{kind} bf16_tflops (burst)",
            "launch_ms": round(sec * 1e3, 4), "flop_per_launch": flop,
            "traffic": recorded_traffic("lm_head_gemm")}


def recorded_traffic(key):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(key)
    if not rec:
        return None
    h = hashlib.sha256()
    for src in rec["sources"]:
        path = os.path.join(ROOT, src)
        if not os.path.exists(path):
            return None
        h.update(open(path, "rb").read())
    return rec["bytes_per_launch"] if h.hexdigest()[:16] == rec["sources_sha256_16"] else None


# ------------------------------------------------------ CPU oracle timing --

def oracle_one_step(config, seed=1000, tokens=None):
    """One fwd + bwd + AdamW step of the CPU oracle on one sequence of the
    workload (batch 1, full depth, width and vocabulary; the first `tokens`
    positions of a T-token stream, all T by default); returns seconds."""
    import numpy as np
    import oracle
    from decoder_only_transformer_step_b200 import inputs
    L, d, H, T, Vr, V, B = CONFIGS[config]
    cfg = oracle.Config(L, d, H, T, V)
    rng = np.random.default_rng(seed)
    params = {}
    for n, s in oracle.param_shapes(cfg):
        params[n] = np.ones(s) if n.endswith("_g") else (0.02 * rng.standard_normal(s) if len(s) == 2 else np.zeros(s))
    m = {n: np.zeros(s) for n, s in oracle.param_shapes(cfg)}
    v = {n: np.zeros(s) for n, s in oracle.param_shapes(cfg)}
    tok, tgt = inputs.zipf_tokens(1, T, n_ids=Vr, seed=seed)
    if tokens is not None:
        tok, tgt = tok[:, :tokens], tgt[:, :tokens]
    t0 = time.perf_counter()
    oracle.train_step(params, m, v, 1, cfg, tok, tgt)
    return time.perf_counter() - t0, tok.size


def host_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        if info:
            return int(info[0].get("num_threads") or os.cpu_count())
    except Exception:
        pass
    return os.cpu_count()


def cpu_baseline(config):
    sec, tokens = oracle_one_step(config)
    return {"value": round(tokens / sec, 2), "unit": "tokens/s", "cores": host_threads(), "kind": "oracle",
            "sample": f"one full training step (fwd+bwd+AdamW, fp64 numpy) on 1 sequence of {tokens} tokens "
                      f"of the same model: {sec:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    L, d, H, T, Vr, V, B = CONFIGS[args.config]
    # warm-up steps of a CPU program only warm caches: at most one is run
    sample = 256
    for _ in range(min(args.warmup, 1)):
        oracle_one_step(args.config, tokens=sample)
    total, tokens = 0.0, 0
    for i in range(args.steps):
        s, t = oracle_one_step(args.config, seed=1000 + i, tokens=sample)
        total += s
        tokens += t
    tps = tokens / total
    cores = host_threads()
    sample = (f"each step: one fwd+bwd+AdamW of the fp64 oracle on the first {sample} tokens of one "
              f"{T}-token sequence (full depth, width and vocabulary)")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(tps, 2), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic Zipf(1.1) token ids", "config": {
            "workload": workload_name(args.config, CONFIGS[args.config]), "batch_per_gpu": B, "seq_len": T,
            "parallelism": "cpu"},
        "cpu_baseline": {"value": round(tps, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(tps, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_kernel(args):
    """One kernel of the step on its own, at a chosen token count (small cases
    for profiler captures): the LM-head GEMM, the attention forward or backward."""
    import torch
    import decoder_only_transformer_step_b200 as gp
    L, d, H, T, Vr, V, B = CONFIGS[args.config]
    hbm = args.kernel in HBM_KERNELS
    # HBM-bound kernels: inputs larger than the 126 MB L2 by default, so the
    # DRAM counters of a capture measure HBM traffic
    M = args.tokens or (131072 if args.kernel in ("ln_fwd", "ln_bwd") else 32768 if args.kernel == "colsum"
                        else 16384 if args.kernel.startswith("lm_head_ce") or args.kernel in LINEAR_KERNELS
                        else 4096)
    g = torch.Generator(device="cuda").manual_seed(0)
    torch.cuda.synchronize()
    nbytes = 0
    if args.kernel in ("ln_fwd", "ln_bwd"):
        x = torch.randn(M, d, device="cuda", generator=g).to(torch.bfloat16)
        gam = (1 + 0.1 * torch.randn(d, device="cuda", generator=g)).to(torch.bfloat16)
        bet = (0.1 * torch.randn(d, device="cuda", generator=g)).to(torch.bfloat16)
        y = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
        mean, rstd = torch.empty(M, device="cuda"), torch.empty(M, device="cuda")
        gp.gpt2_op_layernorm_fwd_bf16(x, gam, bet, y, mean, rstd, M, d)
        if args.kernel == "ln_fwd":
            fn = lambda: gp.gpt2_op_layernorm_fwd_bf16(x, gam, bet, y, mean, rstd, M, d)  # noqa: E731
            nbytes = M * (4 * d + 8)                       # x in, y out (bf16), mean + rstd out
        else:
            dy = torch.randn(M, d, device="cuda", generator=g).to(torch.bfloat16)
            dx = torch.zeros(M, d, dtype=torch.bfloat16, device="cuda")
            dgb = torch.empty(2 * d, device="cuda")
            scr = torch.empty(gp.gpt2_op_layernorm_bwd_scratch_floats(M, d), device="cuda")
            # accumulate into dx, as the step adds into the residual-stream gradient
            fn = lambda: gp.gpt2_op_layernorm_bwd_bf16(dy, x, mean, rstd, gam, dx, 1, dgb, scr, M, d)  # noqa: E731
            nbytes = M * (8 * d + 8)                       # dy, x, dx in; dx out (bf16); mean + rstd in
        flop = 0.0
    elif args.kernel == "colsum":
        N = 4 * d
        x = torch.randn(M, N, device="cuda", generator=g).to(torch.bfloat16)
        out = torch.empty(N, device="cuda")
        scr = torch.empty(gp.gpt2_op_colsum_scratch_floats(M, N), device="cuda")
        fn = lambda: gp.gpt2_op_colsum_bf16(x, M, N, out, scr)  # noqa: E731
        nbytes = M * N * 2                                 # the bias gradient's input, read once
        flop = 0.0
    elif args.kernel == "adamw":
        # the optimizer pass over every parameter of the model (batch 1: the
        # workspace is not used by this kernel)
        model = gp.GPT2(gp.ModelConfig(L, d, H, T, Vr, V, 1, 0))
        model.init_params(seed=0)
        model.grad.normal_(0.0, 1e-3, generator=g)
        M = model.n_params
        stepno = [0]

        def fn():
            stepno[0] += 1
            model.adamw_step(stepno[0])
        nbytes = 30 * M                                    # p, g, m, v in; p, m, v out (fp32); bf16 shadow out
        flop = 0.0
    elif args.kernel == "decode":
        # eager decode steps of the 124M model at batch 8 after a 128-token prompt
        model = gp.GPT2(gp.ModelConfig(L, d, H, T, Vr, V, 8, 0))
        model.init_params(seed=0)
        cache = gp.KVCache(model, 8, T)
        tok = torch.randint(0, Vr, (8, T), dtype=torch.int32, device="cuda", generator=g)
        cache.prefill(tok, torch.full((8,), 128, dtype=torch.int32, device="cuda"))

        def fn():
            cache.step()
            cache.greedy_advance()
        flop = 2.0 * 8 * (L * 12 * d * d + V * d)
    elif args.kernel in ("lm_head_ce", "lm_head_ce_bwd"):
        # the tied LM head with the fused cross-entropy (op entry points): the
        # forward GEMM with the log-sum-exp epilogue, target count, merge and
        # mean; or the two backward GEMMs with the softmax in their operand staging
        A = torch.randn(M, d, device="cuda", generator=g).to(torch.bfloat16)
        W = (0.02 * torch.randn(V, d, device="cuda", generator=g)).to(torch.bfloat16)
        tgt = torch.randint(0, Vr, (M,), device="cuda", generator=g, dtype=torch.int32)
        scr = torch.empty(gp.gpt2_op_lm_head_ce_scratch_bytes(M, V), dtype=torch.uint8, device="cuda")
        loss, rows = torch.empty(1, device="cuda"), torch.empty(M, device="cuda")
        gp.gpt2_op_lm_head_ce_fwd_bf16(A, W, tgt, M, V, d, Vr, loss, rows, scr)
        if args.kernel == "lm_head_ce":
            fn = lambda: gp.gpt2_op_lm_head_ce_fwd_bf16(A, W, tgt, M, V, d, Vr, loss, rows, scr)  # noqa: E731
            flop = 2.0 * M * V * d
        else:
            dx = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
            dw = torch.empty(V, d, device="cuda")
            fn = lambda: gp.gpt2_op_lm_head_ce_bwd_bf16(A, W, M, V, d, 1.0, dx, dw, 0, scr)  # noqa: E731
            flop = 4.0 * M * V * d
    elif args.kernel in LINEAR_KERNELS:
        # one linear layer of a decoder block with its fused epilogue
        N, K, act = {"qkv": (3 * d, d, 0), "attn_proj": (d, d, 1), "fc": (4 * d, d, 2),
                     "mlp_proj": (d, 4 * d, 1)}[args.kernel]
        A = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
        W = (torch.randn(N, K, device="cuda", generator=g) / math.sqrt(K)).to(torch.bfloat16)
        bias = (0.1 * torch.randn(N, device="cuda", generator=g)).to(torch.bfloat16)
        R = torch.randn(M, N, device="cuda", generator=g).to(torch.bfloat16) if act == 1 else None
        C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        C2 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda") if act == 2 else None
        fn = lambda: gp.gpt2_op_linear_bf16(A, W, bias, R, C, C2, M, N, K, act)  # noqa: E731
        flop = 2.0 * M * N * K
    elif args.kernel == "lm_head":
        A = torch.randn(M, d, device="cuda", generator=g).to(torch.bfloat16)
        W = (0.02 * torch.randn(V, d, device="cuda", generator=g)).to(torch.bfloat16)
        C = torch.empty(M, V, dtype=torch.bfloat16, device="cuda")
        fn = lambda: gp.gpt2_op_gemm_bf16(A, 0, d, W, 0, d, C, 0, V, M, V, d)  # noqa: E731
        flop = 2.0 * M * V * d
    else:
        Bn = max(1, M // T)
        qkv = torch.randn(Bn * T, 3 * d, device="cuda", generator=g).to(torch.bfloat16)
        o = torch.empty(Bn * T, d, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(Bn, H, T, device="cuda")
        gp.gpt2_op_attention_fwd_bf16(qkv, o, lse, Bn, T, H, d // H)
        flop = 2.0 * 2 * Bn * H * T * T * (d // H) / 2
        if args.kernel == "attn_fwd":
            fn = lambda: gp.gpt2_op_attention_fwd_bf16(qkv, o, lse, Bn, T, H, d // H)  # noqa: E731
        else:
            do = torch.randn(Bn * T, d, device="cuda", generator=g).to(torch.bfloat16)
            dqkv = torch.empty(Bn * T, 3 * d, dtype=torch.bfloat16, device="cuda")
            scr = torch.empty(Bn * T * d + Bn * H * T, device="cuda")
            fn = lambda: gp.gpt2_op_attention_bwd_bf16(qkv, o, lse, do, dqkv, scr, Bn, T, H, d // H)  # noqa: E731
            flop *= 2.5
    for _ in range(2):
        fn()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.reps
    rec = {"kernel": args.kernel, "tokens" if args.kernel != "adamw" else "params": M, "ms": round(ms, 4)}
    if hbm:
        peaks, kind = load_peaks()
        gbs = nbytes / (ms / 1e3) / 1e9
        rec.update({"algorithmic_bytes": int(nbytes), "gbs": round(gbs, 1),
                    "frac": round(gbs / peaks["hbm_gbs"], 4), "peak": peaks["hbm_gbs"], "peak_source": kind})
    else:
        rec["tflops"] = round(flop / ms / 1e9, 1)
    print(json.dumps(rec))


def relaunch_per_gpu(n):
    """`bench.py --gpus N` started as a plain process: run the same command as
    N ranks on this node (torchrun, rendezvous on 127.0.0.1), each rank taking
    its own GPU, and return the launcher's exit status."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", choices=["lm_head", "lm_head_ce", "lm_head_ce_bwd", "attn_fwd", "attn_bwd",
                                         *LINEAR_KERNELS,
                                         "decode"] + list(HBM_KERNELS),
                    default=None, help="time one kernel alone instead of the step (profiler captures)")
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="124m", choices=sorted(CONFIGS))
    ap.add_argument("--eager", action="store_true",
                    help="issue the step's kernels one by one instead of replaying the captured CUDA graph")
    ap.add_argument("--accum", type=int, default=32,
                    help="also time optimizer steps with this many accumulated micro-batches (0 or 1: skip)")
    ap.add_argument("--decode-steps", type=int, default=64,
                    help="also time this many greedy KV-cache decode steps at batch 8 (0: skip)")
    ap.add_argument("--zero1", action="store_true",
                    help="N>1: shard the AdamW state (reduce-scatter, own-shard update, all-gather) instead of "
                         "an all-reduce and the full update")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: relaunch this command under torchrun
        sys.exit(relaunch_per_gpu(args.gpus))
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.kernel:
        run_kernel(args)
    elif args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
