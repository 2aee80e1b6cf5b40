#!/usr/bin/env python
"""Benchmark of the layer-streamed NF4 LoRA training step on B200.

Default workload: a Llama-3.1-8B-shaped stack (32 decoder layers, hidden
4096, 32 q / 8 kv heads of 128, SwiGLU 14336, vocab 128256, untied lm_head),
all seven projections NF4 (64-blocks) with LoRA r=16 alpha=32, streamed from
pinned host RAM through stream_buffers=2 device slots under a 4 GB device cap;
batch 4 x seq 512 uniform-random token ids; one SFT step = forward through the
streamed stack, chunked next-token CE, recompute-backward through the stream
producing every LoRA gradient.  Synthetic random-init weights of that
architecture (no checkpoints, no datasets).

Prints one JSON line (rank 0).  `value` is train tokens/s measured on the
device (CUDA events on the compute stream, max over ranks) with the step's
inputs already in HBM; `e2e` is the same metric through the public API with
the token ids copied from pinned host memory and the loss read back every
step.  `roofline` reports the dominant kernel (the fused NF4-dequant GEMM)
against the measured bf16 tensor peak.

Multi-GPU (torchrun): data parallel, one micro-batch per rank (weak scaling),
each rank streaming its own copy of the base over its own host link, LoRA
gradients all-reduced with NCCL after the backward pass.

--impl reference times the CPU oracle (plain fp64 numpy) on this host's
cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS = {
    # Llama-3.1-8B-shaped NF4 stack, batch 4 x seq 512, stream_buffers=2, 4 GB cap
    "llama8b-nf4-stream-sft": dict(hidden=4096, n_q_heads=32, n_kv_heads=8, head_dim=128, intermediate=14336,
                                   rank=16, alpha=32.0, vocab=128256, n_layers=32, kind="nf4", tied=False,
                                   batch=4, seq=512, buffers=2, cap_gb=4.0, task="sft"),
    # Qwen2.5-3B-shaped un-quantised bf16 stack, batch 2 x seq 1024, tied embeddings
    "qwen3b-bf16-stream-sft": dict(hidden=2048, n_q_heads=16, n_kv_heads=2, head_dim=128, intermediate=11008,
                                   rank=16, alpha=32.0, vocab=151936, n_layers=36, kind="bf16", tied=True,
                                   batch=2, seq=1024, buffers=2, cap_gb=0.0, task="sft"),
    # DPO on the 8B NF4 stream: 4 pairs, 256-token shared prompt + 256-token continuations
    "llama8b-nf4-stream-dpo": dict(hidden=4096, n_q_heads=32, n_kv_heads=8, head_dim=128, intermediate=14336,
                                   rank=16, alpha=32.0, vocab=128256, n_layers=32, kind="nf4", tied=False,
                                   batch=8, seq=512, buffers=2, cap_gb=0.0, task="dpo", prompt=256, beta=0.1),
    # the reference-free preference losses on the same stream and pairs
    "llama8b-nf4-stream-simpo": dict(hidden=4096, n_q_heads=32, n_kv_heads=8, head_dim=128, intermediate=14336,
                                     rank=16, alpha=32.0, vocab=128256, n_layers=32, kind="nf4", tied=False,
                                     batch=8, seq=512, buffers=2, cap_gb=0.0, task="simpo", prompt=256, beta=2.0,
                                     gamma=1.0),
    "llama8b-nf4-stream-orpo": dict(hidden=4096, n_q_heads=32, n_kv_heads=8, head_dim=128, intermediate=14336,
                                    rank=16, alpha=32.0, vocab=128256, n_layers=32, kind="nf4", tied=False,
                                    batch=8, seq=512, buffers=2, cap_gb=0.0, task="orpo", prompt=256, lam=0.1),
}
DEFAULT = "llama8b-nf4-stream-sft"
METRIC = "train tokens/s, 8B-shape NF4 streamed LoRA, 1 B200; fused GEMM % bf16 peak"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def gemm_traffic():
    """Per-launch DRAM bytes of the dominant kernel from the committed ncu
    summary (lines "key: value"), if it was taken on the current GEMM source
    (else None)."""
    p = os.path.join(ROOT, "profiles", "gemm_nf4_fwd_traffic.md")
    src = os.path.join(ROOT, "layer_streamed_qlora_b200", "csrc", "gemm.cu")
    if not os.path.exists(p):
        return None
    d = {}
    with open(p) as f:
        for line in f:
            k, sep, v = line.strip().lstrip("-* ").partition(": ")
            if sep and k in ("gemm_cu_sha256", "bytes_per_launch"):
                d[k] = v.strip().strip("`")
    with open(src, "rb") as f:
        h = hashlib.sha256(f.read()).hexdigest()
    if d.get("gemm_cu_sha256") != h or "bytes_per_launch" not in d:
        return None
    return {"bytes_per_launch": float(d["bytes_per_launch"])}


class ClockSampler:
    def __init__(self, dev):
        self.dev = dev
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"soup_bench_clocks_{os.getpid()}_{dev}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,"
                 "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
                 "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                 "clocks_event_reasons.sw_power_cap", "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = max(mx, float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- CPU oracle
HEAD_SAMPLE_TOKENS = 64
HEAD_VOCAB_FRACTION = 8   # the head sample uses 1/8 of the vocab rows; its time scales linearly in V


def oracle_sample_seconds(w, tokens=256, reps=1):
    """Times the CPU oracle (fp64 numpy) on a bounded sample of one step of the
    workload: one decoder layer of its shape, forward + backward for `tokens`
    tokens of one sequence (plus the adapters-off reference forward for DPO);
    the AdamW step over that layer's LoRA factors; and the output head (final
    RMSNorm, logits, log-softmax and dL/dh) for HEAD_SAMPLE_TOKENS tokens over
    1/HEAD_VOCAB_FRACTION of the vocabulary rows.  Weights are random fp64
    (their preparation is not timed).  Returns (layer s, AdamW s, head s)."""
    import numpy as np

    import soup_synth as ss
    from oracle.head import token_logprobs, token_logprobs_bwd
    from oracle.layer import layer_bwd, layer_fwd
    from oracle.optim import adamw_step
    shape = ss.LayerShape(hidden=w["hidden"], n_q_heads=w["n_q_heads"], n_kv_heads=w["n_kv_heads"],
                          head_dim=w["head_dim"], intermediate=w["intermediate"], rank=w["rank"], alpha=w["alpha"])
    g = np.random.default_rng(0)
    W = {p: g.standard_normal(shape.proj_shape(p)) * 0.02 for p in ss.PROJ_NAMES}
    W["norm1"] = 1 + 0.02 * g.standard_normal(shape.hidden)
    W["norm2"] = 1 + 0.02 * g.standard_normal(shape.hidden)
    lora = {}
    for p in ss.PROJ_NAMES:
        o, i = shape.proj_shape(p)
        lora[p] = (g.standard_normal((shape.rank, i)) * 0.02, g.standard_normal((o, shape.rank)) * 0.02)
    moments = {p: [(np.zeros_like(a), np.zeros_like(a)) for a in lora[p]] for p in ss.PROJ_NAMES}
    h = g.standard_normal((1, tokens, shape.hidden))
    dh = g.standard_normal(h.shape)
    Vs = max(1, w["vocab"] // HEAD_VOCAB_FRACTION)
    E = g.standard_normal((Vs, shape.hidden)) * 0.02
    wf = 1 + 0.02 * g.standard_normal(shape.hidden)
    hh = g.standard_normal((1, HEAD_SAMPLE_TOKENS + 1, shape.hidden))
    ids = g.integers(0, Vs, size=(1, HEAD_SAMPLE_TOKENS + 1))
    times, adam, head = [], [], []
    for _ in range(reps):
        t0 = time.perf_counter()
        if w.get("task") == "dpo":  # the adapters-off reference pass of a DPO step
            layer_fwd(h, W, lora, shape, False)
        _, cache = layer_fwd(h, W, lora, shape)
        _, grads = layer_bwd(cache, W, lora, shape, dh)
        t1 = time.perf_counter()
        for p in ss.PROJ_NAMES:
            for j in range(2):
                m, v = moments[p][j]
                adamw_step(lora[p][j], grads[p][j], m, v, 1, 5e-4)
        t2 = time.perf_counter()
        logp, hc = token_logprobs(hh, wf, E, ids, 1e-5)
        token_logprobs_bwd(hc, wf, E, ids, np.full(logp.shape, -1.0 / logp.size))
        t3 = time.perf_counter()
        times.append(t1 - t0)
        adam.append(t2 - t1)
        head.append(t3 - t2)
    return min(times), min(adam), min(head)


def oracle_seconds_per_token(w, t_layer, t_adam, t_head, tokens):
    """Oracle time per token of the whole step: the layer sample covers
    `tokens` tokens of one layer, the AdamW sample one layer's factors once
    per step of the workload's batch * seq tokens (both times the layer
    count), the head sample HEAD_SAMPLE_TOKENS tokens over
    1/HEAD_VOCAB_FRACTION of the vocabulary."""
    return ((t_layer / tokens + t_adam / (w["batch"] * w["seq"])) * w["n_layers"] +
            t_head * HEAD_VOCAB_FRACTION / HEAD_SAMPLE_TOKENS)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=os.cpu_count())
    except Exception:
        return os.cpu_count()


def _sample_text(w, tokens, t=None, ta=None, th=None):
    ref = "reference fwd + " if w.get("task") == "dpo" else ""
    tt = (lambda x: f" ({x:.2f} s)" if x is not None else "")
    return (f"one {w['hidden']}-hidden decoder layer, {ref}fwd+bwd on 1x{tokens} tokens{tt(t)}, the AdamW step of "
            f"its LoRA factors{tt(ta)}, and the output head (final norm, logits, log-softmax, dL/dh) on "
            f"{HEAD_SAMPLE_TOKENS} tokens x {w['vocab'] // HEAD_VOCAB_FRACTION} vocab rows{tt(th)}, fp64 numpy; "
            f"projected to the {w['n_layers']}-layer, {w['vocab']}-vocab step of {w['batch'] * w['seq']} tokens")


def cpu_baseline(w, tokens=256):
    t, ta, th = oracle_sample_seconds(w, tokens)
    per_token_stack = oracle_seconds_per_token(w, t, ta, th, tokens)
    return {"value": 1.0 / per_token_stack, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": _sample_text(w, tokens, t, ta, th)}


def bench_config(w, name, world, kept_layers=None, saved_layers=None, recompute=None):
    cfg = {"workload": name, "global_batch": w["batch"] * world, "seq_len": w["seq"], "layers": w["n_layers"],
           "base": w["kind"], "stream_buffers": w["buffers"], "device_cap_gb": w["cap_gb"],
           "device_cap_bytes": int(w["cap_gb"] * (1 << 30)),
           "parallelism": f"dp{world}" if world > 1 else "single",
           "l2": "inputs larger than L2 (the streamed base, >4 GB per step)",
           "optimizer": "AdamW on the LoRA adapters every step (lr 5e-4, fp32 master + moments)"}
    if kept_layers is not None:
        cfg["kept_qkv_layers"] = kept_layers
    if saved_layers is not None:
        cfg["saved_layers"] = saved_layers
    if recompute is not None:
        cfg["stream_recompute"] = recompute
    return cfg


def run_reference(args, w, name):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    tokens = 256
    for _ in range(args.warmup):  # untimed warm-up samples
        oracle_sample_seconds(w, tokens)
    per, sample_s = [], []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        t, ta, th = oracle_sample_seconds(w, tokens)
        sample_s.append(time.perf_counter() - t0)
        per.append(oracle_seconds_per_token(w, t, ta, th, tokens))
    per_token = statistics.median(per)
    value = 1.0 / per_token
    step_tokens = w["batch"] * w["seq"]
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup,
            # what was actually timed per step (the bounded sample, incl. its
            # untimed weight preparation); the full step is a projection
            "ms_per_step": statistics.median(sample_s) * 1e3,
            "ms_per_step_kind": "wall time of one bounded oracle sample (the timed work of a step of this arm)",
            "projected_ms_per_full_step": per_token * step_tokens * 1e3,
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": bench_config(w, name, args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": "per step: " + _sample_text(w, tokens)},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
# Launch mix of the forward fused NF4 GEMM (one A operand) per layer and
# step: the forward pass runs o, gate|up and down, the recompute o and
# gate|up again; q|k|v (kept from the forward pass) takes a hi + lo A pair,
# another kernel.
PROBE_WEIGHTS = {"qkv": 0, "o": 2, "gate_up": 2, "down": 1}


def probe_shapes(w):
    H, I = w["hidden"], w["intermediate"]
    qkv = (w["n_q_heads"] + 2 * w["n_kv_heads"]) * w["head_dim"]
    return {"qkv": (qkv, H), "o": (H, w["n_q_heads"] * w["head_dim"]), "gate_up": (2 * I, H), "down": (H, I)}


def run_probe_gemm(w):
    """The fused NF4 GEMMs of each projection shape of the workload's layer at
    its token count (random NF4 weights, LoRA r), in the order of
    PROBE_WEIGHTS: per shape a warm-up pass, then one forward (W) and one
    backward (W^T) launch of the fused kernel; an ncu capture of
    `gemm_pair_persistent` with -c 16 lists, per shape, warm-up W, warm-up
    W^T, W, W^T."""
    import torch

    from layer_streamed_qlora_b200 import _lib as L
    T, r = w["batch"] * w["seq"], w["rank"]
    g = torch.Generator(device="cuda").manual_seed(7)
    for name, (N, K) in probe_shapes(w).items():
        W = torch.randn(N, K, device="cuda", generator=g) * 0.02
        codes = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
        absmax = torch.empty((N, K // 64), dtype=torch.float32, device="cuda")
        flag = torch.zeros(1, dtype=torch.int32, device="cuda")
        L.soup_nf4_quantize(W, codes, absmax, flag)
        del W
        wt = L.weight_nf4(codes, absmax, N, K)
        x = torch.randn(T, K, device="cuda", generator=g).bfloat16()
        A = (torch.randn(r, K, device="cuda", generator=g) * 0.02).bfloat16()
        Bm = (torch.randn(N, r, device="cuda", generator=g) * 0.02).bfloat16()
        y = torch.empty(T, N, dtype=torch.bfloat16, device="cuda")
        u = torch.empty(r, T, dtype=torch.bfloat16, device="cuda")
        dy = torch.randn(T, N, device="cuda", generator=g).bfloat16()
        dx = torch.empty(T, K, dtype=torch.bfloat16, device="cuda")
        dA = torch.empty(r, K, device="cuda")
        dB = torch.empty(N, r, device="cuda")
        ws = torch.empty(L.soup_lora_linear_bwd_workspace(T, r, N), dtype=torch.uint8, device="cuda")
        for _ in range(2):
            L.soup_lora_linear_fwd(wt, A, Bm, r, w["alpha"] / r, x, T, y, u)
            L.soup_lora_linear_bwd(wt, A, Bm, r, w["alpha"] / r, x, u, dy, T, dx, dA, dB, ws)
        torch.cuda.synchronize()
        print(f"probe {name}: N={N} K={K} T={T}", flush=True)
    assert L.device_error() == 0
    print(json.dumps({"probe": "fused NF4 GEMMs (W and W^T)", "weights": PROBE_WEIGHTS}))
    return 0


def run_probe_attention(w, reps=20):
    """Times the attention kernels alone (soup_attention_fwd / _bwd, CUDA
    events on the launching stream, after warm-up) at the workload's shape and
    at one 2048-token sequence, random fp16 q|k|v and dO; prints one JSON
    line per shape with TFLOP/s (algorithmic: 4 B Hq d S(S+1)/2 forward, 2.5x
    that backward)."""
    import torch

    from layer_streamed_qlora_b200 import _lib as L
    Hq, Hkv, d = w["n_q_heads"], w["n_kv_heads"], w["head_dim"]
    g = torch.Generator(device="cuda").manual_seed(11)
    for B, S in ((w["batch"], w["seq"]), (1, 2048)):
        T = B * S
        qkv = torch.randn(T, (Hq + 2 * Hkv) * d, device="cuda", generator=g).half()
        dout = torch.randn(T, Hq * d, device="cuda", generator=g).half()
        out = torch.empty(T, Hq * d, device="cuda", dtype=torch.bfloat16)
        out16 = torch.empty(T, Hq * d, device="cuda", dtype=torch.float16)
        lse = torch.empty(Hq, T, device="cuda")
        D = torch.empty(Hq, T, device="cuda")
        dqkv = torch.empty(T, (Hq + 2 * Hkv) * d, device="cuda", dtype=torch.bfloat16)
        fl = 4.0 * B * Hq * d * S * (S + 1) / 2
        res = {"probe": "attention", "batch": B, "seq": S, "n_q_heads": Hq, "n_kv_heads": Hkv}
        for name, fn, flops in (("fwd", lambda: L.soup_attention_fwd(qkv, B, S, Hq, Hkv, out, out16, lse), fl),
                                ("bwd", lambda: L.soup_attention_bwd(qkv, B, S, Hq, Hkv, out16, dout, lse, D, dqkv),
                                 2.5 * fl)):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                fn()
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / reps
            res[name] = {"ms": ms, "TFLOP/s": flops / (ms / 1e3) / 1e12}
        print(json.dumps(res), flush=True)
    assert L.device_error() == 0
    return 0


def spawn_ranks(args):
    """`--gpus N` without a launcher: starts N copies of this command, one
    process per GPU with RANK / LOCAL_RANK / WORLD_SIZE / MASTER_* set (the
    environment torchrun gives), and returns the first nonzero exit code.
    Rank 0 prints the JSON line."""
    import socket
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    procs = []
    for r in range(args.gpus):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(args.gpus),
                   LOCAL_WORLD_SIZE=str(args.gpus), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        env.setdefault("NCCL_DEBUG", "INFO")       # the communicator log (NVLS / transport choice)
        env.setdefault("NCCL_DEBUG_SUBSYS", "INIT")
        procs.append(subprocess.Popen([sys.executable, os.path.abspath(__file__)] + sys.argv[1:], env=env))
    rc = 0
    for pr in procs:
        c = pr.wait()
        rc = rc or c
    return rc


def run_dist_check(args):
    """Launcher check without a GPU workload: every rank joins the process
    group (backend --backend), all-reduces its rank + 1, and rank 0 prints
    the ranks that took part."""
    import datetime

    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1:
        dist.init_process_group(args.backend, timeout=datetime.timedelta(seconds=60))
    t = torch.tensor([float(rank + 1), 1.0])
    if world > 1:
        dist.all_reduce(t)
    if rank == 0:
        print(json.dumps({"dist_check": True, "n_gpus": world, "ranks_joined": int(t[1]),
                          "rank_sum": float(t[0]), "backend": args.backend if world > 1 else None}), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def h2d_link_probe(torch, nbytes=512 << 20, reps=3):
    """Host-link peak for the copy stream's roofline: pinned host -> device
    copies of `nbytes`, as one copy on one stream and split in halves over two
    streams (as the slot ring copies), best of `reps`, GB/s."""
    src = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    half = nbytes // 2
    out = {}
    for name, split in (("one_stream", False), ("two_streams", True)):
        best = 0.0
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            a.record(s1)
            with torch.cuda.stream(s1):
                dst[:half if split else nbytes].copy_(src[:half if split else nbytes], non_blocking=True)
            if split:
                s2.wait_event(a)
                with torch.cuda.stream(s2):
                    dst[half:].copy_(src[half:], non_blocking=True)
                s1.wait_stream(s2)
            b.record(s1)
            torch.cuda.synchronize()
            best = max(best, nbytes / (a.elapsed_time(b) / 1e3) / 1e9)
        out[name] = best
    del src, dst
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default=DEFAULT, choices=sorted(WORKLOADS))
    ap.add_argument("--buffers", type=int, default=0, help="override stream_buffers (2..8)")
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (diagnostics only)")
    ap.add_argument("--source", default="ram", choices=["ram", "disk"],
                    help="stream_source: layer shards in pinned RAM, or files read ahead from disk")
    ap.add_argument("--shard-dir", default="", help="directory for the disk tier's shard files (default: a temp dir)")
    ap.add_argument("--read-ahead", type=int, default=2, help="stream_read_ahead for the disk tier (1..8)")
    ap.add_argument("--recompute", default="auto", choices=["auto", "recompute", "keep"],
                    help="stream_recompute: keep activations for the backward as the cap admits (auto), keep none, "
                         "or keep every layer's")
    ap.add_argument("--no-prompt-dedup", action="store_true",
                    help="preference workloads: lay out both sequences of a pair in full instead of storing and "
                         "computing their shared prompt once")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--probe-gemm", action="store_true",
                    help="run each forward fused NF4 GEMM shape of one layer twice and exit (for an ncu capture)")
    ap.add_argument("--probe-attention", action="store_true",
                    help="time the attention kernels alone at the workload's shape and at seq 2048, and exit")
    ap.add_argument("--dist-check", action="store_true",
                    help="only join the process group of --gpus ranks and report them (launcher check)")
    ap.add_argument("--backend", default="nccl", choices=["nccl", "gloo"],
                    help="process-group backend (gloo: CPU launcher checks)")
    args = ap.parse_args()
    w = dict(WORKLOADS[args.workload])
    if args.buffers:
        w["buffers"] = args.buffers
    if args.layers:
        w["n_layers"] = args.layers
    if args.impl == "reference":
        return run_reference(args, w, args.workload)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return spawn_ranks(args)
    if args.dist_check:
        return run_dist_check(args)
    if args.probe_gemm:
        return run_probe_gemm(w)
    if args.probe_attention:
        return run_probe_attention(w)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group(args.backend, timeout=datetime.timedelta(seconds=120))
    from layer_streamed_qlora_b200 import _lib as L
    from layer_streamed_qlora_b200.model import ModelConfig, StreamedLoRAModel

    cfg = ModelConfig(hidden=w["hidden"], n_q_heads=w["n_q_heads"], n_kv_heads=w["n_kv_heads"],
                      head_dim=w["head_dim"], intermediate=w["intermediate"], rank=w["rank"], alpha=w["alpha"],
                      vocab=w["vocab"], n_layers=w["n_layers"], kind=w["kind"], tied=w["tied"])
    B, S = w["batch"], w["seq"]
    cap = int(w["cap_gb"] * (1 << 30))
    torch.cuda.init()
    L.lib()
    torch.cuda.synchronize()
    free0, total_dev = torch.cuda.mem_get_info()
    torch.cuda.reset_peak_memory_stats()
    t_build = time.time()
    shard_dir = None
    if args.source == "disk":
        import tempfile
        shard_dir = args.shard_dir or tempfile.mkdtemp(prefix="soup_shards_")
    model = StreamedLoRAModel(cfg, B, S, n_buffers=w["buffers"], device_cap_bytes=cap, seed=0, task=w["task"],
                              stream_source=args.source, shard_dir=shard_dir, read_ahead=args.read_ahead,
                              stream_recompute=args.recompute,
                              prompt_dedup=0 if (w["task"] == "sft" or args.no_prompt_dedup) else w["prompt"])
    t_build = time.time() - t_build
    g = torch.Generator().manual_seed(1000 + rank)
    ids_host = torch.randint(0, cfg.vocab, (B, S), generator=g, dtype=torch.int32)
    if w["task"] != "sft":  # preference pairs: rows 2p, 2p+1 share their prompt
        ids_host[1::2, :w["prompt"]] = ids_host[0::2, :w["prompt"]]
    ids_host = ids_host.pin_memory()
    loss_host = torch.zeros(1, dtype=torch.float32).pin_memory()
    model.set_ids(ids_host)
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    from layer_streamed_qlora_b200 import dp

    def step():
        task = w["task"]
        if task == "sft":
            loss = model.sft_step()
        elif task == "dpo":
            loss = model.dpo_step(w["prompt"], w["beta"])
        elif task == "simpo":
            loss = model.simpo_step(w["prompt"], w["beta"], w["gamma"])
        else:
            loss = model.orpo_step(w["prompt"], w["lam"])
        # data parallel: the one exchange of the step, the LoRA gradients
        # summed in place (a no-op on one rank); the optimiser step takes the
        # mean's 1/world as its gradient scale
        world_ = dp.allreduce_sum_(model.grad_flat)
        model.optimizer_step(grad_scale=1.0 / world_)
        return loss

    loss0 = None
    for i in range(max(3, args.warmup)):
        lo = step()
        if i == 0:  # the untrained step's loss (about ln(vocab) for SFT on random ids)
            loss0 = float(lo.item())
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    model.plan.reset_stats()
    torch.cuda.reset_peak_memory_stats()
    clocks = ClockSampler(local)
    clocks.start()
    n0 = L.launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(st)
    for i in range(args.steps):
        if i == 0:  # NVTX range: lets an ncu launch list capture exactly one step
            torch.cuda.nvtx.range_push("soup_step")
        step()
        if i == 0:
            torch.cuda.nvtx.range_pop()
    e1.record(st)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = e0.elapsed_time(e1) / args.steps
    launches = (L.launch_count() - n0) // args.steps
    sstats = model.plan.stats()
    clk = clocks.stop()
    free_after, _ = torch.cuda.mem_get_info()
    peak_alloc = torch.cuda.max_memory_allocated()
    reserved = torch.cuda.memory_reserved()
    # the dominant kernel class event-timed over a second run of the same K
    # steps (the timed region above runs uninstrumented), with its own clocks
    dom_mask = 0b00001 if cfg.kind == "nf4" else 0b00100
    clocks2 = ClockSampler(local)
    clocks2.start()
    L.profile_enable(dom_mask)
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize()
    prof = L.profile_read()
    L.profile_enable(0)
    clk2 = clocks2.stop()
    # per-class breakdown of every profiled kernel class from one extra step
    L.profile_enable(L.PROFILE_ALL)
    step()
    torch.cuda.synchronize()
    prof_all = L.profile_read()
    L.profile_enable(0)

    # end-to-end through the public API: host ids in, loss out, every step
    torch.cuda.synchronize()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(st)
    for _ in range(args.steps):
        model.set_ids(ids_host)
        loss = step()
        loss_host.copy_(loss, non_blocking=True)
        st.synchronize()
    e3.record(st)
    torch.cuda.synchronize()
    ms_e2e = e2.elapsed_time(e3) / args.steps
    if world > 1:
        t = torch.tensor([ms, ms_e2e], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms, ms_e2e = float(t[0]), float(t[1])
    tokens = B * S * world
    value = tokens / (ms / 1e3)
    pk, pk_kind = peaks()
    # dominant kernel: the GEMM class with the most device time
    dom_name, dom = max(((k, v) for k, v in prof.items() if v["launches"]), key=lambda kv: kv[1]["total_ms"])
    achieved = dom["flops"] / (dom["total_ms"] / 1e3) / 1e12 if dom["total_ms"] > 0 else 0.0
    burst = pk.get("bf16_tflops")
    sustained = pk.get("bf16_tflops_sustained", burst)
    tr = gemm_traffic() if dom_name == "nf4_fwd" else None
    roofline = {"bound": "tensor", "kernel": f"gemm {dom_name}", "achieved": achieved, "peak": burst,
                "unit": "TFLOP/s", "frac": achieved / burst if burst else None,
                "traffic": tr.get("bytes_per_launch") if tr else None,
                "peak_kind": f"{pk_kind} burst bf16 (cuBLAS, clock-comparable: this step ran at "
                             f"{clk2['sm_mhz'] if clk2 else 'unsampled'} MHz)",
                "frac_vs_sustained": achieved / sustained if sustained else None,
                "sustained_peak": sustained,
                "sustained_peak_note": "measured in a seconds-long loop under the power cap "
                                       f"(clocks under load: {pk.get('clocks_under_load', 'not recorded')})",
                "timing": "CUDA events around each launch of the class on its stream, over a second run of "
                          "the K timed steps (the timed region itself runs uninstrumented)",
                "sm_mhz_during": clk2["sm_mhz"] if clk2 else None,
                "launches_per_step": dom["launches"] // args.steps,
                "algorithmic_flops_per_launch": dom["flops"] / max(1, dom["launches"]),
                "avg_launch_ms": dom["total_ms"] / max(1, dom["launches"])}
    hbm = pk.get("hbm_gbs")
    kernel_classes = {}
    for k, v in prof_all.items():
        if not v["launches"]:
            continue
        sec = v["total_ms"] / 1e3
        e = {"launches_per_step": v["launches"], "ms_per_step": v["total_ms"]}
        if v["flops"] > 0 and sec > 0:
            e["TFLOP/s"] = v["flops"] / sec / 1e12
        if v["bytes"] > 0 and sec > 0:
            e["GB/s"] = v["bytes"] / sec / 1e9
            if k in L.HBM_CLASSES and hbm:
                e["frac_of_hbm"] = e["GB/s"] / hbm
        kernel_classes[k] = e
    h2d_bytes = sstats["bytes_copied"] / args.steps
    copy_ms = sstats["copy_ms"] / args.steps
    step_flops = sum(v["flops"] for k, v in prof_all.items() if k in L.GEMM_CLASSES)
    link = h2d_link_probe(torch)
    h2d_gbs = (h2d_bytes / 1e9) / (copy_ms / 1e3) if copy_ms > 0 else None
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(bench_config(w, args.workload, world, sum(1 for k in model.keep_plan if k == "qkv"),
                                    sum(1 for k in model.keep_plan if k == "saved"), args.recompute),
                       token_rows_per_step=model.T, prompt_dedup=model.prompt_dedup,
                       head_chunk=model.head_chunk, stream_source=args.source,
                       **({"read_ahead": args.read_ahead} if args.source == "disk" else {})),
        "e2e": {"value": tokens / (ms_e2e / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": ids_host.numel() * 4,
                "d2h_bytes_per_step": 4},
        "gpu_launches": launches,
        "roofline": roofline,
        "kernel_classes": kernel_classes,
        "kernel_classes_note": "one extra step with every profiled launch event-timed (not the timed region); "
                               "GB/s = algorithmic bytes (each operand read once, each output written once)",
        "stream": {"h2d_gb_per_step": h2d_bytes / 1e9, "copies_per_step": sstats["copies"] / args.steps,
                   "reused_per_step": sstats["reuses"] / args.steps,
                   "h2d_gbs": h2d_gbs, "h2d_link_peak_gbs": link,
                   "h2d_frac_of_link": (h2d_gbs / link["two_streams"]) if h2d_gbs and link["two_streams"] else None,
                   "copy_ms_per_step": copy_ms, "stall_ms_per_step": sstats["stall_ms"] / args.steps,
                   "stall_frac": (sstats["stall_ms"] / args.steps) / ms},
        "gemm_tflops_per_step": step_flops / (ms / 1e3) / 1e12,
        "disk": model.disk.stats() if model.disk is not None else None,
        "peak_device_bytes": peak_alloc + sstats["arena_bytes"] + L.static_device_bytes(),
        "device_bytes": {"torch_peak_allocated": peak_alloc, "torch_reserved": reserved,
                         "slot_arena": sstats["arena_bytes"], "library_static": L.static_device_bytes(),
                         "mem_get_info_delta": free0 - free_after,
                         "note": "mem_get_info_delta = free device memory before the model was built minus after "
                                 "the timed steps (includes allocator slack and module loading)"},
        "build_s": t_build,
        "loss_step0": loss0,
        "loss": float(loss_host.item()),
    }
    if clk:
        line["clocks"] = clk
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    model.close()
    if shard_dir and not args.shard_dir:
        import shutil
        shutil.rmtree(shard_dir, ignore_errors=True)
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
