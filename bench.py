#!/usr/bin/env python
"""Throughput of the GPT-2 124M training step on B200.

One step = one optimizer step of the pages' headline workload: micro-batch B=16, T=1024,
32 gradient-accumulation micro-steps (524,288 tokens, loss / 32), then the global-norm
clip and AdamW at lr = get_lr(1000).  Token streams are seeded synthetic Zipf(1.1) ids
(the pages' datasets are not available); weights are the random GPT-2 init.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line on rank 0.  With N > 1 (launched by torchrun) every rank trains an
independent replica on its own token stream (the path has no exchange step in this
build), and value = all ranks' tokens / the slowest rank's device time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GPT-2 124M train tokens/sec (B=16,T=1024, 1 B200); ms/step; MFU vs BF16 peak"
# the headline model and the medium one (GPT-2 350M shape: 24 layers, 1024 channels, 16 heads)
MODELS = {"124m": dict(n_layer=12, n_embd=768, n_head=12, label="GPT-2 124M", micro_batch=16, accum=32),
          "medium": dict(n_layer=24, n_embd=1024, n_head=16, label="GPT-2 medium (L=24, C=1024, H=16)",
                         micro_batch=8, accum=8)}


def flop_per_token(model: str, T: int = 1024, Vp: int = 50304) -> int:
    """Training FLOPs per token: 6 (12 L C^2 + Vp C) for the matrix products (pad columns
    counted) plus 6 L T C for the causal attention products."""
    m = MODELS[model]
    L, C = m["n_layer"], m["n_embd"]
    return 6 * (12 * L * C * C + Vp * C) + 6 * L * T * C


FLOP_PER_TOKEN = flop_per_token("124m")   # 798,031,872


def metric_name(model: str, B: int = 16, T: int = 1024) -> str:
    if model == "124m" and (B, T) == (16, 1024):
        return METRIC
    return f"{MODELS[model]['label']} train tokens/sec (B={B},T={T}, 1 B200); ms/step; MFU vs BF16 peak"
NOMINAL_BF16_TFLOPS = 2250.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--model", default="124m", choices=sorted(MODELS),
                    help="124m: the headline workload; medium: the 24-layer, 1024-channel model")
    ap.add_argument("--micro-batch", type=int, default=None)
    ap.add_argument("--seq", type=int, default=1024)
    ap.add_argument("--accum", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--ddp", action="store_true",
                    help="data-parallel instead of independent replicas: the ranks split each optimizer step's "
                         "micro-steps and average the gradients with one all-reduce before AdamW")
    args = ap.parse_args()
    m = MODELS[args.model]
    # the 124M model at a longer context takes the pages' GPT-3 batch ("3:41:50 – 3:53:37" of the
    # Lecture 9 notes: T = 2048 with B = 32), at most 131072 positions per micro-step; the step
    # keeps its tokens (T = 2048: B = 32, 8 micro-steps of 65,536 tokens)
    if args.micro_batch is None:
        b = 32 if (args.model == "124m" and args.seq > 1024) else m["micro_batch"]
        args.micro_batch = max(1, min(b, 131072 // args.seq))
    if args.accum is None:
        args.accum = max(1, m["micro_batch"] * m["accum"] * 1024 // (args.micro_batch * args.seq))
    return args


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def recorded_traffic(cls: str):
    """DRAM bytes per call of a profiler class, from the ncu launch-list summaries under
    profiles/: (bytes, note).  A figure counts only while the kernel sources it lists still
    hash to the recorded SHA-256; a changed kernel gives (None, reason)."""
    import glob
    import hashlib
    import re
    pat = re.compile(r"<!-- traffic (\w+) bytes_per_call=(\d+) sources=([\w./,]+) sha256=([0-9a-f]{64}) -->")
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        for m in pat.finditer(open(path).read()):
            if m.group(1) != cls:
                continue
            h = hashlib.sha256()
            for f in m.group(3).split(","):
                h.update(open(os.path.join(ROOT, "decoder_only_transformer_train_b200", f), "rb").read())
            name = os.path.basename(path)
            if h.hexdigest() != m.group(4):
                return None, f"{name}: kernel sources changed since the capture"
            return int(m.group(2)), f"{name}: dram__bytes_read.sum + dram__bytes_write.sum per call"
    return None, "no capture recorded"


# ------------------------------------------------------------------ clocks sampling
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        pw = [v for v in (num(r[3]) for r in rows) if v is not None]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "power_w_median": statistics.median(pw) if pw else None, "power_w_max": max(pw) if pw else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ distributed plumbing
def ddp_shape(args, world: int):
    """Data-parallel runs keep the optimizer step's tokens: the accumulation micro-steps are
    split across the ranks ("2:59:25 – 3:10:20 Synchronizing gradients and losses" of the
    Lecture 9 notes: each rank's gradients are averaged once, after its last micro-step)."""
    args.ddp_world = world if (args.ddp and world > 1) else 1
    if args.ddp_world > 1:
        if args.accum % world:
            raise SystemExit(f"--ddp: {args.accum} accumulation micro-steps do not split over {world} ranks")
        args.accum //= world
    return args


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def dist_init(world, backend):
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))


def dist_max(x: float, world: int, device, op: str = "max") -> float:
    """The maximum (or, with op="sum", the sum) of x over the ranks."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def average_gradients(grads, world: int):
    """Data-parallel gradient exchange ("2:46:43 – 2:59:25 Going multi-GPU with DDP" and
    "2:59:25 – 3:10:20 Synchronizing gradients and losses" of the Lecture 9 notes): every
    rank's gradient of its own loss / k_local is replaced, in place, by the mean over the
    ranks, once per optimizer step after the rank's last micro-step.  With k_local micro-steps
    on each of `world` ranks that is the gradient of the global batch's mean loss.  A sum
    followed by one division, so the same code runs on NCCL and on gloo (which has no
    average)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        assert world == 1, "a data-parallel exchange needs a process group"
        return grads
    dist.all_reduce(grads, op=dist.ReduceOp.SUM)
    grads.div_(world)
    return grads


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ CPU oracle baseline
def cpu_oracle_configs():
    """Wall time of the oracle (fp32, as it stands) on the small workloads: the tiny model's
    full step (B=2, T=64: forward, backward, clip, AdamW), the 124M B=1 x T=1024 forward +
    backward on one thread, one 124M step on B=4 x T=1024 on all host threads, the
    classifier-head stress (lm_head + softmax + cross-entropy forward and backward at the
    unpadded vocabulary 50257, timed on 1024 of its 16384 rows and scaled), and the medium
    model's B=1 x T=1024 forward + backward."""
    import torch
    import oracle as O
    from decoder_only_transformer_train_b200 import synthetic as S
    out = {}

    def step(params, cfg, B, T, seed):
        m = {n: torch.zeros_like(t) for n, t in params.items()}
        v = {n: torch.zeros_like(t) for n, t in params.items()}
        x, y = S.token_batch(seed, B, T, cfg.vocab_size)
        t0 = time.perf_counter()
        O.train_step(params, m, v, 1, cfg, [(torch.from_numpy(x), torch.from_numpy(y))], O.get_lr(1000))
        return time.perf_counter() - t0

    out["tiny_step_s"] = round(step(O.init_params(O.TINY, 1, dtype=torch.float32), O.TINY, 2, 64, 2), 4)
    cfg = O.GPT2_124M
    params = O.init_params(cfg, 1, dtype=torch.float32)
    threads = torch.get_num_threads()
    torch.set_num_threads(1)
    try:
        x, y = S.token_batch(3, 1, 1024, cfg.vocab_size)
        t0 = time.perf_counter()
        _, cache = O.forward(params, cfg, torch.from_numpy(x), torch.from_numpy(y))
        O.backward(params, cfg, cache)
        t1 = time.perf_counter() - t0
        del cache
    finally:
        torch.set_num_threads(threads)
    out["gpt2_124m_b1_fwd_bwd_1_thread_s"] = round(t1, 2)
    out["gpt2_124m_tokens_per_s_1_thread"] = round(1024 / t1, 1)
    out["gpt2_124m_b4_step_s"] = round(step(params, cfg, 4, 1024, 2), 2)
    del params
    # classifier head at V=50257: hidden states N(0,1), tied weight N(0,0.02), uniform targets
    # with 1% ignored; 1024 rows of the 16384 (the oracle's cost is linear in the rows)
    g = torch.Generator().manual_seed(7)
    rows, V, C = 1024, 50257, 768
    h = torch.randn(rows, C, generator=g)
    W = torch.randn(V, C, generator=g) * 0.02
    y = torch.randint(0, V, (rows,), generator=g)
    y[torch.rand(rows, generator=g) < 0.01] = O.IGNORE_INDEX
    t0 = time.perf_counter()
    z = h @ W.t()
    _, lse, count = O.cross_entropy_forward(z, y)
    dz = O.cross_entropy_backward(z, y, lse, count, 1.0)
    _ = dz @ W
    _ = dz.t() @ h
    out["c4_classifier_50257_s"] = round((time.perf_counter() - t0) * (16384 / rows), 2)
    out["c4_sample"] = f"{rows} of 16384 rows, scaled"
    del z, dz, W
    mcfg = O.Config(n_layer=24, n_embd=1024, n_head=16)
    mparams = O.init_params(mcfg, 1, dtype=torch.float32)
    x, y = S.token_batch(4, 1, 1024, mcfg.vocab_size)
    t0 = time.perf_counter()
    _, cache = O.forward(mparams, mcfg, torch.from_numpy(x), torch.from_numpy(y))
    O.backward(mparams, mcfg, cache)
    out["c5_medium_b1_fwd_bwd_s"] = round(time.perf_counter() - t0, 2)
    out["threads"] = threads
    return out


def cpu_oracle_sample(seq: int, samples: int = 1, model: str = "124m", seqs_per_step: int = 512):
    """Times the CPU oracle (fp32, as it stands) on B=1 x `seq` tokens of the same model:
    forward + backward per sample, plus one clip + AdamW step amortised over the
    `seqs_per_step` sequences (micro-batch x accumulation steps) of an optimizer step."""
    import torch
    import oracle as O
    from decoder_only_transformer_train_b200 import synthetic as S
    m = MODELS[model]
    cfg = O.Config(n_layer=m["n_layer"], n_embd=m["n_embd"], n_head=m["n_head"], block_size=max(1024, seq))
    params = O.init_params(cfg, 1, dtype=torch.float32)
    x, y = S.token_batch(3, 1, seq, cfg.vocab_size)
    x, y = torch.from_numpy(x), torch.from_numpy(y)
    t0 = time.perf_counter()
    grads = None
    for _ in range(samples):
        _, cache = O.forward(params, cfg, x, y)
        grads = O.backward(params, cfg, cache, grad_scale=1.0 / 32, grads=grads)
        del cache
    t_fb = (time.perf_counter() - t0) / samples
    m = {n: torch.zeros_like(t) for n, t in params.items()}
    v = {n: torch.zeros_like(t) for n, t in params.items()}
    t1 = time.perf_counter()
    O.optimizer_step(params, grads, m, v, 1, cfg, lr=O.get_lr(1000))
    t_opt = time.perf_counter() - t1
    per_micro = t_fb + t_opt / seqs_per_step
    return seq / per_micro, torch.get_num_threads(), t_fb, t_opt


# ------------------------------------------------------------------ reference arm
def run_reference(args, world, rank):
    """The oracle, as it stands, on the host cores: each step is a bounded sample of the
    workload (one B=1 x T sequence forward + backward, plus its share of an optimizer step)."""
    if rank != 0:
        return
    import torch
    tok_s, threads, t_fb, t_opt = None, None, None, None
    rates = []
    for i in range(args.warmup + args.steps):
        r, threads, t_fb, t_opt = cpu_oracle_sample(args.seq, model=args.model,
                                                    seqs_per_step=args.micro_batch * args.accum)
        if i >= args.warmup:
            rates.append(r)
    value = statistics.mean(rates)
    ms = args.micro_batch * args.seq * args.accum / value * 1000.0
    line = {
        "metric": metric_name(args.model, args.micro_batch, args.seq), "impl": "reference", "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        # each timed step is one B=1 sequence plus its share of the optimizer step; ms_per_step
        # is that rate extrapolated to the whole optimizer step, which was not run
        "extrapolated": True, "timed_samples": args.steps,
        "timed_sample": f"B=1 x T={args.seq} forward+backward plus 1/{args.micro_batch * args.accum} of clip+AdamW",
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(args),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"{MODELS[args.model]['label']} fp32 CPU oracle, B=1 x T={args.seq} forward+backward "
                                   f"({t_fb:.2f} s) plus 1/{args.micro_batch * args.accum} of clip+AdamW "
                                   f"({t_opt:.2f} s) per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(args):
    dw = getattr(args, "ddp_world", 1)
    tokens = args.micro_batch * args.seq * args.accum * dw
    steps_txt = f"{args.accum} accumulation micro-steps" + (f" on each of {dw} data-parallel ranks" if dw > 1 else "")
    return {"workload": f"{MODELS[args.model]['label']} training step: B={args.micro_batch} x T={args.seq}, "
                        f"{steps_txt} ({tokens} tokens), global-norm clip 1.0, AdamW at lr=get_lr(1000)",
            "micro_batch": args.micro_batch, "seq_len": args.seq, "grad_accum_steps": args.accum,
            "tokens_per_step": tokens,
            "parallelism": f"ddp{dw}" if dw > 1 else ("replicas" if args.gpus > 1 else "single-gpu"),
            "l2": "inputs larger than L2 (every micro-step moves several GB of parameters and activations)"}


# ------------------------------------------------------------------ our arm
def run_ours(args, world, rank, local):
    import numpy as np
    import torch
    from decoder_only_transformer_train_b200 import binding as BD
    from decoder_only_transformer_train_b200 import synthetic as S

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_init(world, "nccl")
    B, T, k = args.micro_batch, args.seq, args.accum
    mdl = MODELS[args.model]
    cfg = BD.Config(n_layer=mdl["n_layer"], n_embd=mdl["n_embd"], n_head=mdl["n_head"], block_size=max(1024, T),
                    vocab_size=50257, padded_vocab_size=50304,
                    max_batch=B, grad_accum_steps=k, precision=BD.GPT2_BF16)
    stream = torch.cuda.Stream(device)
    model = BD.GPT2(cfg, seed=1, stream=stream.cuda_stream)
    lr = float(BD.lib().gpt2_lr_cosine(1000, 6e-4, 715, 19073, 0.1))
    # each rank its own seeded token stream: k micro-batches of B x T (+1 for the targets)
    run = S.zipf_tokens(3 + rank, k * B * T + 1, 50257)
    x_host = run[:-1].reshape(k, B, T).astype(np.int32)
    y_host = run[1:].reshape(k, B, T).astype(np.int32)
    x_dev = torch.from_numpy(x_host).to(device)
    y_dev = torch.from_numpy(y_host).to(device)
    ddp = getattr(args, "ddp_world", 1) > 1
    grads = model.grad_tensor() if ddp else None

    def grad_sync():
        # data-parallel: every rank's gradient (of its loss / k) averaged across ranks, once
        # per optimizer step, on the model's stream before the clip and AdamW
        if ddp:
            average_gradients(grads, world)

    def step():
        model.zero_grad()
        for i in range(k):
            model.forward(x_dev[i], y_dev[i], sync_loss=False)
            model.backward()
        grad_sync()
        model.adamw_step(lr, sync_norm=False)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize(device)
    first_loss = model.get_loss()

    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize(device)
    launches0 = int(BD.lib().gpt2_kernel_launches())
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            step()
    ev1.record(stream)
    torch.cuda.synchronize(device)
    launches = int(BD.lib().gpt2_kernel_launches()) - launches0
    barrier(world)
    clk = clocks.stop()
    ms_total = ev0.elapsed_time(ev1)
    ms_max = dist_max(ms_total, world, device)
    tokens = world * args.steps * k * B * T
    value = tokens / (ms_max / 1000.0)
    last_loss = model.get_loss()
    if ddp:   # the logged loss is the mean over the ranks, like the gradients
        first_loss = dist_max(first_loss / world, world, device, op="sum")
        last_loss = dist_max(last_loss / world, world, device, op="sum")

    # per-kernel-class event timing of one more step (roofline of the dominant kernel)
    with torch.cuda.stream(stream):
        model.profile_start()
        step()
        prof = model.profile_stop()
    torch.cuda.synchronize(device)

    # end to end through the public API with host buffers: pinned token/target copies in,
    # loss and grad norm out, every step
    e2e = None
    if not args.no_e2e:
        xp = torch.from_numpy(x_host).pin_memory()
        yp = torch.from_numpy(y_host).pin_memory()

        def step_host():
            model.zero_grad()
            for i in range(k):
                model.forward_host(xp[i], yp[i], sync_loss=False)
                model.backward()
            model.get_loss()
            grad_sync()
            return model.adamw_step(lr, sync_norm=True)

        barrier(world)
        torch.cuda.synchronize(device)
        t0 = time.perf_counter()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(args.steps):
                step_host()
        e1.record(stream)
        torch.cuda.synchronize(device)
        wall = time.perf_counter() - t0
        ms_e2e = dist_max(max(e0.elapsed_time(e1), wall * 1000.0), world, device)
        e2e = {"value": tokens / (ms_e2e / 1000.0), "unit": "tokens/s",
               "h2d_bytes_per_step": int(2 * k * B * T * 4), "d2h_bytes_per_step": 8}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r, threads, t_fb, t_opt = cpu_oracle_sample(T, model=args.model, seqs_per_step=B * k)
        cpu = {"value": r, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"{MODELS[args.model]['label']} fp32 CPU oracle, B=1 x T={T} forward+backward ({t_fb:.2f} s) plus "
                         f"1/{B * k} of clip+AdamW ({t_opt:.2f} s)"}
        if args.model == "124m" and T == 1024:
            cpu["other_workloads"] = cpu_oracle_configs()

    if rank == 0:
        pk = peaks()
        tensor_classes = ("gemm_fwd", "gemm_bwd", "lm_head_fwd", "lm_head_bwd", "attn_fwd", "attn_bwd")
        dom = max(prof, key=lambda c: prof[c]["ms"])
        d = prof[dom]
        if dom in tensor_classes:
            achieved = d["flops"] / (d["ms"] / 1e3) / 1e12
            peak = pk["bf16_tflops_sustained"]
            roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": None, "kernel": dom,
                    "launches": d["launches"], "avg_launch_ms": d["ms"] / max(1, d["launches"]),
                    "peak_kind": f"{pk['source']} sustained dense bf16"}
        else:
            achieved = d["bytes"] / (d["ms"] / 1e3) / 1e9
            peak = pk["hbm_gbs"]
            roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                    "traffic": None, "kernel": dom, "launches": d["launches"],
                    "avg_launch_ms": d["ms"] / max(1, d["launches"]), "peak_kind": f"{pk['source']} HBM copy"}
        roof["traffic"], roof["traffic_note"] = recorded_traffic(dom)
        step_ms = sum(p["ms"] for p in prof.values())
        kernels = {}
        for c, p in prof.items():
            if p["launches"] == 0:
                continue
            ent = {"ms": round(p["ms"], 3), "share": round(p["ms"] / step_ms, 4), "launches": p["launches"]}
            if p["flops"] > 0:
                ent["tflops"] = round(p["flops"] / (p["ms"] / 1e3) / 1e12, 1)
            if p["bytes"] > 0:
                ent["gbs"] = round(p["bytes"] / (p["ms"] / 1e3) / 1e9, 1)
            kernels[c] = ent
        per_gpu = value / world
        fpt = flop_per_token(args.model, args.seq)
        line = {
            "metric": metric_name(args.model, args.micro_batch, args.seq), "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "strong" if ddp else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(args),
            "mfu": {"vs_nominal_2250": per_gpu * fpt / (NOMINAL_BF16_TFLOPS * 1e12),
                    "vs_measured_sustained": per_gpu * fpt / (pk["bf16_tflops_sustained"] * 1e12),
                    "flop_per_token": fpt},
            "roofline": roof, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
            "clocks": clk, "gpu_launches": launches,
            "loss": {"after_warmup": first_loss, "after_timed": last_loss},
        }
        print(json.dumps(line), flush=True)
    del grads
    model.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    args = parse()
    world, rank, local = dist_setup()
    if world > 1:
        args.gpus = world
    ddp_shape(args, world)
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
