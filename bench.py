#!/usr/bin/env python
"""Throughput of the Llama training step (forward + backward + AdamW) on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

Default workload: the ~350M-parameter decoder (vocab 32000, d_model 1024, 20
layers, 16 heads, SwiGLU 2730, context 2048, batch 8 = 16384 tokens per step),
bf16 compute with fp32 master weights, synthetic Zipf(1.1) tokens.  Prints one
JSON line on rank 0.

Our arm: W untimed steps, then K steps timed with CUDA events on the
library's stream, bracketed by a barrier and a synchronize, max over ranks.
The library runs on its own stream, where llm_step captures the step into a
CUDA graph on its second call and replays it afterwards (the warm-up steps
include the capture).
With N > 1 GPUs every rank runs an independent replica on its own batch
(weak scaling; no gradient exchange is part of the timed step), or, with
--dp allreduce|overlap|sharded|sharded-overlap, one model trained
data-parallel: the same weights on every rank, each rank's own batch, and the
NCCL gradient exchange (one all-reduce, one per layer bucket overlapped with
the backward, reduce-scatter + sharded AdamW + all-gather, or that per bucket
overlapped with the backward) inside every timed step.
The roofline object is for the dominant kernel (the tcgen05 GEMM): its
algorithmic FLOPs over the summed device time of its launches, taken with CUDA
events around every GEMM launch over K more steps run right after the timed
region as individual launches (events cannot time nodes of a replayed graph;
the kernels are the same).  e2e repeats the timed loop through the same C ABI
with the step's tokens and targets copied from pinned host memory each step
and the loss read back each step (one step in flight: the host reads step i's
loss after launching step i + 1).  cpu_baseline times the float64 CPU oracle
on a bounded sample of the same workload.

Decode (--decode): generation throughput of the same workload's model with a
key/value cache: a forward over the whole context (the prefill), then K timed
llm_decode steps at positions --pos, --pos + 1, ... (each step one new position
for every sequence, the weights and every cached key/value row up to it read
once); value = sequences x K / time.  Its roofline is HBM bytes per step
(bf16 weights, K/V rows read, K/V row and logits written) over the step's time
against the measured copy bandwidth; e2e adds top-k sampling with the
token ids and uniforms copied from pinned host memory and the sampled ids read
back every step; cpu_baseline is the float64 oracle decoding one sequence.

Reference arm (--impl reference): the float64 CPU oracle, each step a fixed
fraction of the workload (a token prefix of one sequence, forward and
backward, plus AdamW over the same fraction of the parameters), scaled to
tokens/s of the full step; rank 0 only.
"""
import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "training tokens/sec (fwd+bwd+AdamW) on 1 B200; % of tensor/HBM roofline"
# DRAM bytes (read + write) per tcgen05 GEMM launch, averaged over the 243
# GEMM launches of one 350M step (profiles/gemm_dram_traffic_step_350m.md);
# valid only for the GEMM sources that were captured, identified by hash.
GEMM_TRAFFIC = {"bytes_per_launch": 178.3e6, "workload": "350m-v32000-d1024-l20-bf16",
                "sha256": {"gemm_tc.cu": "8a92a32c71372280371fe8dfc5e064b978fc84dc97facb3787daa2a1bfb0cb36",
                           "tcgen05.cuh": "3ec0ac326a7fbd3690692656fd8581d42175193edc7eb03dbfaf27afa97b1c4a"}}


def gemm_traffic(workload):
    """The captured GEMM traffic per launch if the GEMM sources are unchanged
    since the capture and the workload is the captured one, else None."""
    import hashlib
    if workload != GEMM_TRAFFIC["workload"]:
        return None
    for name, want in GEMM_TRAFFIC["sha256"].items():
        path = os.path.join(ROOT, "scratch_llama_decoder_b200", "csrc", name)
        try:
            with open(path, "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != want:
                    return None
        except OSError:
            return None
    return GEMM_TRAFFIC["bytes_per_launch"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="c5")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the other workloads' step timings (per_config)")
    ap.add_argument("--kernel", default=None, choices=["gemm", "attention"],
                    help="time one hot-path kernel through the C ABI instead of the step")
    ap.add_argument("--shape", default="16384,3072,1024",
                    help="gemm: M,N,K; attention: batch,ctx,n_head,n_kv_head,head_dim")
    ap.add_argument("--fwd-impl", type=int, default=2, choices=[0, 1, 2],
                    help="attention forward kernels: 2 tcgen05, 1 mma, 0 CUDA cores")
    ap.add_argument("--bwd-impl", type=int, default=2, choices=[0, 1, 2],
                    help="attention backward kernels: 2 tcgen05, 1 mma, 0 CUDA cores")
    ap.add_argument("--decode", action="store_true",
                    help="time llm_decode (KV-cache generation) instead of the training step")
    ap.add_argument("--pos", type=int, default=1024, help="first decoded position (--decode)")
    ap.add_argument("--orient", default="kn", choices=["kn", "kk", "nn"],
                    help="gemm operand majorness: kn = x.W (forward), kk = dy.W^T (dgrad), "
                         "nn = x^T.dy (wgrad)")
    # options of the training step (defaults: the step as benchmarked)
    ap.add_argument("--clip", type=float, default=0.0,
                    help="gradient clipping threshold (0: off)")
    ap.add_argument("--clip-mode", default="l2", choices=["l2", "linf"])
    ap.add_argument("--dropout", type=float, default=0.0, help="inverted dropout rate")
    ap.add_argument("--rope-scale", type=float, default=1.0,
                    help="RoPE position interpolation factor")
    ap.add_argument("--recompute", action="store_true",
                    help="keep only layer inputs; recompute activations in the backward")
    ap.add_argument("--ctx", type=int, default=None, help="override the context length")
    ap.add_argument("--batch", type=int, default=None, help="override the batch")
    ap.add_argument("--dp", default="none",
                    choices=["none", "allreduce", "overlap", "sharded", "sharded-overlap"],
                    help="with --gpus N > 1: one model trained data-parallel (gradient "
                         "all-reduce, the same per layer bucket overlapped with the backward, a "
                         "sharded optimiser, or that sharded optimiser with per-bucket "
                         "reduce-scatters overlapped with the backward) instead of N independent "
                         "replicas")
    return ap.parse_args(argv)


def step_options(args):
    """(config overrides, options applied to the context, label suffix) of the
    step's options; empty for the step as benchmarked."""
    over, opts = {}, {}
    if args.ctx is not None:
        over["ctx"] = int(args.ctx)
    if args.batch is not None:
        over["batch"] = int(args.batch)
    if args.recompute:
        over["recompute"] = 1
    if args.clip > 0:
        opts["clip"] = (float(args.clip), args.clip_mode)
    if args.dropout > 0:
        opts["dropout"] = float(args.dropout)
    if args.rope_scale != 1.0:
        opts["rope_scale"] = float(args.rope_scale)
    parts = [f"{k}{v}" for k, v in over.items()]
    if "clip" in opts:
        parts.append(f"clip-{opts['clip'][1]}{opts['clip'][0]:g}")
    parts += [f"{k}{opts[k]:g}" for k in ("dropout", "rope_scale") if k in opts]
    return over, opts, ("+" + "+".join(parts)) if parts else ""


def apply_options(model, opts):
    if "clip" in opts:
        thr, mode = opts["clip"]
        model.set_grad_clip_mode(1 if mode == "linf" else 0)
        model.set_grad_clip(thr)
    if "dropout" in opts:
        model.set_dropout(opts["dropout"], 0x5EED)
    if "rope_scale" in opts:
        model.set_rope_scale(opts["rope_scale"])


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def step_flops(cfg):
    """Algorithmic FLOPs of one step: 6 * matmul params * tokens plus causal
    attention (QK^T and PV, forward and twice in backward)."""
    V, d, L, H, Hkv, h, T, B = (cfg[k] for k in ("vocab", "d_model", "n_layer", "n_head",
                                                 "n_kv_head", "d_ff", "ctx", "batch"))
    hd = d // H
    kvd = Hkv * hd
    M = L * (d * (d + 2 * kvd) + d * d + 3 * d * h) + d * V
    N = B * T
    attn = 12 * L * B * H * (T * (T + 1) / 2) * hd
    return 6.0 * M * N + attn, attn


def step_bytes(cfg):
    """HBM bytes of one step in the roofline's memory term (a model: what a
    step must move at least once with the activations it keeps for the
    backward).  Per token and layer: the saved activations -- the float32
    residual inputs x and x1, and in the activation type xn1, q|k|v, o, xn2,
    a|b and u, plus the float32 rstd pair and the log-sum-exps -- written once
    by the forward and read once by the backward, and the float32 residual
    gradient read and written at each of the layer's two residual joins.  Per
    step: the low-precision weights read by the forward and by the data
    gradients, the float32 weight gradients written, AdamW's 28 bytes per
    parameter, the logits written, read by the cross-entropy, its gradient
    written and read by the two lm_head GEMMs (four passes), and the embedding
    rows gathered and their gradient rows read and written."""
    V, d, L, H, Hkv, h, T, B = (cfg[k] for k in ("vocab", "d_model", "n_layer", "n_head",
                                                 "n_kv_head", "d_ff", "ctx", "batch"))
    hd = d // H
    kvd = Hkv * hd
    ab = 2 if cfg["compute"] == "bf16" else 4
    N = B * T
    saved = 8 * d + ab * (d + (d + 2 * kvd) + d + d + 2 * h + h) + 8 + 4 * H
    per_tok_layer = 2 * saved + 16 * d
    M = L * (d * (d + 2 * kvd) + d * d + 3 * d * h) + d * V
    P = V * d + L * (2 * d + d * (d + 2 * kvd) + d * d + 3 * d * h) + d + d * V
    per_step = 2 * ab * M + 4 * M + 28 * P + 4 * N * V * ab + 2 * N * d * 4 + V * d * 4
    return N * L * per_tok_layer + per_step


FP32_SIMT_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
# nominal dense TF32 / BF16 tensor rates (1.1 and 2.25 PFLOP/s): a float32
# workload's contractions are bounded by the TF32 rate at best
TF32_OF_BF16 = 1.1 / 2.25


def step_roofline(cfg, pk, step_ms):
    """The step against max(FLOPs / tensor peak, bytes / HBM bandwidth)."""
    F, F_attn = step_flops(cfg)
    peak = pk.get("bf16_tflops_sustained", pk.get("bf16_tflops"))
    if cfg["compute"] != "bf16":
        peak = peak * TF32_OF_BF16
    byt = step_bytes(cfg)
    t_tensor = F / (peak * 1e12) * 1e3
    t_hbm = byt / (pk["hbm_gbs"] * 1e9) * 1e3
    t_roof = max(t_tensor, t_hbm)
    return {"flops": F, "attention_flops": F_attn, "bytes": byt,
            "t_tensor_ms": t_tensor, "t_hbm_ms": t_hbm,
            "bound": "tensor" if t_tensor >= t_hbm else "hbm",
            "tensor_peak_tflops": peak,
            "frac_of_tensor_bound": t_tensor / step_ms,
            "frac_of_roofline": t_roof / step_ms}


# ------------------------------------------------------------------ clocks
class Clocks:
    """nvidia-smi sampled every 200 ms while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.out = None

    def start(self):
        try:
            self.out = open(os.devnull if False else f"/tmp/clocks_{os.getpid()}.csv", "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.idx), "-lms", "200"], stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def wait_first(self, timeout_s=5.0):
        """Return once the sampler has written its first line (or on time-out),
        so that a short timed region still gets samples."""
        if not self.proc:
            return
        t0 = time.time()
        while time.time() - t0 < timeout_s:
            try:
                if os.path.getsize(self.out.name) > 0:
                    return
            except OSError:
                pass
            time.sleep(0.02)

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = []
        for line in open(self.out.name):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.out.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows)}


# --------------------------------------------------------------- oracle leg
def oracle_sample_rate(cfg, tokens, reps=1, warmup=0, opts=None):
    """Tokens/s of the float64 oracle on a fraction f = tokens / (B*T) of the
    step: forward + backward of the first `tokens` positions of one sequence,
    plus AdamW over the same fraction of the parameters, with the step's
    options (dropout, RoPE scaling, clipping of that gradient share).  Returns
    (tokens/s, seconds per sample, cores)."""
    import numpy as np
    import oracle as O
    from oracle import train_terms as TT
    from synth import make_batch
    opts = opts or {}
    c = dict(cfg, batch=1, ctx=min(cfg["ctx"], tokens))
    if "rope_scale" in opts:
        c["rope_scale"] = opts["rope_scale"]
    S = c["ctx"]
    lay = O.param_layout(c)
    rng = np.random.default_rng(5)
    n = O.n_params(c)
    p = rng.standard_normal(n) * cfg["init_std"]
    for name, off, r, k in lay:
        if name.split(".")[-1] in ("g1", "g2", "gf"):
            p[off:off + r * k] = 1.0
    tok, tgt = make_batch(c, seed=11)
    frac = S / float(cfg["batch"] * cfg["ctx"])
    n_adam = max(1, int(n * frac))
    g = rng.standard_normal(n_adam) * 1e-3
    m = np.zeros(n_adam)
    v = np.zeros(n_adam)
    times = []
    for it in range(warmup + reps):
        t0 = time.perf_counter()
        drop = (float(np.float32(opts["dropout"])), 0x5EED, it) if "dropout" in opts else None
        O.forward_backward(c, p, tok, tgt, want_logits=False, dropout=drop)
        gc = TT.clip(g, opts["clip"][0], opts["clip"][1])[0] if "clip" in opts else g
        O.adamw(p[:n_adam], gc, m, v, 1, cfg["lr"], cfg["wd"])
        dt = time.perf_counter() - t0
        if it >= warmup:
            times.append(dt)
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    t = statistics.median(times)
    return S / t, t, cores, S


def sample_tokens_for(cfg, budget_s, opts=None):
    """Prefix length whose oracle sample takes about budget_s seconds (probed
    on a 16-token prefix, assuming linear cost in tokens)."""
    _, t16, _, _ = oracle_sample_rate(cfg, 16, opts=opts)
    per_tok = t16 / 16.0
    S = int(max(16, min(cfg["ctx"], budget_s / max(per_tok, 1e-9))))
    return S


# ------------------------------------------------------------ rank helpers
def max_over_ranks(x, world, device=None):
    """The largest of a per-rank value over all ranks (all_reduce MAX on
    `device`: the GPU under NCCL, the CPU under gloo); x itself at world 1."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_step, steps, world, ms):
    """Whole-job throughput: the units all ranks processed over the time the
    slowest rank took (ms, already the max over ranks)."""
    return units_per_step * steps * world / (ms / 1e3)


# --------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist
    from scratch_llama_decoder_b200 import LlamaStep
    from synth import get_config, make_batch, make_params

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    over, opts, suffix = step_options(args)
    cfg = get_config(args.config, **over)
    workload = cfg["name"] + suffix
    # the library's own stream (not the legacy default stream), so llm_step
    # runs as a replayed CUDA graph after its first two calls
    stream = torch.cuda.Stream(device=dev)
    model = LlamaStep(cfg, device=dev, stream=stream)
    apply_options(model, opts)
    dp_mode = args.dp if world > 1 else "none"
    # replicas start from their own weights; a data-parallel model is one
    # model, the same weights on every rank (each rank its own data)
    p_host = make_params(cfg, model.layout,
                         seed=1001 + cfg["index"] + (7919 * rank if dp_mode == "none" else 0))
    tok_h, tgt_h = make_batch(cfg, seed=1000 + cfg["index"] + 7919 * rank)
    stepper = None
    if dp_mode in ("sharded", "sharded-overlap"):
        from scratch_llama_decoder_b200.dp import ShardedDataParallelStep
        stepper = ShardedDataParallelStep(model, model.n_params,
                                          overlap=dp_mode == "sharded-overlap")
        P, G, Mo, Vo = stepper.buffers()  # padded; the moments are this rank's chunk
        P[:model.n_params].copy_(torch.from_numpy(p_host))
    else:
        if dp_mode != "none":
            from scratch_llama_decoder_b200.dp import DataParallelStep
            stepper = DataParallelStep(model, overlap=dp_mode == "overlap")
        P = torch.tensor(p_host, device=dev)
        G = torch.zeros_like(P)
        Mo = torch.zeros_like(P)
        Vo = torch.zeros_like(P)
    tok = torch.tensor(tok_h, device=dev)
    tgt = torch.tensor(tgt_h, device=dev)
    loss = torch.zeros(1, device=dev)
    lr, wd = cfg["lr"], cfg["wd"]
    N = cfg["batch"] * cfg["ctx"]

    def barrier():
        if world > 1:
            dist.barrier()

    def train_step(t):
        # every step of this run, timed or not, goes through here (with a
        # sharded optimiser the moments are chunk-sized: llm_step must not
        # see them)
        if stepper is None:
            model.step(P, G, Mo, Vo, t, tok, tgt, lr, wd, loss)
        else:
            stepper.step(P, G, Mo, Vo, t, tok, tgt, lr, wd, loss)

    def step_launches():
        return model.last_launch_count() if stepper is None else stepper.last_launches

    torch.cuda.synchronize()  # inputs written on the default stream are in place
    t = 0
    # the warm-up steps (>= 3) run the step once as launches, then capture the
    # step graph and replay it; the timed steps are replays
    for _ in range(args.warmup):
        t += 1
        train_step(t)
    st = model.status()
    assert st == 0, f"warm-up step failed with status {st}"
    launches_per_step = step_launches()

    clocks = Clocks(local_rank)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    clocks.wait_first()
    # one event before the first step and one after each: the headline is
    # first to last, the per-step times give the median and best step
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    ev[0].record(stream)
    for k in range(args.steps):
        t += 1
        train_step(t)
        ev[k + 1].record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = ev[0].elapsed_time(ev[-1])
    per_step = sorted(ev[k].elapsed_time(ev[k + 1]) for k in range(args.steps))
    # GEMM roofline: the same K steps again as individual launches, each
    # tensor-core GEMM bracketed by CUDA events on the library's stream (the
    # kernels are the ones the graph replays; events cannot time graph nodes)
    model.set_kernel_timing(True)
    for _ in range(args.steps):
        t += 1
        train_step(t)
    classes = model.read_kernel_class_timing()
    g_ms, g_flops, g_launch = model.read_kernel_timing()
    model.set_kernel_timing(False)
    # clocks sampled over the timed region and the GEMM-timing pass after it
    clk = clocks.stop()
    st = model.status()
    assert st == 0, f"timed step failed with status {st}"
    final_loss = float(loss.item())
    ms = max_over_ranks(ms, world, dev)

    # ---- e2e: same API, host buffers, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        tok_pin = torch.tensor(tok_h).pin_memory()
        tgt_pin = torch.tensor(tgt_h).pin_memory()
        loss_pin = torch.zeros(1).pin_memory()
        barrier()
        torch.cuda.synchronize()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            # two untimed steps: the step graph without timing events is
            # captured here, outside the timed loop
            for _ in range(2):
                t += 1
                tok.copy_(tok_pin, non_blocking=True)
                tgt.copy_(tgt_pin, non_blocking=True)
                train_step(t)
                loss_pin.copy_(loss, non_blocking=True)
                stream.synchronize()
            # one step in flight: step i + 1's inputs are copied (behind step
            # i on the stream, so step i has read its own) and its graph
            # launched before the host reads step i's loss from its pinned slot
            loss_slots = [torch.zeros(1).pin_memory() for _ in range(2)]
            done = [torch.cuda.Event() for _ in range(2)]
            seen = []
            f0.record(stream)
            for i in range(args.steps):
                t += 1
                tok.copy_(tok_pin, non_blocking=True)
                tgt.copy_(tgt_pin, non_blocking=True)
                train_step(t)
                loss_slots[i % 2].copy_(loss, non_blocking=True)
                done[i % 2].record(stream)
                if i > 0:
                    done[(i - 1) % 2].synchronize()
                    seen.append(float(loss_slots[(i - 1) % 2].item()))
            f1.record(stream)
            done[(args.steps - 1) % 2].synchronize()
            seen.append(float(loss_slots[(args.steps - 1) % 2].item()))
            assert len(seen) == args.steps and all(x == x for x in seen), seen
        torch.cuda.synchronize()
        barrier()
        ems = f0.elapsed_time(f1)
        ems = max_over_ranks(ems, world, dev)
        e2e = {"value": job_rate(N, args.steps, world, ems), "unit": "tokens/s",
               "h2d_bytes_per_step": int(tok_pin.numel() * 4 + tgt_pin.numel() * 4),
               "d2h_bytes_per_step": 4}

    if rank != 0:
        return None
    pk, src = peaks()
    F, F_attn = step_flops(cfg)
    step_s = ms / 1e3 / args.steps
    value = job_rate(N, args.steps, world, ms)
    peak_tc = pk.get("bf16_tflops_sustained", pk.get("bf16_tflops"))
    achieved = (g_flops / (g_ms / 1e3)) / 1e12 if g_ms > 0 else 0.0
    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16"
        if cfg["compute"] == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": workload, "tokens_per_step": N, "batch": cfg["batch"],
                   "seq_len": cfg["ctx"],
                   "parallelism": ("single GPU" if world == 1 else f"replicas x{world}"
                                   if dp_mode == "none" else f"dp{world} ({dp_mode})"), "l2": "inputs larger than L2 (saved activations of "
                   "several GB per step; no flush)"},
        "roofline": {"bound": "tensor", "kernel": "tcgen05 GEMM (all projection GEMMs of the "
                     "step)", "achieved": achieved, "peak": peak_tc, "unit": "TFLOP/s",
                     "frac": achieved / peak_tc if peak_tc else None,
                     "traffic": gemm_traffic(workload),
                     "launches": g_launch, "ms_total": g_ms,
                     "peak_source": f"{src} bf16_tflops_sustained"},
        "step_roofline": step_roofline(cfg, pk, step_s * 1e3),
        "kernels": kernel_rates(classes, args.steps, pk, src),
        "gpu_launches": launches_per_step * args.steps,
        # this rank's steps (rank 0): median and best step, as tokens/s per GPU
        "per_step": {"median_ms": per_step[len(per_step) // 2], "best_ms": per_step[0],
                     "median_tokens_per_s_per_gpu": N / (per_step[len(per_step) // 2] / 1e3),
                     "best_tokens_per_s_per_gpu": N / (per_step[0] / 1e3)},
        "loss": final_loss,
        "clocks": clk,
        "e2e": e2e,
    }
    if world == 1 and not args.no_per_config and args.config == "c5" and not suffix:
        # the other workloads, each timed the same way in this process (their
        # own context, stream and clock record)
        model.close()
        del P, G, Mo, Vo, model
        torch.cuda.empty_cache()
        out["per_config"] = {}
        for name in PER_CONFIG:
            r = time_workload(name, args.steps, max(3, args.warmup), dev, local_rank, pk)
            out["per_config"][r.pop("workload")] = r
    if world == 1 and not args.no_cpu_baseline:
        S = sample_tokens_for(cfg, 12.0, opts)
        rate, tsec, cores, S = oracle_sample_rate(cfg, S, opts=opts)
        out["cpu_baseline"] = {
            "value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"float64 oracle: forward+backward of a {S}-token prefix of one "
                      f"sequence plus AdamW over {S}/{N} of the parameters "
                      f"({tsec:.1f} s), scaled to tokens/s"}
    return out


def kernel_rates(classes, steps, pk, src):
    """Per kernel class: device time per step (CUDA events around every
    launch, individual launches on one stream), algorithmic work per step and
    the rate against the class's bound (TFLOP/s against the sustained bf16
    peak for the contractions, GB/s against the measured copy bandwidth for
    the memory-bound passes)."""
    from scratch_llama_decoder_b200._lib import KERNEL_CLASSES
    peak_tc = pk.get("bf16_tflops_sustained", pk.get("bf16_tflops"))
    out = {}
    for name, unit in KERNEL_CLASSES:
        ms, work, n = classes.get(name, (0.0, 0.0, 0))
        if n == 0 or ms <= 0:
            continue
        if unit == "flop" and name == "gemm_cuda_core":
            # float32 FMA on CUDA cores: 148 SMs x 128 lanes x 2 FLOPs x 1.965 GHz
            rate, peak, u = work / (ms / 1e3) / 1e12, FP32_SIMT_TFLOPS, "TFLOP/s"
            ps = "nominal float32 CUDA-core FMA rate"
        elif unit == "flop" and name == "gemm_tf32":
            # three tf32 products per float32 product: the bound is a third of
            # the tf32 rate (the bf16 peak times the nominal tf32/bf16 ratio)
            rate, peak, u = work / (ms / 1e3) / 1e12, peak_tc * TF32_OF_BF16 / 3, "TFLOP/s"
            ps = f"{src} bf16_tflops_sustained x 1.1/2.25 / 3 (3xTF32)"
        elif unit == "flop":
            rate, peak, u = work / (ms / 1e3) / 1e12, peak_tc, "TFLOP/s"
            ps = f"{src} bf16_tflops_sustained"
        else:
            rate, peak, u = work / (ms / 1e3) / 1e9, pk["hbm_gbs"], "GB/s"
            ps = f"{src} hbm_gbs"
        out[name] = {"ms_per_step": ms / steps, "launches_per_step": n / steps,
                     "work_per_step": work / steps, "work_unit": unit, "achieved": rate,
                     "peak": peak, "unit": u, "frac": rate / peak if peak else None,
                     "peak_source": ps}
    return out


PER_CONFIG = ("c2", "c3", "c4")


def time_workload(name, steps, warmup, dev, local_rank, pk):
    """One workload's training step timed as the headline is: its own stream
    (graph replays after the warm-up), an event before the first timed step
    and after each, clocks sampled over the timed region."""
    import torch
    from scratch_llama_decoder_b200 import LlamaStep
    from synth import get_config, make_batch, make_params
    cfg = get_config(name)
    stream = torch.cuda.Stream(device=dev)
    model = LlamaStep(cfg, device=dev, stream=stream)
    P = torch.tensor(make_params(cfg, model.layout), device=dev)
    G, Mo, Vo = (torch.zeros_like(P) for _ in range(3))
    tok_h, tgt_h = make_batch(cfg)
    tok, tgt = torch.tensor(tok_h, device=dev), torch.tensor(tgt_h, device=dev)
    loss = torch.zeros(1, device=dev)
    N = cfg["batch"] * cfg["ctx"]
    torch.cuda.synchronize()
    t = 0
    for _ in range(warmup):
        t += 1
        model.step(P, G, Mo, Vo, t, tok, tgt, cfg["lr"], cfg["wd"], loss)
    assert model.status() == 0, name
    launches = model.last_launch_count()
    clocks = Clocks(local_rank)
    torch.cuda.synchronize()
    clocks.start()
    clocks.wait_first()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    ev[0].record(stream)
    for k in range(steps):
        t += 1
        model.step(P, G, Mo, Vo, t, tok, tgt, cfg["lr"], cfg["wd"], loss)
        ev[k + 1].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    assert model.status() == 0, name
    # kernel classes: the same steps again as individual timed launches
    model.set_kernel_timing(True)
    for _ in range(steps):
        t += 1
        model.step(P, G, Mo, Vo, t, tok, tgt, cfg["lr"], cfg["wd"], loss)
    classes = model.read_kernel_class_timing()
    model.read_kernel_timing()
    model.set_kernel_timing(False)
    ms = ev[0].elapsed_time(ev[-1]) / steps
    per_step = sorted(ev[k].elapsed_time(ev[k + 1]) for k in range(steps))
    roof = step_roofline(cfg, pk, ms)
    src = "measured" if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")) else "fallback"
    out = {"workload": cfg["name"], "ms_per_step": ms, "value": N / (ms / 1e3),
           "unit": "tokens/s", "dtype": "bf16" if cfg["compute"] == "bf16" else "f32",
           "tokens_per_step": N, "frac_of_roofline": roof["frac_of_roofline"],
           "step_roofline": roof, "median_ms": per_step[len(per_step) // 2],
           "best_ms": per_step[0], "gpu_launches": launches * steps,
           "loss": float(loss.item()), "clocks": clk,
           "kernels": kernel_rates(classes, steps, pk, src),
           "l2": "inputs larger than L2 (saved activations of the step); no flush"}
    model.close()
    del P, G, Mo, Vo, model
    torch.cuda.empty_cache()
    return out


def decode_bytes(cfg, pos):
    """HBM bytes of one decode step at position pos: the unpadded bf16 weight
    matrices, the float32 embedding rows and RMSNorm gains, every cached key
    and value row 0..pos (read) and the new row (written), the q row, and the
    float32 logits (written)."""
    V, d, L, H, Hkv, h, B = (cfg[k] for k in ("vocab", "d_model", "n_layer", "n_head",
                                              "n_kv_head", "d_ff", "batch"))
    hd = d // H
    kvd = Hkv * hd
    esz = 2 if cfg["compute"] == "bf16" else 4
    weights = (L * (d * (d + 2 * kvd) + d * d + 2 * d * h + h * d) + d * V) * esz
    small = B * d * 4 + (2 * L + 1) * d * 4
    kv = L * B * ((pos + 1) * 2 * kvd + (d + 2 * kvd)) * esz
    return weights + small + kv + B * V * 4, weights, kv


def oracle_decode_rate(cfg, budget_s=10.0):
    """The float64 oracle decoding one sequence from position 0 for about
    budget_s seconds; returns (tokens/s, seconds, cores, positions)."""
    import numpy as np
    import oracle as O
    from oracle import decode as OD
    from synth import make_batch, make_params
    c1 = dict(cfg, batch=1)
    p = make_params(cfg, O.param_layout(cfg)).astype(np.float64)
    tok, _ = make_batch(cfg)
    cache = OD.KVCache(c1)
    n, t0 = 0, time.time()
    while n < cfg["ctx"] and (time.time() - t0 < budget_s or n < 2):
        OD.decode_step(c1, p, cache, tok[0, n:n + 1], n)
        n += 1
    dt = time.time() - t0
    return n / dt, dt, os.cpu_count(), n


def run_decode(args, rank, world, local_rank):
    import numpy as np
    import torch
    from scratch_llama_decoder_b200 import LlamaStep
    from synth import get_config, make_batch, make_params

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = get_config(args.config)
    B, T, V = cfg["batch"], cfg["ctx"], cfg["vocab"]
    if args.pos + args.warmup + args.steps > T:
        raise SystemExit(f"--pos + --warmup + --steps must be <= ctx ({T})")
    stream = torch.cuda.Stream(device=dev)
    model = LlamaStep(cfg, device=dev, stream=stream)
    p_host = make_params(cfg, model.layout, seed=1001 + cfg["index"] + 7919 * rank)
    tok_h, _ = make_batch(cfg, seed=1000 + cfg["index"] + 7919 * rank)
    tok_h = tok_h.reshape(B, T)
    P = torch.tensor(p_host, device=dev)
    tok_all = torch.tensor(tok_h, device=dev)
    cols = torch.tensor(np.ascontiguousarray(tok_h.T), device=dev)  # [T, B]: row t = ids at t
    tk = torch.empty(B, dtype=torch.int32, device=dev)
    lg = torch.empty(B, V, device=dev)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        model.forward(P, tok_all)  # prefill: every position's keys and values
        pos = args.pos
        for _ in range(args.warmup):  # the second call captures the decode graph
            tk.copy_(cols[pos])
            model.decode(P, tk, pos, logits=lg)
            pos += 1
    st = model.status()
    assert st == 0, f"warm-up decode failed with status {st}"
    launches = model.last_launch_count()
    first = pos
    clocks = Clocks(local_rank)
    torch.cuda.synchronize()
    clocks.start()
    clocks.wait_first()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with torch.cuda.stream(stream):
        ev[0].record(stream)
        for k in range(args.steps):
            tk.copy_(cols[pos])
            model.decode(P, tk, pos, logits=lg)
            pos += 1
            ev[k + 1].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = max_over_ranks(ev[0].elapsed_time(ev[-1]), world, dev)
    per_step = sorted(ev[k].elapsed_time(ev[k + 1]) for k in range(args.steps))
    st = model.status()
    assert st == 0, f"timed decode failed with status {st}"
    byt = [decode_bytes(cfg, q) for q in range(first, pos)]
    alg = sum(b[0] for b in byt) / args.steps

    # e2e: ids and uniforms from pinned host memory, decode + top-k sampling,
    # sampled ids back to the host every step
    e2e = None
    if not args.no_e2e:
        ids_pin = torch.tensor(tok_h[:, 0]).pin_memory()
        uni_pin = torch.rand(B).pin_memory()
        out_pin = torch.zeros(B, dtype=torch.int32).pin_memory()
        ud = torch.empty(B, device=dev)
        od = torch.empty(B, dtype=torch.int32, device=dev)
        with torch.cuda.stream(stream):
            model.forward(P, tok_all)
            q = args.pos
            for _ in range(2):  # untimed: graph capture for these buffers
                tk.copy_(ids_pin, non_blocking=True)
                model.decode(P, tk, q, logits=lg)
                q += 1
            stream.synchronize()
            f0 = torch.cuda.Event(enable_timing=True)
            f1 = torch.cuda.Event(enable_timing=True)
            n_e2e = min(args.steps, T - q)
            f0.record(stream)
            for _ in range(n_e2e):
                tk.copy_(ids_pin, non_blocking=True)
                ud.copy_(uni_pin, non_blocking=True)
                model.decode(P, tk, q, logits=lg)
                model.sample(lg, 0.8, 40, ud, out=od)
                out_pin.copy_(od, non_blocking=True)
                stream.synchronize()
                ids_pin.copy_(out_pin)  # the sampled ids are the next step's input
                q += 1
            f1.record(stream)
        torch.cuda.synchronize()
        ems = f0.elapsed_time(f1)
        e2e = {"value": B * n_e2e / (ems / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": 8 * B,
               "d2h_bytes_per_step": 4 * B, "sampling": "temperature 0.8, top-k 40"}
        assert model.status() == 0
    if rank != 0:
        return None
    pk, src = peaks()
    peak = pk.get("hbm_gbs")
    gbs = alg / (ms / 1e3 / args.steps) / 1e9
    out = {
        "metric": "decode tokens/sec (KV cache, one position per sequence per step) on 1 B200; "
                  "% of HBM roofline",
        "value": job_rate(B, args.steps, world, ms), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if cfg["compute"] == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": cfg["name"], "batch": B, "ctx": T,
                   "positions": [first, pos - 1],
                   "l2": "weights and cache (> 1 GB per step) larger than L2; no flush"},
        "roofline": {"bound": "hbm", "kernel": "decode step (all kernels)", "achieved": gbs,
                     "peak": peak, "unit": "GB/s", "frac": gbs / peak if peak else None,
                     "traffic": None, "bytes_per_step": alg,
                     "weight_bytes": byt[0][1], "kv_bytes_first": byt[0][2],
                     "peak_source": f"{src} hbm_gbs"},
        "gpu_launches": launches * args.steps,
        # this rank's positions: median and best decode step (the later
        # positions read more cached keys and values)
        "per_step": {"median_ms": per_step[len(per_step) // 2], "best_ms": per_step[0]},
        "clocks": clk,
        "e2e": e2e,
    }
    if world == 1 and not args.no_cpu_baseline:
        rate, secs, cores, n = oracle_decode_rate(cfg)
        out["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": cores,
                               "kind": "oracle",
                               "sample": f"float64 oracle decoding positions 0..{n - 1} of one "
                                         f"sequence ({secs:.1f} s)"}
    return out


def run_reference(args, rank):
    if rank != 0:
        return None
    from synth import get_config
    over, opts, suffix = step_options(args)
    cfg = get_config(args.config, **over)
    budget = max(1.0, 150.0 / max(1, args.steps + args.warmup))
    S = sample_tokens_for(cfg, budget, opts)
    rate, tsec, cores, S = oracle_sample_rate(cfg, S, reps=args.steps, warmup=args.warmup,
                                              opts=opts)
    N = cfg["batch"] * cfg["ctx"]
    return {
        "impl": "reference", "metric": METRIC, "value": rate, "unit": "tokens/s", "n_gpus": 1,
        # a step of this arm is a bounded sample (S tokens); ms_per_step is the
        # full step's time at the sampled rate, sample_ms the sample's own time
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": N / rate * 1e3,
        "sample_ms": tsec * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": cfg["name"] + suffix, "tokens_per_step": N,
                   "batch": cfg["batch"], "seq_len": cfg["ctx"], "parallelism": "host CPU"},
        "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: forward+backward of a {S}-token prefix of one "
                                   f"sequence plus AdamW over {S}/{N} of the parameters"},
        "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_kernel(args):
    """Device time of one hot-path kernel shape (CUDA events, after warm-up)."""
    import ctypes as C
    import torch
    import scratch_llama_decoder_b200 as P
    torch.cuda.set_device(0)
    p = lambda t: C.c_void_p(t.data_ptr())
    g = torch.Generator(device="cuda").manual_seed(0)
    if args.kernel == "gemm":
        M, N, K = (int(x) for x in args.shape.split(","))
        ak, bk = {"kn": (1, 0), "kk": (1, 1), "nn": (0, 0)}[args.orient]
        A = torch.randn((M, K) if ak else (K, M), device="cuda", generator=g).to(torch.bfloat16)
        B = torch.randn((N, K) if bk else (K, N), device="cuda", generator=g).to(torch.bfloat16)
        Cm = torch.empty(M, N, device="cuda")
        flag = torch.zeros(1, dtype=torch.int32, device="cuda")

        def call():
            rc = P.lib.llm_kernel_gemm_bf16(M, N, K, p(A), A.shape[1], ak, p(B), B.shape[1], bk,
                                            p(Cm), N, 1, p(flag), None)
            assert rc == 0
        flops = 2.0 * M * N * K
    else:
        Bt, T, H, Hkv, hd = (int(x) for x in args.shape.split(","))
        w = (H + 2 * Hkv) * hd
        qkv = torch.randn(Bt * T, w, device="cuda", generator=g).to(torch.bfloat16)
        o = torch.empty(Bt * T, H * hd, device="cuda", dtype=torch.bfloat16)
        do = torch.randn(Bt * T, H * hd, device="cuda", generator=g).to(torch.bfloat16)
        dqkv = torch.empty_like(qkv)
        lse = torch.empty(Bt, H, T, device="cuda")
        Dv = torch.empty(Bt, H, T, device="cuda")

        def fwd():
            assert P.lib.llm_kernel_attention_fwd_bf16(p(qkv), p(o), p(lse), Bt, T, H, Hkv, hd,
                                                       args.fwd_impl, None) == 0

        def bwd():
            assert P.lib.llm_kernel_attention_bwd_bf16(p(qkv), p(o), p(do), p(lse), p(Dv),
                                                       p(dqkv), Bt, T, H, Hkv, hd, args.bwd_impl,
                                                       None) == 0
        causal = Bt * H * (T * (T + 1) / 2) * hd
        res = {}
        for name, fn, fl in (("fwd", fwd, 4.0 * causal), ("bwd", bwd, 8.0 * causal)):
            for _ in range(args.warmup):
                fwd()
                fn()
            torch.cuda.synchronize()
            tot = 0.0
            for _ in range(args.steps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                if name == "bwd":
                    fwd()
                e0.record()
                fn()
                e1.record()
                torch.cuda.synchronize()
                tot += e0.elapsed_time(e1)
            ms = tot / args.steps
            res[name] = {"ms": ms, "tflops": fl / (ms / 1e3) / 1e12}
        print(json.dumps({"kernel": "attention", "shape": args.shape, "fwd_impl": args.fwd_impl,
                          "bwd_impl": args.bwd_impl, **res}), flush=True)
        return
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        call()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    print(json.dumps({"kernel": args.kernel, "shape": args.shape, "orient": args.orient,
                      "ms": ms, "tflops": flops / (ms / 1e3) / 1e12}), flush=True)


def main():
    args = parse()
    if args.steps < 1 or args.warmup < 0:
        raise SystemExit("bench.py: --steps must be >= 1 and --warmup >= 0")
    if args.kernel:
        run_kernel(args)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        out = run_reference(args, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    if world > 1:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        out = (run_decode if args.decode else run_ours)(args, rank, world, local_rank)
        if out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
