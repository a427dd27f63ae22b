#!/usr/bin/env python
"""GPT-2 124M training-step benchmark on B200 (one process per GPU).

A step is one whole optimizer step of the training hot path: 32 micro-steps
of forward + backward (B=16, T=1024: 524,288 tokens, loss scaled 1/32), the
global-norm clip and AdamW, all in libgpt2's kernels.  Inputs are seeded
synthetic Zipf(1.1) token streams (the pages' dataset is not available), made
resident in HBM before the timed region; the step's working set (about 10 GB
of activations) is far larger than the 126 MB L2, so no flush is needed.

    python bench.py [--gpus N --steps K --warmup W] [--workload t1024|t512]
    python bench.py --impl reference ...   # the CPU oracle, timed on host cores

Prints ONE JSON line (rank 0).  With N > 1 (torchrun) every rank trains its own
replica on its own data (the step has no cross-GPU exchange here): the
whole-job value is the tokens of all ranks over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

NCORES = len(os.sched_getaffinity(0))
for _v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
    os.environ.setdefault(_v, str(NCORES))

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "GPT-2 124M train tokens/s (fwd+bwd+AdamW, bf16) on 1 B200; MFU %"
WORKLOADS = {
    # name: (micro-batch B, sequence T, micro-steps per optimizer step)
    "t1024": (16, 1024, 32),   # GPT-2 124M, B=16 x T=1024, accumulated to 524,288 tokens
    "t512": (32, 512, 32),     # same model at short context, B=32 x T=512
}
N_PARAMS = 124_475_904
L, C, V, VP = 12, 768, 50257, 50304
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "bf16_sustained_sm_mhz": 1300.0}  # the sustained figure settles at about 1.3 GHz
# DRAM bytes (read + write) per launch of the 2-SM GEMM kernel, averaged over
# the captured launches of the ncu launch list of the default workload
# (dram__bytes_read.sum + dram__bytes_write.sum, one pass, this build)
GEMM_TRAFFIC_BYTES_PER_LAUNCH = 238.3e6


def flops_per_token(T: int) -> float:
    """6N + 6*L*T*C: matmul FLOPs of forward+backward plus causal attention
    (score count halved; forward 2 matmuls, backward 4)."""
    return 6.0 * N_PARAMS + 6.0 * L * T * C


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        return self.summarize(out)

    @staticmethod
    def summarize(out: str):
        """The median SM clock over the busy samples (above half the maximum),
        the maximum, and every slowdown reason seen active, from the CSV rows
        of the query above."""
        rows = [r.split(",") for r in out.strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = max((float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()), default=None)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip().lower() == "active"})
        busy = [s for s in sm if mx and s > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(busy) if busy else None, "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------- CPU oracle

SAMPLE_B = 2  # sequences per timed oracle sample (about 15 s of host time at T=1024)


def oracle_sample(T: int, seed: int):
    """The oracle as it stands, fp32, on a slice of one micro-step of the
    workload: forward + backward of SAMPLE_B x T tokens, and one AdamW update
    over all parameters.  Returns (seconds for the fwd+bwd, seconds for AdamW)."""
    from decoder_only_transformer_02_b200 import synthetic as S
    from oracle import gpt2_oracle as O
    cfg = O.GPT2_124M
    flat = O.init_params(cfg, 1234, dtype=np.float32)
    (tok, tgt), = S.token_batches("zipf", V, SAMPLE_B, T, 1, seed=seed)
    t0 = time.perf_counter()
    st = O.forward(flat, cfg, tok, tgt)
    g = O.backward(st, 1.0)
    t1 = time.perf_counter()
    O.adamw_step(flat, g, np.zeros_like(flat), np.zeros_like(flat), 1, 6e-4, cfg)
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1


def cpu_baseline(B, T, accum, seed=7):
    t_smp, t_adam = oracle_sample(T, seed)
    step_s = accum * B / SAMPLE_B * t_smp + t_adam
    return {"value": accum * B * T / step_s, "unit": "tokens/s", "cores": NCORES, "kind": "oracle",
            "sample": f"forward+backward of {SAMPLE_B} x {T} tokens ({t_smp:.2f} s) and one AdamW update over "
                      f"{N_PARAMS} params ({t_adam:.2f} s), NumPy fp32; optimizer step = {accum * B} sequences "
                      f"+ 1 update, extrapolated"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    B, T, accum = WORKLOADS[args.workload]
    from decoder_only_transformer_02_b200 import synthetic as S  # noqa: F401
    # amortised optimizer cost, measured once
    _, t_adam = oracle_sample(T, 99)
    for w in range(args.warmup):
        oracle_sample_fwd_bwd(T, 100 + w)
    times = []
    for k in range(args.steps):
        times.append(oracle_sample_fwd_bwd(T, 200 + k))
    t_smp = sum(times) / len(times)
    step_s = accum * B / SAMPLE_B * t_smp + t_adam
    value = accum * B * T / step_s
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_smp * 1e3, "higher_is_better": True,
        "step": f"one sampled forward+backward of {SAMPLE_B} x {T} tokens (the timed unit); the value "
                f"extrapolates to the {accum * B * T}-token optimizer step, {step_s:.0f} s",
        "ms_per_optimizer_step_extrapolated": step_s * 1e3,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic (Zipf 1.1 token stream)",
        "config": workload_config(args.workload),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": NCORES, "kind": "oracle",
                         "sample": f"each step: forward+backward of {SAMPLE_B} x {T} tokens by the NumPy fp32 "
                                   f"oracle (mean {t_smp:.2f} s); AdamW over all params measured once "
                                   f"({t_adam:.2f} s); "
                                   f"optimizer step = {accum * B} sequences + 1 update, extrapolated"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def oracle_sample_fwd_bwd(T, seed):
    from decoder_only_transformer_02_b200 import synthetic as S
    from oracle import gpt2_oracle as O
    cfg = O.GPT2_124M
    global _ORACLE_FLAT
    if "_ORACLE_FLAT" not in globals():
        _ORACLE_FLAT = O.init_params(cfg, 1234, dtype=np.float32)
    (tok, tgt), = S.token_batches("zipf", V, SAMPLE_B, T, 1, seed=seed)
    t0 = time.perf_counter()
    st = O.forward(_ORACLE_FLAT, cfg, tok, tgt)
    O.backward(st, 1.0)
    return time.perf_counter() - t0


def workload_config(name):
    B, T, accum = WORKLOADS[name]
    return {"workload": f"gpt2-124m optimizer step: B={B} x T={T} x {accum} micro-steps = {B * T * accum} tokens, "
                        f"vocab {VP}, clip 1.0, AdamW, warmup+cosine LR",
            "micro_batch": B, "seq_len": T, "grad_accum": accum, "global_batch_tokens": B * T * accum,
            "parallelism": "replicas only (one independent replica per GPU)",
            "l2": "working set (~10 GB of activations) >> 126 MB L2; no flush needed"}


# -------------------------------------------------------------------- ours

def max_over_ranks(x, world, device):
    """The largest of every rank's x (every rank must call it, in the same
    order): the slowest rank's time is the job's time."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world, steps, tokens_per_step, ms):
    """Whole-job throughput: the tokens of all ranks (each trains its own
    replica on its own data) over the slowest rank's time."""
    return world * steps * tokens_per_step / (ms / 1e3)


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        print(json.dumps({"metric": METRIC, "error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    from decoder_only_transformer_02_b200 import gpt2 as G
    from decoder_only_transformer_02_b200 import synthetic as S

    B, T, accum = WORKLOADS[args.workload]
    if args.B or args.accum:
        # a smaller case of the same step (profiling captures only; not a bench line)
        B, accum = args.B or B, args.accum or accum
    tok_per_step = B * T * accum
    stream = torch.cuda.current_stream()
    m = G.GPT2(G.GPT2Config(L, 12, C, V, VP, 1024, B, T, G.GPT2_BF16), seed=1234 + rank, stream=stream)

    # device-resident inputs for every warm-up and timed step
    nsteps = args.warmup + args.steps
    toks = np.empty((nsteps, accum, B, T), dtype=np.int32)
    tgts = np.empty_like(toks)
    for s in range(nsteps):
        stream_ids = S.zipf_stream(tok_per_step + 1, V, 1.1, seed=1235 + 1000 * rank + s)
        for k, (x, y) in enumerate(S.micro_batches(stream_ids, B, T, accum)):
            toks[s, k], tgts[s, k] = x, y
    d_tok = torch.from_numpy(toks).cuda()
    d_tgt = torch.from_numpy(tgts).cuda()

    def step(s):
        m.zero_grad()
        for k in range(accum):
            m.forward_backward(d_tok[s, k], d_tgt[s, k], 1.0 / accum)
        m.adamw_step(G.lr_at(1000 + s))

    for s in range(args.warmup):
        step(s)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    launches0 = m.kernel_launches
    clocks = ClockSampler(local)
    clocks.start()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    ev0.record(stream)
    for s in range(args.warmup, nsteps):
        step(s)
    ev1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    launches = m.kernel_launches - launches0
    ms = ev0.elapsed_time(ev1)
    # per-kernel-class device times: the same step sequence once more, with a
    # CUDA event pair around every launch (eager launches, no graph replay)
    prof_steps = min(args.steps, 3)
    m.set_timing(True)
    m.get_timing()  # reset
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    for s in range(args.warmup, args.warmup + prof_steps):
        step(s)
    p1.record(stream)
    torch.cuda.synchronize()
    timing = m.get_timing()
    m.set_timing(False)
    prof_ms = p0.elapsed_time(p1) / prof_steps
    loss = m.last_loss()
    ms = max_over_ranks(ms, world, "cuda")
    value = job_tokens_per_s(world, args.steps, tok_per_step, ms)

    # end to end through the public C ABI from pinned HOST buffers: every step
    # copies its tokens to the device and reads the loss and norm back
    e2e_steps = args.steps
    h_tok = torch.empty((e2e_steps + 1, accum * B * T), dtype=torch.int32).pin_memory()
    h_tgt = torch.empty_like(h_tok).pin_memory()
    for s in range(e2e_steps + 1):
        ids = S.zipf_stream(tok_per_step + 1, V, 1.1, seed=777 + 1000 * rank + s)
        h_tok[s] = torch.from_numpy(ids[:-1])
        h_tgt[s] = torch.from_numpy(ids[1:])
    m.train_step(h_tok[0], h_tgt[0], accum, B, T, G.lr_at(2000))  # warm-up
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s in range(1, e2e_steps + 1):
        e_loss, e_norm = m.train_step(h_tok[s], h_tgt[s], accum, B, T, G.lr_at(2000 + s))
    e1.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(e0.elapsed_time(e1), world, "cuda")
    e2e = {"value": job_tokens_per_s(world, e2e_steps, tok_per_step, e_ms), "unit": "tokens/s",
           "h2d_bytes_per_step": int(2 * tok_per_step * 4), "d2h_bytes_per_step": 8,
           "api": "gpt2_train_step (host int32 token/target buffers, pinned)"}

    peaks, peak_kind = load_peaks()
    fpt = flops_per_token(T)
    mfu = value * fpt / (world * peaks["bf16_tflops"] * 1e12)
    mfu_sus = value * fpt / (world * peaks["bf16_tflops_sustained"] * 1e12)
    per_step = {}
    for k, d in timing.items():
        if d["ops"] == 0:
            continue
        e = {"ms_per_step": d["ms"] / prof_steps, "ops_per_step": d["ops"] / prof_steps}
        if d["flops"] > 0:
            e["tflops"] = d["flops"] / (d["ms"] / 1e3) / 1e12
        if d["bytes"] > 0:
            e["gbs"] = d["bytes"] / (d["ms"] / 1e3) / 1e9
        per_step[k] = e
    g = timing["matmul"]
    achieved = g["flops"] / (g["ms"] / 1e3) / 1e12
    peak = peaks["bf16_tflops_sustained"]
    roofline = {"kernel": "tc_gemm_kernel (tcgen05 bf16 GEMM, all matmul shapes of the step)", "bound": "tensor",
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_source": f"{peak_kind} bf16_tflops_sustained (kernel timed inside a long step)",
                "traffic": GEMM_TRAFFIC_BYTES_PER_LAUNCH,
                "traffic_unit": "bytes per launch (mean over the class's launches in an ncu launch list)",
                "timed_by": f"CUDA events around every launch, {prof_steps} instrumented steps of the same "
                            f"sequence run eagerly right after the timed region ({prof_ms:.1f} ms/step instrumented)",
                "per_launch": {"flops": g["flops"] / g["ops"], "ms": g["ms"] / g["ops"]}}

    # the GEMM rate per SM clock against the sustained peak's own clock
    peak_mhz = peaks.get("bf16_sustained_sm_mhz") or peaks.get("sm_mhz_sustained")
    if clk and clk.get("sm_mhz") and peak_mhz:
        roofline["frac_per_clock"] = (achieved / clk["sm_mhz"]) / (peak / peak_mhz)
        roofline["frac_per_clock_note"] = (f"TFLOP/s per median SM MHz ({clk['sm_mhz']:.0f}) over the sustained "
                                           f"peak per its own SM MHz ({peak_mhz:.0f})")

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded Zipf 1.1 token streams)",
        "config": workload_config(args.workload) if not (args.B or args.accum) else
        {"workload": f"smaller profiling case B={B} x T={T} x {accum} (not the benchmark workload)"},
        "mfu": mfu, "mfu_sustained_peak": mfu_sus,
        "flops_per_token": fpt, "flops_convention": "6N + 6*L*T*C (causal attention, halved score count)",
        "mfu_noncausal": value * (fpt + 6.0 * L * T * C) / (world * peaks["bf16_tflops"] * 1e12),
        "peak_bf16_tflops": peaks["bf16_tflops"], "peak_source": peak_kind,
        "final_loss": loss, "roofline": roofline, "kernels": per_step, "e2e": e2e, "clocks": clk,
        "gpu_launches": launches, "micro_step_launch": "CUDA graph replay (captured on second use)",
    }
    m.close()
    if world == 1 and not (args.B or args.accum) and not args.no_sub_records:
        del d_tok, d_tgt
        torch.cuda.empty_cache()
        subs = {}
        if args.workload == "t1024":
            subs["t512"] = sub_record_workload(G, S, torch, "t512", peaks)
        subs["attention"] = sub_record_attention(G, torch, peaks)
        line["sub_records"] = subs
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(B, T, accum)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------ sub-records

def sub_record_workload(G, S, torch, name, peaks, steps=3, warmup=3):
    """The same optimizer step on another workload of the pages (one GPU):
    tokens/s, MFU and per-class device times, timed like the headline."""
    B, T, accum = WORKLOADS[name]
    tok_per_step = B * T * accum
    stream = torch.cuda.current_stream()
    m = G.GPT2(G.GPT2Config(L, 12, C, V, VP, 1024, B, T, G.GPT2_BF16), seed=4321, stream=stream)
    n = warmup + steps
    toks = np.empty((n, accum, B, T), dtype=np.int32)
    tgts = np.empty_like(toks)
    for s in range(n):
        ids = S.zipf_stream(tok_per_step + 1, V, 1.1, seed=5000 + s)
        for k, (x, y) in enumerate(S.micro_batches(ids, B, T, accum)):
            toks[s, k], tgts[s, k] = x, y
    d_tok, d_tgt = torch.from_numpy(toks).cuda(), torch.from_numpy(tgts).cuda()

    def step(s):
        m.zero_grad()
        for k in range(accum):
            m.forward_backward(d_tok[s, k], d_tgt[s, k], 1.0 / accum)
        m.adamw_step(G.lr_at(1000 + s))

    for s in range(warmup):
        step(s)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s in range(warmup, n):
        step(s)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    m.set_timing(True)
    m.get_timing()
    step(warmup)
    timing = m.get_timing()
    m.set_timing(False)
    m.close()
    value = tok_per_step / (ms / 1e3)
    return {"config": workload_config(name), "value": value, "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
            "warmup": warmup, "mfu": value * flops_per_token(T) / (peaks["bf16_tflops"] * 1e12),
            "kernels_ms_per_step": {k: d["ms"] for k, d in timing.items() if d["ops"]}}


def sub_record_attention(G, torch, peaks, reps=5):
    """The standalone causal attention workload: B=8, H=12, d=64, T in
    {1024, 2048, 4096} and, beyond it, 8192; forward and backward timed
    separately with CUDA events around each call; L2 flushed (256 MB write)
    before every timed call."""
    from decoder_only_transformer_02_b200.synthetic import normal_array
    st = torch.cuda.current_stream()
    flush = torch.empty(64 << 20, dtype=torch.float32, device="cuda")
    out = {"B": 8, "H": 12, "d": 64, "flops_convention": "causal: fwd 2*B*H*T^2*d, bwd 2x fwd",
           "l2": "flushed before every timed call"}
    for T in (1024, 2048, 4096, 8192):
        B, H = 8, 12
        Cc = 64 * H
        qkv = torch.from_numpy(normal_array((B, T, 3 * Cc), 3)).to(torch.bfloat16).cuda()
        do = torch.from_numpy(normal_array((B, T, Cc), 4)).to(torch.bfloat16).cuda()
        o = torch.empty(B, T, Cc, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(B, H, T, dtype=torch.float32, device="cuda")
        dqkv = torch.empty_like(qkv)
        wk = torch.empty(G.attention_workspace_floats(B, T, H), dtype=torch.float32, device="cuda")
        fwd = lambda: G.attention_forward(qkv, o, lse, B, T, H, stream=st)
        bwd = lambda: G.attention_backward(qkv, o, do, lse, dqkv, wk, B, T, H, stream=st)
        for _ in range(3):
            fwd()
            bwd()
        G.check_device_error(st)
        t = {"fwd": 0.0, "bwd": 0.0}
        for _ in range(reps):
            for part, call in (("fwd", fwd), ("bwd", bwd)):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(st)
                call()
                e1.record(st)
                torch.cuda.synchronize()
                t[part] += e0.elapsed_time(e1) / reps
        G.check_device_error(st)
        f = 2.0 * B * H * T * T * 64
        out[f"T{T}"] = {"fwd_ms": t["fwd"], "bwd_ms": t["bwd"], "fwd_tflops": f / (t["fwd"] / 1e3) / 1e12,
                        "bwd_tflops": 2 * f / (t["bwd"] / 1e3) / 1e12,
                        "fwd_frac_of_burst_peak": f / (t["fwd"] / 1e3) / 1e12 / peaks["bf16_tflops"],
                        "bwd_frac_of_burst_peak": 2 * f / (t["bwd"] / 1e3) / 1e12 / peaks["bf16_tflops"]}
        del qkv, do, o, lse, dqkv, wk
    return out


# ------------------------------------------------------- standalone operators

def run_op(args):
    """One operator of the step alone, timed with CUDA events (burst peak).
    matmul: D[M,N] = A B^T in the forward / dgrad / wgrad layout of the model.
    attention: causal fwd+bwd, B=8, H=12, d=64 (the standalone attention workload)."""
    import torch
    from decoder_only_transformer_02_b200 import gpt2 as G
    from decoder_only_transformer_02_b200.synthetic import normal_array
    torch.cuda.set_device(0)
    peaks, kind = load_peaks()
    st = torch.cuda.current_stream()
    out = {"op": args.op, "peak_source": kind}
    if args.op == "matmul":
        M, N, K = (int(x) for x in args.shape.split(","))
        a_mn, b_mn = {"fwd": (0, 0), "dgrad": (0, 1), "wgrad": (1, 1)}[args.layout]
        A = torch.from_numpy(normal_array((K, M) if a_mn else (M, K), 1)).to(torch.bfloat16).cuda()
        Bm = torch.from_numpy(normal_array((K, N) if b_mn else (N, K), 2)).to(torch.bfloat16).cuda()
        epi = args.epi if args.epi >= 0 else (5 if args.layout == "wgrad" else 0)
        f32_out = epi in (1, 2, 5)
        o = torch.zeros(M, N, dtype=torch.float32 if f32_out else torch.bfloat16, device="cuda")
        o2 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda") if epi == 3 else None
        aux = torch.from_numpy(normal_array((M, N), 5)).to(torch.bfloat16).cuda() if epi == 4 else None
        resid = torch.from_numpy(normal_array((M, N), 6)).cuda() if epi == 2 else None
        bias = torch.from_numpy(normal_array((N,), 7)).cuda() if epi in (0, 1, 2, 3) else None
        wsb = G.matmul_workspace_bytes(M, N, K) if epi == 5 else 0
        ws = torch.empty(max(1, wsb // 4), dtype=torch.float32, device="cuda")
        call = lambda: G.matmul_bf16(A, M if a_mn else K, a_mn, Bm, N if b_mn else K, b_mn, M, N, K, epi, bias=bias,
                                     resid=resid, out=o, out2=o2, aux=aux, ldc=N, work=ws if wsb else None,
                                     work_bytes=wsb, stream=st)
        work = 2.0 * M * N * K
        out.update(shape=[M, N, K], layout=args.layout, epilogue=epi, splitk_workspace_bytes=wsb)
    else:
        B, H, T = 8, 12, args.T
        Cc = 64 * H
        qkv = torch.from_numpy(normal_array((B, T, 3 * Cc), 3)).to(torch.bfloat16).cuda()
        do = torch.from_numpy(normal_array((B, T, Cc), 4)).to(torch.bfloat16).cuda()
        o = torch.empty(B, T, Cc, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(B, H, T, dtype=torch.float32, device="cuda")
        dqkv = torch.empty_like(qkv)
        wk = torch.empty(G.attention_workspace_floats(B, T, H), dtype=torch.float32, device="cuda")
        fwd = lambda: G.attention_forward(qkv, o, lse, B, T, H, stream=st)
        bwd = lambda: G.attention_backward(qkv, o, do, lse, dqkv, wk, B, T, H, stream=st)
        if args.part == "fwd":
            call, work = fwd, 2.0 * B * H * T * T * 64
        elif args.part == "bwd":
            fwd()
            call, work = bwd, 4.0 * B * H * T * T * 64
        else:
            call, work = (lambda: (fwd(), bwd())), 6.0 * B * H * T * T * 64
        out.update(B=B, H=H, T=T, d=64, part=args.part, flops_convention="causal: fwd 2*B*H*T^2*d, bwd 2x fwd")
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(args.steps):
        call()
    e1.record(st)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    tf = work / (ms / 1e3) / 1e12
    out.update(ms_per_call=ms, tflops=tf, peak_bf16_tflops=peaks["bf16_tflops"], frac=tf / peaks["bf16_tflops"])
    print(json.dumps(out), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", choices=["matmul", "attention"], default=None)
    ap.add_argument("--shape", default="16384,3072,768")
    ap.add_argument("--layout", choices=["fwd", "dgrad", "wgrad"], default="fwd")
    ap.add_argument("--epi", type=int, default=-1,
                    help="matmul epilogue (0 bf16+bias, 1 fp32, 2 fp32 residual, 3 GELU, 4 GELU', 5 accumulate)")
    ap.add_argument("--T", type=int, default=1024)
    ap.add_argument("--part", choices=["fwd", "bwd", "both"], default="both")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="t1024")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sub-records", action="store_true", help="skip the t512 and attention sub-records")
    ap.add_argument("--B", type=int, default=0, help="override the micro-batch (small profiling cases only)")
    ap.add_argument("--accum", type=int, default=0, help="override the micro-steps (small profiling cases only)")
    args = ap.parse_args()
    if args.op:
        return run_op(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
