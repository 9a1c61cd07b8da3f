"""Benchmark: GPT-2 124M training step (forward + backward + clip + AdamW) on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = gpt_forward_loss + gpt_backward + gpt_clip_adamw_step over one
16 x 1024 batch of synthetic Zipf(1.0) tokens (bf16 operands, fp32 master
weights).  `value` is whole-job train tokens/s with inputs resident in HBM;
`e2e` repeats the measurement through the public API with the batch copied
from pinned host memory and the loss read back every step.  With N > 1 the
N ranks run independent replicas (the step has no exchange on one GPU);
time is the max over ranks.  The CPU oracle is timed on a bounded sample as
`cpu_baseline`; `--impl reference` times only the oracle.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from scratch_decoder_only_b200 import configs as CF  # noqa: E402
from scratch_decoder_only_b200 import synthetic as S  # noqa: E402

WL = CF.GPT2_124M
METRIC = "train tokens/sec (fwd+bwd+AdamW) GPT-2 124M bf16, MFU %; decode tok/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        d["source"] = "measured"
        return d
    d = dict(PEAKS_FALLBACK)
    d["source"] = "fallback"
    return d


def flops_per_token(mc: CF.ModelConfig, T: int) -> float:
    """6 N (matmul weights incl. embeddings) + causal attention 6 L C (T+1)."""
    return 6.0 * mc.num_params() + 6.0 * mc.n_layers * mc.d_model * (T + 1)


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        return self.summarize(self.lines)

    @staticmethod
    def summarize(lines):
        """Median SM clock, max SM clock and the throttle reasons seen active in
        nvidia-smi CSV lines of FIELDS (malformed lines are skipped)."""
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- oracle arm

def _oracle_cfg(mc):
    from oracle import gpt_oracle as O
    return O.OracleConfig(vocab=mc.vocab, vocab_padded=mc.vocab_padded, d_model=mc.d_model,
                          n_heads=mc.n_heads, d_mlp=mc.d_mlp, n_layers=mc.n_layers, max_seq=mc.max_seq,
                          tied=mc.tied)


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


class OracleTrainer:
    """The oracle training the workload's model on a bounded sample per step:
    1 row x `seq` tokens forward + backward, then clip + AdamW over all
    parameters (fp64), with the parameters and the AdamW moments carried from
    step to step.  step(seq) returns (seconds of fwd+bwd, seconds of the
    optimiser)."""

    def __init__(self, wl):
        from oracle import gpt_oracle as O
        self.O, self.wl = O, wl
        self.cfg = _oracle_cfg(wl.model)
        self.p = O.init_params(self.cfg, wl.init_seed).astype(np.float64)
        self.m = np.zeros_like(self.p)
        self.v = np.zeros_like(self.p)
        self.t = 0

    def step(self, seq):
        O, hp = self.O, self.wl.adamw
        tok, tgt, _ = S.make_batch(self.wl, batch=1, seq=seq)
        t0 = time.perf_counter()
        _, g = O.loss_and_grads(self.cfg, self.p, tok, tgt)
        t1 = time.perf_counter()
        self.t += 1
        self.p, self.m, self.v, _, _ = O.clip_adamw_step(self.p, g, self.m, self.v, self.t, hp.lr, hp.beta1,
                                                         hp.beta2, hp.eps, hp.weight_decay, hp.clip_norm)
        t2 = time.perf_counter()
        return t1 - t0, t2 - t1


def oracle_sample_step(seq=256):
    """One bounded oracle step of the workload (the `cpu_baseline` of our arm):
    1 row x `seq` tokens, forward + backward + clip + AdamW over all parameters.
    Returns (seconds, tokens, threads)."""
    tr = OracleTrainer(WL)
    fb, opt = tr.step(seq)
    return fb + opt, seq, _blas_threads()


# wall-clock budget of the reference arm's W + K steps (the sample per step is
# sized from a calibration step to fit it)
REF_BUDGET_S = 150.0
REF_SEQS = (256, 128, 64, 32, 16)


def ref_sample_seq(fb0, opt, per_step_budget, seqs=None):
    """Largest sample length whose predicted step time (forward + backward
    linear in the tokens, measured as fb0 seconds at seqs[0]; the optimiser
    fixed at opt seconds) fits the per-step budget; the smallest one when none
    does."""
    seqs = seqs or REF_SEQS
    for seq in seqs:
        if opt + fb0 * seq / seqs[0] <= per_step_budget:
            return seq
    return seqs[-1]


def run_reference(args, rank, world):
    if rank != 0:
        return
    tr = OracleTrainer(WL)
    # calibration: the first warm-up step, on the longest sample
    fb0, opt = tr.step(REF_SEQS[0])
    seq = ref_sample_seq(fb0, opt, REF_BUDGET_S / max(1, args.warmup - 1 + args.steps))
    for _ in range(args.warmup - 1):
        tr.step(seq)
    times = []
    for _ in range(args.steps):
        fb, op = tr.step(seq)
        times.append(fb + op)
    total = sum(times)
    toks = seq * args.steps
    value = toks / total
    threads = _blas_threads()
    sample = (f"1 row x {seq} tokens of the {WL.name} step per timed step (fwd+bwd+clip+AdamW over all params, "
              f"fp64 numpy), {args.steps} timed steps after {max(1, args.warmup)} warm-up; the sample length "
              f"is chosen from a {REF_SEQS[0]}-token calibration step so the run fits about {REF_BUDGET_S:.0f} s")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WL.name, "global_batch": WL.batch * world, "seq_len": WL.seq,
                                            "parallelism": "none (CPU oracle on the host cores)",
                                            "timed_sample": f"one row x {seq} tokens of this workload per step"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- multi-rank timing

def max_over_ranks(x: float, world: int, device=None) -> float:
    """Slowest rank's value (the job's time): all-reduce MAX over the group."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank_step: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank_step * steps / (max_ms / 1000.0)


# ----------------------------------------------------------------------------- our arm

# DRAM bytes per GEMM launch at the headline size: the ncu capture of a
# batch-4 step (dram__bytes_read.sum + dram__bytes_write.sum over its 147
# gemm_tc_kernel launches: 40.50 MB per launch) scaled by the 4x token count
# (profiles/train_step_gpt2_124m_b4_dram_traffic.txt); the algorithmic bytes
# per launch at batch 16 are 162.0 MB (23.82 GB over the 147 launches).
GEMM_TRAFFIC_BYTES_PER_LAUNCH = 162.0e6
GEMM_ALGO_BYTES_PER_LAUNCH = 162.0e6


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from scratch_decoder_only_b200.gpt import GPT

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    mc = WL.model
    B, T = args.batch or WL.batch, WL.seq
    tok, tgt, _ = S.make_batch(WL, batch=B, seed=WL.data_seed + rank)
    d_tok = torch.from_numpy(tok).to(dev)
    d_tgt = torch.from_numpy(tgt).to(dev)
    model = GPT(mc, WL.init_seed)
    hp = WL.adamw
    loss = torch.zeros(1, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        model.train_step(d_tok, d_tgt, None, hp, loss)

    def barrier():
        if world > 1:
            dist.barrier()

    # warm-up: the first W - 1 steps with per-kernel events (they fill the
    # profiling event pool), the last without, which captures the step's CUDA
    # graph that the timed steps replay
    model.profile_enable(True)
    for _ in range(args.warmup - 1):
        step()
    torch.cuda.synchronize()
    model.profile_enable(False)
    step()
    torch.cuda.synchronize()

    # timed region: K steps, inputs resident in HBM (working set >> L2), no
    # per-kernel events in the stream (they would lengthen the step)
    clocks = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    n0 = model.kernel_launches()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    n1 = model.kernel_launches()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    clk = clocks.stop()
    barrier()

    # second timed region of K steps with a CUDA event pair around every
    # kernel class on the model's stream: per-kernel durations for the roofline
    model.profile_enable(True)
    torch.cuda.synchronize()
    barrier()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms_prof = max_over_ranks(e0.elapsed_time(e1), world, dev)
    barrier()
    prof = model.profile_read()
    model.profile_enable(False)
    final_loss = float(loss.item())
    status = model.status()

    tokens_per_step = B * T
    value = job_throughput(tokens_per_step, args.steps, world, ms)
    ms_step = ms / args.steps
    fpt = flops_per_token(mc, T)
    peaks = load_peaks()
    mfu = fpt * tokens_per_step / (ms_step / 1000.0) / (peaks["bf16_tflops"] * 1e12)
    mfu_sust = fpt * tokens_per_step / (ms_step / 1000.0) / (peaks["bf16_tflops_sustained"] * 1e12)

    # dominant kernel: the tcgen05 GEMMs (all GEMM launches of the step)
    g_ms = sum(v["ms"] for k, v in prof.items() if k.startswith("gemm"))
    g_fl = sum(v["flops"] for k, v in prof.items() if k.startswith("gemm"))
    g_n = sum(v["launches"] for k, v in prof.items() if k.startswith("gemm"))
    achieved = g_fl / (g_ms / 1000.0) / 1e12 if g_ms > 0 else 0.0
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops_sustained"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops_sustained"],
                "traffic": GEMM_TRAFFIC_BYTES_PER_LAUNCH if B == WL.batch else None,
                "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum over the 147 GEMM launches of "
                                  "a batch-4 step, per launch, x4 for batch 16 "
                                  "(profiles/train_step_gpt2_124m_b4_dram_traffic.txt)",
                "algorithmic_bytes_per_launch": GEMM_ALGO_BYTES_PER_LAUNCH,
                "kernel": "gemm_tc (all GEMM launches)", "launches": g_n,
                "avg_launch_ms": g_ms / max(1, g_n), "peak_source": peaks["source"] + " sustained",
                "measured": "CUDA events around each launch in a second timed region of the same K steps "
                            "(ms_per_step %.3f there)" % (ms_prof / args.steps)}
    kernels = {k: {"launches": v["launches"], "ms_per_step": v["ms"] / args.steps,
                   "share_of_step": v["ms"] / ms_prof if ms_prof > 0 else None,
                   "tflops": (v["flops"] / (v["ms"] / 1000) / 1e12) if v["flops"] and v["ms"] else None,
                   "gbs": (v["bytes"] / (v["ms"] / 1000) / 1e9) if v["bytes"] and v["ms"] else None,
                   "hbm_frac": ((v["bytes"] / (v["ms"] / 1000) / 1e9) / peaks["hbm_gbs"])
                   if v["bytes"] and v["ms"] else None}
               for k, v in prof.items()}

    # end-to-end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        h_tok = torch.from_numpy(tok).pin_memory()
        h_tgt = torch.from_numpy(tgt).pin_memory()
        h_loss = torch.zeros(1, dtype=torch.float32).pin_memory()
        for _ in range(1):
            d_tok.copy_(h_tok, non_blocking=True)
            d_tgt.copy_(h_tgt, non_blocking=True)
            step()
            h_loss.copy_(loss, non_blocking=True)
        torch.cuda.synchronize()
        barrier()
        k2 = args.steps   # the same number of steps as the headline region
        e0.record(stream)
        for _ in range(k2):
            d_tok.copy_(h_tok, non_blocking=True)
            d_tgt.copy_(h_tgt, non_blocking=True)
            step()
            h_loss.copy_(loss, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        ms2 = max_over_ranks(e0.elapsed_time(e1), world, dev)
        e2e = {"value": job_throughput(tokens_per_step, k2, world, ms2), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h_tok.numel() * 4 + h_tgt.numel() * 4), "d2h_bytes_per_step": 4,
               "steps": k2}

    # greedy decode (secondary metric) and the other training workloads
    decode = None
    if not args.no_decode:
        decode = bench_decode(torch, dev, args)
    configs = None
    if not args.no_configs and B == WL.batch:
        configs = bench_configs(torch, dev, args)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, n, threads = oracle_sample_step()
        cpu = {"value": n / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": "1 row x 256 tokens of the GPT-2 124M step (fwd+bwd+clip+AdamW over all 124.5M "
                         "params), numpy fp64, one step"}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic (Zipf(1.0) tokens, random init)",
                "config": {"workload": WL.name, "global_batch": B * world, "seq_len": T,
                           "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                           "l2": "working set > L2 (no flush needed)"},
                "mfu": mfu, "mfu_sustained_peak": mfu_sust, "flops_per_step": fpt * tokens_per_step,
                "roofline": roofline, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": n1 - n0, "clocks": clk, "decode": decode, "other_workloads": configs,
                "final_loss": final_loss, "status": status}
        print(json.dumps(line), flush=True)
    model.close()


def bench_configs(torch, dev, args):
    """The other training workloads, timed the same way (CUDA events over K
    steps after W warm-up steps, inputs resident): the tiny byte model (fp32,
    100 timed steps), the packed model (bf16, block-diagonal attention, loss
    scale 2^15) and the byte-level 30M model (bf16, 32 x 1024).  MFU counts 6N
    + attention FLOPs (causal pairs; the packed model's from its documents)."""
    from scratch_decoder_only_b200.gpt import GPT
    peaks = load_peaks()
    res = {}
    for wl, steps in ((CF.TINY_BYTE, 100), (CF.PACKED_SMALL, args.steps), (CF.BYTE_30M, args.steps)):
        mc = wl.model
        tok, tgt, seg = S.make_batch(wl)
        d_tok, d_tgt = torch.from_numpy(tok).to(dev), torch.from_numpy(tgt).to(dev)
        d_seg = None if seg is None else torch.from_numpy(seg).to(dev)
        model = GPT(mc, wl.init_seed)
        loss = torch.zeros(1, dtype=torch.float32, device=dev)
        for _ in range(max(3, args.warmup)):
            model.train_step(d_tok, d_tgt, d_seg, wl.adamw, loss)
        torch.cuda.synchronize()
        times = []
        e = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        e[0].record()
        for i in range(steps):
            model.train_step(d_tok, d_tgt, d_seg, wl.adamw, loss)
            e[i + 1].record()
        torch.cuda.synchronize()
        times = [e[i].elapsed_time(e[i + 1]) for i in range(steps)]
        ms = float(np.mean(times))
        B, T = tok.shape
        if seg is None:
            pairs = B * T * (T + 1) / 2.0
        else:
            pairs = 0.0
            for b in range(B):
                _, counts = np.unique(seg[b], return_counts=True)
                pairs += float(np.sum(counts * (counts + 1) / 2.0))
        flops = 6.0 * mc.num_params() * B * T + 12.0 * mc.n_layers * mc.d_model * pairs
        entry = {"workload": wl.name, "tokens_per_s": B * T / (ms / 1000.0), "ms_per_step": ms,
                 "ms_per_step_median": float(np.median(times)), "steps": steps, "final_loss": float(loss.item()),
                 "flops_per_step": flops}
        if mc.precision != "fp32":
            entry["mfu"] = flops / (ms / 1000.0) / (peaks["bf16_tflops"] * 1e12)
        res[wl.name] = entry
        model.close()
    return res


def decode_bytes(mc: CF.ModelConfig, B: int, Tp: int, n_new: int) -> float:
    """Algorithmic HBM bytes of one greedy decode call: the bf16 matmul weights
    (tied head included) once for the prefill and once per later token, the
    K and V rows of the cache each step reads (bf16), and the fp32 logits."""
    C, F, L, Vp = mc.d_model, mc.d_mlp, mc.n_layers, mc.vocab_padded
    w = 2.0 * (L * (4 * C * C + 2 * F * C) + Vp * C)
    kv = sum(B * L * 2 * (Tp + s + 1) * C * 2.0 for s in range(n_new - 1))
    return n_new * w + kv + n_new * B * Vp * 4.0


def bench_decode(torch, dev, args):
    from scratch_decoder_only_b200.gpt import GPT
    wl = CF.GPT2_DECODE
    res = {}
    hbm = load_peaks()["hbm_gbs"]
    model = GPT(wl.model, wl.init_seed)
    for B in (1, 32):
        prompt = torch.from_numpy(S.make_prompts(wl, B, 128)).to(dev)
        out = torch.empty((B, 384), dtype=torch.int32, device=dev)
        model.greedy_decode(prompt, 8, out[:, :8])
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        model.greedy_decode(prompt, 384, out)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        nbytes = decode_bytes(wl.model, B, 128, 384)
        gbs = nbytes / (ms / 1000.0) / 1e9
        res[f"b{B}"] = {"tok_per_s": B * 384 / (ms / 1000.0), "ms": ms, "bytes": nbytes, "gbs": gbs,
                        "hbm_frac": gbs / hbm,
                        "ceiling_tok_per_s": B * 384 / (nbytes / (hbm * 1e9))}
    model.close()
    return res


def decode_profile(torch, dev, batches=(1, 32), n_new=17):
    """Per-kernel critical path of greedy decode (CUPTI kernel records through
    torch.profiler): with programmatic dependent launch a kernel starts while
    its predecessor drains, so each kernel is charged end_k - end_(k-1) in
    stream order.  The projections are labelled by their place in the step
    (q/k/v with LN1, output, fc with LN2, fc2; then the head with the final
    LN).  Prints a table per batch; not a bench value."""
    from torch.profiler import profile, ProfilerActivity
    from scratch_decoder_only_b200.gpt import GPT
    wl = CF.GPT2_DECODE
    model = GPT(wl.model, wl.init_seed)
    for B in batches:
        prompt = torch.from_numpy(S.make_prompts(wl, B, 128)).to(dev)
        model.greedy_decode(prompt, n_new)
        torch.cuda.synchronize()
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            model.greedy_decode(prompt, n_new)
            torch.cuda.synchronize()
        evs = sorted([e for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA],
                     key=lambda e: e.time_range.start)
        # a greedy step ends with its argmax (which also embeds the next token
        # and advances the step); the first one closes the prefill
        adv = [i for i, e in enumerate(evs) if "argmax" in e.name]
        evs = evs[adv[0] + 1: adv[-1] + 1]   # the replayed steps
        nsteps = len(adv) - 1
        labelled, nmma = [], 0
        names = ["q/k/v + LN1", "out", "fc + LN2", "fc2"]
        for e in evs:
            k = e.name.split("(")[0].replace("void ", "")
            if "argmax" in k:
                nmma = 0
            if "dec_mma" in k:
                k = "dec_mma " + (names[nmma % 4] if nmma < 4 * wl.model.n_layers else "head + final LN")
                nmma += 1
            elif "argmax" in k:
                k = "argmax + next embedding + step advance"
            labelled.append((e.time_range.start, e.time_range.end, k))
        agg, tot = critical_path(labelled)
        order = list(agg)
        tot /= nsteps
        print(f"batch {B}: {nsteps} steps, critical path {tot:.1f} us per step ({B / tot * 1e6:.0f} tok/s)")
        print(f"  {'kernel':48s} {'per step':>9s} {'us/step':>9s} {'us each':>8s} {'share':>6s}")
        for k in sorted(order, key=lambda k: -agg[k][1]):
            n, t, _ = agg[k]
            print(f"  {k[:48]:48s} {n // nsteps:9d} {t / nsteps:9.1f} {t / n:8.2f} {100 * t / nsteps / tot:5.1f}%")
    model.close()


def critical_path(evs):
    """Charge each kernel record end_k - max(end_0..end_(k-1)) in start order:
    with programmatic dependent launch a kernel starts while its predecessor
    drains, so its own duration overstates what it adds to the chain.
    Returns {name: [launches, total_us, summed_duration_us]} and the total."""
    agg = {}
    prev_end = evs[0][0] if evs else 0.0
    for start, end, name in evs:
        d = max(0.0, end - prev_end)
        prev_end = max(prev_end, end)
        a = agg.setdefault(name, [0, 0.0, 0.0])
        a[0] += 1
        a[1] += d
        a[2] += end - start
    return agg, sum(v[1] for v in agg.values())


def train_profile(torch, dev, steps=3):
    """Per-kernel critical path of the graph-replayed training step (CUPTI
    kernel records through torch.profiler), headline workload.  Prints a
    table; not a bench value."""
    from torch.profiler import profile, ProfilerActivity
    from scratch_decoder_only_b200.gpt import GPT
    tok, tgt, _ = S.make_batch(WL)
    d_tok, d_tgt = torch.from_numpy(tok).to(dev), torch.from_numpy(tgt).to(dev)
    model = GPT(WL.model, WL.init_seed)
    loss = torch.zeros(1, dtype=torch.float32, device=dev)
    for _ in range(3):   # the first call captures the step's graph
        model.train_step(d_tok, d_tgt, None, WL.adamw, loss)
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        for _ in range(steps):
            model.train_step(d_tok, d_tgt, None, WL.adamw, loss)
        torch.cuda.synchronize()
    evs = sorted(((e.time_range.start, e.time_range.end, e.name.split("(")[0].replace("void ", ""))
                  for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA), key=lambda r: r[0])
    agg, tot = critical_path(evs)
    print(f"{WL.name}: {steps} steps, critical path {tot / steps:.1f} us per step")
    print(f"  {'kernel':60s} {'per step':>8s} {'us/step':>9s} {'us each':>8s} {'dur each':>9s}")
    for k, (n, t, dur) in sorted(agg.items(), key=lambda kv: -kv[1][1]):
        print(f"  {k[:60]:60s} {n // steps:8d} {t / steps:9.1f} {t / n:8.2f} {dur / n:9.2f}")
    model.close()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the other training workloads")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=None, help="override the batch (profiling of small cases)")
    ap.add_argument("--decode-profile", action="store_true",
                    help="print the per-kernel critical path of greedy decode and exit (no bench line)")
    ap.add_argument("--train-profile", action="store_true",
                    help="print the per-kernel critical path of the training step and exit (no bench line)")
    args = ap.parse_args()
    if args.decode_profile:
        import torch
        decode_profile(torch, torch.device("cuda", 0))
        return
    if args.train_profile:
        import torch
        torch.cuda.set_device(0)
        train_profile(torch, torch.device("cuda", 0))
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
