"""Decode throughput of the B200 decode-step library on the 7B-shape Llama-2 workload.

One step = six single-token decode steps through the C ABI: the fp32 path and
the Q8_0 (GS=64) path, each at positions 0, 512 and 2048 of a KV cache
prefilled with N(0,1), token 1 (dim 4096, hidden 11008, 32 layers, 32 heads,
32 KV heads, vocab 32000, seq_len 4096, untied classifier, weights N(0,0.02)
from seed 3; both weight sets resident).  value = tokens decoded per second,
timed on the device with CUDA events between barriers, max over ranks.  Each
rank (one per GPU) runs an independent replica: batch-1 decode does not shard.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--impl reference times the CPU oracle on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
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

import synth  # noqa: E402

SPEC = synth.L7B  # --layers N swaps in the same widths with N layers (small profiling case)
GS = 64
POSITIONS = (0, 512, 2048)
TOKEN = 1
METRIC = "decode tokens/s at batch 1 (fp32 & Q8_0) on 1 B200; achieved HBM GB/s vs peak"
UNIT = "tokens/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
# fp32 FMA peak from unit counts and clock: 148 SMs x 128 FP32 lanes x 2 flop x 1.965 GHz
FP32_FMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


# ------------------------------------------------------------ byte accounting --

def bytes_per_token(q80: bool, pos: int, spec=None, gs=GS) -> float:
    """Algorithmic bytes of one decode step: every weight once, the KV cache for
    positions 0..pos (K and V, fp32), the embedding row; activations ignored."""
    d, h, L, H, Hkv, V, S = (spec or SPEC).cfg
    kvd = Hkv * (d // H)
    kv = 8.0 * L * (pos + 1) * kvd
    mats = L * (2 * d * d + 2 * d * kvd + 3 * d * h) + V * d
    if not q80:
        return 4.0 * (mats + L * 2 * d + d + d) + kv
    return (1 + 4.0 / gs) * (mats + d) + 4.0 * (2 * L * d + d) + kv


def q40_bytes_per_token(pos: int, spec=None, gs=GS) -> float:
    """Algorithmic bytes of one Q4_0 decode step: every weight once as 4-bit codes
    plus one fp32 scale per group, the embedding row (int8-wide codes and scales),
    the norm gains, the fp32 KV cache for positions 0..pos."""
    d, h, L, H, Hkv, V, S = (spec or SPEC).cfg
    kvd = Hkv * (d // H)
    mats = L * (2 * d * d + 2 * d * kvd + 3 * d * h) + V * d
    return (0.5 + 4.0 / gs) * mats + (1 + 4.0 / gs) * d + 4.0 * (2 * L * d + d) + 8.0 * L * (pos + 1) * kvd


def kernel_bytes(kind: int, q80, pos: int, spec=None, gs=GS) -> float:
    """Algorithmic bytes of one launch of step kernel `kind` (the numbering of
    l2c_time_kernel: 0 RMSNorm+QKV+RoPE, 1 attention, 2 wo, 3 RMSNorm+W1/W3+SwiGLU,
    4 W2, 5 final RMSNorm+classifier): its weights once (Q8_0: codes plus fp32
    group scales), plus the vectors it reads and writes; attention: K and V of
    positions 0..pos, q and the output.  q80: 0 fp32, 1 Q8_0, 2 Q4_0 (half a
    byte per weight plus the scales)."""
    spec = spec or SPEC
    d, h, L, H, Hkv, V, S = spec.cfg
    kvd = Hkv * (d // H)
    bpw = ((0.5 if int(q80) == 2 else 1.0) + 4.0 / gs) if q80 else 4.0
    if kind == 0:
        return (d + 2 * kvd) * d * bpw + 4.0 * (2 * d + d + 2 * kvd)
    if kind == 1:
        return 8.0 * (pos + 1) * kvd + 4.0 * 2 * d
    if kind == 2:
        return d * d * bpw + 4.0 * 3 * d
    if kind == 3:
        return 2 * h * d * bpw + 4.0 * (2 * d + h)
    if kind == 4:
        return d * h * bpw + 4.0 * (h + 2 * d)
    return V * d * bpw + 4.0 * (2 * d + V)


KERNEL_NAMES = ("rmsnorm_qkv_rope", "attention", "wo_residual", "rmsnorm_w13_swiglu", "w2_residual",
                "final_norm_classifier")


def pct(xs, q):
    xs = sorted(xs)
    i = (len(xs) - 1) * q
    lo, hi = int(i), min(int(i) + 1, len(xs) - 1)
    return xs[lo] + (xs[hi] - xs[lo]) * (i - lo)


def w13_bytes(q80: bool, spec=None, gs=GS) -> float:
    """Algorithmic bytes of one W1/W3 launch: both weight matrices, the RMSNorm
    gain, the input x and the output hb."""
    spec = spec or SPEC
    d, h = spec.dim, spec.hidden_dim
    w = 2 * h * d * (1 + 4.0 / gs) if q80 else 2 * h * d * 4.0
    return w + 4.0 * (2 * d + h)


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def traffic_record(kernel_key: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the kernel source as it is now (else None)."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    src = os.path.join(ROOT, "decode_llama_step_02_b200", "csrc", "kernels.cuh")
    try:
        rec = json.load(open(p))
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
        if rec.get("kernels_cuh_sha256") != sha:
            return None
        return rec["kernels"][kernel_key]["dram_bytes_per_launch_full"]
    except Exception:
        return None


# ------------------------------------------------------------------- clocks --

class ClockSampler:
    """nvidia-smi clocks and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            # nvidia-smi takes a moment to start: let its first sample arrive before
            # the timed region opens, then keep only samples taken inside it
            t_end = time.time() + 5.0
            while not self.rows and time.time() < t_end and self.proc.poll() is None:
                time.sleep(0.02)
            self.rows.clear()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.rows.append(parts)

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


# ------------------------------------------------------------------ setup ----

def device_blob(torch, spec=None, chunk=1 << 27):
    """The seeded fp32 blob generated on the host in chunks and uploaded."""
    spec = spec or SPEC
    n = synth.blob_floats(spec)
    dev = torch.empty(n, dtype=torch.float32, device="cuda")
    host = torch.empty(chunk, dtype=torch.float32).pin_memory()
    hn = host.numpy()
    for s in range(0, n, chunk):
        m = min(chunk, n - s)
        synth.blob_into(spec, hn[:m], start=s)
        dev[s:s + m].copy_(host[:m], non_blocking=False)
    return dev


def make_decoder(torch, l2c):
    blob = device_blob(torch)
    dec = l2c.Decoder(SPEC.cfg, blob, SPEC.shared_weights)
    del blob
    torch.cuda.empty_cache()
    dec.enable_q80(GS)
    k, v = synth.kv_prefill(SPEC, seq=0, n_pos=max(POSITIONS))
    dec.kv_load(k, v)
    del k, v
    return dec


def one_step(dec):
    for q80 in (False, True):
        for p in POSITIONS:
            dec.forward_ptr(TOKEN, p, q80)


# ----------------------------------------------------------- CPU oracle ------

def oracle_sample(steps_per_variant=3, pos=512):
    """The CPU oracle on the 7B-shape model at `pos`: `steps_per_variant` fp32
    steps, then as many Q8_0 steps.  Returns (tokens, seconds, setup seconds,
    seconds per fp32 step, seconds per Q8_0 step)."""
    import oracle
    t0 = time.perf_counter()
    blob = synth.blob(SPEC)
    m = oracle.Model(SPEC.cfg, blob, SPEC.shared_weights)
    k, v = synth.kv_prefill(SPEC, seq=0, n_pos=pos)
    m.kv_load(k, v)
    del k, v
    m.enable_q80(GS)
    setup = time.perf_counter() - t0
    per = []
    for q80 in (False, True):
        t1 = time.perf_counter()
        for _ in range(steps_per_variant):
            m.forward(TOKEN, pos, q80=q80)
        per.append((time.perf_counter() - t1) / steps_per_variant)
    m.close()
    return 2 * steps_per_variant, steps_per_variant * (per[0] + per[1]), setup, per[0], per[1]


# ---------------------------------------------------------- ranks (N > 1) ----

def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The largest of every rank's x (all ranks call it; one all-reduce)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, seconds_max: float) -> float:
    """Units per second of the whole job: every rank's units over the slowest rank's time."""
    return units_per_rank * world / seconds_max


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# ------------------------------------------------------------------ arms -----

def run_reference(args, rank):
    """The CPU oracle as the reference arm: each step decodes one fp32 and one
    Q8_0 token of the 7B-shape model at pos 512 on the host cores."""
    if rank != 0:
        return 0
    import oracle
    cores = host_cores()
    blob = synth.blob(SPEC)
    m = oracle.Model(SPEC.cfg, blob, SPEC.shared_weights)
    k, v = synth.kv_prefill(SPEC, seq=0, n_pos=512)
    m.kv_load(k, v)
    del k, v
    m.enable_q80(GS)
    for _ in range(args.warmup):
        m.forward(TOKEN, 512, q80=False)
        m.forward(TOKEN, 512, q80=True)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        m.forward(TOKEN, 512, q80=False)
        m.forward(TOKEN, 512, q80=True)
    dt = time.perf_counter() - t0
    val = 2 * args.steps / dt
    sample = "each step: one fp32 and one Q8_0 decode step of the 7B-shape model at pos 512 (KV prefilled N(0,1))"
    out = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (CPU oracle)",
        "data": "synthetic", "config": workload_config(),
        "cpu_baseline": {"value": val, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)
    return 0


def workload_config():
    return {
        "workload": "Llama-2 7B-shape single-token decode, batch 1: dim 4096, hidden 11008, 32 layers, "
                    "32 heads, 32 KV heads, vocab 32000, seq_len 4096, untied classifier; fp32 and Q8_0 "
                    "GS=64 weight sets resident; KV cache prefilled N(0,1); token 1 at positions 0, 512, 2048",
        "tokens_per_step": 2 * len(POSITIONS),
        "positions": list(POSITIONS),
        "variants": ["fp32", "q8_0 gs=64"],
        "l2": "inputs larger than L2 (33.9 GB of weights streamed per step)",
        "parallelism": "replicas (one independent decoder per GPU)",
    }


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import __graft_entry__
    __graft_entry__.build()
    import decode_llama_step_02_b200 as l2c

    torch.cuda.set_device(local_rank)
    dec = make_decoder(torch, l2c)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()


    # warm-up (captures both step graphs)
    for _ in range(max(args.warmup, 1)):
        one_step(dec)
    dec.sync()

    # ---- device-timed region
    launches_per_token = 1 + 5 * SPEC.n_layers + 1
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            one_step(dec)
        e1.record(stream)
        torch.cuda.synchronize()
    barrier()
    dec.sync()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    tokens = 2 * len(POSITIONS) * args.steps * world
    value = whole_job_rate(2 * len(POSITIONS) * args.steps, world, ms / 1e3)

    # ---- per (variant, position) breakdown: every replay timed on its own
    peak, peak_kind = measured_peak()
    reps = max(50, args.steps)
    variants = {}
    for q80 in (False, True):
        for p in POSITIONS:
            for _ in range(3):
                dec.forward_ptr(TOKEN, p, q80)
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
            torch.cuda.synchronize()
            for a, b in evs:
                a.record(stream)
                dec.forward_ptr(TOKEN, p, q80)
                b.record(stream)
            torch.cuda.synchronize()
            ts = [a.elapsed_time(b) for a, b in evs]
            t = statistics.median(ts)
            by = bytes_per_token(q80, p)
            variants[f"{'q8_0' if q80 else 'fp32'}@pos{p}"] = {
                "ms_per_token_median": t, "ms_p10": pct(ts, 0.1), "ms_p90": pct(ts, 0.9), "replays": reps,
                "tokens_per_s": 1e3 / t, "bytes_per_token": by,
                "gbs": by / t / 1e6, "frac_of_measured_hbm": by / t / 1e6 / peak,
                "frac_of_8tbs_roofline": by / t / 1e6 / NOMINAL_HBM_GBS,
                "roofline_tokens_per_s_8tbs": NOMINAL_HBM_GBS * 1e9 / by,
            }
    dec.sync()

    # ---- every kernel of the step, run alone back to back (l2c_time_kernel:
    # 2 * n_layers launches on the handle's stream, launch i on layer i % n_layers,
    # programmatic dependent launch between them as in the step graph)
    kpos = POSITIONS[-1]
    kernels = {}
    for q80 in (False, True):
        dec.forward_ptr(TOKEN, kpos, q80)  # the handle's state: position kpos
        rows = {}
        for kind, name in enumerate(KERNEL_NAMES):
            iters = 2 * SPEC.n_layers if kind != 5 else 8
            dec.time_kernel(kind, q80, max(4, iters // 4))  # warm
            kms = dec.time_kernel(kind, q80, iters)
            by = kernel_bytes(kind, q80, kpos)
            rows[name] = {"avg_launch_us": 1e3 * kms, "bytes_per_launch": by, "gbs": by / kms / 1e6,
                          "frac_of_measured_hbm": by / kms / 1e6 / peak, "launches_timed": iters}
        kernels["q8_0" if q80 else "fp32"] = rows
    kernels["note"] = (f"each kernel alone, back to back over the layers' weights, at pos {kpos} "
                       f"(attention reads K/V of positions 0..{kpos})")

    # ---- dominant kernel: RMSNorm + W1/W3 + SwiGLU (44% of the fp32 step's bytes)
    def kernel_roofline(q80: bool):
        row = kernels["q8_0" if q80 else "fp32"]["rmsnorm_w13_swiglu"]
        avg_ms = row["avg_launch_us"] / 1e3
        ach = w13_bytes(q80) / avg_ms / 1e6
        key = "k_gemv_q8<W13>" if q80 else "k_gemv_f32<W13>"
        return {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                "traffic": traffic_record(key), "kernel": key, "algorithmic_bytes_per_launch": w13_bytes(q80),
                "avg_launch_ms": avg_ms, "peak_kind": peak_kind}

    roof = kernel_roofline(False)
    roof_q8 = kernel_roofline(True)

    # ---- end to end through the public API: per token, logits back to pinned host memory
    host = torch.empty(SPEC.vocab_size, dtype=torch.float32).pin_memory()
    barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for q80 in (False, True):
            for p in POSITIONS:
                lg = dec.forward(TOKEN, p, q80)
                host.copy_(lg, non_blocking=True)
        torch.cuda.synchronize()
    e2e_s = max_over_ranks(time.perf_counter() - t0, world)
    barrier()
    e2e = {"value": tokens / e2e_s, "unit": UNIT,
           "h2d_bytes_per_step": 2 * len(POSITIONS) * 8,          # token + position per decode step
           "d2h_bytes_per_step": 2 * len(POSITIONS) * SPEC.vocab_size * 4}

    # ---- the hot path's other rows on this GPU, device-timed, not part of `value`:
    # a 128-token prompt on this decoder (l2c_prefill), then the GQA-7B batch of
    # 32 sequences (l2c_forward_batch) on a second model once this one is freed
    def ev():
        return torch.cuda.Event(enable_timing=True)

    rows = {}
    if not args.no_rows:
        rows["prefill_7b_128_tokens"] = measure_prefill(torch, dec, ev, stream)
        rows["q4_0_weights"] = measure_q40(torch, dec, stream, peak)
        rows["q8_0_int8_kv_cache"] = measure_kv8(torch, dec, stream, peak)
    dec.close()
    dec = None
    torch.cuda.empty_cache()
    if not args.no_rows:
        rows["batch_gqa7b_32_sequences"] = measure_batch(torch, l2c, ev, stream, peak, args.layers, reps=5)

    # ---- CPU oracle beside it (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ntok, dt, setup, s32, s8 = oracle_sample()
        cpu = {"value": ntok / dt, "unit": UNIT, "cores": host_cores(), "kind": "oracle",
               "sample": f"3 fp32 and 3 Q8_0 decode steps of the 7B-shape model at pos 512 "
                         f"({dt:.1f} s of compute: {s32:.2f} s per fp32 step, {s8:.2f} s per Q8_0 step; "
                         f"{setup:.0f} s to generate the weights, prefill the cache and quantize, not counted)",
               "s_per_step_fp32": s32, "s_per_step_q8_0": s8}

    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32 | i8*i8->i32 with f64 group sums", "data": "synthetic",
        "config": workload_config(), "roofline": roof, "roofline_q8_0": roof_q8,
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_token * 2 * len(POSITIONS) * args.steps,
        "clocks": clk.summary(), "variants": variants, "kernels": kernels, "rows": rows,
        "context": "pages' CPU figures: ~110 tok/s 15M int8 on an M1 MacBook Air; ~0.8 tok/s 7B fp32 on a "
                   "16-core Ryzen 9 7950X; ~4 tok/s 7B on a 96-thread server",
    }
    if rank == 0:
        print(json.dumps(out), flush=True)
    return 0


# ------------------------------------------------- supplementary configs ----

def run_extra(args):
    """The other workloads of the measurement plan, one JSON line each (not bench
    lines): tiny, 15M and 110M decoded with forced uniform tokens over all their
    positions, timed in buckets of 64 positions; the GQA-7B batch of 32 ragged
    sequences (Q8_0 GS=64) as one batched step."""
    import torch

    import __graft_entry__
    __graft_entry__.build()
    import decode_llama_step_02_b200 as l2c

    peak, peak_kind = measured_peak()
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    stream = torch.cuda.current_stream()

    def ev():
        return torch.cuda.Event(enable_timing=True)

    small = ((synth.TINY, 0, (False,)), (synth.M15, 32, (False, True)), (synth.M110, 64, (False, True)))
    for spec, gs, variants in (small if args.extra in ("all", "small") else ()):
        dec = l2c.Decoder(spec.cfg, torch.from_numpy(synth.blob(spec)).cuda(), spec.shared_weights)
        if gs:
            dec.enable_q80(gs)
        S = spec.seq_len
        toks = synth.tokens(spec.seed, 2, S, spec.vocab_size)
        for q80 in variants:
            for p in range(8):  # warm-up, captures the step graph
                dec.forward_ptr(int(toks[p]), p, q80)
            dec.sync()
            buckets = []
            for b0 in range(0, S, 64):
                a, b = ev(), ev()
                a.record(stream)
                for p in range(b0, min(S, b0 + 64)):
                    dec.forward_ptr(int(toks[p]), p, q80)
                b.record(stream)
                torch.cuda.synchronize()
                n = min(S, b0 + 64) - b0
                us = 1e3 * a.elapsed_time(b) / n
                by = bytes_per_token(q80, b0 + n // 2, spec, gs or GS)
                buckets.append({"pos": [b0, b0 + n - 1], "us_per_token": us, "tokens_per_s": 1e6 / us,
                                "bytes_per_token_mid": by, "gbs": by / us / 1e3})
            dec.sync()
            # secondary datum: the same positions with L2 flushed before each
            # timed step (a write of twice the L2 size outside the events)
            flush = torch.empty(2 * l2 // 4, dtype=torch.float32, device="cuda")
            flushed = []
            for b0 in range(0, S, 64):
                ts = []
                for p in range(b0, min(S, b0 + 64), 8):
                    flush.fill_(1.0)
                    a, b = ev(), ev()
                    a.record(stream)
                    dec.forward_ptr(int(toks[p]), p, q80)
                    b.record(stream)
                    torch.cuda.synchronize()
                    ts.append(1e3 * a.elapsed_time(b))
                flushed.append({"pos": [b0, min(S, b0 + 64) - 1], "us_per_token_median": statistics.median(ts),
                                "steps": len(ts)})
            del flush
            dec.sync()
            weights = bytes_per_token(q80, 0, spec, gs or GS)
            resident = weights < l2
            for bk in buckets:
                bk["frac_of_measured_hbm"] = None if resident else bk["gbs"] / peak
            print(json.dumps({
                "extra": True, "config": spec.name, "variant": f"q8_0 gs={gs}" if q80 else "fp32",
                "shape": dict(zip(("dim", "hidden", "layers", "heads", "kv_heads", "vocab", "seq_len"), spec.cfg)),
                "inputs": "forced tokens uniform in [0, vocab) (stream 2), positions 0..seq_len-1 in order",
                "timing": "CUDA events around 64 consecutive decode steps through the C ABI, host launch included",
                "l2_resident": bool(resident), "l2_bytes": l2, "peak_gbs": peak, "peak_kind": peak_kind,
                "buckets": buckets,
                "l2_flushed": {"how": "2x L2 bytes written before each timed step; events around the step only",
                               "buckets": flushed}}), flush=True)
        dec.close()

    if args.extra in ("all", "prefill"):
        run_prefill(torch, l2c, ev, stream)
    if args.extra not in ("all", "batch"):
        return 0
    for line in measure_batch(torch, l2c, ev, stream, peak, args.layers, reps=10):
        print(json.dumps(line), flush=True)
    return 0


def measure_batch(torch, l2c, ev, stream, peak, layers=0, reps=10):
    """GQA-7B, 32 sequences at positions U[0, 2047] on caches prefilled N(0,1):
    one batched step (l2c_forward_batch), Q8_0 and fp32, timed with CUDA events
    around `reps` steps.  Returns one record per variant."""
    spec, B = synth.GQA7B, 32
    if layers:
        spec = dataclasses.replace(spec, name=f"GQA-7B-width-{layers}L", n_layers=layers)
    blob = device_blob(torch, spec)
    dec = l2c.Decoder(spec.cfg, blob, spec.shared_weights, max_batch=B)
    del blob
    torch.cuda.empty_cache()
    dec.enable_q80(GS)
    toks = synth.tokens(spec.seed, 0, B, spec.vocab_size)
    pos = synth.positions(spec.seed, 0, B, spec.seq_len)
    for sq in range(B):
        if pos[sq]:
            k, v = synth.kv_prefill(spec, seq=sq, n_pos=int(pos[sq]))
            dec.kv_load(k, v, seq=sq)
            del k, v
    tk = torch.from_numpy(toks.astype(np.int32)).cuda()
    ps = torch.from_numpy(pos.astype(np.int32)).cuda()
    out = torch.empty((B, spec.vocab_size), dtype=torch.float32, device="cuda")
    d, h, L, H, Hkv, V, S = spec.cfg
    kvd = Hkv * (d // H)
    kvbytes = float(sum(8.0 * L * (int(p) + 1) * kvd for p in pos))
    lines = []
    for q80 in (True, False):
        for _ in range(3):
            dec.forward_batch(tk, ps, out, q80=q80)
        dec.sync()
        a, b = ev(), ev()
        a.record(stream)
        for _ in range(reps):
            dec.forward_batch(tk, ps, out, q80=q80)
        b.record(stream)
        torch.cuda.synchronize()
        dec.sync()
        ms = a.elapsed_time(b) / reps
        wbytes = bytes_per_token(q80, -1, spec, GS)  # weights only (pos -1: no KV)
        by = wbytes + kvbytes
        line = {
            "extra": True, "config": spec.name + " batch 32", "variant": f"q8_0 gs={GS}" if q80 else "fp32",
            "ms_per_step": ms, "tokens_per_s": B / ms * 1e3, "bytes_per_step": by, "weight_bytes": wbytes,
            "kv_bytes": kvbytes, "gbs": by / ms / 1e6, "frac_of_measured_hbm": by / ms / 1e6 / peak,
            "frac_of_8tbs": by / ms / 1e6 / NOMINAL_HBM_GBS,
            "inputs": "tokens uniform (stream 2), positions uniform in [0, 2047] (stream 3), caches prefilled N(0,1)",
            "timing": f"CUDA events around {reps} batched steps (l2c_forward_batch), device-resident inputs"}
        if not q80:
            fl = 2.0 * B * matvec_params(spec)
            line["gemm_flops_per_step"] = fl
            line["gemm_tflops"] = fl / ms / 1e9
            line["frac_of_fp32_fma_peak"] = fl / ms / 1e9 / FP32_FMA_TFLOPS
        lines.append(line)
    dec.close()
    return lines


def matvec_params(spec) -> float:
    """Weights one token multiplies: every matvec of the step (classifier included)."""
    d, h, L, H, Hkv, V, S = spec.cfg
    kvd = Hkv * (d // H)
    return float(L * (2 * d * d + 2 * d * kvd + 3 * d * h) + V * d)


def run_prefill(torch, l2c, ev, stream):
    """A 128-token prompt on the 7B shape, fp32 and Q8_0 GS=64 (one JSON line each)."""
    blob = device_blob(torch)
    dec = l2c.Decoder(SPEC.cfg, blob, SPEC.shared_weights)
    del blob
    torch.cuda.empty_cache()
    dec.enable_q80(GS)
    for line in measure_prefill(torch, dec, ev, stream):
        print(json.dumps(line), flush=True)
    dec.close()


def kv8_bytes_per_token(pos: int, spec=None, gs=GS) -> float:
    """Algorithmic bytes of one Q8_0 step reading the int8 KV cache: the Q8_0
    weights and vectors, plus codes (1 byte) and one fp32 scale per head row
    for K and V of positions 0..pos."""
    d, h, L, H, Hkv, V, S = (spec or SPEC).cfg
    kvd = Hkv * (d // H)
    return bytes_per_token(True, -1, spec, gs) + 2.0 * L * (pos + 1) * (kvd + 4 * Hkv)


def measure_kv8(torch, dec, stream, peak, reps=20):
    """The Q8_0 step with the int8 KV cache (l2c_enable_kv8: every row already in
    the cache is quantized) at the bench positions: the median of `reps`
    individually timed graph replays per position.  Leaves the cache on."""
    dec.enable_kv8()
    out = {}
    for p in POSITIONS:
        for _ in range(3):
            dec.forward_ptr(TOKEN, p, True)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        torch.cuda.synchronize()
        for a, b in evs:
            a.record(stream)
            dec.forward_ptr(TOKEN, p, True)
            b.record(stream)
        torch.cuda.synchronize()
        t = statistics.median([a.elapsed_time(b) for a, b in evs])
        by = kv8_bytes_per_token(p)
        out[f"pos{p}"] = {"ms_per_token_median": t, "tokens_per_s": 1e3 / t, "bytes_per_token": by,
                          "gbs": by / t / 1e6, "frac_of_measured_hbm": by / t / 1e6 / peak,
                          "frac_of_8tbs_roofline": by / t / 1e6 / NOMINAL_HBM_GBS, "replays": reps}
    dec.sync()
    return out


def measure_q40(torch, dec, stream, peak, reps=20):
    """The Q4_0 step (l2c_enable_q40, GS as the Q8_0 step) at the bench positions:
    the median of `reps` individually timed graph replays per position, and each
    kernel alone at the last position (l2c_time_kernel), as for the main variants."""
    dec.enable_q40(GS)
    out = {}
    for p in POSITIONS:
        for _ in range(3):
            dec.forward_ptr(TOKEN, p, q40=True)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        torch.cuda.synchronize()
        for a, b in evs:
            a.record(stream)
            dec.forward_ptr(TOKEN, p, q40=True)
            b.record(stream)
        torch.cuda.synchronize()
        ts = [a.elapsed_time(b) for a, b in evs]
        t = statistics.median(ts)
        by = q40_bytes_per_token(p)
        out[f"pos{p}"] = {"ms_per_token_median": t, "ms_p10": pct(ts, 0.1), "ms_p90": pct(ts, 0.9),
                          "tokens_per_s": 1e3 / t, "bytes_per_token": by,
                          "gbs": by / t / 1e6, "frac_of_measured_hbm": by / t / 1e6 / peak,
                          "frac_of_8tbs_roofline": by / t / 1e6 / NOMINAL_HBM_GBS, "replays": reps}
    kpos = POSITIONS[-1]
    dec.forward_ptr(TOKEN, kpos, q40=True)
    kern = {}
    for kind, name in enumerate(KERNEL_NAMES):
        iters = 2 * SPEC.n_layers if kind != 5 else 8
        dec.time_kernel(kind, 2, max(4, iters // 4))  # warm
        kms = dec.time_kernel(kind, 2, iters)
        by = kernel_bytes(kind, 2, kpos)
        kern[name] = {"avg_launch_us": 1e3 * kms, "bytes_per_launch": by, "gbs": by / kms / 1e6,
                      "frac_of_measured_hbm": by / kms / 1e6 / peak, "launches_timed": iters}
    out["kernels_pos%d" % kpos] = kern
    # the Q4_0 W1/W3 kernel against the copy peak (weights at half a byte plus the scales)
    d, h = SPEC.dim, SPEC.hidden_dim
    wb = 2 * h * d * (0.5 + 4.0 / GS) + 4.0 * (2 * d + h)
    avg_ms = kern["rmsnorm_w13_swiglu"]["avg_launch_us"] / 1e3
    out["roofline_w13"] = {"bound": "hbm", "achieved": wb / avg_ms / 1e6, "peak": peak, "unit": "GB/s",
                           "frac": wb / avg_ms / 1e6 / peak, "traffic": traffic_record("k_gemv_q8<W13,Q4_0>"),
                           "kernel": "k_gemv_q8<W13,Q4_0>", "algorithmic_bytes_per_launch": wb,
                           "avg_launch_ms": avg_ms}
    out["gs"] = GS
    dec.sync()
    return out


def measure_prefill(torch, dec, ev, stream, n=128, reps=3):
    """A prompt of n tokens at positions 0..n-1 of sequence 0 (l2c_prefill: GEMM
    chunks of 32 tokens), fp32 and Q8_0, timed with CUDA events around whole calls
    (median of reps).  Overwrites the cache rows 0..n-1.  Returns one record per
    variant."""
    toks = synth.tokens(SPEC.seed, 4, n, SPEC.vocab_size)
    last = torch.empty(SPEC.vocab_size, dtype=torch.float32, device="cuda")
    lines = []
    for q80 in (False, True):
        dec.prefill(toks, 0, q80=q80, logits_last=last)  # warm-up: buffers, module loading
        ts = []
        for _ in range(reps):
            a, b = ev(), ev()
            a.record(stream)
            dec.prefill(toks, 0, q80=q80, logits_last=last)
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        ms = statistics.median(ts)
        fl = 2.0 * n * matvec_params(SPEC)
        line = {"extra": True, "config": SPEC.name + " prefill", "variant": f"q8_0 gs={GS}" if q80 else "fp32",
                "prompt_tokens": n, "chunks": (n + 31) // 32, "ms_per_prompt": ms, "tokens_per_s": n / ms * 1e3,
                "matvec_flops": fl, "tflops": fl / ms / 1e9,
                "decode_equivalent": "the same prompt fed token by token costs n decode steps (see the bench line)",
                "timing": f"CUDA events around l2c_prefill, median of {reps}; weights larger than L2"}
        if not q80:
            line["frac_of_fp32_fma_peak"] = fl / ms / 1e9 / FP32_FMA_TFLOPS
        lines.append(line)
    return lines


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rows", action="store_true",
                    help="skip the prefill and batched-step records of the bench line")
    ap.add_argument("--extra", nargs="?", const="all", choices=("all", "small", "batch", "prefill"),
                    help="the other workloads (small: tiny, 15M, 110M position curves; batch: GQA-7B batch 32; "
                         "prefill: a 128-token 7B prompt), not bench lines")
    ap.add_argument("--layers", type=int, default=0,
                    help="profiling case: the 7B widths with this many layers (not a bench line)")
    args = ap.parse_args()
    if args.layers:
        global SPEC
        SPEC = dataclasses.replace(synth.L7B, name=f"7B-width-{args.layers}L", n_layers=args.layers)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        return run_reference(args, rank)
    if args.extra:
        return run_extra(args)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    try:
        return run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
