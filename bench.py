#!/usr/bin/env python3
"""Benchmark: generated tokens/s of early-skipping generation on B200.

One bench step = one whole generation (esd_generate) of the workload: prompt
of P tokens + G masked positions, blocks of `block` positions, `n_unmask`
tokens per denoising step; each block starts with a dense refresh step and
continues with early-skipping sparse steps (score, top-k, gather, sparse
layers with partial attention and K/V scatter, fused head, remask).

Default workload: the 8B-class bf16 model at batch 1 (32 layers, d 4096, 32x128
heads, FFN 12288, vocab 126464), prompt 512 + 256 generated tokens in blocks of
32, 1 token per step (256 steps), skip layer 4, keep 25% (k = 192 of 768).
Weights are random N(0, 0.02) drawn on the device from the seeded generator.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 8b|8b32|1b]
    python bench.py --impl reference      # the CPU oracle on a bounded sample

Under torchrun (N > 1) each rank runs the workload on its own GPU with its own
sequences (the path shards by sequence; no data-path collective): value is the
tokens of all ranks over the slowest rank's device time.
"""
from __future__ import annotations

import argparse
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

WORKLOADS = {
    "8b": dict(dims=synth.M8B, run=synth.M8B_RUN, seq=synth.M8B_SEQ,
               name="8B-class bf16 masked-diffusion transformer, batch 1, prompt 512 + 256 generated, "
                    "blocks of 32, 1 token/step, skip layer 4, keep 25%"),
    "8b32": dict(dims=synth.M8B, run=synth.M8B_RUN, seq=synth.M8B32_SEQ,
                 name="8B-class bf16, batch 32, prompt 1024 + 512 generated, blocks of 64, "
                      "2 tokens/step, skip layer 4"),
    "1b": dict(dims=synth.M1B, run=synth.M1B_RUN, seq=synth.M1B_SEQ,
               name="1B-class bf16, batch 1, prompt 256 + 256 generated, blocks of 32, "
                    "1 token/step, skip layer 4, keep 20%"),
}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained", p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- oracle sample
def oracle_sample(wl: dict, max_seconds: float = 30.0) -> dict:
    """Time the CPU oracle on a bounded sample of the workload and extrapolate
    to a whole generation: one dense layer over all rows, one sparse layer over
    the selected rows, scoring + selection of one sequence, and the head over
    a slice of the vocabulary (scaled to the full vocabulary)."""
    import torch

    import oracle as O

    dims, run, seq = wl["dims"], wl["run"], wl["seq"]
    B, P, G = seq["batch"], seq["prompt"], seq["gen"]
    L = P + G
    k = O.keep_count(run.keep_ratio, L)
    threads = len(os.sched_getaffinity(0))
    torch.set_num_threads(threads)
    # one layer's weights, drawn from the seeded generator (layer 0's stream offsets)
    lay = [e for e in synth.weight_layout(dims) if e[1] == 0]
    lw = {name: O.store(synth.weight_f32(0, off, shape).astype(np.float64), dims.dtype)
          for name, _, shape, off in lay}
    vslice = max(256, dims.vocab // 16)
    wout_off = [e for e in synth.weight_layout(dims) if e[0] == "w_out"][0][3]
    w_out = O.store(synth.weight_f32(0, wout_off, (vslice, dims.d)).astype(np.float64), dims.dtype)
    hd = dataclass_replace_vocab(dims, vslice)
    x = O.store(synth.normal(7, 0, L * dims.d).reshape(L, dims.d), dims.dtype)
    hc = O.store(x + 0.01 * synth.normal(7, L * dims.d, L * dims.d).reshape(L, dims.d), dims.dtype)
    conf = synth.uniform(8, 0, L) ** 0.2
    t = {}
    t0 = time.perf_counter()
    _, kk, vv = O.dense_layer(x, lw, dims)
    t["dense_layer"] = time.perf_counter() - t0
    idx = O.topk_select(O.importance(x, hc, conf, run), k)
    t0 = time.perf_counter()
    s = O.importance(x, hc, conf, run)
    idx = O.topk_select(s, k)
    t["select"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    xs = O.sparse_layer(x[idx], idx, kk, vv, lw, dims)
    t["sparse_layer"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    O.head(xs, w_out, hd)
    t["head_sel"] = (time.perf_counter() - t0) * dims.vocab / vslice
    n_dense_layers = run.skip_layer
    n_sparse_layers = dims.n_layers - run.skip_layer
    # per sequence; B sequences run one after another in the oracle
    sparse_step = B * (n_dense_layers * t["dense_layer"] + n_sparse_layers * t["sparse_layer"]
                       + t["select"] + t["head_sel"])
    dense_step = B * (dims.n_layers * t["dense_layer"] + t["head_sel"] * L / k)
    steps_per_block = seq["block"] // seq["n_unmask"]
    n_blocks = G // seq["block"]
    gen_time = n_blocks * (dense_step + (steps_per_block - 1) * sparse_step)
    return {"value": B * G / gen_time, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": (f"one dense layer ({L} rows), one sparse layer ({k} rows), scoring + top-k "
                       f"of one sequence, head over {vslice} of {dims.vocab} vocabulary rows "
                       f"(scaled); extrapolated to {n_blocks} dense + "
                       f"{n_blocks * (steps_per_block - 1)} sparse steps x {B} sequences"),
            "seconds": {k_: round(v, 3) for k_, v in t.items()}}


def dataclass_replace_vocab(dims, vocab):
    import dataclasses
    return dataclasses.replace(dims, vocab=vocab, mask_id=vocab - 1)


# ---------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="8b", choices=sorted(WORKLOADS))
    ap.add_argument("--keep", type=float, default=None, help="override the keep ratio")
    ap.add_argument("--blocks", type=int, default=None, help="generate only this many blocks")
    ap.add_argument("--prompt", type=int, default=None,
                    help="override the prompt length (with --blocks, keeps L for profiling cases)")
    ap.add_argument("--layers", type=int, default=None,
                    help="override the layer count (small profiling cases only)")
    ap.add_argument("--vocab", type=int, default=None,
                    help="override the vocabulary (small profiling cases only)")
    ap.add_argument("--micro", action="store_true",
                    help="the kernel microbenchmark (B 16, S 4096, d 4096, bf16) instead")
    ap.add_argument("--no-dense-baseline", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()

    import dataclasses

    wl = dict(WORKLOADS[args.workload])
    if args.keep is not None:
        wl["run"] = dataclasses.replace(wl["run"], keep_ratio=args.keep)
    if args.blocks is not None:
        wl["seq"] = dict(wl["seq"], gen=args.blocks * wl["seq"]["block"])
    if args.prompt is not None:
        wl["seq"] = dict(wl["seq"], prompt=args.prompt)
    if args.layers is not None:
        wl["dims"] = dataclasses.replace(wl["dims"], n_layers=args.layers)
        wl["name"] += f" [profiling case: {args.layers} layers]"
    if args.vocab is not None:
        wl["dims"] = dataclasses.replace(wl["dims"], vocab=args.vocab, mask_id=args.vocab - 1)
        wl["name"] += f" [profiling case: vocab {args.vocab}]"

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        return run_reference(args, wl)
    if args.micro:
        return run_micro(args)

    import torch
    import torch.distributed as dist

    import synth.gpu as sgpu
    import token_skipping_sparse_step_b200 as esd

    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))

    dims, run, seq = wl["dims"], wl["run"], wl["seq"]
    B, P, G, blk, nu = seq["batch"], seq["prompt"], seq["gen"], seq["block"], seq["n_unmask"]
    L = P + G
    weights = sgpu.model_weights(dims)
    ed = esd.make_dims(dims.n_layers, dims.d, dims.n_heads, dims.head_dim, dims.ffn, dims.vocab,
                       dims.mask_id, dims.rope_theta, dims.rms_eps, dims.dtype)
    er = esd.make_run(run.score_mode, run.alpha, run.lam, run.skip_layer, run.keep_ratio,
                      run.refresh_interval, B, L)
    ctx = esd.Context(ed, weights, er)
    k = ctx.keep_count(L)
    # each rank draws its own sequences (sequence sharding across replicas)
    prompt_np = synth.prompt_ids(dims, B, P, seed=synth.SEED_PROMPT + 1000 * rank)
    prompt_host = torch.from_numpy(prompt_np).pin_memory()
    prompt_dev = prompt_host.to("cuda")
    out_dev = torch.empty((B, G), dtype=torch.int32, device="cuda")
    out_host = torch.empty((B, G), dtype=torch.int32).pin_memory()
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        ctx.generate(prompt_dev, G, blk, nu, out=out_dev)

    # the dominant kernel: the gate/up GEMM of the sparse layers (rows = B*k)
    ctx.profile_enable(esd.K_GEMM_GATE_UP, B * k, B * k)
    ctx.profile_read(reset=True)
    props = torch.cuda.get_device_properties(local_rank)
    sampler = ClockSampler(f"GPU-{props.uuid}" if hasattr(props, "uuid") else str(local_rank))
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.2)
    l0 = ctx.launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        ctx.generate(prompt_dev, G, blk, nu, out=out_dev)
    e1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier()
    launches = ctx.launch_count() - l0
    ms = e0.elapsed_time(e1)
    prof_ms, prof_n = ctx.profile_read(reset=True)
    ctx.profile_enable(-1)
    t = torch.tensor([ms], dtype=torch.float64, device="cuda")
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_max = float(t.item())
    tokens = world * B * G * args.steps
    value = tokens / (ms_max / 1e3)

    # end to end through the public call with host buffers (prompt H2D and the
    # generated ids D2H inside the timed region)
    barrier()
    torch.cuda.synchronize()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for _ in range(args.steps):
        ctx.generate(prompt_host, G, blk, nu, out=out_host)
    e3.record(stream)
    torch.cuda.synchronize()
    t2 = torch.tensor([e2.elapsed_time(e3)], dtype=torch.float64, device="cuda")
    if world > 1:
        dist.all_reduce(t2, op=dist.ReduceOp.MAX)
    e2e_value = tokens / (float(t2.item()) / 1e3)
    assert torch.equal(out_host, out_dev.cpu()), "host and device generations differ"

    # per-step times (caches filled by the last generation)
    tok = torch.full((B, L), dims.mask_id, dtype=torch.int32, device="cuda")
    tok[:, :P] = prompt_dev
    msk = torch.zeros((B, L), dtype=torch.uint8, device="cuda")
    msk[:, P:] = 1

    def step_ms(dense, reps=5):
        ctx.denoise_step(tok.clone(), msk.clone(), P, P + blk, nu, force_dense=True)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        tt, mm = tok.clone(), msk.clone()
        a.record(stream)
        for _ in range(reps):
            ctx.denoise_step(tt, mm, P, P + blk, nu, force_dense=dense)
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    ms_dense, ms_sparse = step_ms(True), step_ms(False)

    dense_baseline = None
    if not args.no_dense_baseline:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        ctx.generate(prompt_dev, G, blk, nu, out=out_dev, vanilla=True)
        b.record(stream)
        torch.cuda.synchronize()
        dms = a.elapsed_time(b)
        dense_baseline = {"value": round(B * G / (dms / 1e3), 2), "unit": "tokens/s",
                          "what": "dense every-token recompute (every step a full refresh), same kernels"}

    hbm, tf_burst, tf_sus, peak_src = peaks()
    F, d = dims.ffn, dims.d
    M = B * k
    alg_bytes = (2 * F * d + M * d + M * F) * 2
    alg_flops = 2.0 * M * (2 * F) * d
    avg_s = (prof_ms / max(prof_n, 1)) / 1e3
    bound = "hbm" if alg_flops / alg_bytes < (tf_sus * 1e12) / (hbm * 1e9) else "tensor"
    if bound == "hbm":
        achieved = alg_bytes / avg_s / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4), "traffic": None}
    else:
        achieved = alg_flops / avg_s / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": tf_sus, "unit": "TFLOP/s",
                "frac": round(achieved / tf_sus, 4), "traffic": None}
    roof.update({"kernel": f"tc_gemm gate/up + SwiGLU, sparse layers (M={M}, N={2 * F}, K={d})",
                 "launches": prof_n, "avg_us": round(avg_s * 1e6, 2),
                 "algorithmic_bytes": alg_bytes, "algorithmic_flops": alg_flops,
                 "peak_source": f"{peak_src} ({'sustained' if bound == 'tensor' else 'copy'})"})

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample(wl)

    line = {
        "metric": "generated tokens/s", "value": round(value, 2), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_max / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl["name"], "batch_per_gpu": B, "prompt": P, "gen": G,
                   "block": blk, "tokens_per_step": nu, "skip_layer": run.skip_layer,
                   "keep_ratio": run.keep_ratio, "k": k, "score": run.score_mode,
                   "step": "one whole generation (esd_generate)",
                   "l2": "inputs larger than L2: every denoising step streams the 16 GB of weights"},
        "ms_per_denoise_step": {"dense": round(ms_dense, 3), "sparse": round(ms_sparse, 3)},
        "e2e": {"value": round(e2e_value, 2), "unit": "tokens/s", "h2d_bytes_per_step": B * P * 4,
                "d2h_bytes_per_step": B * G * 4},
        "gpu_launches": int(launches),
        "roofline": roof,
        "dense_recompute": dense_baseline,
        "cpu_baseline": None if cpu is None else {k_: cpu[k_] for k_ in ("value", "unit", "cores", "kind", "sample")},
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    ctx.close()
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_micro(args) -> int:
    """Isolated sparse-step pieces at the microbenchmark shape (B 16, S 4096,
    d 4096, 32 x 128 heads, bf16; inputs per the recipe of synth.micro_inputs):
    score + top-k + gather, partial attention of k queries over S keys, and the
    row scatter into a cache, for k in {64, 256, 1024}. Each launch is timed
    alone with CUDA events after a 256 MB write that flushes L2."""
    import torch

    import synth.gpu as sg
    import token_skipping_sparse_step_b200 as esd

    hbm, tf_burst, tf_sus, peak_src = peaks()
    B, S, d = synth.MICRO["batch"], synth.MICRO["seq"], synth.MICRO["d"]
    H, hd = synth.MICRO["n_heads"], synth.MICRO["head_dim"]
    dims = synth.ModelDims(2, d, H, hd, 256, 1024, 1023, 5e5, 1e-6, "bf16")
    ctx = esd.Context(esd.make_dims(2, d, H, hd, 256, 1024, 1023, 5e5, 1e-6, "bf16"),
                      sg.model_weights(dims), esd.make_run("es", 0.5, 0.5, 1, 0.25, 0, B, S))
    x, h, conf = sg.micro_inputs(B, S, d)
    kc = torch.empty((B * S, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    sg.fill_normal(kc, 22, 0)
    sg.fill_normal(vc, 23, 0)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def timed(fn, reps):
        for _ in range(args.warmup):
            fn()
        tot = 0.0
        for _ in range(reps):
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            tot += a.elapsed_time(b)
        return tot / reps / 1e3  # seconds

    reps = max(args.steps, 5)
    out = {}
    for k in synth.MICRO["ks"]:
        sc = torch.empty(B * S, dtype=torch.float32, device="cuda")
        idx = torch.empty(B * k, dtype=torch.int32, device="cuda")
        xs = torch.empty((B * k, d), dtype=torch.bfloat16, device="cuda")

        def select():
            ctx.importance_select(x, h, conf, B, S, k, idx, scores_out=sc)
            ctx.gather_rows(x, idx, B, S, k, xs, None)

        t = timed(select, reps)
        by = 2 * B * S * d * 2 + 8 * B * S + 2 * B * k * d * 2
        out[f"select_k{k}"] = {"us": round(t * 1e6, 1), "GB/s": round(by / t / 1e9, 1),
                               "frac_hbm": round(by / t / 1e9 / hbm, 3), "bytes": by}

        def scatter():
            ctx.gather_rows(x, idx, B, S, k, xs, h)

        t = timed(scatter, reps)
        by = 3 * B * k * d * 2
        out[f"scatter_k{k}"] = {"us": round(t * 1e6, 1), "GB/s": round(by / t / 1e9, 1),
                                "frac_hbm": round(by / t / 1e9 / hbm, 3), "bytes": by}
        q = xs  # k selected rows per sequence as queries
        o = torch.empty_like(q)

        def attend():
            ctx.partial_attention(q, kc, vc, B, S, k, o)

        t = timed(attend, reps)
        fl = 4.0 * B * k * S * d
        by = 2 * B * S * d * 2 + 2 * B * k * d * 2
        tf = fl / t / 1e12
        out[f"attention_k{k}"] = {"us": round(t * 1e6, 1), "TFLOP/s": round(tf, 1),
                                  "GB/s": round(by / t / 1e9, 1),
                                  "frac_tensor": round(tf / tf_burst, 3),
                                  "frac_hbm": round(by / t / 1e9 / hbm, 3),
                                  "bound": "hbm" if fl / by < tf_burst * 1e3 / hbm else "tensor"}
    ctx.sync_check()
    line = {"metric": "microbenchmark of the sparse-step pieces", "unit": "see entries",
            "config": {"workload": "B 16, S 4096, d 4096, 32 x 128 heads, bf16; x ~ N(0,1), cache = x + "
                                   "N(0, 0.01^2) on 90% of rows, fresh N(0,1) on 10%, conf ~ Beta(5,1)",
                       "l2": "256 MB write between timed launches"},
            "peaks": {"hbm_gbs": hbm, "bf16_tflops": tf_burst, "source": peak_src},
            "results": out}
    print(json.dumps(line), flush=True)
    ctx.close()
    return 0


def run_reference(args, wl) -> int:
    """The oracle as it stands on the host cores: each step one bounded sample
    of the workload, extrapolated to a whole generation."""
    vals = []
    t_all = time.perf_counter()
    res = None
    for i in range(args.warmup + args.steps):
        res = oracle_sample(wl)
        if i >= args.warmup:
            vals.append(res["value"])
    v = statistics.median(vals) if vals else res["value"]
    seq = wl["seq"]
    line = {
        "metric": "generated tokens/s", "value": round(v, 4), "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "impl": "reference",
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl["name"], "batch_per_gpu": seq["batch"], "prompt": seq["prompt"],
                   "gen": seq["gen"]},
        "cpu_baseline": {"value": round(v, 4), "unit": "tokens/s", "cores": res["cores"],
                         "kind": "oracle", "sample": res["sample"]},
        "e2e": {"value": round(v, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "wall_s": round(time.perf_counter() - t_all, 1),
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
