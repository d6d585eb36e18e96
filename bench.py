#!/usr/bin/env python
"""Benchmark of the B200 GPTQ layer solver.

One step = one whole layer solve through the C ABI on inputs resident in HBM:
S = 0; S += X X^T over all calibration tokens (gptq_hessian_accumulate);
gptq_prepare_hinv; gptq_quantize_layer (codes packed, scales, zeros, g_idx).
The metric is weights quantized per second (out * in per step), with the
per-step split and the roofline of the dominant kernel (the Hessian SYRK on
the tensor cores).  Inputs are seeded synthetic stand-ins for the pages'
calibration set (128 sequences x 2048 tokens) and a Llama-7B-shaped layer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     # the CPU oracle, timed on the host

With N > 1 (torchrun, one process per GPU) every rank solves its own
independent copy of the layer (layers are independent problems; there is no
data-path collective): value = all ranks' weights / max-over-ranks time.
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

METRIC = "GPTQ layer-solve weights/sec and ms/layer (4096×4096, 4-bit g128), % of roofline"
UNIT = "weights/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def strip_comments(src):
    """C/C++ source without comments and blank space, so that a change to a
    comment alone keeps a kernel's recorded counters valid."""
    import re
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def kernel_sources_sha256(texts=None):
    """Hash of the code (comments excluded) the SYRK kernel is built from."""
    import hashlib
    h = hashlib.sha256()
    for name in ("tc_gemm.cu", "gemm.cuh", "common.cuh"):
        if texts is None:
            with open(os.path.join(ROOT, "post_weight_quantization_13_b200", "csrc", name)) as f:
                src = f.read()
        else:
            src = texts[name]
        h.update(strip_comments(src).encode())
    return h.hexdigest()


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=150)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama7b_q_proj")
    ap.add_argument("--tokens", type=int, default=0,
                    help="calibration tokens (default: the workload's); smaller for profiling")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-dequant", action="store_true")
    ap.add_argument("--block-size", type=int, default=0,
                    help="lazy-batch width of the sweep (default: the workload's)")
    ap.add_argument("--desc-act", action="store_true",
                    help="process columns in act-order (default: the workload's, off)")
    ap.add_argument("--unsampled", action="store_true",
                    help="with --impl reference: time one whole oracle layer solve instead of samples")
    return ap.parse_args()


def quant_of(wl, args):
    """The workload's quantization settings with the command-line overrides."""
    import dataclasses
    q = wl.quant[0]
    if getattr(args, "block_size", 0):
        q = dataclasses.replace(q, block_size=args.block_size)
    if getattr(args, "desc_act", False):
        q = dataclasses.replace(q, desc_act=True)
    return q


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, enabled=True):
        self.proc = None
        self.path = None
        if not enabled:
            return
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    rows.append((float(parts[0]), float(parts[1]), float(parts[2]), parts[4:8]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "samples": len(rows), "reasons": reasons}


def gpu_id_for(dev):
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev)


# ------------------------------------------------------------------ CPU oracle
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((p.get("num_threads", 1) for p in threadpool_info()), default=1)
    except Exception:
        return len(os.sched_getaffinity(0))


def oracle_setup(wl, layer, q, W, X):
    """Untimed setup for the sampled oracle: a full-size U and perm."""
    import numpy as np
    import oracle as O
    S, nt = O.hessian([np.asarray(X[:, :2048])])
    prep = O.prepare(S, nt, q.damp_percent, q.desc_act)
    return dict(S=S, nt=nt, U=prep["U"], perm=prep["perm"])


# The one sampling recipe both oracle legs use (the GPU line's cpu_baseline
# and the reference arm): the Hessian over SAMPLE_TOKENS tokens, the whole
# prepare, and the sweep of SAMPLE_ROWS rows over all columns, each part
# scaled to the whole layer.  The reference arm times the prepare (which has
# no smaller sample) once and shrinks the other two parts when many steps
# are asked for, so that its whole run stays within REFERENCE_BUDGET_S.
SAMPLE_TOKENS = 32768
SAMPLE_ROWS = 4096
REFERENCE_BUDGET_S = 150.0


def oracle_sample(wl, layer, q, W, X, setup, tokens=SAMPLE_TOKENS, rows=SAMPLE_ROWS, t_prepare=None):
    """The float64 oracle, as it stands, on a bounded sample of one layer
    solve, scaled to the whole layer: the Hessian over ``tokens`` tokens
    (x all/tokens), the whole prepare (unscaled; timed here unless its time
    ``t_prepare`` is given), and the column sweep of ``rows`` rows over all
    columns (x out/rows).  Returns (weights/s, detail)."""
    import numpy as np
    import oracle as O
    n = wl.tokens
    tokens = min(tokens, X.shape[1], n)
    t0 = time.perf_counter()
    O.hessian([np.asarray(X[:, :tokens])])
    t_h = time.perf_counter() - t0
    if t_prepare is None:
        t0 = time.perf_counter()
        O.prepare(setup["S"], setup["nt"], q.damp_percent, q.desc_act)
        t_p = time.perf_counter() - t0
    else:
        t_p = t_prepare
    r = min(rows, layer.out)
    Wp = np.asarray(W[:r], dtype=np.float64)[:, setup["perm"]]
    t0 = time.perf_counter()
    O.sweep_blocked(Wp, setup["U"], q.bits, q.group_size, q.sym, q.block_size)
    t_s = time.perf_counter() - t0
    sh, ss = n / tokens, layer.out / r
    total = t_h * sh + t_p + t_s * ss
    sample = (f"Hessian over {tokens} of {n} tokens (x{sh:.0f}), the whole {layer.in_}x{layer.in_} "
              f"prepare (x1{', timed once' if t_prepare is not None else ''}), sweep of {r} of "
              f"{layer.out} rows (x{ss:.0f}); {t_h + t_s + (0 if t_prepare is not None else t_p):.2f} s measured")
    return layer.out * layer.in_ / total, dict(
        cores=_blas_threads(), sample=sample, est_s_per_layer=total,
        split_s=dict(hessian=t_h * sh, prepare=t_p, sweep=t_s * ss))


def O_prepare_once(setup, q):
    """One oracle prepare of the layer (the reference arm times it once)."""
    import oracle as O
    O.prepare(setup["S"], setup["nt"], q.damp_percent, q.desc_act)


def oracle_unsampled(wl, layer, q, W, X):
    """One whole layer solve by the oracle, nothing sampled: the Hessian over
    every token (in 16384-token chunks), the prepare and the sweep of every
    row.  Returns (seconds, split)."""
    import numpy as np
    import oracle as O
    t0 = time.perf_counter()
    S = np.zeros((layer.in_, layer.in_), np.float64)
    for c0 in range(0, X.shape[1], 16384):
        O.hessian_accumulate(S, X[:, c0:c0 + 16384])
    t1 = time.perf_counter()
    prep = O.prepare(S, X.shape[1], q.damp_percent, q.desc_act)
    t2 = time.perf_counter()
    Wd = np.asarray(W, np.float64)
    Wd[:, prep["dead"]] = 0.0
    O.sweep_blocked(Wd[:, prep["perm"]], prep["U"], q.bits, q.group_size, q.sym, q.block_size)
    t3 = time.perf_counter()
    return t3 - t0, dict(hessian=t1 - t0, prepare=t2 - t1, sweep=t3 - t2)


def config_of(wl, layer, q, world, x_bytes=None):
    """The line's config, identical in both arms."""
    return {"workload": wl.name, "out": layer.out, "in": layer.in_, "tokens": wl.tokens,
            "bits": q.bits, "group_size": q.group_size, "sym": q.sym, "desc_act": q.desc_act,
            "damp_percent": q.damp_percent, "block_size": q.block_size, "x_dtype": wl.x_dtype,
            "l2": ("inputs larger than L2 (X %.2f GiB)" % ((x_bytes if x_bytes is not None else
                   layer.in_ * wl.tokens * (2 if wl.x_dtype == "float16" else 4)) / 2**30)),
            "parallelism": f"replicas x{world}"}


def run_reference(args):
    """--impl reference: the CPU oracle (float64 numpy) on the host cores,
    each step one bounded sample of the same layer solve (the recipe the GPU
    line's cpu_baseline uses).  With --unsampled: one whole layer solve by the
    oracle instead, timed once, beside the recipe's estimate."""
    import gen
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    wl = gen.WORKLOADS[args.workload]
    layer = wl.layers[0]
    q = quant_of(wl, args)
    W = gen.weight(wl, layer)
    if getattr(args, "unsampled", False):
        X = gen.x_full(wl, layer.site)
        setup = oracle_setup(wl, layer, q, W, X)
        v_est, d_est = oracle_sample(wl, layer, q, W, X, setup)
        secs, split = oracle_unsampled(wl, layer, q, W, X)
        print(json.dumps({"impl": "reference", "unsampled": True, "config": config_of(wl, layer, q, world),
                          "seconds_per_layer": secs, "split_s": split, "cores": _blas_threads(),
                          "recipe_estimate_s": d_est["est_s_per_layer"], "recipe_split_s": d_est["split_s"],
                          "recipe_sample": d_est["sample"]}), flush=True)
        return
    X = gen.x_full(wl, layer.site, tokens=min(SAMPLE_TOKENS, wl.tokens))
    setup = oracle_setup(wl, layer, q, W, X)
    vals, detail = [], None
    t_run = time.perf_counter()
    t0 = time.perf_counter()
    O_prepare_once(setup, q)
    t_prep = time.perf_counter() - t0
    tokens, rows = SAMPLE_TOKENS, SAMPLE_ROWS
    n_samples = args.warmup + args.steps
    for i in range(n_samples):
        t0 = time.perf_counter()
        v, detail = oracle_sample(wl, layer, q, W, X, setup, tokens, rows, t_prepare=t_prep)
        if i == 0 and n_samples > 1:
            # the rest of the run within the budget: shrink tokens and rows
            left = REFERENCE_BUDGET_S - (time.perf_counter() - t_run)
            f = min(1.0, max(left, 0.0) / ((n_samples - 1) * (time.perf_counter() - t0)))
            tokens, rows = max(1024, int(SAMPLE_TOKENS * f)), max(16, int(SAMPLE_ROWS * f))
        if i >= args.warmup:
            vals.append(v)
    t_run = time.perf_counter() - t_run
    v = statistics.median(vals)
    line = {"metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * layer.out * layer.in_ / v,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": config_of(wl, layer, q, world),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": detail["cores"], "kind": "oracle",
                             "sample": detail["sample"],
                             "note": ("value and ms_per_step are the whole layer's oracle time "
                                      "estimated from each step's sample; the run itself took "
                                      f"{t_run:.1f} s for {args.warmup + args.steps} samples")},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ ranks
def max_over_ranks(x: float, pg, device) -> float:
    """The maximum of x over all ranks (x itself without a process group).
    Every rank must call it at the same point."""
    if pg is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, weights_per_layer: int, layers: int, elapsed_ms: float) -> float:
    """Weights/s of the whole job: every rank solves ``layers`` layers of
    ``weights_per_layer`` weights in ``elapsed_ms`` (the slowest rank's time)."""
    return world * weights_per_layer * layers / (elapsed_ms / 1e3)


# ------------------------------------------------------------------ GPU
def run_ours(args):
    import numpy as np
    import torch

    import gen
    import post_weight_quantization_13_b200 as g

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    wl = gen.WORKLOADS[args.workload]
    if args.tokens:
        import dataclasses
        wl = dataclasses.replace(wl, tokens=args.tokens)
    layer = wl.layers[0]
    q = quant_of(wl, args)
    cfg = g.GptqConfig(**q.as_dict())
    out, in_ = layer.out, layer.in_
    n_tok = wl.tokens

    # inputs: generated on the host (pinned), copied once; resident in HBM
    Wh = torch.from_numpy(gen.weight(wl, layer)).pin_memory()
    tdt = {"float16": torch.float16, "float32": torch.float32}[wl.x_dtype]
    Xh = torch.empty((in_, n_tok), dtype=tdt, pin_memory=True)
    gen.x_full(wl, layer.site, out=Xh.numpy())
    W = Wh.to(dev)
    X = Xh.to(dev)
    S = torch.zeros((in_, in_), dtype=torch.float32, device=dev)
    ws = torch.empty(g.gptq_workspace_bytes(out, in_, cfg), dtype=torch.uint8, device=dev)
    U = torch.empty((in_, in_), dtype=torch.float32, device=dev)
    perm = torch.empty(in_, dtype=torch.int32, device=dev)
    dead = torch.empty(in_, dtype=torch.uint8, device=dev)
    ng = 1 if q.group_size == -1 else in_ // q.group_size
    scales = torch.empty((out, ng), dtype=torch.float32, device=dev)
    zeros = torch.empty((out, ng), dtype=torch.int32, device=dev)
    g_idx = torch.empty(in_, dtype=torch.int32, device=dev)
    qweight = torch.empty((out, in_ * q.bits // 32), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    phase_ms = {"hessian": [], "prepare": [], "quantize": [], "syrk": []}

    def step(record=False):
        e0, es, e1, e2, e3 = ev(), ev(), ev(), ev(), ev()
        e0.record(stream)
        S.zero_()
        es.record(stream)
        n = g.gptq_hessian_accumulate(S, X, 0, stream)
        e1.record(stream)
        g.gptq_prepare_hinv(S, n, cfg, U, perm, dead, ws, stream)
        e2.record(stream)
        g.gptq_quantize_layer(W, U, perm, dead, cfg, scales, zeros, g_idx, ws, qweight=qweight,
                              stream=stream)
        e3.record(stream)
        return (e0, es, e1, e2, e3) if record else None

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)

    sampler = ClockSampler(gpu_id_for(local), enabled=not args.no_clocks)
    time.sleep(0.3)
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    launches0 = g.gptq_kernel_launches()
    start, end = ev(), ev()
    marks = []
    start.record(stream)
    for _ in range(args.steps):
        marks.append(step(record=True))
    end.record(stream)
    torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    launches = g.gptq_kernel_launches() - launches0
    clocks = sampler.stop()
    elapsed = start.elapsed_time(end)  # ms
    for e0, es, e1, e2, e3 in marks:
        phase_ms["hessian"].append(e0.elapsed_time(e1))
        phase_ms["syrk"].append(es.elapsed_time(e1))
        phase_ms["prepare"].append(e1.elapsed_time(e2))
        phase_ms["quantize"].append(e2.elapsed_time(e3))
    elapsed = max_over_ranks(elapsed, pg, dev)
    ms_step = elapsed / args.steps
    value = job_throughput(world, out * in_, args.steps, elapsed)

    # the dominant kernel: one tcgen05 SYRK launch per step, timed alone
    hess_ms = statistics.mean(phase_ms["syrk"])
    flops = in_ * (in_ + 1) * n_tok
    peaks, peak_src = load_peaks()
    # the burst peak for a timed region under a second (the GPU has not yet
    # settled at its power cap), the sustained one for a longer run
    burst = elapsed < 1000.0
    peak_key = "bf16_tflops" if burst else "bf16_tflops_sustained"
    peak = peaks.get(peak_key, PEAKS_FALLBACK[peak_key])
    achieved = flops / (hess_ms / 1e3) / 1e12
    # whole-step roofline: each step at the slower of its tensor-core and HBM
    # floors (a1 Hessian and a4 factorisation on tensor cores, a6 lazy
    # update and the gathers/packing on HBM), against the measured peaks
    bw = peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"]) * 1e9
    pf = peak * 1e12
    nblk = -(-in_ // 128)
    terms = {"a1_hessian": flops / pf, "a4_factor": (2.0 / 3.0) * in_ ** 3 / pf,
             "a6_lazy_update": 4.0 * out * in_ * max(nblk - 1, 0) / bw,
             "a2_a3_a7_bytes": (8.0 * in_ * in_ + out * in_ * (2 + 4 + q.bits / 8)) / bw}
    t_roof = sum(terms.values()) * 1e3
    step_roof = {"t_roof_ms": t_roof, "frac": t_roof / ms_step,
                 "terms_ms": {k: v * 1e3 for k, v in terms.items()}}
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tpath):
        with open(tpath) as f:
            t = json.load(f).get(f"hessian_syrk:{wl.name}")
        # counters taken on an older build of the kernel no longer apply; X is
        # read once per drain, so the traffic scales with the tokens
        if t and t.get("kernel_sources_sha256") == kernel_sources_sha256():
            traffic = int(t.get("bytes_per_launch") * n_tok // t.get("tokens", n_tok))

    # e2e: host buffers in, results out, every step, through the same ABI
    # calls.  Calibration tokens arrive as host batches (chunk-major pinned
    # buffers, as a data loader hands them over); each batch is copied on a
    # copy stream into one of two device buffers while the previous batch is
    # accumulated, so the host link and the SYRK overlap.
    e2e = None
    if not args.no_e2e:
        outs_h = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                  for t in (qweight, scales, zeros, g_idx, perm)]
        outs_d = [qweight, scales, zeros, g_idx, perm]
        chunk = min(n_tok, 32768)
        nch = -(-n_tok // chunk)
        Xc = [torch.empty((in_, min(chunk, n_tok - c * chunk)), dtype=tdt, pin_memory=True)
              for c in range(nch)]
        for c in range(nch):
            Xc[c].copy_(Xh[:, c * chunk:c * chunk + Xc[c].shape[1]])
        Xd = [torch.empty((in_, chunk), dtype=tdt, device=dev) for _ in range(2)]
        cstream = torch.cuda.Stream(dev)
        ready = [torch.cuda.Event() for _ in range(2)]
        free = [torch.cuda.Event() for _ in range(2)]
        w_ready = torch.cuda.Event()

        q_done = torch.cuda.Event()

        def e2e_step():
            S.zero_()
            n = 0
            for c in range(nch):
                b = c % 2
                cstream.wait_event(free[b])
                with torch.cuda.stream(cstream):
                    xd = Xd[b][:, :Xc[c].shape[1]]
                    xd.copy_(Xc[c], non_blocking=True)
                    ready[b].record(cstream)
                stream.wait_event(ready[b])
                n = g.gptq_hessian_accumulate(S, xd, n, stream)
                free[b].record(stream)
            cstream.wait_event(q_done)  # the previous step's quantize is done with W
            with torch.cuda.stream(cstream):
                W.copy_(Wh, non_blocking=True)
                w_ready.record(cstream)
            g.gptq_prepare_hinv(S, n, cfg, U, perm, dead, ws, stream)
            stream.wait_event(w_ready)
            g.gptq_quantize_layer(W, U, perm, dead, cfg, scales, zeros, g_idx, ws, qweight=qweight,
                                  stream=stream)
            q_done.record(stream)
            for h, d in zip(outs_h, outs_d):
                h.copy_(d, non_blocking=True)

        for bi in range(2):
            free[bi].record(stream)
        q_done.record(stream)
        e2e_step()
        torch.cuda.synchronize(dev)
        if pg:
            pg.barrier()
        s0, s1 = ev(), ev()
        s0.record(stream)
        cstream.wait_stream(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        s1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(s0.elapsed_time(s1), pg, dev)
        h2d = sum(t.numel() * t.element_size() for t in Xc) + Wh.numel() * Wh.element_size()
        d2h = sum(t.numel() * t.element_size() for t in outs_d)
        e2e = {"value": job_throughput(world, out * in_, args.e2e_steps, e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e_ms / args.e2e_steps, "steps": args.e2e_steps,
               "pipeline": f"{nch} host batches of {chunk} tokens, copy overlapped with the SYRK"}

    # dequantisation of the solved layer back to fp16 (HBM-bound), each launch
    # timed alone after an L2 flush (a read of 256 MiB, so that no dirty lines
    # are left for the timed kernel to write back)
    deq = None
    if not args.no_dequant:
        Wq = torch.empty((out, in_), dtype=torch.float16, device=dev)
        flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)
        times = []
        for it in range(8):
            flush.sum()
            d0, d1 = ev(), ev()
            d0.record(stream)
            g.gptq_dequantize_layer(qweight, scales, zeros, g_idx, q.bits, Wq, stream)
            d1.record(stream)
            torch.cuda.synchronize(dev)
            if it >= 3:
                times.append(d0.elapsed_time(d1))
        dq_ms = statistics.median(times)
        dq_bytes = (out * in_ * q.bits // 8 + out * ng * 8 + in_ * 4 + out * in_ * 2)
        bw_peak = peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])
        deq = {"kernel": "dequant_kernel<f16>", "ms": dq_ms, "bytes": dq_bytes,
               "GB/s": dq_bytes / (dq_ms / 1e3) / 1e9, "peak": bw_peak,
               "frac": dq_bytes / (dq_ms / 1e3) / 1e9 / bw_peak, "bound": "hbm",
               "note": "each launch timed alone (launch latency included) after reading 256 MiB to clear L2"}
        del flush

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        setup = oracle_setup(wl, layer, q, Wh.numpy(), Xh.numpy())
        v, d = oracle_sample(wl, layer, q, Wh.numpy(), Xh.numpy(), setup)
        cpu = {"value": v, "unit": UNIT, "cores": d["cores"], "kind": "oracle", "sample": d["sample"],
               "est_s_per_layer": d["est_s_per_layer"], "split_s": d["split_s"]}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": config_of(wl, layer, q, world, Xh.numel() * Xh.element_size()),
            "split_ms": {k: statistics.mean(v) for k, v in phase_ms.items()},
            "roofline": {"kernel": "tc_gemm_kernel<f16> (Hessian S += X X^T, tcgen05)",
                         "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "frac_of_sustained_peak": achieved / peaks.get(
                             "bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"]),
                         "peak_source": (f"{peak_src} bf16 {'burst' if burst else 'sustained'} "
                                         f"(timed region {elapsed / 1e3:.2f} s; fp16 dense rate = bf16)"),
                         "flops_per_launch": flops},
            "step_roofline": step_roof,
            "dequant": deq,
            "gpu_launches": launches,
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if pg:
        pg.destroy_process_group()


def run_block(args):
    """A whole decoder block (4 activation sites, 7 layers) through
    solve_block: one Hessian and one prepare per site, the layers of a site
    quantized concurrently.  Prints one JSON line; rank 0 of N replicas."""
    import torch

    import gen
    import post_weight_quantization_13_b200 as g

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
        pg = dist
    wl = gen.WORKLOADS[args.workload]
    n_tok = args.tokens or wl.tokens
    q = quant_of(wl, args)
    acts = {}
    for site in wl.sites:
        Xh = torch.empty((site.in_, n_tok), dtype=torch.float16, pin_memory=True)
        gen.x_full(wl, site, tokens=n_tok, out=Xh.numpy())
        acts[site.name] = Xh.to(dev)
        del Xh
    layers = [(l.name, torch.from_numpy(gen.weight(wl, l)).to(dev), l.site) for l in wl.layers]
    weights = sum(W.shape[0] * W.shape[1] for _, W, _ in layers)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    for _ in range(args.warmup):
        g.solve_block(layers, acts, q.as_dict())
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(gpu_id_for(local), enabled=not args.no_clocks)
    if pg:
        pg.barrier()
    launches0 = g.gptq_kernel_launches()
    e0, e1 = ev(), ev()
    e0.record()
    for _ in range(args.steps):
        g.solve_block(layers, acts, q.as_dict())
    e1.record()
    torch.cuda.synchronize(dev)
    launches = g.gptq_kernel_launches() - launches0
    clocks = sampler.stop()
    elapsed = max_over_ranks(e0.elapsed_time(e1), pg, dev)
    ms_step = elapsed / args.steps

    # the same block on one stream, and as seven independent layer solves
    # (each with its own Hessian and prepare), one timed pass each
    def timed(fn):
        torch.cuda.synchronize(dev)
        a, b = ev(), ev()
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize(dev)
        return max_over_ranks(a.elapsed_time(b), pg, dev)

    one_stream_ms = timed(lambda: g.solve_block(layers, acts, q.as_dict(), streams=False))
    naive_ms = timed(lambda: [g.solve_layer(W, acts[site], q.as_dict(), with_codes=False)
                              for _, W, site in layers])
    peaks, peak_src = load_peaks()
    pf = peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"]) * 1e12
    syrk_floor = sum(s.in_ * (s.in_ + 1) * n_tok for s in wl.sites) / pf * 1e3
    if rank == 0:
        line = {
            "metric": METRIC, "value": job_throughput(world, weights, args.steps, elapsed),
            "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": {"workload": wl.name, "layers": [(l.name, l.out, l.in_, l.site) for l in wl.layers],
                       "tokens": n_tok, "bits": q.bits, "group_size": q.group_size,
                       "desc_act": q.desc_act, "parallelism": f"replicas x{world}",
                       "l2": "inputs larger than L2"},
            "block_roofline": {"syrk_floor_ms": syrk_floor, "frac": syrk_floor / ms_step,
                               "peak_source": f"{peak_src} bf16 sustained"},
            "compare_ms": {"one_stream": one_stream_ms, "seven_independent_solves": naive_ms},
            "gpu_launches": launches, "clocks": clocks, "e2e": None, "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)
    if pg:
        pg.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "llama7b_block":
        run_block(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
