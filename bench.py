"""Training-step throughput of the decoder on B200s (tokens/s and MFU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One process per GPU (torchrun for N > 1, NCCL).  A step is grad_accum x
(forward + backward) micro-batches plus the optimizer step, over the
workload's synthetic Zipf(1.1) token stream, with random-init weights.
Default workload: the 12-layer d=768 bf16 decoder, 32 x 1024 = 32K tokens per
step, tied vocab 50304.

Rank 0 prints one JSON line.  `value` is whole-job tokens/s with the inputs
already in HBM (CUDA events on the model's stream, barrier + synchronize on
both sides, max over ranks).  `e2e` repeats the measurement through the same
public calls with pinned host buffers, copying each step's tokens/targets in
and its loss out inside the timed region.  `roofline` is the dominant kernel
class (by time) from CUDA events bracketing every kernel in a second timed
pass of the same steps.  `cpu_baseline` times the fp64 oracle on a bounded
sample on the host cores.  `--impl reference` times that oracle as the
reference arm on the same metric.
"""

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synthetic import tokens_and_targets, workload  # noqa: E402

SPEC_BF16_FLOPS = 2.25e15           # B200 dense bf16 spec (the metric's denominator)
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "training tokens/sec and MFU (% of B200 dense BF16 peak) at 1 GPU"
L2_NOTE = "no L2 flush: a step's working set (weights, activations, logits chunk) is > 10 GB, far above the 126 MB L2"


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "roofline_traffic_gpt2s_bf16.json")
GEMM_SOURCES = ["gemm_tc.cuh", "gemm_common.cuh"]
# the GEMM host code inside gpt.cu: tensor maps, launch, tile width and split-K choice
GEMM_DISPATCH = ("static int make_tmap_gen(", "// ======================================================================== arena plan")


def gemm_sources_sha():
    """sha256 of what decides a GEMM launch's DRAM traffic besides its shape:
    the GEMM kernel sources and gpt.cu's GEMM dispatch code."""
    import hashlib
    csrc = os.path.join(ROOT, "gpt_pretraining_step_decoder_b200", "csrc")
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    with open(os.path.join(csrc, "gpt.cu"), encoding="utf-8") as fh:
        src = fh.read()
    a, b = src.index(GEMM_DISPATCH[0]), src.index(GEMM_DISPATCH[1])
    h.update(src[a:b].encode("utf-8"))
    return h.hexdigest()


def gemm_launch_signature(prof, steps):
    """The step's GEMM call plan: per GEMM scope label, launches and FLOPs
    (2*M*N*K summed) per step."""
    return {k: [round(v["launches"] / steps, 3), round(v["flops"] / steps)]
            for k, v in sorted(prof.items()) if k.startswith("gemm")}


def recorded_traffic(workload_name, signature):
    """DRAM bytes per GEMM launch from the committed ncu summary, if it was
    taken on this workload with the current GEMM sources and the same GEMM
    launches per step; else None."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("workload") != workload_name or rec.get("sources_sha256") != gemm_sources_sha():
        return None
    if rec.get("gemm_launches") != signature:
        return None
    return rec.get("dram_bytes_per_launch")


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
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
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ oracle timing
def oracle_sample(w, seed):
    """fp64 oracle: one full step on one sequence at the workload's length."""
    from oracle.step import OracleTrainer
    from synthetic import init_params
    ws = dict(w, micro_batch=1, grad_accum=1)
    if ws["x0_rows"] or ws["v_rows"]:
        ws["x0_rows"] = min(ws["x0_rows"], 1 << 16)
        ws["v_rows"] = min(ws["v_rows"], 1 << 15)
    params = init_params(ws, seed=seed)
    tr = OracleTrainer(ws, params)
    tok, tgt = tokens_and_targets(1, ws["seq_len"], ws["vocab"], seed)
    return tr, tok, tgt


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(w, seconds=20.0):
    tr, tok, tgt = oracle_sample(w, w["seed"])
    steps, t0 = 0, time.perf_counter()
    while True:
        tr.forward_loss(tok, tgt)
        tr.backward_step(1e-3)
        steps += 1
        el = time.perf_counter() - t0
        if el > seconds or steps >= 3:
            break
    return {"value": steps * w["seq_len"] / el, "unit": "tokens/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"fp64 NumPy oracle, {steps} full step(s) (forward, backward, updates) on one "
                      f"{w['seq_len']}-token sequence of the same workload, tables (if any) cut to "
                      f"64K/32K rows; {el:.1f} s of host time"}


def run_reference(args, w, rank, world):
    """The reference arm: the fp64 oracle as it stands, on the host cores."""
    if rank != 0:
        return
    tr, tok, tgt = oracle_sample(w, w["seed"])
    for _ in range(args.warmup):
        tr.forward_loss(tok, tgt)
        tr.backward_step(1e-3)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        tr.forward_loss(tok, tgt)
        tr.backward_step(1e-3)
    el = time.perf_counter() - t0
    value = args.steps * w["seq_len"] / el
    sample = (f"fp64 NumPy oracle, one {w['seq_len']}-token sequence per step (forward, backward, "
              f"AdamW), warmup {args.warmup}, timed {args.steps}")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_json(w, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "kind": "oracle", "cores": blas_threads(),
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_json(w, world):
    return {"workload": f"{w['name']}: {w['n_layer']} layers, d {w['d_model']}, {w['n_head']}x{w['head_dim']} heads, "
                        f"ReLU^2 MLP {w['d_ff']}, vocab {w['vocab']} ({'tied' if w['tie_embeddings'] else 'untied'}), "
                        f"bigram tables {w['x0_rows']}/{w['v_rows']} rows",
            "tokens_per_step": w["micro_batch"] * w["seq_len"] * w["grad_accum"] * world,
            "seq_len": w["seq_len"], "micro_batch": w["micro_batch"], "grad_accum": w["grad_accum"],
            "parallelism": f"dp{world}", "l2": L2_NOTE}


# ------------------------------------------------------------------ our arm
def run_ours(args, w, rank, world, dist):
    import torch
    import gpt_pretraining_step_decoder_b200 as g

    dev = torch.device("cuda", torch.cuda.current_device())
    from gpt_pretraining_step_decoder_b200 import dp
    cfg = g.make_config(**w)
    model = g.Model(cfg, seed=w["seed"])  # identical replicas on every rank
    A, B, T, V = w["grad_accum"], w["micro_batch"], w["seq_len"], w["vocab"]
    n_micro = A * (args.warmup + args.steps)
    host_tok, host_tgt = [], []
    for i in range(n_micro):
        tok, tgt = tokens_and_targets(B, T, V, dp.rank_stream_seed(w["seed"], rank), w["zipf_s"], w["repeat_frac"],
                                      micro=i)
        host_tok.append(torch.from_numpy(tok).pin_memory())
        host_tgt.append(torch.from_numpy(tgt).pin_memory())
    dev_tok = [t.to(dev) for t in host_tok]
    dev_tgt = [t.to(dev) for t in host_tgt]
    stream = model.stream
    lr = args.lr

    def step(i, tok_src, tgt_src):
        if world > 1:
            dp.train_step(model, [(tok_src[i * A + a], tgt_src[i * A + a]) for a in range(A)], lr)
            return
        for a in range(A):
            model.forward_loss(tok_src[i * A + a], tgt_src[i * A + a])
            model.backward_step(lr)

    def timed(fn_step, first, count):
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for i in range(first, first + count):
            fn_step(i)
        ev1.record(stream)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        ms = ev0.elapsed_time(ev1)
        if dist is not None:
            t = torch.tensor([ms], dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ms = float(t.item())
        return ms

    # warm-up
    for i in range(args.warmup):
        step(i, dev_tok, dev_tgt)
    torch.cuda.synchronize()
    st = model.sync_status()
    if st != g.GPT_OK:
        raise RuntimeError(f"device error after warm-up: {st} {g.gpt_last_error()}")

    # timed region: inputs resident in HBM
    l0 = g.gpt_launch_count()
    with ClockSampler(torch.cuda.current_device()) as clk:
        ms = timed(lambda i: step(i, dev_tok, dev_tgt), args.warmup, args.steps)
    launches = g.gpt_launch_count() - l0
    clocks = clk.summary()
    tokens_per_step = A * B * T * world
    value = tokens_per_step * args.steps / (ms / 1e3)
    loss = float(model.loss.item())

    # second timed pass with every kernel bracketed by CUDA events (roofline)
    g.gpt_profile_enable(model.h, 1)
    ms_prof = timed(lambda i: step(i, dev_tok, dev_tgt), args.warmup, args.steps)
    prof = g.gpt_profile_read(model.h)
    g.gpt_profile_enable(model.h, 0)

    # end-to-end through the public calls with pinned host buffers
    in_tok = [torch.empty_like(dev_tok[0]) for _ in range(A)]
    in_tgt = [torch.empty_like(dev_tgt[0]) for _ in range(A)]
    loss_host = torch.empty(1, dtype=torch.float32).pin_memory()

    def e2e_step(i):
        for a in range(A):
            in_tok[a].copy_(host_tok[i * A + a], non_blocking=True)
            in_tgt[a].copy_(host_tgt[i * A + a], non_blocking=True)
            if world == 1:
                model.forward_loss(in_tok[a], in_tgt[a])
                model.backward_step(lr)
                loss_host.copy_(model.loss, non_blocking=True)
        if world > 1:
            # the same data-parallel step as the device-resident pass (gradient
            # average, table exchange after every backward, optimizer step)
            dp.train_step(model, list(zip(in_tok, in_tgt)), lr, loss_host=loss_host)

    ms_e2e = timed(e2e_step, args.warmup, args.steps)
    st = model.sync_status()
    if st != g.GPT_OK:
        raise RuntimeError(f"device error in timed steps: {st} {g.gpt_last_error()}")

    if rank != 0:
        return
    f_tok, f_tok_causal = g.gpt_flops_per_token(cfg)
    peaks, peak_src = measured_peaks()
    tok_s_gpu = value / world
    mfu_spec = tok_s_gpu * f_tok / SPEC_BF16_FLOPS
    mfu_meas = tok_s_gpu * f_tok / (peaks["bf16_tflops_sustained"] * 1e12)
    total_ms = sum(v["ms"] for v in prof.values())
    # every contraction runs on the same tcgen05 GEMM kernel: one class for the roofline
    classes = {k: v for k, v in prof.items() if not k.startswith("gemm")}
    gemms = [v for k, v in prof.items() if k.startswith("gemm")]
    if gemms:
        classes["gemm"] = {f: sum(v[f] for v in gemms) for f in ("scopes", "launches", "ms", "flops", "bytes")}
    dom_name, dom = max(classes.items(), key=lambda kv: kv[1]["ms"])
    if dom["flops"] > 0:
        achieved = dom["flops"] / (dom["ms"] / 1e3) / 1e12
        roof = {"bound": "tensor", "kernel": dom_name, "achieved": achieved,
                "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops_sustained"],
                "traffic": (recorded_traffic(w["name"], gemm_launch_signature(prof, args.steps))
                            if dom_name == "gemm" else None),
                "peak_source": f"{peak_src} bf16 sustained (cuBLAS loop under the power cap)"}
    else:
        achieved = dom["bytes"] / (dom["ms"] / 1e3) / 1e9
        roof = {"bound": "hbm", "kernel": dom_name, "achieved": achieved, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                "peak_source": f"{peak_src} HBM copy"}
    roof["launches_per_step"] = dom["launches"] / args.steps
    roof["share_of_step"] = dom["ms"] / total_ms if total_ms else None
    roof["per_launch"] = (f"{dom_name}: algorithmic FLOPs (2*M*N*K per contraction) or bytes of every launch in "
                          "the step, summed, over the summed CUDA-event time of those launches; traffic = DRAM "
                          "bytes per launch from the committed ncu summary (null unless taken with the same GEMM "
                          "kernel and dispatch sources and the same GEMM launches per step)")
    breakdown = {k: {"ms_per_step": v["ms"] / args.steps, "launches_per_step": v["launches"] / args.steps,
                     "tflops": (v["flops"] / (v["ms"] / 1e3) / 1e12) if v["flops"] and v["ms"] else None,
                     "gbs": (v["bytes"] / (v["ms"] / 1e3) / 1e9) if v["bytes"] and v["ms"] else None}
                 for k, v in sorted(prof.items(), key=lambda kv: -kv[1]["ms"])}
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w["dtype"] == "bf16" else "f32",
        "data": "synthetic (Zipf(1.1) token stream, random-init weights)",
        "config": config_json(w, world),
        "mfu": {"formula": mfu_spec, "causal": tok_s_gpu * f_tok_causal / SPEC_BF16_FLOPS,
                "of_measured_sustained": mfu_meas, "flops_per_token": f_tok,
                "flops_per_token_causal": f_tok_causal, "peak_spec_flops": SPEC_BF16_FLOPS},
        "loss_last": loss,
        "roofline": roof,
        "breakdown": breakdown,
        "profiled_ms_per_step": ms_prof / args.steps,
        "e2e": {"value": tokens_per_step * args.steps / (ms_e2e / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(A * (host_tok[0].numel() + host_tgt[0].numel()) * 4),
                "d2h_bytes_per_step": int(A * 4)},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if world == 1 and not args.no_tables:
        # the standalone table calls on the full-size x0 table (2,097,152 x 768 bf16) of the
        # tables workload, one micro-batch (N = 32768) and one accumulated step (N = 196608);
        # run after the timed region, on a fresh table
        tb = table_bandwidth(workload("gpt2s_tables_bf16"), 5, 3, tables=("x0",))
        line["tables"] = {"results": [{k: r[k] for k in ("call", "table", "n", "u_over_n", "us", "gbs",
                                                         "frac_of_measured_hbm", "frac_of_8tbs")}
                                      for r in tb["results"]],
                          "peak_source": tb["peak_source"], "l2": tb["l2"], "target": "0.70 of 8 TB/s"}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ table kernels
def table_bandwidth(w, steps, warmup, tables=("x0", "v")):
    """Achieved HBM bandwidth of the standalone bigram-table calls on the
    full-size tables (2,097,152 x d and 1,048,576 x d bf16), rows hashed from
    the workload's token stream; one micro-batch (N = B*T) and a whole
    accumulated step (N = A*B*T).  L2 is flushed (a 256 MB write) before every
    timed call; each call is bracketed by CUDA events on the launching stream.
    Algorithmic bytes: gather N*d*2 read + N*d*2 written + N*4 ids; update
    N*d*4 gradient + U*(2*d*2 + 2*4) rows and states read and written + N*4
    ids + 4*N*4 sorting, U = distinct rows."""
    import torch
    import gpt_pretraining_step_decoder_b200 as g
    dev = torch.device("cuda", torch.cuda.current_device())
    st = torch.cuda.current_stream()
    d = w["d_model"]
    B, T, A, V = w["micro_batch"], w["seq_len"], w["grad_accum"], w["vocab"]
    peaks, peak_src = measured_peaks()
    toks = [torch.from_numpy(tokens_and_targets(B, T, V, w["seed"], w["zipf_s"], w["repeat_frac"], micro=i)[0]).to(dev)
            for i in range(A)]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    results = []
    with ClockSampler(0) as clk:
        for name, R in (("x0", w["x0_rows"]), ("v", w["v_rows"])):
            if not R or name not in tables:
                continue
            table = (torch.randn((R, d), device=dev) * 0.02).to(torch.bfloat16)
            state = torch.zeros(R, dtype=torch.float32, device=dev)
            for n_micro in (1, A):
                n = n_micro * B * T
                rows = torch.empty(n, dtype=torch.int32, device=dev)
                for i in range(n_micro):
                    g.ngram_hash(toks[i], B, T, V, w["hash_p1"], w["hash_p2"], R, rows[i * B * T:(i + 1) * B * T])
                out = torch.empty((n, d), dtype=torch.bfloat16, device=dev)
                grad = torch.randn((n, d), dtype=torch.float32, device=dev)
                ws_bytes = g.ngram_sparse_update_workspace_bytes(n, d)
                ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
                nupd = torch.zeros(1, dtype=torch.int32, device=dev)
                upd = torch.empty(n, dtype=torch.int32, device=dev)
                g.ngram_sparse_update(table, state, R, d, g.DTYPE_BF16, rows, grad, n, 1e-4, 0.95, 1e-10,
                                      upd, nupd, ws, ws_bytes)
                torch.cuda.synchronize()
                U = int(nupd.item())
                calls = {
                    "ngram_gather": (lambda: g.ngram_gather(rows, n, table, R, d, g.DTYPE_BF16, out, 0),
                                     2.0 * n * d * 2 + 4.0 * n),
                    "ngram_sparse_update": (lambda: g.ngram_sparse_update(table, state, R, d, g.DTYPE_BF16, rows, grad,
                                                                          n, 1e-4, 0.95, 1e-10, None, None, ws,
                                                                          ws_bytes),
                                            4.0 * n * d + U * (2.0 * d * 2 + 8) + 4.0 * n + 16.0 * n),
                }
                for cname, (fn, nbytes) in calls.items():
                    times = []
                    for it in range(warmup + steps):
                        flush.zero_()
                        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                        e0.record(st)
                        fn()
                        e1.record(st)
                        torch.cuda.synchronize()
                        if it >= warmup:
                            times.append(e0.elapsed_time(e1))
                    if g.ngram_sync_status() != g.GPT_OK:
                        raise RuntimeError(f"{cname}: device error {g.gpt_last_error()}")
                    us = 1e3 * float(np.median(times))
                    gbs = nbytes / (us * 1e-6) / 1e9
                    results.append({"call": cname, "table": f"{name} {R}x{d} bf16", "n": n, "distinct_rows": U,
                                    "u_over_n": U / n, "us": us, "algorithmic_bytes": nbytes, "gbs": gbs,
                                    "frac_of_measured_hbm": gbs / peaks["hbm_gbs"], "frac_of_8tbs": gbs / 8000.0})
                del out, grad, ws, upd
            del table, state
            torch.cuda.empty_cache()
    del flush
    torch.cuda.empty_cache()
    return {"metric": "bigram table calls: achieved HBM bandwidth (algorithmic bytes / CUDA-event time)",
            "unit": "GB/s", "workload": w["name"], "hbm_peak_gbs": peaks["hbm_gbs"], "peak_source": f"{peak_src} HBM copy",
            "steps": steps, "warmup": warmup, "l2": "flushed (256 MB write) before every timed call",
            "results": results, "clocks": clk.summary()}


def run_tables(args, w):
    print(json.dumps(table_bandwidth(w, args.steps, args.warmup)), flush=True)


def run_muon(args, w):
    """Muon inside the training step: the workload with matrix_optimizer =
    muon (the q, k, v blocks, projection and MLP weights of every layer on
    Muon, batched by shape; the embedding on AdamW).  Reports the Muon part of
    the optimizer step from CUDA events bracketing its kernels (momentum and
    normalisation, ns_steps x three batched Newton-Schulz GEMMs and two
    elementwise kernels per shape group, the step), the whole training step's
    time with Muon on, and the Newton-Schulz GEMM rate.  Newton-Schulz FLOPs per
    matrix with R = min(out, in), C = max(out, in): ns_steps * (2 R^2 C [X X^T]
    + 2 R^3 [A A] + 2 R^2 C [B X]).  Inputs exceed L2 (no flush)."""
    import torch
    import gpt_pretraining_step_decoder_b200 as g
    dev = torch.device("cuda", 0)
    w = dict(w, matrix_optimizer="muon")
    model = g.Model(g.make_config(**w), seed=w["seed"])
    A, B, T, V = w["grad_accum"], w["micro_batch"], w["seq_len"], w["vocab"]
    toks = [tuple(torch.from_numpy(x).to(dev) for x in tokens_and_targets(B, T, V, w["seed"], w["zipf_s"],
                                                                        w["repeat_frac"], micro=i))
            for i in range(A)]
    st = model.stream

    def step():
        for tok, tgt in toks:
            model.forward_loss(tok, tgt)
            model.backward_step(args.lr)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clk:
        e0.record(st)
        for _ in range(args.steps):
            step()
        e1.record(st)
        torch.cuda.synchronize()
    step_ms = e0.elapsed_time(e1) / args.steps
    g.gpt_profile_enable(model.h, 1)
    for _ in range(args.steps):
        step()
    prof = g.gpt_profile_read(model.h)
    g.gpt_profile_enable(model.h, 0)
    if model.sync_status() != g.GPT_OK:
        raise RuntimeError(f"Muon step: device error {g.gpt_last_error()}")
    mu = {k: v for k, v in prof.items() if k.startswith("muon")}
    ms = sum(v["ms"] for v in mu.values()) / args.steps
    ns_ms = sum(v["ms"] for k, v in mu.items() if k.startswith("muon.")) / args.steps
    ns_flops = sum(v["flops"] for k, v in mu.items() if k.startswith("muon.")) / args.steps
    peaks, peak_src = measured_peaks()
    tflops = ns_flops / (ns_ms * 1e-3) / 1e12 if ns_ms else None
    d, f, L = w["d_model"], w["d_ff"], w["n_layer"]
    line = {"metric": "Muon optimizer step over the block matrices inside the training step (CUDA-event time)",
            "unit": "ms", "value": ms, "workload": w["name"], "matrices": 6 * L, "ns_steps": w.get("muon_ns_steps", 5),
            "training_step_ms": step_ms, "share_of_step": ms / step_ms,
            "ns_gemm_ms": ns_ms, "ns_gemm_flops": ns_flops, "tflops": tflops, "peak_tflops": peaks["bf16_tflops"],
            "frac_of_peak": (tflops / peaks["bf16_tflops"]) if tflops else None,
            "peak_source": f"{peak_src} bf16 burst",
            "launches_per_step": sum(v["launches"] for v in mu.values()) / args.steps,
            "steps": args.steps, "warmup": args.warmup, "l2": "no flush: W, M, G of the matrices exceed L2",
            "clocks": clk.summary()}
    print(json.dumps(line), flush=True)


def run_fp8(args, w):
    """The FP8 GEMM path against the bf16 one on the same products: the
    up-projection (N*d -> d_ff) and the LM-head logits chunk (8192 x vocab)
    of the workload, e4m3 operands with per-tensor scales (fp32 output) vs
    bf16 operands, CUDA events around each call; outputs exceed L2 (no flush).
    FP8 peak: the measured bf16 peak times the nominal fp8/bf16 ratio (2)."""
    import torch
    import gpt_pretraining_step_decoder_b200 as g
    dev = torch.device("cuda", 0)
    st = torch.cuda.current_stream()
    peaks, peak_src = measured_peaks()
    N_tok, d, F, V = w["micro_batch"] * w["seq_len"], w["d_model"], w["d_ff"], w["vocab"]
    shapes = {"up_proj": (N_tok, F, d), "lm_head_chunk": (8192, V, d)}
    ws = torch.empty(g.fp8_quantize_workspace_bytes(), dtype=torch.uint8, device=dev)
    out = []
    for name, (M, N, K) in shapes.items():
        A = torch.randn((M, K), device=dev) * 0.05
        B = torch.randn((N, K), device=dev) * 0.02
        qa = torch.empty((M, K), dtype=torch.uint8, device=dev)
        qb = torch.empty((N, K), dtype=torch.uint8, device=dev)
        sa = torch.empty(1, device=dev)
        sb = torch.empty(1, device=dev)
        g.fp8_quantize(A, g.DTYPE_F32, M * K, qa, sa, ws, ws.numel())
        g.fp8_quantize(B, g.DTYPE_F32, N * K, qb, sb, ws, ws.numel())
        Ab, Bb = A.to(torch.bfloat16), B.to(torch.bfloat16)
        C = torch.empty((M, N), dtype=torch.float32, device=dev)
        calls = {"fp8": lambda: g.gptx_gemm_fp8(M, N, K, qa, K, qb, K, sa, sb, g.DTYPE_F32, C, N),
                 "bf16": lambda: g.gptx_gemm_bf16(M, N, K, Ab, K, 1, Bb, K, 1, C, N, 0, 1, None, 0,
                                                  mode=g.EPI_STORE_F32)}
        rec = {"product": name, "M": M, "N": N, "K": K}
        for cname, fn in calls.items():
            times = []
            for it in range(args.warmup + args.steps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(st)
                fn()
                e1.record(st)
                torch.cuda.synchronize()
                if it >= args.warmup:
                    times.append(e0.elapsed_time(e1))
            us = 1e3 * float(np.median(times))
            tf = 2.0 * M * N * K / (us * 1e-6) / 1e12
            peak = peaks["bf16_tflops"] * (2.0 if cname == "fp8" else 1.0)
            rec[cname] = {"us": us, "tflops": tf, "peak_tflops": peak, "frac": tf / peak}
        rec["speedup"] = rec["bf16"]["us"] / rec["fp8"]["us"]
        out.append(rec)
        del A, B, qa, qb, Ab, Bb, C
    if g.ngram_sync_status() != g.GPT_OK:
        raise RuntimeError(f"fp8 measurement: device error {g.gpt_last_error()}")
    print(json.dumps({"metric": "FP8 (e4m3, per-tensor scales) vs bf16 GEMM on the step's products (CUDA events)",
                      "unit": "TFLOP/s", "workload": w["name"], "results": out,
                      "peak_source": f"{peak_src} bf16 burst; fp8 = 2 x bf16 (nominal ratio)",
                      "steps": args.steps, "warmup": args.warmup}), flush=True)


def parse_override(items):
    out = {}
    for it in items:
        k, v = it.split("=", 1)
        try:
            v = int(v)
        except ValueError:
            try:
                v = float(v)
            except ValueError:
                pass
        out[k] = v
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="gpt2s_bf16")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--lr", type=float, default=1e-4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-tables", action="store_true",
                    help="leave out the table-call bandwidth record of the default line")
    ap.add_argument("--measure", default="step", choices=["step", "tables", "muon", "fp8"],
                    help="step: the training step (default); tables: bandwidth of the bigram-table calls; "
                         "muon: one Muon step over the workload's matrix parameters")
    ap.add_argument("--override", nargs="*", default=[],
                    help="workload field overrides, e.g. n_layer=1 micro_batch=8 (profiling captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = workload(args.workload, **parse_override(args.override))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, w, rank, world)
        return
    if args.measure == "muon":
        import torch
        torch.cuda.set_device(0)
        run_muon(args, workload(args.workload, **parse_override(args.override)))
        return
    if args.measure == "fp8":
        import torch
        torch.cuda.set_device(0)
        run_fp8(args, w)
        return
    if args.measure == "tables":
        import torch
        torch.cuda.set_device(0)
        run_tables(args, workload(args.workload if args.workload != "gpt2s_bf16" else "gpt2s_tables_bf16",
                                  **parse_override(args.override)))
        return
    import torch
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    try:
        run_ours(args, w, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
