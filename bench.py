#!/usr/bin/env python
"""KVpop decode benchmark on B200: decode tokens/s and achieved HBM bandwidth.

One step = one KVpop decode step of every layer of the workload for every
batch row: per layer one kvpop_decode_step call (window append, boundary
scoring, argmin-replace and GQA attention over the bounded cache, fused in one
kernel launch), through the C ABI.  Default workload: Qwen3-4B-shaped,
87.5% compression (36 layers, 32 q / 8 kv heads, d 128, bf16, batch 64,
budget 1024 = 4 sinks + 128 window + 892 long-range, prompt 8192).  Data are
synthetic (seeded), shaped like the pages' workloads; the cache (9.7 GB) is
far larger than L2, so no flush is needed between steps.

`--path prefill-attention` times instead the parallel sparse prefill
attention of one layer of the same shape (kvpop_prefill_attention: prompt
scores, running cutoffs and the masked attention of all 8192 positions) and
prints its own line, with the roofline against the bf16 tensor peak.

Prints one JSON line (rank 0).  `--impl reference` times the CPU oracle
instead (the reference arm).  Multi-GPU: one replica per rank (the path
shards into independent (batch row, KV head) units; no data-path
collective), timed as the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import kvpop_workloads as wl  # noqa: E402

WORKLOADS = {"cr88": wl.QWEN3_4B_CR88, "cr75": wl.QWEN3_4B_CR75, "8b_d32": wl.QWEN3_8B_D32}
METRIC = "decode tokens/s and achieved HBM GB/s (% of peak) at 75%/88% KV compression"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None, help="timed steps (default 200 decode, 10 prefill-attention)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["kvpop", "reference"], default="kvpop")
    ap.add_argument("--path", choices=["decode", "prefill-attention"], default="decode",
                    help="decode (the headline) or the parallel sparse prefill attention of one layer")
    ap.add_argument("--pa-batch", type=int, default=0,
                    help="prefill-attention path: batch rows (default: the workload's; smaller for profiling)")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="cr88")
    ap.add_argument("--e2e-steps", type=int, default=None, help="e2e timed steps (default: --steps)")
    ap.add_argument("--e2e-warmup", type=int, default=None, help="e2e warm-up steps (default: --warmup)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other configurations (75%% compression, 8B with delayed scoring) and the sweep")
    ap.add_argument("--no-sweep", action="store_true", help="skip the bandwidth sweep")
    ap.add_argument("--cpu-workers", type=int, default=0,
                    help="processes of the parallel oracle leg (default: min(host CPUs, 16))")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--input-sets", type=int, default=32, help="distinct decode input sets, cycled")
    ap.add_argument("--graph", action="store_true",
                    help="capture one step (all layers' launches) per input set in CUDA graphs and replay them")
    ap.add_argument("--log-decay", type=float, default=None,
                    help="temporal decay: ln(gamma) <= 0 for every KV head (default: no decay)")
    ap.add_argument("--layers", type=int, default=0,
                    help="override the layer count (small cases for ncu captures; renames the workload)")
    return ap.parse_args()


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ---------------------------------------------------------------------------
# algorithmic bytes
# ---------------------------------------------------------------------------

def attention_bytes(w: wl.Workload) -> int:
    """Bytes one attention launch (one layer, all units) must move at steady
    state: every occupied slot row [k | v] once, q in, output out."""
    es = 2 if w.dtype == "bf16" else 4
    units = w.batch * w.n_kv_heads
    slots = w.sinks + w.window + w.delay + w.topk
    return units * slots * 2 * w.head_dim * es + 2 * w.batch * w.n_q_heads * w.head_dim * es


def step_bytes(w: wl.Workload) -> int:
    """Algorithmic HBM bytes of one whole decode step (all layers, all rows):
    K/V read + q + out + new K/V write + boundary K/V read + replace copy +
    long-range score scan, per (batch row, layer); scorer weights once."""
    es = 2 if w.dtype == "bf16" else 4
    d, Hkv, Hq = w.head_dim, w.n_kv_heads, w.n_q_heads
    per_row_layer = (Hkv * (w.sinks + w.window + w.delay + w.topk) * 2 * d * es
                     + Hq * d * es + Hq * d * es
                     + Hkv * 3 * 2 * d * es
                     + Hkv * w.topk * 8)
    weights = w.n_layers * Hkv * (w.scorer_hidden * 2 * d + 2 * w.scorer_hidden + 1) * 4
    return w.batch * w.n_layers * per_row_layer + weights


# DRAM bytes (read + write) of one decode_kernel launch, from one ncu capture
# of `bench.py --layers 2 --steps 2 --warmup 1` (the cr88 shape, 2 layers),
# valid only for the kernel sources whose hash is recorded with it.
TRAFFIC_CAPTURE = {"workload": "qwen3_4b_cr88_b64_B1024",
                   "sources_sha256": "9b3c42ad75e0dfdd3a80099795cac9f95def999cb44b67e34a6f3c33d411fb84",
                   "dram_bytes": 280_001_792 + 6_511_872, "algorithmic_bytes": 274_452_512}


# ncu capture of the prefill attention's tensor-core kernel (the small case of
# profiles/sparse_attn_tcp_kernel_cr88_b4_full.md: 4 rows x 8 KV heads =
# 32 units, prompt 8192): DRAM read + write of one launch.  Traffic grows with
# the units a launch covers (every unit reads its own q, k, v and writes its
# own output), so a launch of U units moves dram_bytes * U / 32.
PA_TRAFFIC_CAPTURE = {"workload": "qwen3_4b_cr88_b64_B1024", "units": 32,
                      "kernel_sha256": "beca722c9380e6e50b89152aefac4c8391a573c3bc8487aa3d4ab72b68a25f90",
                      "dram_bytes": 403_797_248 + 239_627_520}


def _strip_code(src: str) -> str:
    import re
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(ln.strip() for ln in src.splitlines() if ln.strip())


def mma_kernel_sha256() -> str:
    """sha256 of the prefill attention's tensor-core kernel (its section of
    kvpop_prefill_attn.cu with its launcher, comments and blank lines removed)."""
    import hashlib
    with open(os.path.join(ROOT, "fixed_budget_kv_kvpop_b200", "csrc", "kvpop_prefill_attn.cu")) as fh:
        src = fh.read()
    a = src.index("bf16 attention on tcgen05: persistent, two row blocks per work item")
    b = src.index("int launch_attn_f32(")
    return hashlib.sha256(_strip_code(src[a:b]).encode()).hexdigest()


def kernel_sources_sha256() -> str:
    """sha256 of the decode kernel's code: its two source files with comments
    and blank lines removed (a comment edit does not change the kernel)."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in ("kvpop_decode.cu", "kvpop_internal.cuh"):
        with open(os.path.join(ROOT, "fixed_budget_kv_kvpop_b200", "csrc", f)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update("\n".join(ln.strip() for ln in src.splitlines() if ln.strip()).encode())
    return h.hexdigest()


def measured_traffic(w: wl.Workload, abytes: int):
    """ncu DRAM bytes per launch scaled to this workload's launch (traffic grows
    with the cache rows a launch reads), or None when the capture was taken
    on other kernel sources or another shape family."""
    c = TRAFFIC_CAPTURE
    if not c["dram_bytes"] or not w.name.startswith(c["workload"]):
        return None
    if kernel_sources_sha256() != c["sources_sha256"]:
        return None
    return c["dram_bytes"] * abytes / c["algorithmic_bytes"]


# ---------------------------------------------------------------------------
# clocks sampling during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and reference arm)
# ---------------------------------------------------------------------------

class OracleSample:
    """A bounded sample of the workload on the CPU oracle: `n_units` units of
    the workload's shape (prompt of P tokens prefilled, untimed), stepped one
    decode token at a time."""

    def __init__(self, w: wl.Workload, n_units: int, max_steps: int, seed: int = 1):
        import numpy as np
        from oracle import kvpop_oracle as orc
        self.orc = orc
        one = w.replace(batch=1, n_layers=1)
        k, v = wl.prompt_kv(one, 0, master=seed)
        qd, kd, vd = wl.decode_inputs_batched(one, 0, max_steps, master=seed)
        w1, b1, w2, b2 = wl.scorer_weights(one, master=seed)
        self.units = []
        G = w.group
        for u in range(n_units):
            h = u % w.n_kv_heads
            k_all = np.concatenate([k[0, h].double().numpy(), kd[:, 0, h].double().numpy()])
            v_all = np.concatenate([v[0, h].double().numpy(), vd[:, 0, h].double().numpy()])
            q_steps = qd[:, 0, h * G:(h + 1) * G].double().numpy()
            s = orc.unit_scores_mlp(k_all, v_all, w1[0, h].double().numpy(), b1[0, h].double().numpy(),
                                    w2[0, h].double().numpy(), float(b2[0, h]))
            unit = orc.OracleUnit(k_all, v_all, s, w.sinks, w.window, w.delay, w.topk, w.prefill,
                                  check_simulator=False)
            self.units.append((unit, q_steps))
        self.i = 0

    def step(self):
        for unit, q_steps in self.units:
            unit.step(q_steps[self.i])
        self.i += 1


def host_info():
    """The host the CPU oracle runs on: logical CPUs and the CPU model."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


def cpu_threads_limit():
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(limits=1)
    except Exception:
        return None


def oracle_tokens_per_s(w: wl.Workload, seconds: float):
    """Times the oracle's decode steps on a bounded sample; returns
    (tokens/s, description)."""
    units_per_token = w.n_layers * w.n_kv_heads
    n_units, max_steps = 4, 400
    lim = cpu_threads_limit()
    sample = OracleSample(w, n_units, max_steps)
    t0 = time.perf_counter()
    steps = 0
    while steps < max_steps and (time.perf_counter() - t0 < seconds or steps < 2):
        sample.step()
        steps += 1
    dt = time.perf_counter() - t0
    if lim is not None:
        lim.unregister() if hasattr(lim, "unregister") else None
    unit_steps = n_units * steps
    tok_s = unit_steps / units_per_token / dt
    desc = (f"{n_units} (batch row, KV head) units of the {w.name} shape, prompt {w.prefill} prefilled "
            f"untimed, {steps} decode steps each timed ({unit_steps} unit-steps, {dt:.1f} s); one decode "
            f"token = {units_per_token} unit-steps (all layers and KV heads of one batch row)")
    return tok_s, desc


def _oracle_worker(w, seed, seconds, max_steps, barrier, results):
    """One process of the parallel oracle leg: one unit of the workload's
    shape, prefilled (untimed), then decode steps for `seconds` after every
    worker is ready."""
    import threadpoolctl
    with threadpoolctl.threadpool_limits(limits=1):
        sample = OracleSample(w, 1, max_steps, seed=seed)
        barrier.wait(timeout=600)
        t0 = time.perf_counter()
        steps = 0
        while steps < max_steps and (time.perf_counter() - t0 < seconds or steps < 2):
            sample.step()
            steps += 1
        results.put((steps, time.perf_counter() - t0))


def oracle_parallel_tokens_per_s(w: wl.Workload, seconds: float, workers: int):
    """The oracle on `workers` host cores at once: one process per core
    (started with spawn, safe after CUDA initialisation), each stepping its
    own unit of the workload's shape.  Units are independent, so the
    throughput is the sum of the processes' unit-step rates.  Returns
    (tokens/s, cores used, description)."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    barrier = ctx.Barrier(workers)
    results = ctx.Queue()
    max_steps = 4000
    procs = [ctx.Process(target=_oracle_worker, args=(w, 100 + i, seconds, max_steps, barrier, results))
             for i in range(workers)]
    for p_ in procs:
        p_.start()
    got = [results.get(timeout=900) for _ in procs]
    for p_ in procs:
        p_.join(timeout=60)
    units_per_token = w.n_layers * w.n_kv_heads
    rate = sum(st / dt for st, dt in got)          # unit-steps per second, all processes together
    steps = sum(st for st, _ in got)
    mean_dt = sum(dt for _, dt in got) / len(got)
    desc = (f"{workers} processes on {workers} host cores, each one (batch row, KV head) unit of the {w.name} "
            f"shape (prompt {w.prefill} prefilled untimed), stepped for {mean_dt:.1f} s on average after all "
            f"were ready ({steps} unit-steps in all); one decode token = {units_per_token} unit-steps")
    return rate / units_per_token, workers, desc


def run_reference(args, w, rank, world):
    if rank != 0:
        return
    units_per_token = w.n_layers * w.n_kv_heads
    n_units = 2
    lim = cpu_threads_limit()
    sample = OracleSample(w, n_units, args.warmup + args.steps + 1)
    for _ in range(args.warmup):
        sample.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        sample.step()
    dt = time.perf_counter() - t0
    tok_s = n_units * args.steps / units_per_token / dt
    desc = (f"each step: one decode step of {n_units} units of the {w.name} shape on the CPU oracle "
            f"(prompt {w.prefill} prefilled untimed); tokens = unit-steps / {units_per_token}")
    line = {
        "impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": w.name, "sample": desc},
        "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": desc,
                         "host": host_info()},
        "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# Multi-GPU: independent replicas, one per rank (no data-path collective)
# ---------------------------------------------------------------------------

def max_over_ranks(value: float, world: int, torch, device) -> float:
    """The slowest rank's time: every rank must call this at the same point
    (one all-reduce, MAX); device 'cuda' under NCCL, 'cpu' under gloo."""
    if world <= 1:
        return value
    t = torch.tensor([value], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(batch: int, steps: int, world: int, elapsed_ms: float) -> float:
    """Whole-job decode tokens/s: every rank decodes `batch` rows for `steps`
    steps, and the job takes the slowest rank's time."""
    return batch * steps * world / (elapsed_ms / 1e3)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

MLSTM_DIMS = (16, 16)   # mLSTM scorer of the bench: Hedgehog projection p, value size dv


def build_cache(w: wl.Workload, torch, log_decay=None, prompt=None, scorer="mlp"):
    """A cache for every layer of `w`, each layer prefilled with `prompt`
    tokens (default: the workload's prompt) in one kvpop_prefill call.
    scorer: 'mlp' (the workload's MLP) or 'mlstm' (the stateful scorer with
    seeded weights, p = dv = 16)."""
    import fixed_budget_kv_kvpop_b200 as kp
    P = w.prefill if prompt is None else prompt
    weights = tuple(t.cuda() for t in wl.scorer_weights(w))
    w1, b1, w2, b2 = weights
    extra = {}
    if scorer == "mlstm":
        packed = wl.mlstm_weights(w, *MLSTM_DIMS).cuda()
        weights = weights + (packed,)
        extra = dict(scorer="mlstm", mlstm_p=MLSTM_DIMS[0], mlstm_dv=MLSTM_DIMS[1], mlstm_w=packed)
    decay = None
    if log_decay is not None:
        decay = torch.full((w.n_layers, w.n_kv_heads), float(log_decay), dtype=torch.float32, device="cuda")
        weights = weights + (decay,)
    cfg = kp.make_config(batch=w.batch, n_layers=w.n_layers, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                         head_dim=w.head_dim, sinks=w.sinks, window=w.window, topk=w.topk, delay=w.delay,
                         ref_context=w.prefill, compression_ratio=w.compression_ratio,
                         max_prefill_chunk=P, dtype=w.dtype, scorer_hidden=w.scorer_hidden,
                         w1=w1, b1=b1, w2=w2, b2=b2, log_decay=decay, **extra)
    cache = kp.KVPopCache(cfg, keepalive=weights)
    stream = torch.cuda.current_stream()
    prefill_ms = []
    for layer in range(w.n_layers):
        k, v = wl.prompt_kv(w, layer, n_tokens=P, device="cuda")
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        cache.prefill(layer, k, v, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        prefill_ms.append(e0.elapsed_time(e1))
        del k, v
    torch.cuda.synchronize()
    return cache, prefill_ms


def prefill_summary(w: wl.Workload, prefill_ms):
    """The prefill build (one kvpop_prefill per layer, whole prompt in one
    chunk): time per layer, prompt tokens per second, and the fp64 rate of its
    scorer (2 * 2d * hidden flops for every token that leaves the window)."""
    ms = statistics.median(prefill_ms)
    eligible = max(0, w.prefill - w.window - w.delay - w.sinks)
    flops = w.batch * w.n_kv_heads * eligible * 2.0 * (2 * w.head_dim) * w.scorer_hidden
    return {"ms_per_layer": ms, "prompt_tokens_per_s": w.batch * w.prefill / (ms / 1e3),
            "scorer_fp64_tflops_lower_bound": flops / (ms / 1e3) / 1e12, "layers_timed": len(prefill_ms),
            "note": "one-off per prompt, not in the decode tokens/s; the TFLOP/s figure divides the scorer's "
                    "flops by the whole prefill time (select, move and write included)"}


def smi_index(torch):
    dev = torch.cuda.current_device()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        try:
            return int(vis.split(",")[dev])
        except (ValueError, IndexError):
            return dev
    return dev


def time_decode(w, cache, steps, warmup, torch, world, input_sets=32, graph=False):
    """Times `steps` decode steps (every layer, every batch row) after
    `warmup` untimed ones, on the current stream, with CUDA events around the
    launches and nvidia-smi sampling the clocks; the time is the max over
    ranks.  Returns the measurement as a dict."""
    stream = torch.cuda.current_stream()
    L = w.n_layers
    NI = max(1, min(input_sets, steps + warmup))
    qs, ks, vs = [], [], []
    for layer in range(L):
        q, k, v = wl.decode_inputs_batched(w, layer, NI, device="cuda")
        qs.append(q); ks.append(k); vs.append(v)
    outs = [torch.empty_like(qs[0][0]) for _ in range(L)]
    torch.cuda.synchronize()

    def launch_step(j, st):
        for layer in range(L):
            cache.decode_step(layer, qs[layer][j], ks[layer][j], vs[layer][j], outs[layer], stream=st)

    graphs = []

    def one_step(i):
        if graphs:
            graphs[i % len(graphs)].replay()
        else:
            launch_step(i % NI, stream)

    for i in range(warmup):
        one_step(i)
    torch.cuda.synchronize()
    if graph:
        # Capture (not run) one step per input set.  Each replay advances the
        # layers' device-side counters like an eager step; only the library's
        # host mirrors (used for argument validation) run ahead.
        for j in range(min(NI, 4)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                launch_step(j, torch.cuda.current_stream())
            graphs.append(g)
        for i in range(3):
            one_step(i)
        torch.cuda.synchronize()
    st, bits = cache.get_error()
    if st != 0:
        raise RuntimeError(f"device error after warm-up: status {st} bits {bits}")
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(smi_index(torch))
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    start.record(stream)
    for s in range(steps):
        one_step(warmup + s)
    end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    elapsed_ms = start.elapsed_time(end)
    st, bits = cache.get_error()
    if st != 0:
        raise RuntimeError(f"device error in timed region: status {st} bits {bits}")
    elapsed_ms = max_over_ranks(elapsed_ms, world, torch, "cuda")
    peak, peak_kind = measured_peaks()
    sbytes = step_bytes(w)
    step_gbs = sbytes * steps / (elapsed_ms / 1e3) / 1e9
    # The timed region holds nothing but these launches, back to back on one
    # stream (no event between them, so programmatic dependent launch can
    # overlap one launch's tail with the next one's prologue): the average
    # launch duration is the region's duration over the launch count.
    n_launches = L * steps
    del graphs
    return {"elapsed_ms": elapsed_ms, "ms_per_step": elapsed_ms / steps,
            "tokens_per_s": replica_throughput(w.batch, steps, world, elapsed_ms),
            "step_bytes": sbytes, "achieved_gbs": step_gbs, "peak_gbs": peak, "frac": step_gbs / peak,
            "frac_of_8tbs": step_gbs / 8000.0, "peak_kind": peak_kind,
            "mean_launch_us": elapsed_ms / n_launches * 1e3, "launches": n_launches,
            "bytes_per_launch": sbytes // L, "clocks": clocks, "input_sets": len(graphs) if graph else NI}


def run_gpu(args, w, rank, world, torch):
    t_setup = time.perf_counter()
    cache, prefill_ms = build_cache(w, torch, args.log_decay)
    torch.cuda.synchronize()
    setup_s = time.perf_counter() - t_setup
    m = time_decode(w, cache, args.steps, args.warmup, torch, world, args.input_sets, args.graph)
    L = w.n_layers
    abytes = m["bytes_per_launch"]
    attn_gbs = abytes / (m["mean_launch_us"] / 1e6) / 1e9

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, w, cache, torch, world)

    res = {
        "metric": METRIC, "value": m["tokens_per_s"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": m["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "layers": w.n_layers, "q_heads": w.n_q_heads,
                   "kv_heads": w.n_kv_heads, "head_dim": w.head_dim, "sinks": w.sinks, "window": w.window,
                   "topk": w.topk, "delay": w.delay, "budget": w.budget, "prompt": w.prefill,
                   "compression": round(w.compression_ratio, 4), "parallelism": f"replicas x{world}",
                   "l2": "no flush: inputs (cache %.1f GB) larger than L2" % (w.n_layers * attention_bytes(w) / 1e9),
                   "input_sets": m["input_sets"], "log_decay": args.log_decay, "cuda_graph": bool(args.graph)},
        "hbm": {k: m[k] for k in ("step_bytes", "achieved_gbs", "peak_gbs", "frac", "frac_of_8tbs", "peak_kind")},
        "roofline": {"kernel": "decode_kernel (fused append + attend, one launch per layer)",
                     "bound": "hbm", "achieved": attn_gbs,
                     "peak": m["peak_gbs"], "unit": "GB/s", "frac": attn_gbs / m["peak_gbs"],
                     "traffic": measured_traffic(w, abytes),
                     "bytes_per_launch": abytes, "mean_launch_us": m["mean_launch_us"],
                     "launches": m["launches"], "peak_kind": m["peak_kind"]},
        "gpu_launches": m["launches"],
        "prefill": prefill_summary(w, prefill_ms),
        "clocks": m["clocks"],
        "setup_s": setup_s,
    }
    if e2e is not None:
        res["e2e"] = e2e
    del cache
    torch.cuda.empty_cache()
    return res


def other_config(args, w, torch, world, prompt=None, note=None, scorer="mlp"):
    """Decode throughput of another configuration, timed like the headline
    (same steps and warm-up; no e2e or CPU leg)."""
    t0 = time.perf_counter()
    cache, prefill_ms = build_cache(w, torch, None, prompt, scorer)
    m = time_decode(w, cache, args.steps, args.warmup, torch, world, args.input_sets)
    del cache
    torch.cuda.empty_cache()
    out = {"workload": w.name, "batch": w.batch, "layers": w.n_layers, "budget": w.budget, "delay": w.delay,
           "prompt": w.prefill if prompt is None else prompt, "compression": round(w.compression_ratio, 4),
           "tokens_per_s": m["tokens_per_s"], "ms_per_step": m["ms_per_step"],
           "achieved_gbs": m["achieved_gbs"], "frac": m["frac"], "frac_of_8tbs": m["frac_of_8tbs"],
           "mean_launch_us": m["mean_launch_us"], "bytes_per_launch": m["bytes_per_launch"],
           "launches": m["launches"], "clocks": m["clocks"], "prefill_ms_per_layer": statistics.median(prefill_ms),
           "wall_s": time.perf_counter() - t0}
    if note:
        out["note"] = note
    return out


SWEEP_CACHE_CAP = 80e9   # bytes of cache a sweep point may hold (HBM is 180 GB)


def sweep_plan(budgets=wl.SWEEP_BUDGETS, batches=wl.SWEEP_BATCHES, cap=SWEEP_CACHE_CAP):
    """The bandwidth sweep on the Qwen3-8B shape: per (budget, batch) the
    workload, the layers it runs (36, or fewer when the 36-layer cache would
    exceed `cap`), and the prompt it prefills (budget + 256 tokens: a decode
    step reads the whole bounded cache, whose size does not depend on how
    long the prompt was once the long-range slots are full)."""
    plan = []
    for B in budgets:
        for b in batches:
            w = wl.sweep_point(B, b)
            per_layer = attention_bytes(w)
            layers = max(1, min(w.n_layers, int(cap // per_layer)))
            plan.append({"budget": B, "batch": b, "workload": w.replace(n_layers=layers), "layers": layers,
                         "full_cache_gb": per_layer * w.n_layers / 1e9, "prompt": B + 256})
    return plan


def run_sweep(args, torch, world):
    points = []
    for pt in sweep_plan():
        w = pt["workload"]
        notes = [f"prompt shortened from {w.prefill} to {pt['prompt']} tokens: the decode step reads the full "
                 "bounded cache either way"]
        if pt["layers"] < 36:
            notes.append(f"layers reduced to {pt['layers']} of 36: the 36-layer cache is "
                         f"{pt['full_cache_gb']:.0f} GB" + (", more than the 180 GB of HBM"
                                                             if pt["full_cache_gb"] > 180 else ""))
        r = other_config(args, w, torch, world, prompt=pt["prompt"], note="; ".join(notes))
        r.update({"budget": pt["budget"], "batch": pt["batch"], "layers_full": 36,
                  "layers_reduced": pt["layers"] < 36})
        points.append(r)
    return {"shape": "Qwen3-8B (36 layers, 32 q / 8 kv heads, d 128, bf16), 4 sinks, window 128, K = B - 132, D 0",
            "points": points}


def run_e2e(args, w, cache, torch, world):
    """Same metric through the C ABI with the step's inputs in pinned HOST
    memory: each step copies q/k/v of all layers host->device, runs the step,
    and copies the outputs device->host, pipelined over two buffers and three
    streams (copy-in, compute, copy-out)."""
    L = w.n_layers
    K = max(1, args.e2e_steps if args.e2e_steps is not None else args.steps)
    WU = max(1, args.e2e_warmup if args.e2e_warmup is not None else args.warmup)
    NI = 4
    hq = [torch.empty((L,) + (w.batch, w.n_q_heads, w.head_dim), dtype=w.torch_dtype()).pin_memory()
          for _ in range(NI)]
    hk = [torch.empty((L, w.batch, w.n_kv_heads, w.head_dim), dtype=w.torch_dtype()).pin_memory()
          for _ in range(NI)]
    hv = [torch.empty_like(hk[0]).pin_memory() for _ in range(NI)]
    for i in range(NI):
        for layer in range(L):
            q, k, v = wl.decode_inputs(w, layer, 10_000 + i)
            hq[i][layer].copy_(q); hk[i][layer].copy_(k); hv[i][layer].copy_(v)
    hout = [torch.empty_like(hq[0]).pin_memory() for _ in range(2)]
    dq = [torch.empty_like(hq[0], device="cuda") for _ in range(2)]
    dk = [torch.empty_like(hk[0], device="cuda") for _ in range(2)]
    dv = [torch.empty_like(hk[0], device="cuda") for _ in range(2)]
    dout = [torch.empty_like(hq[0], device="cuda") for _ in range(2)]
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()

    def step(s, first):
        b = s % 2
        with torch.cuda.stream(s_in):
            if not first[b]:
                s_in.wait_event(ev_cmp[b])
            dq[b].copy_(hq[s % NI], non_blocking=True)
            dk[b].copy_(hk[s % NI], non_blocking=True)
            dv[b].copy_(hv[s % NI], non_blocking=True)
            ev_in[b].record(s_in)
        s_cmp.wait_event(ev_in[b])
        if not first[b]:
            s_cmp.wait_event(ev_out[b])
        for layer in range(L):
            cache.decode_step(layer, dq[b][layer], dk[b][layer], dv[b][layer], dout[b][layer], stream=s_cmp)
        ev_cmp[b].record(s_cmp)
        s_out.wait_event(ev_cmp[b])
        with torch.cuda.stream(s_out):
            hout[b].copy_(dout[b], non_blocking=True)
            ev_out[b].record(s_out)
        first[b] = False

    first = [True, True]
    for s in range(WU):
        step(s, first)
    torch.cuda.synchronize()
    start.record(s_in)
    for s in range(K):
        step(WU + s, first)
    end.record(s_out)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    ms = max_over_ranks(ms, world, torch, "cuda")
    es = 2 if w.dtype == "bf16" else 4
    h2d = L * w.batch * (w.n_q_heads + 2 * w.n_kv_heads) * w.head_dim * es
    d2h = L * w.batch * w.n_q_heads * w.head_dim * es
    return {"value": replica_throughput(w.batch, K, world, ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": K, "warmup": WU, "ms_per_step": ms / K,
            "note": "same step count and warm-up as the device-timed region; the copies of step s+1 and s-1 "
                    "overlap step s's launches (two buffers, three streams), so e2e can come out at or even "
                    "slightly below the device-only step time"}


PA_METRIC = "prefill attention tokens/s under the running top-k mask (one layer: scores, cutoffs, attention)"


def prefill_attention_flops(w: wl.Workload) -> float:
    """Algorithmic flops of one layer's prefill attention: 2 * d for q.k and
    2 * d for p.v per attended (position, query head) pair; position q attends
    to min(q + 1, S + W + D + K) tokens."""
    B = w.sinks + w.window + w.delay + w.topk
    pairs = sum(min(q + 1, B) for q in range(w.prefill))
    return 4.0 * w.head_dim * pairs * w.n_q_heads * w.batch


def oracle_prefill_rows_per_s(w: wl.Workload, seconds: float):
    """The oracle's per-position computation (running top-k at q, attended set,
    attention) on rows sampled evenly over one unit's prompt."""
    import numpy as np
    from oracle import kvpop_oracle as orc
    one = w.replace(batch=1, n_layers=1)
    k, v = wl.prompt_kv(one, 0, master=1)
    q = wl.prompt_queries(one, 0, master=1)
    w1, b1, w2, b2 = wl.scorer_weights(one, master=1)
    G = w.group
    kk, vv = k[0, 0].double().numpy(), v[0, 0].double().numpy()
    qq = q[0, :G].double().numpy().transpose(1, 0, 2)
    s = orc.unit_scores_mlp(kk, vv, w1[0, 0].double().numpy(), b1[0, 0].double().numpy(),
                            w2[0, 0].double().numpy(), float(b2[0, 0]))
    rows = np.linspace(0, w.prefill - 1, 2048).astype(int)
    lim = cpu_threads_limit()   # one core, as the line's "cores" says
    t0 = time.perf_counter()
    done = 0
    for qp in rows:
        T = orc.running_topk(s, int(qp), w.sinks, w.window, w.delay, w.topk)
        A = orc.attended_positions(int(qp), w.sinks, w.window, w.delay, T)
        orc.attention(qq[qp], kk[A], vv[A])
        done += 1
        if time.perf_counter() - t0 > seconds:
            break
    dt = time.perf_counter() - t0
    if lim is not None and hasattr(lim, "unregister"):
        lim.unregister()
    tok_s = done / dt / w.n_kv_heads
    desc = (f"{done} prompt positions of one (batch row, KV head) unit of the {w.name} shape, spread evenly "
            f"over the {w.prefill}-token prompt, scores untimed ({dt:.1f} s); one prompt token = "
            f"{w.n_kv_heads} unit-rows (all KV heads of one batch row, one layer)")
    return tok_s, desc


def run_prefill_attention(args, w, torch):
    import fixed_budget_kv_kvpop_b200 as kp
    steps = args.steps if args.steps is not None else 10
    one = w.replace(name=w.name + "_L1", n_layers=1)
    if args.pa_batch:
        one = one.replace(name=f"{w.name}_L1_b{args.pa_batch}", batch=args.pa_batch)
    weights = tuple(t.cuda() for t in wl.scorer_weights(one))
    w1, b1, w2, b2 = weights
    cfg = kp.make_config(batch=one.batch, n_layers=1, n_q_heads=one.n_q_heads, n_kv_heads=one.n_kv_heads,
                         head_dim=one.head_dim, sinks=one.sinks, window=one.window, topk=one.topk,
                         delay=one.delay, ref_context=one.prefill, compression_ratio=one.compression_ratio,
                         max_prefill_chunk=1, dtype=one.dtype, scorer_hidden=one.scorer_hidden,
                         w1=w1, b1=b1, w2=w2, b2=b2)
    cache = kp.KVPopCache(cfg, keepalive=weights)
    n = one.prefill
    k, v = wl.prompt_kv(one, 0, device="cuda")
    q = wl.prompt_queries(one, 0, device="cuda")
    out = torch.empty_like(q)
    lse = torch.empty((one.batch, one.n_q_heads, n), dtype=torch.float32, device="cuda")
    ws = torch.empty(cache.prefill_attention_workspace_bytes(n), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(max(args.warmup, 3)):
        cache.prefill_attention(0, q, k, v, out, lse, ws, stream=stream)
    torch.cuda.synchronize()
    st, bits = cache.get_error()
    if st != 0:
        raise RuntimeError(f"device error after warm-up: status {st} bits {bits}")
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        cache.prefill_attention(0, q, k, v, out, lse, ws, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    # the attention kernel alone: the same call from the cutoffs the calls
    # above left in the workspace (no scoring, no cutoff kernel)
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for _ in range(steps):
        cache.prefill_attention_from_cutoffs(0, q, k, v, out, lse, ws, stream=stream)
    e3.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1) / steps
    attn_ms = e2.elapsed_time(e3) / steps
    st, bits = cache.get_error()
    if st != 0:
        raise RuntimeError(f"device error in timed region: status {st} bits {bits}")
    flops = prefill_attention_flops(one)
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peak, kind = float(json.load(f)["bf16_tflops"]), "measured (burst)"
    except Exception:
        peak, kind = 1590.0, "fallback"
    achieved = flops / (attn_ms / 1e3) / 1e12
    call_tflops = flops / (ms / 1e3) / 1e12
    cap = PA_TRAFFIC_CAPTURE
    units = one.batch * one.n_kv_heads
    traffic = None
    if w.name.startswith(cap["workload"]) and mma_kernel_sha256() == cap["kernel_sha256"]:
        traffic = cap["dram_bytes"] * units / cap["units"]
    esize = 2 if one.dtype == "bf16" else 4
    io_bytes = (2 * q.numel() + 2 * k.numel()) * esize   # q, k, v read; output written
    res = {
        "metric": PA_METRIC, "value": one.batch * n / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1,
        "steps": steps, "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": one.dtype, "data": "synthetic",
        "config": {"workload": one.name, "batch": one.batch, "layers": 1, "q_heads": one.n_q_heads,
                   "kv_heads": one.n_kv_heads, "head_dim": one.head_dim, "sinks": one.sinks,
                   "window": one.window, "topk": one.topk, "delay": one.delay, "prompt": n,
                   "l2": "no flush: q, k, v (%.1f GB) larger than L2" % ((q.numel() + 2 * k.numel()) * esize / 1e9)},
        "roofline": {"kernel": "the masked attention kernel alone (bf16: tcgen05, TMEM accumulators)",
                     "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic, "flops_per_launch": flops, "peak_kind": kind,
                     "mean_launch_ms": attn_ms, "attention_io_bytes": io_bytes,
                     "note": "CUDA events around kvpop_prefill_attention_from_cutoffs calls (one attention "
                             "launch each, the cutoffs of the timed calls reused); traffic = the attention "
                             "kernel's DRAM bytes per launch from an ncu capture of 32 units, scaled by units"},
        "whole_call": {"ms": ms, "tflops": call_tflops, "frac": call_tflops / peak,
                       "kernels": "prompt scorer + cutoff_kernel + attention"},
        "gpu_launches": 3 * steps + steps,
        "clocks": clocks,
    }
    if not args.no_cpu_baseline:
        v_, desc = oracle_prefill_rows_per_s(one, args.cpu_seconds)
        res["cpu_baseline"] = {"value": v_, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": desc,
                               "host": host_info()}
    return res


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = WORKLOADS[args.workload]
    if args.layers and args.layers != w.n_layers:
        w = w.replace(name=f"{w.name}_L{args.layers}", n_layers=args.layers)
    if args.impl == "reference":
        if args.steps is None:
            args.steps = 200
        run_reference(args, w, rank, world)
        return
    import torch
    torch.cuda.set_device(local)
    if args.path == "prefill-attention":
        if world > 1 and rank != 0:
            return
        print(json.dumps(run_prefill_attention(args, w, torch)), flush=True)
        return
    if args.steps is None:
        args.steps = 200
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        res = run_gpu(args, w, rank, world, torch)
        # The other configurations of the metric, timed the same way (single
        # GPU runs only: under torchrun every rank would have to repeat them).
        if world == 1 and not args.no_extras:
            extras = {}
            for key in ("cr75", "cr88", "8b_d32"):
                if WORKLOADS[key].name != w.name and not args.layers:
                    extras[key] = other_config(args, WORKLOADS[key], torch, world)
            res["configs"] = extras
            # the stateful mLSTM scorer with delayed readout on the headline shape
            res["mlstm"] = other_config(
                args, w, torch, world, scorer="mlstm",
                note=f"mLSTM scorer (p = {MLSTM_DIMS[0]}, dv = {MLSTM_DIMS[1]}, seeded weights): per layer and step "
                     "one mlstm_step_kernel (state update with the new token, delayed readout of the boundary "
                     "token, argmin decision) and one decode_kernel")
            res["mlstm"]["gpu_launches"] = 2 * res["mlstm"]["launches"]
            if not args.no_sweep:
                res["sweep"] = run_sweep(args, torch, world)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            v1, desc1 = oracle_tokens_per_s(w, args.cpu_seconds)
            single = {"value": v1, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": desc1}
            workers = args.cpu_workers or max(1, min(os.cpu_count() or 1, 16))
            try:
                vp, cores, descp = oracle_parallel_tokens_per_s(w, args.cpu_seconds, workers)
                res["cpu_baseline"] = {"value": vp, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                       "sample": descp, "single_core": single, "host": host_info()}
            except Exception as exc:   # the single-core figure still stands
                single.update({"host": host_info(), "parallel_leg_failed": repr(exc)[:200]})
                res["cpu_baseline"] = single
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
