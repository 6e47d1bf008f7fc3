"""Benchmark: one sparse-prefill attention layer per step (index build + block-sparse attention).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama8b] [--impl ours|reference]

Default workload: the Llama-3-8B-shaped layer at 128K context (S=131072, Hq=32,
Hkv=8, d=128, b=128, gamma=0.9, tau=0.1, bf16), seeded synthetic inputs.  A step
is fp_build_index + fp_sparse_attn on inputs resident in HBM; value is the
dense-equivalent throughput 2*Hq*d*S^2 / t (TFLOP/s) summed over ranks, and
ms_per_step is ms per layer.  Inputs (Q 1 GiB, K and V 256 MiB each) exceed the
126 MB L2, so no flush is needed between steps.  Under torchrun every rank runs
an independent replica (the layer does not shard on one node here).

--impl reference times the fp64 CPU oracle on the host cores on bounded samples
of the same workload (rank 0 only) and prints the same JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from dynamic_block_sparse_last_b200 import synth  # noqa: E402

METRIC = "sparse-prefill ms/layer & dense-equiv TFLOPS at S=128K; % of HBM/TC roofline"
UNIT = "dense-equiv TFLOP/s"
# the library's switch of the q-bar . k-bar logits to the tensor cores (kLgTensorMinN in
# index_kernels.cuh): from n = 640 blocks two k_split_tf32 launches precede k_qa_logits
LOGITS_TENSOR_MIN_N = 640


def kernels_per_step(S: int, b: int) -> int:
    """Launches of the library's kernels per layer step: k_score_last, k_head_stats,
    k_qpool, k_qa_logits (plus two k_split_tf32 on the tensor-core path), k_cut,
    k_sparse_attn."""
    n = (S + b - 1) // b
    return 6 + (2 if n >= LOGITS_TENSOR_MIN_N else 0)
ATTN_SRC = os.path.join(ROOT, "dynamic_block_sparse_last_b200", "csrc", "attn_kernel.cuh")


FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    """Roofline denominators: the measured copy bandwidth (GB/s) and bf16 GEMM
    throughput (TFLOP/s, burst and sustained) from MEASURED_PEAKS.json beside
    this file, else the pool's earlier measurement (source "fallback").  A file
    without positive numbers under those keys counts as absent."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        try:
            d = json.load(open(p))
            hbm, burst = float(d["hbm_gbs"]), float(d["bf16_tflops"])
            sus = float(d.get("bf16_tflops_sustained", burst))
            if hbm > 0 and burst > 0 and sus > 0:
                return {"hbm_gbs": hbm, "bf16_tflops": burst, "bf16_tflops_sustained": sus, "source": "measured"}
        except (ValueError, TypeError, KeyError, json.JSONDecodeError):
            pass
        return dict(FALLBACK_PEAKS, source="fallback (MEASURED_PEAKS.json unreadable)")
    return dict(FALLBACK_PEAKS, source="fallback")


def attn_traffic_record():
    """Per-launch DRAM bytes of the attention kernel from a committed ncu summary,
    or None when the kernel source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "attn_traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p))
    sha = hashlib.sha256(open(ATTN_SRC, "rb").read()).hexdigest()
    if rec.get("kernel_src_sha256") != sha:
        return None
    return rec


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


def computed_chunk_tiles(row_ptr, col, Hq: int, S: int, b: int) -> int:
    """128 x 128 query-tile x key-chunk tiles the attention kernel computes for
    an index in CSR form (rows h*n + r): a tile attends to every chunk of its
    listed blocks up to its own position; with b = 64 a tile holds two query
    blocks and a chunk two key blocks, so it computes the chunks of the union
    of both lists."""
    n = (S + b - 1) // b
    nq = (S + 127) // 128
    total = 0
    for h in range(Hq):
        lists = [col[row_ptr[h * n + r]: row_ptr[h * n + r + 1]] for r in range(n)]
        for qc in range(nq):
            if b >= 128:
                per, r = b // 128, qc * 128 // b
                total += (len(lists[r]) - 1) * per + qc % per + 1
            else:
                blocks = np.concatenate([lists[r] for r in (2 * qc, 2 * qc + 1) if r < n])
                total += len({int(c) // 2 for c in blocks if int(c) // 2 <= qc})
    return total


def attention_peak(bf16_peak: float, int8_peak=None) -> float:
    """Tensor peak for the attention's contractions.  bf16: the bf16 peak.
    W8A8 (int8_peak given): Q.K^T (half the FLOPs) runs at the int8 peak and
    P.V at the bf16 peak, so the roofline time of F FLOPs is
    F/2/P_i8 + F/2/P_bf16 and the effective peak 2 / (1/P_i8 + 1/P_bf16)."""
    if int8_peak is None:
        return bf16_peak
    return 2.0 / (1.0 / int8_peak + 1.0 / bf16_peak)


def int8_gemm_peak(dev, n: int = 8192, sustain_s: float = 1.5):
    """Measured int8 tensor throughput on this GPU: torch._int_mm (int8 x int8
    -> int32, a library GEMM) at n^3.  burst = best of 10 single launches;
    sustained = mean over a loop of about sustain_s seconds (the power-capped
    figure, for kernels timed inside a long step).  TOPS = 2 n^3 / t.
    Returns a dict, or None when the library call is unavailable."""
    try:
        a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev)
        b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev)
        for _ in range(3):
            torch._int_mm(a, b)
        torch.cuda.synchronize(dev)
        best = float("inf")
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._int_mm(a, b)
            e1.record()
            torch.cuda.synchronize(dev)
            best = min(best, e0.elapsed_time(e1))
        reps = max(10, int(sustain_s * 1e3 / best))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            torch._int_mm(a, b)
        e1.record()
        torch.cuda.synchronize(dev)
        mean = e0.elapsed_time(e1) / reps
        flops = 2.0 * n ** 3
        del a, b
        return {"burst_tops": flops / (best / 1e3) / 1e12, "sustained_tops": flops / (mean / 1e3) / 1e12,
                "n": n, "reps": reps, "how": "torch._int_mm int8 x int8 -> int32, CUDA events"}
    except (RuntimeError, AttributeError) as e:  # library call missing for this shape or build
        return {"unavailable": str(e).splitlines()[0][:200]}


def index_pass_floors(S: int, Hq: int, b: int, idx_bytes: int, hbm_gbs: float, sm_count: int, sm_mhz: float):
    """The index pass's two floors: its algorithmic bytes at the HBM copy
    bandwidth, and one exponential per (last-block row, causal key) of every
    head at 16 ex2 per clock per SM.  Returns (hbm_floor_ms, n_exp, mufu_floor_ms)."""
    n = (S + b - 1) // b
    nlast = S - (n - 1) * b
    n_exp = Hq * sum(S - nlast + i + 1 for i in range(nlast))
    mufu_ms = n_exp / (16.0 * sm_count * sm_mhz * 1e6) * 1e3
    return idx_bytes / (hbm_gbs * 1e9) * 1e3, n_exp, mufu_ms


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, device=None) -> float:
    """Maximum of a per-rank number over all ranks (identity without a
    process group): every multi-rank time is the slowest rank's."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def make_line(args, w, value, ms_per_step, extra):
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8" if w.int8 else "bf16", "data": "synthetic",
            "config": {"workload": w.name, "S": w.S, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "b": w.b,
                       "gamma": w.gamma, "tau": w.tau, "seed": w.seed, "batch": 1,
                       "l2": "inputs larger than L2 (no flush)", "parallelism": "replicas"}}
    line.update(extra)
    return line


# ----------------------------------------------------------------------------- oracle (CPU)

def oracle_sample(w, P, seed, heads, tiles, threads):
    """A bounded oracle sample of the workload: the full index of `heads`
    query heads (both patterns' kinds) and the attention of `tiles` seeded
    128-row query tiles, spread over `threads` host threads; every item is
    timed by its own thread's CPU clock.  The layer estimate scales the mean
    item times to all Hq heads and Hq*ceil(S/128) tiles (extrapolated).
    Returns a dict with the per-layer CPU seconds, the estimate on `threads`
    cores, and the spread of the item times."""
    import concurrent.futures as cf
    rng = np.random.default_rng(seed)
    nq = (w.S + 127) // 128
    kinds = w.head_kinds()
    vs = [h for h in range(w.Hq) if kinds[h] == "vs"]
    qa = [h for h in range(w.Hq) if kinds[h] != "vs"]
    pick = []
    for i in range(heads):
        pool = (vs if i % 2 == 0 else qa) or list(range(w.Hq))
        pick.append(int(pool[int(rng.integers(0, len(pool)))]))
    tile_list = [(int(rng.integers(0, w.Hq)), int(rng.integers(0, nq))) for _ in range(tiles)]

    def index_item(h):
        t0 = time.thread_time()
        o = P.build_index_head(h, w.gamma, w.tau, want_scores=False)
        return time.thread_time() - t0, o["rows"]

    def tile_item(t, rows_of):
        h, qc = t
        lo, hi = qc * 128, min(qc * 128 + 128, w.S)
        t0 = time.thread_time()
        for r in range(lo // w.b, (hi - 1) // w.b + 1):  # the tile's query blocks
            P.attn_rows(h, max(lo, r * w.b), min(hi, (r + 1) * w.b), rows_of[r])
        return time.thread_time() - t0

    wall0 = time.perf_counter()
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        idx_res = list(ex.map(index_item, pick))
        # attention tiles use the rows of a head whose index was just built (same kind of
        # structure), so no extra index is built inside the timed items
        rows_by_head = {h: rows for h, (_, rows) in zip(pick, idx_res)}
        tile_list = [(pick[i % len(pick)], qc) for i, (_, qc) in enumerate(tile_list)]
        tile_t = list(ex.map(lambda t: tile_item(t, rows_by_head[t[0]]), tile_list))
    wall = time.perf_counter() - wall0
    head_t = [t for t, _ in idx_res]
    layer_cpu_s = float(np.mean(head_t)) * w.Hq + float(np.mean(tile_t)) * w.Hq * nq
    spread = {"index_head_s": [float(min(head_t)), float(np.median(head_t)), float(max(head_t))],
              "tile_s": [float(min(tile_t)), float(np.median(tile_t)), float(max(tile_t))]}
    desc = (f"oracle (fp64, one head or tile per thread) on {threads} host threads: full index of {heads} heads "
            f"(vertical-slash and query-aware kinds, {np.mean(head_t):.2f} s CPU each) and {tiles} seeded 128-row "
            f"attention tiles ({np.mean(tile_t):.3f} s CPU each), each timed by its thread's CPU clock; "
            f"extrapolated to {w.Hq} heads and {w.Hq * nq} tiles; per-layer = CPU seconds / {threads} cores")
    return {"layer_cpu_s": layer_cpu_s, "layer_s": layer_cpu_s / threads, "threads": threads, "wall_s": wall,
            "spread_min_median_max": spread, "desc": desc}


def oracle_problem(w, x):
    from oracle import oracle as orc
    if w.int8:
        return orc.OracleProblem(x["q"], x["k"], x["v"], w.b, q8=x["q8"], k8=x["k8"],
                                 q_scale=x["q_scale"], k_scale=x["k_scale"])
    return orc.OracleProblem(x["q"], x["k"], x["v"], w.b)


def run_reference(args, w):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    x = synth.make_inputs(w)
    P = oracle_problem(w, x)
    dense = synth.dense_equiv_flops(w.S, w.Hq, w.d)
    threads = max(1, min(8, os.cpu_count() or 1))
    for s in range(args.warmup):
        oracle_sample(w, P, 500 + s, heads=1, tiles=2, threads=threads)
    per_layer, cpu_s, wall = [], [], 0.0
    res = None
    for s in range(args.steps):
        res = oracle_sample(w, P, 1000 + s, heads=2, tiles=threads, threads=threads)
        wall += res["wall_s"]
        per_layer.append(res["layer_s"])
        cpu_s.append(res["layer_cpu_s"])
    layer_s = float(np.mean(per_layer))
    value = dense / layer_s / 1e12
    cpu = {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
           "sample": f"{args.steps} steps, each: " + res["desc"],
           "layer_cpu_s_one_thread": float(np.mean(cpu_s)),
           "layer_s_spread_over_steps": [float(min(per_layer)), float(np.median(per_layer)), float(max(per_layer))],
           "host_cpus": os.cpu_count()}
    line = make_line(args, w, value, layer_s * 1e3,
                     {"impl": "reference", "cpu_baseline": cpu,
                      "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
                      "reference_note": f"fp64 oracle on {threads} host threads, {args.steps} bounded samples "
                                        f"({wall:.1f} s), ms_per_step = extrapolated ms per layer"})
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- CUDA path

def time_layer(fp, w, qq, kk, v, qs, ks, dt, args, dev, stream, world):
    """Warm-up, then args.steps timed steps of fp_build_index + fp_sparse_attn
    on `stream` (CUDA events around each stage and around the whole region,
    barrier + synchronize on both sides, clocks sampled meanwhile)."""
    out = torch.empty(w.Hq, w.S, w.d, dtype=torch.bfloat16, device=dev)
    idx = fp.fp_index_create(w.S, w.Hq, w.Hkv, w.d, w.b)

    def step():
        fp.fp_build_index(qq, kk, w.S, w.Hq, w.Hkv, w.d, w.b, w.gamma, w.tau, dt, qs, ks, idx, stream)
        fp.fp_sparse_attn(qq, kk, v, qs, ks, idx, out, stream)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            step()
    stream.synchronize()
    assert fp.fp_get_device_error(stream) == fp.FP_OK
    exp = fp.fp_index_export(idx, stream)
    n = (w.S + w.b - 1) // w.b
    chunks = computed_chunk_tiles(exp["row_ptr"], exp["col"], w.Hq, w.S, w.b)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t_start.record(stream)
        for s in range(args.steps):
            ev[s][0].record(stream)
            fp.fp_build_index(qq, kk, w.S, w.Hq, w.Hkv, w.d, w.b, w.gamma, w.tau, dt, qs, ks, idx, stream)
            ev[s][1].record(stream)
            fp.fp_sparse_attn(qq, kk, v, qs, ks, idx, out, stream)
            ev[s][2].record(stream)
        t_end.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if world > 1:
        torch.distributed.barrier()
    assert fp.fp_get_device_error(stream) == fp.FP_OK
    return {"idx": idx, "out": out, "exp": exp, "clocks": clocks, "chunks": chunks,
            "attn_flops": chunks * 4.0 * 128 * 128 * 128,
            "density": exp["nnz"] / (w.Hq * n * (n + 1) / 2),
            "total_ms": t_start.elapsed_time(t_end),
            "index_ms": float(np.mean([e[0].elapsed_time(e[1]) for e in ev])),
            "attn_ms": float(np.mean([e[1].elapsed_time(e[2]) for e in ev]))}


def run_ours(args, w):
    world, rank, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    from dynamic_block_sparse_last_b200 import fp

    x = synth.make_inputs(w)
    q, k, v = x["q"].to(dev), x["k"].to(dev), x["v"].to(dev)
    if w.int8:
        qq, kk = x["q8"].to(dev), x["k8"].to(dev)
        qs, ks = x["q_scale"].to(dev), x["k_scale"].to(dev)
        dt = fp.FP_QK_INT8
    else:
        qq, kk, qs, ks, dt = q, k, None, None, fp.FP_QK_BF16
    stream = torch.cuda.Stream(device=dev)
    L = time_layer(fp, w, qq, kk, v, qs, ks, dt, args, dev, stream, world)
    idx, out, exp, clocks = L["idx"], L["out"], L["exp"], L["clocks"]
    chunks, attn_flops, density = L["chunks"], L["attn_flops"], L["density"]
    index_ms, attn_ms = L["index_ms"], L["attn_ms"]
    total_ms = max_over_ranks(L["total_ms"], dev)
    ms_per_step = total_ms / args.steps
    dense = synth.dense_equiv_flops(w.S, w.Hq, w.d)
    value = world * dense * args.steps / (total_ms / 1e3) / 1e12

    # end to end through the host-to-host prefill call (fp_prefill_run) with
    # pinned host buffers: every step copies Q, K, V (and int8 scales) in and
    # the output out, overlapped with the compute in KV-head groups
    h_q = x["q8"].pin_memory() if w.int8 else x["q"].pin_memory()
    h_k = x["k8"].pin_memory() if w.int8 else x["k"].pin_memory()
    h_v = x["v"].pin_memory()
    h_qs = x["q_scale"].pin_memory() if w.int8 else None
    h_ks = x["k_scale"].pin_memory() if w.int8 else None
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    pipe = fp.Prefill(w.S, w.Hq, w.Hkv, w.d, w.b, dt, args.e2e_groups)
    e2e_steps = max(2, min(20, args.steps))  # the timed region's step count
    # one run alone (its latency: nothing before or after it to overlap with)
    pipe.run(h_q, h_k, h_v, h_qs, h_ks, w.gamma, w.tau, h_out, stream)
    l0, l1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    l0.record(stream)
    pipe.run(h_q, h_k, h_v, h_qs, h_ks, w.gamma, w.tau, h_out, stream)
    l1.record(stream)
    # e2e_steps runs queued back to back (consecutive runs overlap), one wait
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for it in range(e2e_steps):
        pipe.enqueue(h_q, h_k, h_v, h_qs, h_ks, w.gamma, w.tau, h_out, stream)
    pipe.wait(stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    assert fp.fp_get_device_error(stream) == fp.FP_OK
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, dev)
    latency_ms = max_over_ranks(l0.elapsed_time(l1), dev)
    nbytes = lambda t: 0 if t is None else t.numel() * t.element_size()
    h2d = nbytes(h_q) + nbytes(h_k) + nbytes(h_v) + nbytes(h_qs) + nbytes(h_ks)
    d2h = nbytes(h_out)
    e2e = {"value": world * dense / (e2e_ms / 1e3) / 1e12, "unit": UNIT, "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "api": "fp_prefill_enqueue",
           "steps": e2e_steps, "head_groups": pipe.groups, "single_run_latency_ms": latency_ms}
    pipe.free()

    peaks = load_peaks()
    bf16_peak = peaks["bf16_tflops_sustained"]
    src = ("measured bf16 sustained (MEASURED_PEAKS.json)" if peaks["source"] == "measured"
           else f"{peaks['source']}: 1.4 PFLOP/s sustained")
    i8 = int8_gemm_peak(dev) if (w.int8 or not args.no_w8a8) else None
    i8_sus = i8.get("sustained_tops") if i8 else None
    if w.int8 and i8_sus:
        peak = attention_peak(bf16_peak, i8_sus)
        src += f"; int8 Q.K^T at the measured int8 sustained {i8_sus:.0f} TOPS, bf16 P.V: 2/(1/P_i8 + 1/P_bf16)"
    elif w.int8:
        peak = attention_peak(bf16_peak, 2.0 * bf16_peak)
        src += "; int8 measurement unavailable: int8 at the nominal 2x of bf16"
    else:
        peak = attention_peak(bf16_peak)
    achieved = attn_flops / (attn_ms / 1e3) / 1e12
    trec = attn_traffic_record() if not w.int8 else None  # the record is of the bf16 kernel
    roof = {"kernel": "k_sparse_attn<int8>" if w.int8 else "k_sparse_attn", "bound": "tensor",
            "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": (trec["dram_bytes_per_launch"] if trec else None),
            "peak_source": src,
            "algorithmic_flops_per_launch": attn_flops,
            "note": "algorithmic FLOPs = 4*128^3 per computed 128x128 query-key chunk tile"}
    # index pass against HBM: K once, Q of the query-aware heads once (pooled after the pattern
    # decision), the last query block of every head
    elt = 1 if w.int8 else 2
    qa_heads = int((exp["pattern"] == 1).sum())
    idx_bytes = (w.Hkv * w.S * w.d + qa_heads * w.S * w.d + w.Hq * w.b * w.d) * elt
    idx_gbs = idx_bytes / (index_ms / 1e3) / 1e9
    # the pass's floors: its bytes at the HBM copy bandwidth, and its exponentials at the MUFU
    # rate and the SM clock sampled during the run
    hbm_floor_ms, n_exp, mufu_floor_ms = index_pass_floors(
        w.S, w.Hq, w.b, idx_bytes, peaks["hbm_gbs"], torch.cuda.get_device_properties(dev).multi_processor_count,
        clocks.get("sm_mhz") or 1965.0)
    extra = {"roofline": roof,
             "index_pass": {"ms": index_ms, "algorithmic_bytes": idx_bytes, "achieved_gbs": idx_gbs,
                            "frac_of_hbm": idx_gbs / peaks["hbm_gbs"], "qa_heads": qa_heads,
                            "bytes_note": "K + Q of the query-aware heads + the last query block, each read once",
                            "hbm_floor_ms": hbm_floor_ms,
                            "exponentials": n_exp, "mufu_floor_ms": mufu_floor_ms},
             "attn_ms": attn_ms, "density": density, "chunks": chunks,
             "e2e": e2e, "clocks": clocks, "gpu_launches": kernels_per_step(w.S, w.b) * args.steps,
             "gpu": torch.cuda.get_device_name(dev)}
    extra["int8_peak"] = i8
    # compact forms of the same index on the device (not part of the step): CSR rows and the
    # per-(KV head, query block) union lists with head masks
    rp = torch.empty(w.Hq * ((w.S + w.b - 1) // w.b) + 1, dtype=torch.int32, device=dev)
    col = torch.empty(max(1, int(exp["nnz"])), dtype=torch.int32, device=dev)
    gp = torch.empty(w.Hkv * ((w.S + w.b - 1) // w.b) + 1, dtype=torch.int32, device=dev)
    fp.fp_index_group_lists(idx, gp, None, None, stream)
    torch.cuda.synchronize(dev)
    gtot = int(gp[-1])
    gc = torch.empty(max(1, gtot), dtype=torch.int32, device=dev)
    gm = torch.empty(max(1, gtot), dtype=torch.int32, device=dev)
    ct = []
    for _ in range(5):
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record(stream)
        fp.fp_index_csr(idx, rp, col, stream)
        e1.record(stream)
        fp.fp_index_group_lists(idx, gp, gc, gm, stream)
        e2.record(stream)
        torch.cuda.synchronize(dev)
        ct.append((e0.elapsed_time(e1), e1.elapsed_time(e2)))
    extra["compact_lists"] = {"csr_ms": float(np.median([a for a, _ in ct])),
                              "group_lists_ms": float(np.median([b for _, b in ct])),
                              "nnz": int(exp["nnz"]), "group_entries": gtot,
                              "note": "device CSR and per-group union lists of the timed index; the attention "
                                      "reads the padded rows, so neither is part of the step"}
    del rp, col, gp, gc, gm
    if not w.int8 and not args.no_w8a8 and w.b == 128 and w.S % 256 == 0:
        # the same layer at b = 256 (two 128-row halves per block share one list)
        wb = synth.Workload(w.name + "_b256", S=w.S, Hq=w.Hq, Hkv=w.Hkv, d=w.d, b=256, gamma=w.gamma, tau=w.tau,
                            n_vertical=w.n_vertical, n_topics=w.n_topics, seed=w.seed)
        Lb = time_layer(fp, wb, qq, kk, v, qs, ks, dt, args, dev, stream, world)
        msb = max_over_ranks(Lb["total_ms"], dev) / args.steps
        achb = Lb["attn_flops"] / (Lb["attn_ms"] / 1e3) / 1e12
        extra["b256"] = {"workload": wb.name, "ms_per_layer": msb, "index_ms": Lb["index_ms"],
                         "attn_ms": Lb["attn_ms"], "value": world * dense / (msb / 1e3) / 1e12, "unit": UNIT,
                         "density": Lb["density"], "chunks": Lb["chunks"],
                         "roofline": {"kernel": "k_sparse_attn", "bound": "tensor", "achieved": achb,
                                      "peak": peak, "unit": "TFLOP/s", "frac": achb / peak, "peak_source": src},
                         "clocks": Lb["clocks"], "gpu_launches": kernels_per_step(wb.S, wb.b) * args.steps}
        Lb["idx"].free()
    if not w.int8 and not args.no_w8a8:
        # the W8A8 variant of the same layer: Q and K quantised per head from these bf16 tensors
        del q, k, qq, kk
        wq = synth.Workload(w.name + "_w8a8", S=w.S, Hq=w.Hq, Hkv=w.Hkv, d=w.d, b=w.b, gamma=w.gamma, tau=w.tau,
                            n_vertical=w.n_vertical, n_topics=w.n_topics, seed=w.seed, int8=True)
        q8, q_sc = synth.quantize_per_head(x["q"])
        k8, k_sc = synth.quantize_per_head(x["k"])
        q8, k8, q_sc, k_sc = q8.to(dev), k8.to(dev), q_sc.to(dev), k_sc.to(dev)
        idx.free()
        L8 = time_layer(fp, wq, q8, k8, v, q_sc, k_sc, fp.FP_QK_INT8, args, dev, stream, world)
        ms8 = max_over_ranks(L8["total_ms"], dev) / args.steps
        pk8 = attention_peak(bf16_peak, i8_sus if i8_sus else 2.0 * bf16_peak)
        ach8 = L8["attn_flops"] / (L8["attn_ms"] / 1e3) / 1e12
        extra["w8a8"] = {"workload": wq.name, "ms_per_layer": ms8, "index_ms": L8["index_ms"],
                         "attn_ms": L8["attn_ms"], "value": world * dense / (ms8 / 1e3) / 1e12, "unit": UNIT,
                         "density": L8["density"], "chunks": L8["chunks"],
                         "roofline": {"kernel": "k_sparse_attn<int8>", "bound": "tensor", "achieved": ach8,
                                      "peak": pk8, "unit": "TFLOP/s", "frac": ach8 / pk8,
                                      "peak_source": ("int8 Q.K^T at the measured int8 sustained TOPS and bf16 P.V "
                                                      "at the bf16 sustained peak: 2/(1/P_i8 + 1/P_bf16)"
                                                      if i8_sus else "int8 at the nominal 2x of bf16")},
                         "clocks": L8["clocks"]}
        extra["w8a8"]["gpu_launches"] = kernels_per_step(wq.S, wq.b) * args.steps
        L8["idx"].free()
        del q8, k8
        idx = None
    if world == 1 and not args.no_cpu_baseline and rank == 0:
        P = oracle_problem(w, x)
        threads = max(1, min(16, os.cpu_count() or 1))
        res = oracle_sample(w, P, 7, heads=4, tiles=64, threads=threads)
        dense = synth.dense_equiv_flops(w.S, w.Hq, w.d)
        extra["cpu_baseline"] = {"value": dense / res["layer_s"] / 1e12, "unit": UNIT, "cores": threads,
                                 "kind": "oracle", "sample": res["desc"],
                                 "value_one_thread": dense / res["layer_cpu_s"] / 1e12,
                                 "spread_min_median_max": res["spread_min_median_max"],
                                 "sample_wall_s": res["wall_s"], "host_cpus": os.cpu_count()}
    if rank == 0:
        print(json.dumps(make_line(args, w, value, ms_per_step, extra)), flush=True)
    if idx is not None:
        idx.free()
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


SHARE_EPS = 0.05  # head-pattern sharing threshold reported in the sweep (half of tau)


def run_sweep(args):
    """The S x b x gamma sweep on the 128K generator (Hq=32, Hkv=8): one JSON
    line per point with density next to time (not the headline line).  At
    b = 128 each line also carries the block size the content rule chooses
    from that index (fp_choose_block_size) and the layer with head-pattern
    sharing (fp_index_share, eps = SHARE_EPS): its density, sharing time and
    attention time."""
    from dynamic_block_sparse_last_b200 import fp
    dev = torch.device("cuda", 0)
    cache = {}
    for w in synth.sweep_workloads():
        if w.S not in cache:
            cache.clear()
            x = synth.make_inputs(w)
            cache[w.S] = (x["q"].to(dev), x["k"].to(dev), x["v"].to(dev))
        q, k, v = cache[w.S]
        out = torch.empty_like(q)
        idx = fp.fp_index_create(w.S, w.Hq, w.Hkv, w.d, w.b)

        def build():
            fp.fp_build_index(q, k, w.S, w.Hq, w.Hkv, w.d, w.b, w.gamma, w.tau, fp.FP_QK_BF16, None, None, idx)

        for _ in range(args.warmup):
            build()
            fp.fp_sparse_attn(q, k, v, None, None, idx, out)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
        for e in ev:
            e[0].record()
            build()
            e[1].record()
            fp.fp_sparse_attn(q, k, v, None, None, idx, out)
            e[2].record()
        torch.cuda.synchronize()
        assert fp.fp_get_device_error() == fp.FP_OK
        n = (w.S + w.b - 1) // w.b
        nnz = fp.fp_index_nnz(idx)
        idx_ms = float(np.median([e[0].elapsed_time(e[1]) for e in ev]))
        attn_ms = float(np.median([e[1].elapsed_time(e[2]) for e in ev]))
        layer = idx_ms + attn_ms
        line = {"sweep": w.name, "S": w.S, "b": w.b, "gamma": w.gamma,
                "density": nnz / (w.Hq * n * (n + 1) / 2), "index_ms": idx_ms, "attn_ms": attn_ms,
                "ms_per_layer": layer,
                "dense_equiv_tflops": synth.dense_equiv_flops(w.S, w.Hq, w.d) / (layer / 1e3) / 1e12}
        if w.b == 128:
            bsel, rho = fp.fp_choose_block_size(idx, w.gamma)
            line["adaptive_block"] = {"b": bsel, "rho": rho}
            # head-pattern sharing on the same index: lists replaced by class unions
            sh = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
            for e in sh:
                build()
                e[0].record()
                fp.fp_index_share(idx, SHARE_EPS)
                e[1].record()
                fp.fp_sparse_attn(q, k, v, None, None, idx, out)
                e[2].record()
            torch.cuda.synchronize()
            assert fp.fp_get_device_error() == fp.FP_OK
            cls = fp.fp_index_classes(idx)
            line["shared"] = {"eps": SHARE_EPS, "classes": int(len(set(cls.tolist()))),
                              "density": fp.fp_index_nnz(idx) / (w.Hq * n * (n + 1) / 2),
                              "share_ms": float(np.median([e[0].elapsed_time(e[1]) for e in sh])),
                              "attn_ms": float(np.median([e[1].elapsed_time(e[2]) for e in sh]))}
        print(json.dumps(line), flush=True)
        idx.free()
    return 0


def run_rope_pool(args):
    """The rotary-embedding epilogue with block pooling (fp_rope_pool) at the
    workload's shape against HBM, and the index build on its means
    (fp_build_index_pooled) beside the one that pools Q and K itself.  One JSON
    line; not the headline."""
    from dynamic_block_sparse_last_b200 import fp
    dev = torch.device("cuda", 0)
    w = synth.WORKLOADS[args.workload]
    x = synth.make_prerope_inputs(w)
    q_in, k_in = x["q_in"].to(dev), x["k_in"].to(dev)
    cos, sin = x["cos"].to(dev), x["sin"].to(dev)
    n = (w.S + w.b - 1) // w.b
    q, k = torch.empty_like(q_in), torch.empty_like(k_in)
    qbar = torch.empty(w.Hq, n, w.d, device=dev)
    kbar = torch.empty(w.Hkv, n, w.d, device=dev)
    idx = fp.fp_index_create(w.S, w.Hq, w.Hkv, w.d, w.b)

    def rope():
        fp.fp_rope_pool(q_in, k_in, cos, sin, w.S, w.Hq, w.Hkv, w.d, w.b, q, k, qbar, kbar)

    def build():
        fp.fp_build_index(q, k, w.S, w.Hq, w.Hkv, w.d, w.b, w.gamma, w.tau, fp.FP_QK_BF16, None, None, idx)

    def build_pooled():
        fp.fp_build_index_pooled(q, k, qbar, kbar, w.S, w.Hq, w.Hkv, w.d, w.b, w.gamma, w.tau, idx)

    res = {}
    for name, fn in (("rope_pool", rope), ("index", build), ("index_pooled", build_pooled)):
        for _ in range(max(3, args.warmup)):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for e0, e1 in ev:
            e0.record()
            fn()
            e1.record()
        torch.cuda.synchronize()
        res[name] = float(np.median([e0.elapsed_time(e1) for e0, e1 in ev]))
    assert fp.fp_get_device_error() == fp.FP_OK
    peaks = load_peaks()
    # algorithmic bytes: every Q and K element read and written once (bf16),
    # the cos/sin tables read once, the means written
    nbytes = (w.Hq + w.Hkv) * w.S * w.d * 4 + w.S * (w.d // 2) * 4 * 2 + (w.Hq + w.Hkv) * n * w.d * 4
    gbs = nbytes / (res["rope_pool"] / 1e3) / 1e9
    print(json.dumps({"metric": "rotary epilogue with block pooling (GB/s) and index build on its means (ms)",
                      "config": {"workload": w.name, "S": w.S, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "b": w.b},
                      "steps": args.steps, "rope_pool_ms": res["rope_pool"], "rope_pool_bytes": nbytes,
                      "rope_pool_gbs": gbs, "rope_pool_frac_of_hbm": gbs / peaks["hbm_gbs"],
                      "hbm_peak_gbs": peaks["hbm_gbs"], "index_ms": res["index"],
                      "index_pooled_ms": res["index_pooled"], "gpu": torch.cuda.get_device_name(dev)}), flush=True)
    idx.free()
    return 0


def run_profile_case(args):
    """One layer of a given shape, for profiler captures of a small case:
    --profile-case S:Hq:Hkv:b[:int8] on the 128K layer's generator (64
    vertical positions, 32 topics, seed 2, gamma 0.9, tau 0.1); warm-up, then
    --steps builds + attentions on one stream.  Prints one JSON line with the
    mean times per stage (not a bench line)."""
    from dynamic_block_sparse_last_b200 import fp
    parts = args.profile_case.split(":")
    S, Hq, Hkv, b = (int(v) for v in parts[:4])
    int8 = len(parts) > 4 and parts[4] == "int8"
    w = synth.Workload(f"profile_S{S}_Hq{Hq}_Hkv{Hkv}_b{b}" + ("_int8" if int8 else ""), S=S, Hq=Hq, Hkv=Hkv, b=b,
                       n_vertical=64, n_topics=32, seed=2, int8=int8)
    dev = torch.device("cuda", 0)
    x = synth.make_inputs(w)
    v = x["v"].to(dev)
    if int8:
        qq, kk = x["q8"].to(dev), x["k8"].to(dev)
        qs, ks, dt = x["q_scale"].to(dev), x["k_scale"].to(dev), fp.FP_QK_INT8
    else:
        qq, kk, qs, ks, dt = x["q"].to(dev), x["k"].to(dev), None, None, fp.FP_QK_BF16
    stream = torch.cuda.Stream(device=dev)
    L = time_layer(fp, w, qq, kk, v, qs, ks, dt, args, dev, stream, 1)
    print(json.dumps({"profile_case": w.name, "index_ms": L["index_ms"], "attn_ms": L["attn_ms"],
                      "density": L["density"], "chunks": L["chunks"], "steps": args.steps,
                      "warmup": args.warmup}), flush=True)
    L["idx"].free()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama8b", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-w8a8", action="store_true", help="skip the W8A8 sub-record of the default line")
    ap.add_argument("--e2e-groups", type=int, default=0,
                    help="KV-head groups of the host-to-host pipeline (0 = one KV head per group)")
    ap.add_argument("--sweep", action="store_true", help="S x b x gamma sweep (one line per point)")
    ap.add_argument("--rope-pool", action="store_true",
                    help="time the rotary epilogue with block pooling and the index build on its means")
    ap.add_argument("--profile-case", default="",
                    help="S:Hq:Hkv:b[:int8] -- one small layer for profiler captures (not a bench line)")
    args = ap.parse_args()
    if args.profile_case:
        return run_profile_case(args)
    if args.warmup < 3:
        args.warmup = 3
    if args.sweep:
        return run_sweep(args)
    if args.rope_pool:
        return run_rope_pool(args)
    w = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
