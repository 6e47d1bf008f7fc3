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
# k_score_last, k_row_stats, k_block_mass, k_kbar, k_pattern, k_qbar, k_qa_logits, k_cut, k_sparse_attn
KERNELS_PER_STEP = 9
ATTN_SRC = os.path.join(ROOT, "dynamic_block_sparse_last_b200", "csrc", "attn_kernel.cuh")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


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


def attention_peak(bf16_peak: float, int8: bool) -> float:
    """Tensor peak for the attention's contractions: bf16 for both, or for W8A8
    Q.K^T (half the FLOPs) as int8 at the nominal 2x of bf16 and P.V as bf16,
    whose roofline time F/2/(2P) + F/2/P makes an effective peak of 4/3 P."""
    return bf16_peak * 4.0 / 3.0 if int8 else bf16_peak


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

def oracle_sample(w, x, P, step, tiles_per_step=1):
    """One bounded oracle sample: the full index of one head plus attention of
    `tiles_per_step` 128-row tiles of that head; returns (seconds, extrapolated
    seconds per layer, description)."""
    h = step % w.Hq
    nq = (w.S + 127) // 128
    t0 = time.perf_counter()
    o = P.build_index_head(h, w.gamma, w.tau, want_scores=False)
    t1 = time.perf_counter()
    rng = np.random.default_rng(1000 + step)
    tile_t = []
    for _ in range(tiles_per_step):
        qc = int(rng.integers(0, nq))
        lo, hi = qc * 128, min(qc * 128 + 128, w.S)
        s = time.perf_counter()
        for r in range(lo // w.b, (hi - 1) // w.b + 1):  # the tile's query blocks
            P.attn_rows(h, max(lo, r * w.b), min(hi, (r + 1) * w.b), o["rows"][r])
        tile_t.append(time.perf_counter() - s)
    t2 = time.perf_counter()
    per_layer = (t1 - t0) * w.Hq + float(np.mean(tile_t)) * w.Hq * nq
    desc = (f"oracle index of head {h} ({t1 - t0:.2f} s) x {w.Hq} heads + {tiles_per_step} attention "
            f"tile(s) of 128 rows ({np.mean(tile_t):.2f} s mean) x {w.Hq * nq} tiles; 1 thread; extrapolated")
    return t2 - t0, per_layer, desc


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
    for s in range(args.warmup):
        oracle_sample(w, x, P, s)
    per_layer, wall, desc = [], 0.0, ""
    for s in range(args.steps):
        t, pl, desc = oracle_sample(w, x, P, args.warmup + s)
        wall += t
        per_layer.append(pl)
    layer_s = float(np.mean(per_layer))
    value = dense / layer_s / 1e12
    cpu = {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc}
    line = make_line(args, w, value, layer_s * 1e3,
                     {"impl": "reference", "cpu_baseline": cpu,
                      "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
                      "reference_note": f"fp64 oracle on host cores, {args.steps} bounded samples "
                                        f"({wall:.1f} s), ms_per_step = extrapolated ms per layer"})
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- CUDA path

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
    out = torch.empty_like(q)
    idx = fp.fp_index_create(w.S, w.Hq, w.Hkv, w.d, w.b)
    stream = torch.cuda.Stream(device=dev)

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
    attn_flops = chunks * 4.0 * 128 * 128 * 128
    density = exp["nnz"] / (w.Hq * n * (n + 1) / 2)

    # timed region: K steps, events around each stage on the launching stream
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
    total_ms = t_start.elapsed_time(t_end)
    index_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in ev]))
    attn_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in ev]))
    assert fp.fp_get_device_error(stream) == fp.FP_OK
    total_ms = max_over_ranks(total_ms, dev)
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
    src = (f"{peaks['source']} bf16 sustained (MEASURED_PEAKS.json)" if peaks["source"] == "measured"
           else "fallback 1.4 PFLOP/s sustained")
    peak = attention_peak(bf16_peak, w.int8)
    if w.int8:
        src += "; int8 Q.K^T at the nominal 2x (4.5 vs 2.25 PFLOP/s dense), bf16 P.V: 4/3 of it"
    achieved = attn_flops / (attn_ms / 1e3) / 1e12
    trec = attn_traffic_record() if not w.int8 else None  # the record is of the bf16 kernel
    roof = {"kernel": "k_sparse_attn<int8>" if w.int8 else "k_sparse_attn", "bound": "tensor",
            "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": (trec["dram_bytes_per_launch"] if trec else None),
            "peak_source": src,
            "algorithmic_flops_per_launch": attn_flops,
            "note": "algorithmic FLOPs = 4*128^3 per computed 128x128 query-key chunk tile"}
    # index pass against HBM: K once, Q of query-aware heads, the last query block
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
                            "hbm_floor_ms": hbm_floor_ms,
                            "exponentials": n_exp, "mufu_floor_ms": mufu_floor_ms},
             "attn_ms": attn_ms, "density": density, "chunks": chunks,
             "e2e": e2e, "clocks": clocks, "gpu_launches": KERNELS_PER_STEP * args.steps,
             "gpu": torch.cuda.get_device_name(dev)}
    if world == 1 and not args.no_cpu_baseline and rank == 0:
        P = oracle_problem(w, x)
        t, per_layer, desc = oracle_sample(w, x, P, 0)
        extra["cpu_baseline"] = {"value": synth.dense_equiv_flops(w.S, w.Hq, w.d) / per_layer / 1e12,
                                 "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc,
                                 "host_cpus": os.cpu_count()}
    if rank == 0:
        print(json.dumps(make_line(args, w, value, ms_per_step, extra)), flush=True)
    idx.free()
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def run_sweep(args):
    """The S x b x gamma sweep on the 128K generator (Hq=32, Hkv=8): one JSON
    line per point with density next to time (not the headline line)."""
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
        for _ in range(args.warmup):
            fp.fp_build_index(q, k, w.S, w.Hq, w.Hkv, w.d, w.b, w.gamma, w.tau, fp.FP_QK_BF16, None, None, idx)
            fp.fp_sparse_attn(q, k, v, None, None, idx, out)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
        for e in ev:
            e[0].record()
            fp.fp_build_index(q, k, w.S, w.Hq, w.Hkv, w.d, w.b, w.gamma, w.tau, fp.FP_QK_BF16, None, None, idx)
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
        print(json.dumps({"sweep": w.name, "S": w.S, "b": w.b, "gamma": w.gamma,
                          "density": nnz / (w.Hq * n * (n + 1) / 2), "index_ms": idx_ms, "attn_ms": attn_ms,
                          "ms_per_layer": layer,
                          "dense_equiv_tflops": synth.dense_equiv_flops(w.S, w.Hq, w.d) / (layer / 1e3) / 1e12}),
              flush=True)
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


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama8b", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-groups", type=int, default=0,
                    help="KV-head groups of the host-to-host pipeline (0 = one KV head per group)")
    ap.add_argument("--sweep", action="store_true", help="S x b x gamma sweep (one line per point)")
    ap.add_argument("--rope-pool", action="store_true",
                    help="time the rotary epilogue with block pooling and the index build on its means")
    args = ap.parse_args()
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
