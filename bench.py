"""Benchmark: quantized attention forward (INT8 QK^T, FP8 PV) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--n N] [--causal]

Workload (default): the kernel-sweep configuration at its longest length,
B=1, H=32, N=32768, d=128, fp16, HND, non-causal, seeded synthetic inputs
(Q, V ~ N(0,1); K ~ N(0,1) plus a per-channel offset ~ N(0, 3^2)).

A step is one pass of the whole path on device-resident inputs: sage_quant_qkv
(K mean, Q/K INT8, V e4m3 in one cooperative launch) and sage_attn_fwd.  TOPS =
4*B*H*N^2*d / time (halved when causal).  Inputs (3 x 256 MiB) exceed the
126 MB L2, so no flush is needed between steps.  Rank 0 prints one JSON line.

Multi-GPU (torchrun): every rank runs its own copy of the workload (independent
problems, no data-path collective; weak scaling); the time is the max over ranks.
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
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "attention TOPS at hd128, seq 1K–32K (1×B200); % of INT8/FP8 tensor peak"
UNIT = "TOPS"
NOMINAL_INT8_OVER_BF16 = 2.0  # 4.5 POPS dense INT8/FP8 vs 2.25 PFLOP/s dense bf16 (datasheet ratio)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="sage", choices=["sage", "reference"])
    ap.add_argument("--n", type=int, default=32768)
    ap.add_argument("--causal", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=1536,
                    help="query rows of the oracle sample (cpu_baseline and every reference step)")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the per-length / per-workload attention measurements")
    ap.add_argument("--granularity", default="block", choices=["block", "thread"],
                    help="INT8 scale granularity of Q/K: per block (the method as stated) or "
                         "per thread (a scale per Q token and per 32-token K block)")
    return ap.parse_args()


def workload(args):
    from quantized_attention_06_b200.inputs import sweep_workload
    return sweep_workload(args.n)


def config(w, args, n_gpus):
    return {"workload": f"sweep B={w.batch} H={w.heads_q} N={w.seqlen} d={w.head_dim} "
                        f"{w.dtype} {w.layout} {'causal' if args.causal else 'non-causal'}",
            "batch": w.batch, "heads": w.heads_q, "seq_len": w.seqlen, "head_dim": w.head_dim,
            "causal": bool(args.causal), "layout": w.layout, "n_gpus": n_gpus,
            "l2": "inputs (3 x 256 MiB) larger than the 126 MB L2; no flush",
            "step": "sage_quant_qkv + sage_attn_fwd",
            "granularity": getattr(args, "granularity", "block")}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p["bf16_tflops"], p.get("bf16_tflops_sustained"), p.get("hbm_gbs"), "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


# ---------------------------------------------------------------- CPU oracle baseline
# The oracle is plain NumPy.  It is timed on all of the host's cores: a process pool
# (started with spawn, one single-threaded worker per core) splits the sampled query
# rows; every worker repeats the head's quantization (part of the sample) and then
# computes its rows exactly as oracle.attention_head defines them.

_POOL_HEAD = {}


def _pool_init(q, k, v):
    _POOL_HEAD.update(q=q, k=k, v=v)


def _pool_rows(task):
    import oracle as orc
    rows, causal, qblk, kblk = task
    h = _POOL_HEAD
    orc.attention_head(h["q"], h["k"], h["v"], causal=causal, rows=rows, qblk=qblk, kblk=kblk)
    return len(rows)


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def orc_blocks(args):
    thread = getattr(args, "granularity", "block") == "thread"
    return (1, 32) if thread else (128, 64)


class OraclePool:
    """A spawn-started pool of single-threaded oracle workers over one head."""

    def __init__(self, w, args):
        import multiprocessing as mp
        from dataclasses import replace
        from quantized_attention_06_b200.inputs import generate
        # one head drawn with the workload's recipe and seed (timing sample only)
        x = generate(replace(w, batch=1, heads_q=1, heads_kv=1))
        self.q, self.k, self.v = x["q"][0, 0], x["k"][0, 0], x["v"][0, 0]
        self.w, self.args = w, args
        self.cores = os.cpu_count() or 1
        for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
            os.environ[var] = "1"          # read by the spawned workers' NumPy
        ctx = mp.get_context("spawn")
        self.pool = ctx.Pool(self.cores, initializer=_pool_init, initargs=(self.q, self.k, self.v))
        qb, kb = orc_blocks(args)
        # warm the workers (imports, first quantization) before any timing
        self.pool.map(_pool_rows, [(np.arange(1), False, qb, kb)] * self.cores)

    def sample(self, rows):
        """Time `rows` evenly spaced query rows (plus the head's quantization in every
        worker).  Returns (TOPS, seconds, description)."""
        w, args = self.w, self.args
        sel = np.linspace(0, w.seqlen - 1, rows).astype(np.int64)
        qb, kb = orc_blocks(args)
        chunks = [c for c in np.array_split(sel, self.cores) if len(c)]
        t0 = time.perf_counter()
        self.pool.map(_pool_rows, [(c, bool(args.causal), qb, kb) for c in chunks])
        dt = time.perf_counter() - t0
        n_keys = (sel + 1).sum() if args.causal else rows * w.seqlen
        ops = 4.0 * n_keys * w.head_dim
        desc = (f"one head: quantization (Q, K, V; repeated by each of {len(chunks)} workers) "
                f"plus {rows} evenly spaced query rows against "
                f"{'their causal prefix' if args.causal else f'all {w.seqlen} keys'}, "
                f"oracle.attention_head (fp64)")
        return ops / dt / 1e12, dt, desc

    def close(self):
        self.pool.close()
        self.pool.join()


def max_over_ranks(values, device):
    """Element-wise max of each rank's `values` over all ranks (the slowest rank sets
    the job's time); every rank calls it at the same point.  Without a process group
    (one rank) the values come back unchanged."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(x) for x in values]
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_rate(ops_per_rank, world, ms):
    """Whole-job TOPS: every rank runs the same workload (weak scaling), so the job
    does ops_per_rank * world in the slowest rank's `ms` milliseconds."""
    return ops_per_rank * world / (ms * 1e-3) / 1e12


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    w = workload(args)
    pool = OraclePool(w, args)
    times = []
    for i in range(args.warmup + args.steps):
        tops, dt, sample = pool.sample(args.cpu_rows)
        if i >= args.warmup:
            times.append(tops)
    pool.close()
    val = statistics.median(times)
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config(w, args, world),
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": pool.cores, "kind": "oracle",
                             "sample": sample, "nproc": os.cpu_count(), "cpu_model": cpu_model()},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


class Clocks:
    """nvidia-smi sampler running while the timed region runs."""

    def __init__(self, dev_index):
        self.dev = dev_index
        self.proc = None
        # the per-sample log; SAGE_CLOCKS_DIR keeps it somewhere chosen, else a temp dir
        import tempfile
        base = os.environ.get("SAGE_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(base, f"clocks_bench_{os.getpid()}.csv")

    def __enter__(self):
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.dev}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            self.proc.wait()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, mx, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                    power.append(float(parts[3]))
                except ValueError:
                    continue
                for nm, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(nm)
        load = [s for s in sm if mx and s > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# ---------------------------------------------------------------- the metric's range
# The metric spans seq 1K-32K at hd128 and the workloads of the other four configs.
# Each point is timed on its own: inputs drawn on the device (same distributions as
# inputs.py, seeded), quantized once, then the attention kernel alone (the kernel
# figure, `attn`) and the whole step of three calls (`step`) are timed with CUDA
# events around each launch.  Where the operands fit in L2, a 512 MiB buffer is
# written between timed launches, so no launch starts with a warm L2.

def _device_inputs(w, dev, seqlens=None):
    import torch
    g = torch.Generator(device=dev).manual_seed(1000 + w.seed)
    if w.varlen:
        total = int(sum(seqlens))
        qs, ks = (total, w.heads_q, w.head_dim), (total, w.heads_kv, w.head_dim)
    elif w.layout == "NHD":
        qs, ks = ((w.batch, w.seqlen, w.heads_q, w.head_dim), (w.batch, w.seqlen, w.heads_kv, w.head_dim))
    else:
        qs, ks = ((w.batch, w.heads_q, w.seqlen, w.head_dim), (w.batch, w.heads_kv, w.seqlen, w.head_dim))
    dt = torch.float16 if w.dtype == "fp16" else torch.bfloat16
    q = torch.randn(qs, generator=g, device=dev)
    k = torch.randn(ks, generator=g, device=dev)
    v = torch.randn(ks, generator=g, device=dev)
    if w.tail_frac > 0:
        q = torch.where(torch.rand(qs, generator=g, device=dev) < w.tail_frac, q * w.tail_scale, q)
        k = torch.where(torch.rand(ks, generator=g, device=dev) < w.tail_frac, k * w.tail_scale, k)
    off_shape = [1] * k.dim()
    off_shape[-1] = w.head_dim
    off_shape[-2 if (w.layout == "NHD" or w.varlen) else 1] = w.heads_kv
    k = k + torch.randn(off_shape, generator=g, device=dev) * w.k_offset_sigma
    return q.to(dt), k.to(dt), v.to(dt)


def measure_point(w, causal, dev, peak, pv="fp8", granularity="block", reps=10, seqlens=None):
    import torch
    from quantized_attention_06_b200 import api
    q, k, v = _device_inputs(w, dev, seqlens)
    cu = None
    if w.varlen:
        cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    layout = "NHD" if (w.layout == "NHD" or w.varlen) else "HND"
    z = api.quant_qkv(q, k, v, layout, cu, granularity=granularity, pv=pv)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()
    operand_bytes = sum(t.numel() * t.element_size() for t in (z.q8, z.k8, z.v8))
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev) if operand_bytes < (256 << 20) else None

    def time_it(fn):
        ts = []
        for i in range(3 + reps):
            if flush is not None:
                flush.fill_(i & 0xFF)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            if i >= 3:
                ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    attn_ms = time_it(lambda: api.attn_fwd(z, is_causal=causal, out=out))
    ws = torch.empty(z.problem.sizes.workspace_qkv + 256, dtype=torch.uint8, device=dev)
    step_ms = time_it(lambda: (api.quant_qkv(q, k, v, layout, cu, problem=z.problem, out=z, workspace=ws),
                               api.attn_fwd(z, is_causal=causal, out=out)))
    assert api.poll_device_status() == 0
    ops = w.ops(causal, seqlens)
    tops = ops / (attn_ms * 1e-3) / 1e12
    return {"workload": w.name, "seq_len": w.seqlen, "causal": causal, "pv": pv,
            "granularity": granularity, "attn_ms": attn_ms, "tops": tops, "frac": tops / peak,
            "step_ms": step_ms, "step_tops": ops / (step_ms * 1e-3) / 1e12,
            "l2": "flushed between launches" if flush is not None else "operands larger than L2"}


def measure_metric_range(args, dev, peak):
    from dataclasses import replace
    import torch
    from quantized_attention_06_b200.inputs import SWEEP_LENGTHS, WORKLOADS, sweep_workload
    res = []
    for n in SWEEP_LENGTHS:
        for causal in (False, True):
            res.append(measure_point(sweep_workload(n), causal, dev, peak))
            torch.cuda.empty_cache()
    res.append(measure_point(sweep_workload(32768), False, dev, peak, pv="fp16"))
    res.append(measure_point(sweep_workload(32768), False, dev, peak, granularity="thread"))
    for causal in (False, True):
        res.append(measure_point(WORKLOADS["prefill"], causal, dev, peak))
    res.append(measure_point(WORKLOADS["dit"], False, dev, peak))
    w = WORKLOADS["gqa_varlen"]
    lens = np.random.default_rng(w.seed).integers(w.varlen_range[0], w.varlen_range[1] + 1,
                                                  size=w.varlen_count)
    res.append(measure_point(replace(w, seqlen=int(lens.max())), True, dev, peak,
                             seqlens=[int(x) for x in lens]))
    torch.cuda.empty_cache()
    return res


def run_sage(args):
    import torch
    import torch.distributed as dist

    from quantized_attention_06_b200 import api
    from quantized_attention_06_b200.inputs import generate

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=120))

    w = workload(args)
    # the oracle's worker pool is spawned before any CUDA work (rank 0, one GPU only)
    pool = OraclePool(w, args) if (rank == 0 and world == 1) else None
    x = generate(w)
    host = {n: torch.from_numpy(x[n]).to(torch.float16).pin_memory() for n in ("q", "k", "v")}
    del x
    q, k, v = (host[n].to(dev) for n in ("q", "k", "v"))
    p = api.Problem.from_tensors(q, k, "HND", granularity=args.granularity)
    z = api.Quantized(p, "HND")
    ws_qk = torch.empty(max(1, p.sizes.workspace_qk // 8), dtype=torch.float64, device=dev)
    ws_v = torch.empty(max(1, p.sizes.workspace_v // 4), dtype=torch.float32, device=dev)
    ws_qkv = torch.empty(p.sizes.workspace_qkv + 256, dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()
    launches_per_step = 2  # quant_fused (Q, K, V in one cooperative launch), attention

    def step(ev=None):
        api.quant_qkv(q, k, v, "HND", problem=p, out=z, workspace=ws_qkv)
        if ev is not None:
            ev[0].record(stream)
        api.attn_fwd(z, is_causal=args.causal, out=out)
        if ev is not None:
            ev[1].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    barrier()
    assert api.poll_device_status() == 0

    # ---- whole-step timing (device events, max over ranks)
    attn_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(local) as clk:
        barrier()
        t_start.record(stream)
        for i in range(args.steps):
            step(attn_ev[i])
        t_end.record(stream)
        barrier()
    total_ms = t_start.elapsed_time(t_end)
    attn_ms = [a.elapsed_time(b) for a, b in attn_ev]
    total_ms, attn_mean = max_over_ranks([total_ms, statistics.mean(attn_ms)], dev)
    assert api.poll_device_status() == 0

    ops = w.ops(args.causal)
    ms_per_step = total_ms / args.steps
    value = job_rate(ops, world, ms_per_step)

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        host_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        e_steps = max(2, args.steps // 2)

        def e2e_step():
            # the public host-buffer call: chunks of heads are copied in, quantized,
            # attended and copied out, with the copies overlapping the kernels
            api.sageattn_host(host["q"], host["k"], host["v"], tensor_layout="HND",
                              is_causal=args.causal, out=host_out, synchronize=False,
                              granularity=args.granularity)

        e2e_step()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e_steps):
            e2e_step()
        e1.record(stream)
        barrier()
        e_ms, = max_over_ranks([e0.elapsed_time(e1) / e_steps], dev)
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        e2e = {"value": job_rate(ops, world, e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": out.numel() * out.element_size(),
               "ms_per_step": e_ms}

    # ---- quantization kernels alone: algorithmic HBM bytes / time
    def timed(fn, reps=5):
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)
    qkv_ms = timed(lambda: api.quant_qkv(q, k, v, "HND", problem=p, out=z, workspace=ws_qkv))
    qk_ms = timed(lambda: api.quant_qk(q, k, "HND", problem=p, out=z, workspace=ws_qk))
    v_ms = timed(lambda: api.quant_v(v, z, workspace=ws_v))
    elems_q = q.numel()
    elems_kv = k.numel()
    qk_bytes = 3.0 * elems_q + 5.0 * elems_kv   # Q: read 2 + write 1; K: 2 reads of 2 + write 1
    v_bytes = 5.0 * elems_kv                      # V: 2 reads of 2 + write 1

    bf16, bf16_sus, hbm, src = peaks()
    peak = bf16 * NOMINAL_INT8_OVER_BF16
    sweep = None
    if not args.no_sweep:
        del q, k, v, out, z, ws_qk, ws_v
        torch.cuda.empty_cache()
        sweep = measure_metric_range(args, dev, peak)
    achieved = ops / (attn_mean * 1e-3) / 1e12
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "attn_fwd_traffic.json")
    if os.path.exists(tpath):
        with open(tpath) as f:
            tr = json.load(f)
        import hashlib
        src_hash = hashlib.sha256(open(os.path.join(ROOT, "quantized_attention_06_b200", "csrc",
                                                    "attn_fwd.cuh"), "rb").read()).hexdigest()[:16]
        if tr.get("source_sha16") == src_hash and tr.get("workload_n") == w.seqlen:
            traffic = tr.get("bytes_per_launch")

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8 QK / e4m3 PV (fp32 softmax)",
            "data": "synthetic", "config": config(w, args, world),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "kernel": "sage_attn_fwd_kernel", "ms_per_launch": attn_mean,
                         "peak_source": f"{src} bf16 burst {bf16} x nominal INT8/FP8:bf16 ratio 2",
                         "frac_of_sustained": (achieved / (bf16_sus * NOMINAL_INT8_OVER_BF16)
                                               if bf16_sus else None),
                         "frac_of_datasheet_4500": achieved / 4500.0},
            "e2e": e2e,
            "quant": {"unit": "GB/s", "hbm_peak": hbm,
                      "quant_qkv": {"ms": qkv_ms,
                                    "achieved": (qk_bytes + v_bytes) / (qkv_ms * 1e-3) / 1e9,
                                    "frac": (qk_bytes + v_bytes) / (qkv_ms * 1e-3) / 1e9 / hbm,
                                    "bytes": qk_bytes + v_bytes, "launches": 1},
                      "quant_qk": {"ms": qk_ms, "achieved": qk_bytes / (qk_ms * 1e-3) / 1e9,
                                   "frac": qk_bytes / (qk_ms * 1e-3) / 1e9 / hbm,
                                   "bytes": qk_bytes},
                      "quant_v": {"ms": v_ms, "achieved": v_bytes / (v_ms * 1e-3) / 1e9,
                                  "frac": v_bytes / (v_ms * 1e-3) / 1e9 / hbm, "bytes": v_bytes}},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk.summary(),
        }
        if sweep is not None:
            line["sweep"] = sweep
        if pool is not None:
            tops, dt, sample = pool.sample(args.cpu_rows)
            pool.close()
            line["cpu_baseline"] = {"value": tops, "unit": UNIT, "cores": pool.cores,
                                    "kind": "oracle", "sample": sample, "seconds": dt,
                                    "nproc": os.cpu_count(), "cpu_model": cpu_model()}
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_sage(args)


if __name__ == "__main__":
    sys.exit(main())
