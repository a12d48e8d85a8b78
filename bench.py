"""Benchmark of the BATQuant W4A4 linear layer on B200: Y = Q(XP) . Q(P^-1 W^T).

One step = the whole online path over one batch: the fused prologue (GPK block
transform + block clip + MXFP4 quantize/pack of X) and the block-scaled MXFP4
GEMM against weights prepared offline. Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

The headline workload defaults to prefill_o, the largest; on one GPU the line also
carries `per_config`, the same figures for the other workloads.

Multi-GPU (torchrun, one process per GPU): every rank runs its own batch of the
same layer (replicated weights, independent token batches, no collective on the
data path) -> weak scaling; time = max over ranks.
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

import numpy as np  # noqa: E402

import workloads as wl  # noqa: E402

METRIC = "W4A4 BAT linear TFLOP/s (% FP4 peak); act-quant prologue GB/s (% HBM)"
METRIC_W4A8 = "W4A8 BAT linear TFLOP/s (% FP8 peak); act-quant prologue GB/s (% HBM)"
PROLOGUE_BYTES_PER_ELT = 2.0 + 0.5 + 1.0 / 32.0  # bf16 in, 4-bit code out, 1/32 scale byte
PROLOGUE8_BYTES_PER_ELT = 2.0 + 1.0 + 1.0 / 32.0  # bf16 in, E4M3 code out, 1/32 scale byte
FP4_OVER_BF16 = 9.0 / 2.25  # nominal dense FP4 / BF16 tensor throughput on B200
FP8_OVER_BF16 = 4.5 / 2.25  # nominal dense FP8 (and FP8 x FP4) / BF16
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu record, if it still describes
    the current kernel source (hash match) and this workload; else None."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[kernel]
        h = hashlib.sha256()
        for fn in rec["files"]:
            with open(os.path.join(ROOT, fn), "rb") as f:
                h.update(f.read())
        if h.hexdigest()[:16] != rec["source_sha256_16"] or rec["workload"] != workload:
            return None
        return int(rec["traffic_bytes"])
    except Exception:
        return None


def max_over_ranks(dist_mod, values, device):
    """Element-wise max of per-rank timings (every rank gets the result)."""
    import torch
    if dist_mod is None:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist_mod.all_reduce(t, op=dist_mod.ReduceOp.MAX)
    return t.tolist()


def job_throughput(units_per_step: float, steps: int, world: int, seconds: float) -> float:
    """Whole-job rate: the units every rank processed over the slowest rank's time."""
    return units_per_step * steps * world / seconds


def rank_batch_seed(rank: int) -> int:
    """Token batch of rank r: seed r (rank 0 uses the workload's own seed 0)."""
    return rank


def rank_inputs(name: str, rank: int):
    """The workload for one rank: weights, factors and clip logits from seed 0 (shared
    by every rank), the token batch X from the rank's own seed."""
    inp = wl.make_inputs(name, seed=0)
    seed = rank_batch_seed(rank)
    x = inp.X if seed == 0 else wl.make_inputs(name, seed=seed, with_weight=False).X
    return inp, x


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# ---------------------------------------------------------------- clocks during the timed region
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="bat_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[4:]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for n, v in zip(names, r[3][1:]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        under = [r for r in rows if r[2] > 200.0]
        loaded = under or rows
        return {"sm_mhz": statistics.median(r[0] for r in loaded),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows), "samples_under_load": len(under),
                "power_w_max": max(r[2] for r in rows)}


# ---------------------------------------------------------------- CPU oracle leg
def oracle_sample(inp, w, budget_s: float, seed: int = 0, act_fmt: str = "e2m1"):
    """Time the oracle (as it stands) on a bounded sample of the layer.

    The sample is `rows` token rows against `cols` weight rows: the oracle's
    transform + clip + quantize of those rows, their dequantization, and the fp64
    dot products. Weight preparation is offline on both sides and not timed.
    Returns (flop/s, seconds, description, threads).
    """
    import oracle
    rng = np.random.default_rng(seed)
    _, wc, ws = oracle.prepare_weight(inp.W, inp.A, inp.B)
    Wd = oracle.dequantize(wc, ws)

    def run(rows, cols):
        t0 = time.perf_counter()
        X = inp.X[rows]
        _, xc, xs = oracle.quantize_act(X, inp.A, inp.B, inp.g_lo, inp.g_hi, fmt=act_fmt)
        Xd = oracle.dequantize(xc, xs, act_fmt)
        oracle.gemm_sampled(Xd, Wd, None, cols)
        return time.perf_counter() - t0

    cols = np.arange(w.N)
    run(rng.integers(0, w.M, size=1), cols)  # first call: page in the dequantized weights
    t1 = run(rng.integers(0, w.M, size=4), cols) / 4
    ncols = w.N
    per = int(max(1, min(w.M, 0.5 * budget_s / max(t1, 1e-6) / 4)))  # rows per timed batch
    if t1 > budget_s:  # a single full row is already over budget: sample columns too
        per, ncols = 1, int(max(1, w.N * budget_s / t1))
    sel = np.sort(rng.choice(w.N, size=ncols, replace=False))
    dt, nrows = 0.0, 0
    while dt < budget_s and nrows < w.M:  # repeat batches until the time budget is used
        rows = rng.choice(w.M, size=per, replace=False)
        dt += run(rows, sel)
        nrows += per
    flops = 2.0 * nrows * ncols * w.K
    desc = (f"{nrows} random token rows x {ncols} weight rows of {w.name} "
            f"(K={w.K}) in batches of {per}: transform+clip+quantize, dequantize, fp64 dot products")
    return flops / dt, dt, desc, oracle.num_threads()


def run_reference(args, w, inp):
    """The oracle timed as the reference arm, on the same config and metric."""
    steps, warm = args.steps, args.warmup
    per_step = max(0.05, min(2.0, args.ref_budget_s / max(1, steps + warm)))
    import oracle
    a8 = args.act == "mxfp8"
    fmt = "e4m3" if a8 else "e2m1"
    if args.shared != 8:
        inp.A, inp.B, _, _ = wl.random_factors(w.K // 32, seed=1, shared=args.shared)
    _, wc, ws = oracle.prepare_weight(inp.W, inp.A, inp.B)
    Wd = oracle.dequantize(wc, ws)
    rng = np.random.default_rng(1)

    nrows = max(1, min(w.M, oracle.num_threads()))  # one token row per oracle thread

    def step(ncols):
        rows = rng.choice(w.M, size=nrows, replace=False)
        cols = np.sort(rng.choice(w.N, size=ncols, replace=False))
        t0 = time.perf_counter()
        _, xc, xs = oracle.quantize_act(inp.X[rows], inp.A, inp.B, inp.g_lo, inp.g_hi, fmt=fmt)
        oracle.gemm_sampled(oracle.dequantize(xc, xs, fmt), Wd, None, cols)
        return time.perf_counter() - t0

    step(w.N)  # page in the dequantized weights
    t_full = step(w.N)
    ncols = int(max(1, min(w.N, w.N * per_step / max(t_full, 1e-6))))
    for _ in range(warm):
        step(ncols)
    total = 0.0
    for _ in range(steps):
        total += step(ncols)
    flops = 2.0 * nrows * ncols * w.K * steps
    value = flops / total / 1e12
    desc = f"per step: {nrows} random token rows x {ncols} weight rows of {w.name} (K={w.K})"
    line = {
        "impl": "reference", "metric": METRIC_W4A8 if a8 else METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": steps, "warmup": warm,
        "ms_per_step": 1e3 * total / steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "M": w.M, "N": w.N, "K": w.K},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- KV-cache store
KV_HEADS, KV_DIM = 8, 128  # Qwen3-8B-class attention: 8 KV heads of 128 channels


def kv_inputs(T: int, seed: int):
    """K and V [T][8][128] bf16: N(0,1) with 2 % of the head channels x20 in K (the
    channel outliers of keys), and the K- and V-path factors and clip logits."""
    rng = np.random.Generator(np.random.PCG64(seed))
    k = rng.standard_normal((T, KV_HEADS, KV_DIM)).astype(np.float32)
    ch = rng.choice(KV_DIM, size=max(1, KV_DIM // 50), replace=False)
    k[:, :, ch] *= 20.0
    v = rng.standard_normal((T, KV_HEADS, KV_DIM)).astype(np.float32)
    fk = wl.random_factors(KV_DIM // 32, seed=seed + 1)
    fv = wl.random_factors(KV_DIM // 32, seed=seed + 2)
    return wl.f32_to_bf16_bits(k), wl.f32_to_bf16_bits(v), fk, fv


def run_kv(args, rank, world, local):
    import torch
    import w4a4_bit_gemm_b200 as bat
    bat.lib()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist
    T = args.kv_tokens
    k_host, v_host, fk, fv = kv_inputs(T, seed=rank_batch_seed(rank))

    def bf16(bits):
        return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(dev)

    def f32(a):
        return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(dev)

    K, V = bf16(k_host), bf16(v_host)
    Ak, Bk, glk, ghk = (f32(a) for a in fk)
    Av, Bv, glv, ghv = (f32(a) for a in fv)
    S = 2 * T  # a paged cache twice the batch: the tokens land on scattered rows
    slots = torch.from_numpy(np.random.default_rng(3).permutation(S)[:T].astype(np.int64)).to(dev)
    ck = bat.KVCache.empty(S, KV_HEADS, KV_DIM, args.kv_format, dev)
    cv = bat.KVCache.empty(S, KV_HEADS, KV_DIM, args.kv_format, dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_view = flush.view(torch.int32)

    def step(Kin, Vin):
        bat.bat_kv_quantize(Kin, Ak, Bk, slots, ck, glk, ghk, stream=stream)
        bat.bat_kv_quantize(Vin, Av, Bv, slots, cv, glv, ghv, stream=stream)

    for i in range(args.warmup):
        flush.fill_(i & 0xFF)
        flush_view.amax()
        step(K, V)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    sampler = ClockSampler(local)
    if not args.no_clocks and rank == 0:
        sampler.start()
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        flush_view.amax()
        ev[i][0].record(stream)
        step(K, V)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    clocks = sampler.stop() if (not args.no_clocks and rank == 0) else None
    t = max_over_ranks(pg, [sum(e0.elapsed_time(e1) * 1e-3 for e0, e1 in ev)], dev)[0]
    assert bat.bat_device_error() == 0, "a kernel reported a failure"
    elems = 2 * T * KV_HEADS * KV_DIM
    per_elt = 2.0 + (1.0 if args.kv_format == "mxfp8" else 0.5) + 1.0 / 32.0
    gbs = per_elt * elems * args.steps * world / t / 1e9
    peaks, peak_src = load_peaks()

    e2e = None
    if not args.no_e2e:
        kh = torch.from_numpy(k_host.view(np.int16).copy()).view(torch.bfloat16).pin_memory()
        vh = torch.from_numpy(v_host.view(np.int16).copy()).view(torch.bfloat16).pin_memory()
        ch_codes = torch.empty_like(ck.codes, device="cpu").pin_memory()
        Kd, Vd = torch.empty_like(K), torch.empty_like(V)

        def e2e_step():
            Kd.copy_(kh, non_blocking=True)
            Vd.copy_(vh, non_blocking=True)
            step(Kd, Vd)
            ch_codes.copy_(ck.codes, non_blocking=True)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        te = max_over_ranks(pg, [e0.elapsed_time(e1) * 1e-3], dev)[0]
        e2e = {"value": per_elt * elems * args.e2e_steps * world / te / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": int(2 * K.numel() * 2),
               "d2h_bytes_per_step": int(ck.codes.numel())}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        rng = np.random.default_rng(0)
        n, dt = 0, 0.0
        while dt < args.cpu_budget_s and n < T:
            rows = rng.choice(T, size=min(64, T), replace=False)
            cc = np.zeros((len(rows), KV_HEADS, KV_DIM), np.uint8)
            cs = np.zeros((len(rows), KV_HEADS, KV_DIM // 32), np.uint8)
            t0 = time.perf_counter()
            ofmt = "e4m3" if args.kv_format == "mxfp8" else "e2m1"
            oracle.kv_quantize(k_host[rows], *fk, ofmt, np.arange(len(rows)), cc, cs)
            oracle.kv_quantize(v_host[rows], *fv, ofmt, np.arange(len(rows)), cc, cs)
            dt += time.perf_counter() - t0
            n += len(rows)
        cpu = {"value": per_elt * 2 * n * KV_HEADS * KV_DIM / dt / 1e9, "unit": "GB/s",
               "cores": oracle.num_threads(), "kind": "oracle",
               "sample": f"{n} random tokens of K and V (8 heads x 128), batches of 64",
               "seconds": round(dt, 2)}

    if rank == 0:
        line = {
            "metric": f"BAT KV-cache store GB/s (% HBM), {args.kv_format}",
            "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": args.kv_format, "data": "synthetic",
            "config": {"workload": f"kv_store T={T}", "tokens": T, "kv_heads": KV_HEADS,
                       "head_dim": KV_DIM, "cache_rows": S, "format": args.kv_format,
                       "l2": "flushed between steps (256 MiB write + read outside the timed events)",
                       "parallelism": f"replicas x{world} (independent token batches)"},
            "gpu_launches": 2 * args.steps * world,
            "roofline": {"bound": "hbm", "achieved": gbs / world, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": gbs / world / peaks["hbm_gbs"], "traffic": None,
                         "kernel": "bat_kv_quantize_kernel", "peak_source": peak_src},
            "clocks": clocks, "e2e": e2e, "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


def run_reference_kv(args):
    """The oracle's KV-cache store timed as the reference arm (same metric as --path kv)."""
    import oracle
    T = args.kv_tokens
    k_host, v_host, fk, fv = kv_inputs(T, seed=rank_batch_seed(0))
    fmt = "e4m3" if args.kv_format == "mxfp8" else "e2m1"
    per_elt = 2.0 + (1.0 if args.kv_format == "mxfp8" else 0.5) + 1.0 / 32.0
    rng = np.random.default_rng(0)
    per_step = max(0.05, min(2.0, args.ref_budget_s / max(1, args.steps + args.warmup)))
    nt = max(1, min(T, 64))
    cc = np.zeros((nt, KV_HEADS, KV_DIM), np.uint8)
    cs = np.zeros((nt, KV_HEADS, KV_DIM // 32), np.uint8)

    def step():
        n, t = 0, 0.0
        while t < per_step:
            rows = rng.choice(T, size=nt, replace=False)
            t0 = time.perf_counter()
            oracle.kv_quantize(k_host[rows], *fk, fmt, np.arange(nt), cc, cs)
            oracle.kv_quantize(v_host[rows], *fv, fmt, np.arange(nt), cc, cs)
            t += time.perf_counter() - t0
            n += nt
        return n, t

    for _ in range(args.warmup):
        step()
    tot_n, tot_t = 0, 0.0
    for _ in range(args.steps):
        n, t = step()
        tot_n += n
        tot_t += t
    value = per_elt * 2 * tot_n * KV_HEADS * KV_DIM / tot_t / 1e9
    desc = f"per step: batches of {nt} random tokens of K and V (8 heads x 128) for about {per_step:.2f} s"
    line = {
        "impl": "reference", "metric": f"BAT KV-cache store GB/s (% HBM), {args.kv_format}",
        "value": value, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"kv_store T={T}", "tokens": T, "kv_heads": KV_HEADS,
                   "head_dim": KV_DIM, "format": args.kv_format},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU leg
PER_CONFIG_ORDER = ("mlp_gate_up", "mlp_down", "decode_qkv", "prefill_o")


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


def oracle_prologue_rate(inp, w, budget_s: float, threads: int, seed: int = 5):
    """The oracle's activation side (transform + clip + MXFP4 quantize) on random token
    rows for about `budget_s` seconds with `threads` OpenMP threads; GB/s at the
    prologue's algorithmic 2.531 bytes per element."""
    import oracle
    prev = oracle.num_threads()
    oracle.set_num_threads(threads)
    try:
        rng = np.random.default_rng(seed)
        per = max(1, min(w.M, 8 * threads))
        oracle.quantize_act(inp.X[:1], inp.A, inp.B, inp.g_lo, inp.g_hi)  # page in
        n, dt = 0, 0.0
        while dt < budget_s and n < 64 * w.M:
            rows = rng.choice(w.M, size=per, replace=False)
            t0 = time.perf_counter()
            oracle.quantize_act(inp.X[rows], inp.A, inp.B, inp.g_lo, inp.g_hi)
            dt += time.perf_counter() - t0
            n += per
        gbs = PROLOGUE_BYTES_PER_ELT * n * w.K / dt / 1e9
        return {"value": gbs, "unit": "GB/s", "cores": threads, "seconds": round(dt, 2),
                "sample": f"{n} random token rows of {w.name} (K={w.K}) in batches of {per}"}
    finally:
        oracle.set_num_threads(prev)


class LinearBench:
    """One workload of the linear layer on one GPU (and its rank's token batch)."""

    def __init__(self, args, name, rank, dev, stream, pg):
        import torch
        import w4a4_bit_gemm_b200 as bat
        self.torch, self.bat, self.args, self.dev, self.stream, self.pg = torch, bat, args, dev, stream, pg
        self.w = w = wl.WORKLOADS[name]
        inp, X_host = rank_inputs(name, rank)
        self.inp, self.X_host = inp, X_host

        def bf16(bits):
            return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(dev)

        def f32(a):
            return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(dev)

        self.X = bf16(X_host)
        self.gl, self.gh = f32(inp.g_lo), f32(inp.g_hi)
        self.a8 = a8 = args.act == "mxfp8"
        gl, gh = self.gl, self.gh
        if args.shared != 8:  # another split: factors of the standard recipe at that size
            inp.A, inp.B, _, _ = wl.random_factors(w.K // 32, seed=1, shared=args.shared)
        self.A, self.B = A, B = f32(inp.A), f32(inp.B)
        if a8:
            self.quantize = lambda Xin, out, s=stream: bat.bat_quantize_act_mxfp8(
                Xin, A, B, gl, gh, Xq=out, stream=s)
            prepare = lambda Win: bat.bat_prepare_weight_gpk(Win, A, B)
        elif args.shared == 8:
            self.quantize = lambda Xin, out, s=stream: bat.bat_quantize_act(
                Xin, A, B, gl, gh, Xq=out, stream=s)
            prepare = lambda Win: bat.bat_prepare_weight(Win, A, B)
        else:
            self.quantize = lambda Xin, out, s=stream: bat.bat_quantize_act_gpk(
                Xin, A, B, gl, gh, Xq=out, stream=s)
            prepare = lambda Win: bat.bat_prepare_weight_gpk(Win, A, B)
        Wdev = bf16(inp.W)
        prepare(Wdev)  # first call: module load, attributes
        torch.cuda.synchronize()
        wp0, wp1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        wp0.record()
        self.Wq = prepare(Wdev)  # offline weight side, timed for information only
        wp1.record()
        torch.cuda.synchronize()
        self.prep_ms = wp0.elapsed_time(wp1)
        del Wdev
        self.Xq = (bat.MXFP8 if a8 else bat.MXFP4).empty(w.M, w.K, dev)
        self.Y = torch.empty(w.M, w.N, dtype=torch.bfloat16, device=dev)
        self.gemm_fn = bat.bat_w4a8_gemm if a8 else bat.bat_mxfp4_gemm
        # W4A4 with the default factor split: the step is the public bat_linear (the
        # quantizer and the GEMM on one stream); otherwise the two calls directly
        self.use_linear = not a8 and args.shared == 8
        self.ws = torch.empty(bat.bat_linear_workspace_bytes(w.M, w.K), dtype=torch.uint8, device=dev)
        self.flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.flush_view = self.flush.view(torch.int32)
        self.launches_per_step = 2

    def step(self):
        if self.use_linear:
            self.bat.bat_linear(self.X, self.Wq, self.A, self.B, self.gl, self.gh, Y=self.Y,
                                out_dtype=self.torch.bfloat16, workspace=self.ws, stream=self.stream,
                                fused=self.args.fused == 1)
        else:
            self.quantize(self.X, self.Xq)
            self.gemm_fn(self.Xq, self.Wq, Y=self.Y, out_dtype=self.torch.bfloat16, stream=self.stream)

    def flush_l2(self, i):
        # write, then read, a buffer twice the L2: the next kernel starts with a cold L2
        # holding only clean lines of unrelated data (no write-back lands on it)
        self.flush.fill_(i & 0xFF)
        self.flush_view.amax()

    def timed_pass(self, K_):
        """K_ steps, an L2 flush before each (outside the events), one event pair per step
        around the step's kernels. Nothing sits between the two kernels on the stream, so
        the GEMM (programmatic stream serialization) sets up while the quantizer finishes.
        Returns the sum of the step times (s)."""
        torch = self.torch
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K_)]
        if self.pg:
            self.pg.barrier()
        torch.cuda.synchronize()
        for i in range(K_):
            self.flush_l2(i)
            ev[i][0].record(self.stream)
            self.step()
            ev[i][1].record(self.stream)
        torch.cuda.synchronize()
        if self.pg:
            self.pg.barrier()
        return sum(e0.elapsed_time(e1) * 1e-3 for e0, e1 in ev)

    def kernel_pass(self, K_):
        """The same steps with an event between the two kernels (which also keeps them
        from overlapping): per-launch durations of the quantizer and the GEMM (s)."""
        torch = self.torch
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K_)]
        torch.cuda.synchronize()
        for i in range(K_):
            self.flush_l2(i)
            ev[i][0].record(self.stream)
            self.quantize(self.X, self.Xq)
            ev[i][1].record(self.stream)
            self.gemm_fn(self.Xq, self.Wq, Y=self.Y, out_dtype=torch.bfloat16, stream=self.stream)
            ev[i][2].record(self.stream)
        torch.cuda.synchronize()
        return ([e[0].elapsed_time(e[1]) * 1e-3 for e in ev],
                [e[1].elapsed_time(e[2]) * 1e-3 for e in ev])

    def run(self, steps, warmup, min_timed_s, sampler=None):
        """Warm-up, then timed passes of exactly `steps` steps until at least
        `min_timed_s` of timed GPU work has accumulated (so the clock record covers the
        load); the headline is the median pass, the max over ranks."""
        torch = self.torch
        for i in range(warmup):
            self.flush_l2(i)
            self.step()
        torch.cuda.synchronize()
        if sampler is not None:
            sampler.start()
        first = max_over_ranks(self.pg, [self.timed_pass(steps)], self.dev)[0]
        passes = int(min(400, max(1, np.ceil(min_timed_s / max(first, 1e-9)))))
        times = [first] + [self.timed_pass(steps) for _ in range(passes - 1)]
        clocks = sampler.stop() if sampler is not None else None
        med = float(np.median(times))
        t_step = max_over_ranks(self.pg, [med], self.dev)[0]
        # per-kernel durations: passes of the same steps until about a quarter of that time
        tp, tg = [], []
        while True:
            a, b = self.kernel_pass(steps)
            tp += a
            tg += b
            if sum(tp) + sum(tg) >= 0.25 * min_timed_s or len(tp) >= 400 * steps:
                break
        mp, mg = max_over_ranks(self.pg, [float(np.mean(tp)), float(np.mean(tg))], self.dev)
        assert self.bat.bat_device_error() == 0, "a kernel reported a stalled wait"
        return {"t_pass": t_step, "passes": passes, "timed_s": float(sum(times)),
                "pro_s": mp, "gemm_s": mg, "clocks": clocks}

    def summary(self, r, steps, world):
        """Figures of one measured workload (throughput of the whole job)."""
        w = self.w
        flop = 2.0 * w.M * w.N * w.K
        peaks, peak_src = load_peaks()
        ratio = FP8_OVER_BF16 if self.a8 else FP4_OVER_BF16
        tc_peak = peaks["bf16_tflops"] * ratio
        step_s = r["t_pass"] / steps
        value = job_throughput(flop, steps, world, r["t_pass"]) / 1e12
        gemm_tf = flop / r["gemm_s"] / 1e12
        pro_bytes = (PROLOGUE8_BYTES_PER_ELT if self.a8 else PROLOGUE_BYTES_PER_ELT) * w.M * w.K
        pro_gbs = pro_bytes / r["pro_s"] / 1e9
        d = {"workload": w.name, "M": w.M, "N": w.N, "K": w.K,
             "step_us": 1e6 * step_s, "linear_tflops": value / world,
             "linear_frac": value / world / tc_peak,
             "gemm_us": 1e6 * r["gemm_s"], "gemm_tflops": gemm_tf, "gemm_frac": gemm_tf / tc_peak,
             "prologue_us": 1e6 * r["pro_s"], "prologue_gbs": pro_gbs,
             "prologue_frac": pro_gbs / peaks["hbm_gbs"], "passes": r["passes"],
             "timed_s": round(r["timed_s"], 3)}
        if w.M <= 64:  # decode: memory-bound on the weight stream
            wbytes = w.N * w.K / 2 + w.N * ((w.K // 32 + 3) // 4) * 4
            d["gemm_weight_stream_gbs"] = wbytes / r["gemm_s"] / 1e9
            d["gemm_weight_stream_frac"] = d["gemm_weight_stream_gbs"] / peaks["hbm_gbs"]
        c = r.get("clocks")
        if c:
            d["clocks"] = c
            if c.get("sm_mhz"):
                d["step_us_x_sm_ghz"] = 1e6 * step_s * c["sm_mhz"] / 1e3
        return d, value, gemm_tf, tc_peak, pro_gbs, peaks, peak_src, ratio

    def e2e(self, world, e2e_steps):
        """End to end through the public API: pinned host X -> device, linear, Y -> pinned
        host. Two lanes (streams, each with its own buffers) take alternate steps, so one
        step's host copies overlap the other's kernels and copies in the other direction,
        as a serving loop would run them; every step still copies its X in from pinned
        host memory and its Y out."""
        torch, bat, w, args = self.torch, self.bat, self.w, self.args
        Xh = torch.from_numpy(self.X_host.view(np.int16).copy()).view(torch.bfloat16).pin_memory()
        lanes = []
        for _ in range(2):
            lanes.append({
                "stream": torch.cuda.Stream(self.dev),
                "Xdev": torch.empty_like(self.X),
                "Y": torch.empty(w.M, w.N, dtype=torch.bfloat16, device=self.dev),
                "Yh": torch.empty(w.M, w.N, dtype=torch.bfloat16).pin_memory(),
                "ws": torch.empty(bat.bat_linear_workspace_bytes(w.M, w.K), dtype=torch.uint8,
                                  device=self.dev),
                "Xq": (bat.MXFP8 if self.a8 else bat.MXFP4).empty(w.M, w.K, self.dev),
            })

        def e2e_step(i):
            ln = lanes[i % 2]
            ls = ln["stream"]
            with torch.cuda.stream(ls):
                ln["Xdev"].copy_(Xh, non_blocking=True)
                if self.use_linear:
                    bat.bat_linear(ln["Xdev"], self.Wq, self.A, self.B, self.gl, self.gh, Y=ln["Y"],
                                   out_dtype=torch.bfloat16, workspace=ln["ws"], stream=ls,
                                   fused=self.args.fused == 1)
                else:
                    self.quantize(ln["Xdev"], ln["Xq"], ls)
                    self.gemm_fn(ln["Xq"], self.Wq, Y=ln["Y"], out_dtype=torch.bfloat16, stream=ls)
                ln["Yh"].copy_(ln["Y"], non_blocking=True)

        for i in range(4):
            e2e_step(i)
        torch.cuda.synchronize()
        if self.pg:
            self.pg.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        for ln in lanes:
            ln["stream"].wait_event(e0)
        for i in range(e2e_steps):
            e2e_step(i)
        for ln in lanes:
            done = torch.cuda.Event()
            done.record(ln["stream"])
            self.stream.wait_event(done)
        e1.record(self.stream)
        torch.cuda.synchronize()
        te = max_over_ranks(self.pg, [e0.elapsed_time(e1) * 1e-3], self.dev)[0]
        flop = 2.0 * w.M * w.N * w.K
        return {"value": job_throughput(flop, e2e_steps, world, te) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": int(self.X.numel() * 2),
                "d2h_bytes_per_step": int(self.Y.numel() * 2)}

    def release(self):
        for k in ("X", "Wq", "Xq", "Y", "ws", "flush", "flush_view"):
            setattr(self, k, None)
        self.torch.cuda.synchronize()
        self.torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="prefill_o", choices=wl.ORDER,
                    help="headline workload (default: the largest, prefill_o)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget-s", type=float, default=8.0)
    ap.add_argument("--ref-budget-s", type=float, default=90.0)
    ap.add_argument("--min-timed-s", type=float, default=0.5,
                    help="repeat timed passes of --steps steps until this much timed GPU work")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="measure only the headline workload")
    ap.add_argument("--fused", type=int, default=0, choices=[0, 1],
                    help="bat_linear's fused argument: 1 lets the GEMM start on each token tile "
                         "as the prologue publishes it; 0 (default, the faster as measured) "
                         "waits for the whole prologue")
    ap.add_argument("--shared", type=int, default=8, choices=[1, 2, 4, 8, 16, 32],
                    help="size s of the shared transform factor (A s x s, each B_b 32/s x 32/s)")
    ap.add_argument("--act", default="mxfp4", choices=["mxfp4", "mxfp8"],
                    help="activation format: MXFP4 (W4A4) or MXFP8 E4M3 (W4A8)")
    ap.add_argument("--path", default="linear", choices=["linear", "kv"],
                    help="linear layer (default) or the KV-cache store (K and V of --kv-tokens tokens)")
    ap.add_argument("--kv-tokens", type=int, default=16384)
    ap.add_argument("--kv-format", default="mxfp8", choices=["mxfp8", "mxfp4"])
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank, world, local = dist_env()
    w = wl.WORKLOADS[args.workload]

    if args.impl == "reference":
        if rank == 0:
            if args.path == "kv":
                run_reference_kv(args)
            else:
                run_reference(args, w, wl.make_inputs(w.name, seed=0))
        return
    if args.path == "kv":
        run_kv(args, rank, world, local)
        return

    import torch
    import w4a4_bit_gemm_b200 as bat

    bat.lib()  # fail loudly if the CUDA library is missing
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist
    stream = torch.cuda.current_stream(dev)
    K_ = args.steps

    # rank r draws its own token batch; weights and transform factors are shared
    lb = LinearBench(args, w.name, rank, dev, stream, pg)
    sampler = ClockSampler(local) if (not args.no_clocks and rank == 0) else None
    r = lb.run(K_, args.warmup, args.min_timed_s, sampler)
    head, value, gemm_tf, tc_peak, pro_gbs, peaks, peak_src, ratio = lb.summary(r, K_, world)
    e2e = None if args.no_e2e else lb.e2e(world, args.e2e_steps)
    inp, a8 = lb.inp, lb.a8
    prep_ms = lb.prep_ms
    lb.release()

    # the other workloads, measured the same way (one GPU, rank 0 only)
    per_config = None
    if world == 1 and not args.no_per_config:
        per_config = {}
        for name in PER_CONFIG_ORDER:
            if name == w.name:
                continue
            o = LinearBench(args, name, rank, dev, stream, None)
            s_o = ClockSampler(local) if not args.no_clocks else None
            ro = o.run(K_, args.warmup, 0.25 * args.min_timed_s, s_o)
            per_config[name] = o.summary(ro, K_, 1)[0]
            o.release()
            del o

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        fl, dt, desc, thr = oracle_sample(inp, w, args.cpu_budget_s,
                                          act_fmt="e4m3" if a8 else "e2m1")
        cpu = {"value": fl / 1e12, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
               "sample": desc, "seconds": round(dt, 2), "cpu_model": cpu_model(),
               "host_cpus": os.cpu_count()}
        if not a8:
            budget = max(1.0, 0.25 * args.cpu_budget_s)
            cpu["prologue_1thread"] = oracle_prologue_rate(inp, w, budget, 1)
            cpu["prologue_all_cores"] = oracle_prologue_rate(inp, w, budget, oracle.num_threads())

    # the library's GEMM routing: CTA pairs on 256 x 256 tiles for MXFP4 activations with
    # more than one 128-row tile, the one-SM kernel otherwise (W4A8, decode split-K)
    if a8:
        gemm_kernel = "bat_mxf4_gemm_kernel<true> (W4A8)"
    elif w.M > 128:
        gemm_kernel = "bat_mxf4_gemm_pair_kernel (cta_group::2)"
    else:
        gemm_kernel = "bat_mxf4_gemm_kernel"
    pro_kernel = "bat_prologue_kernel<..., MXFP8>" if a8 else "bat_prologue_kernel"
    clocks = r["clocks"]
    if rank == 0:
        line = {
            "metric": METRIC_W4A8 if a8 else METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": K_, "warmup": args.warmup,
            "ms_per_step": 1e3 * r["t_pass"] / K_,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "mxfp8 x mxfp4" if a8 else "mxfp4", "data": "synthetic",
            "config": {"workload": w.name, "M": w.M, "N": w.N, "K": w.K, "out": "bf16",
                       "fused": bool(args.fused) and not a8 and args.shared == 8,
                       "transform": f"GPK A {args.shared}x{args.shared} shared, "
                                    f"B_b {32 // args.shared}x{32 // args.shared} private",
                       "l2": "flushed between steps (256 MiB write + read outside the timed events)",
                       "timing": f"median of {r['passes']} passes of {K_} steps "
                                 f"({r['timed_s']:.3f} s of timed steps)",
                       "parallelism": f"replicas x{world} (independent token batches)"},
            # timed passes: quantizer + GEMM per step
            "gpu_launches": lb.launches_per_step * K_ * r["passes"] * world,
            "roofline": {"bound": "tensor", "achieved": gemm_tf, "peak": tc_peak,
                         "unit": "TFLOP/s", "frac": gemm_tf / tc_peak,
                         "traffic": recorded_traffic(gemm_kernel, w.name),
                         "kernel": gemm_kernel,
                         "peak_source": f"{peak_src} bf16 burst x {ratio:g} (nominal "
                                        f"{'FP8' if a8 else 'FP4'}/BF16)"},
            "prologue": {"bound": "hbm", "achieved": pro_gbs, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": pro_gbs / peaks["hbm_gbs"],
                         "us_per_launch": head["prologue_us"],
                         "traffic": recorded_traffic(pro_kernel, w.name),
                         "kernel": pro_kernel, "peak_source": peak_src},
            "linear_frac": head["linear_frac"],
            "gemm_us_per_launch": head["gemm_us"],
            "prepare_weight_ms": prep_ms,
            "clocks": clocks,
            "step_us_x_sm_ghz": head.get("step_us_x_sm_ghz"),
            "per_config": per_config,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
