"""Benchmark of the W4A4 quantized linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload I] [--impl kq|reference]

A step is one pass of the whole online path over one batch of M tokens: per-token
centring, block transform, MXFP4 quantization and the low-rank input (quantize kernels),
then the block-scaled FP4 GEMM with the fused low-rank and rank-1 branches. The weights
are prepared once, offline (reported separately as prepare_ms, not in tokens/s).

Default workload: the video-DiT-shaped long sequence (M = 2 x 17550 = 35100 tokens, K=3072,
N=3072, Kronecker 4x4 (x) 8x8 block transform, per-token centring with the rank-1 restore,
rank-64 branch), bf16 output: the largest of the five workloads, and it fits one GPU. Inputs are seeded synthetic
data (see the ``synthetic`` package) already resident in HBM; rotating buffer sets
(activations, workspace, outputs and weight copies, together > 2x the 126 MB L2) keep
successive steps from hitting in L2. Steps are replayed from a CUDA graph; timing uses CUDA events on
the launching stream, max over ranks. For N > 1 every rank runs its own batch (tokens
are independent: weak scaling, no collective on the data path).

One JSON line is printed by rank 0.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A4 linear tokens/s; quantize HBM GB/s and GEMM FP4 TFLOPS as % of roofline"
DEFAULT_WORKLOAD = 5
# each phase-isolated timing replays its graph for at least this long
PHASE_MIN_S = 0.1


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16": float(p["bf16_tflops"]),
                "bf16_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


def max_over_ranks(value: float, dist, device) -> float:
    """The largest of every rank's value (timings are reported as the slowest rank's).
    Every rank must call it, in the same order as its other collectives."""
    import torch
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_rows(M: int, rank: int, world: int) -> tuple[int, int]:
    """[begin, end) of the token rows rank `rank` owns when a global batch of M tokens is
    split over `world` replicas (tokens are independent: no exchange is needed)."""
    base, extra = divmod(M, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def quantize_comparator(kq, torch, args, w, inp, sets, R, dev) -> dict:
    """The quantize kernel alone (rank 0, no centring) on this workload's M x K, once with a
    Kronecker block transform and once with SmoothQuant's per-channel scaling, over the same
    rotating activations (KroQuant section 02 reports its kernel up to 14 % faster than
    SmoothQuant's on MI350). Times are CUDA-event graph replays, microseconds per call."""
    from synthetic import make_transform, workload as wl
    Tk = make_transform(wl(w.index, transform="kron"))
    Lk = kq.Layer(w.K, w.N, 0, False, Tk)
    Ls = kq.Layer(w.K, w.N, 0, False, {"kind": "none"})
    wk = torch.zeros(kq.weights_bytes(Lk), dtype=torch.uint8, device=dev)  # not read (Kronecker)
    X0 = sets[0]["X"].float()
    Wf = inp["W"].to(dev).float()
    tiny = torch.finfo(torch.float32).tiny
    s = (X0.abs().amax(dim=0).clamp_min(tiny) / Wf.abs().amax(dim=1).clamp_min(tiny)).sqrt()
    inv_s = (1.0 / s.double()).float().contiguous()
    acts = [torch.empty(kq.act_bytes(Lk, w.M), dtype=torch.uint8, device=dev) for _ in range(R)]
    calls = {
        "kroquant": lambda j: kq.quantize_act(Lk, wk, sets[j]["X"], acts[j]),
        "smoothquant": lambda j: kq.smooth_quantize_act(Ls, inv_s, sets[j]["X"], acts[j]),
    }
    out = {}
    for name, fn in calls.items():
        for j in range(R):
            fn(j)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="relaxed"):
            for j in range(R):
                fn(j)
        g.replay()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        reps = max(10, int(np.ceil(PHASE_MIN_S * 1e3 / max(a.elapsed_time(b), 1e-3))))
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            g.replay()
        b.record()
        torch.cuda.synchronize()
        out[name] = a.elapsed_time(b) * 1e3 / (reps * R)
        del g
    return {"what": "quantize kernel alone, rank 0, no centring: Kronecker (KroQuant) vs "
                    "per-channel scaling (SmoothQuant, alpha 0.5), same MXFP4 encoder and pipeline",
            "shape": f"M={w.M} K={w.K}", "kroquant_us": out["kroquant"],
            "smoothquant_us": out["smoothquant"],
            "smoothquant_over_kroquant": out["smoothquant"] / out["kroquant"]}


def measured_traffic(kernel: str, workload_label: str):
    """DRAM bytes per launch of `kernel` (read + write) from the committed ncu capture
    (profiles/dram_traffic.json) with its note, or None when there is none for this workload
    or a source file of the kernel has changed since it was taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            recs = [r for r in json.load(f).get("records", [])
                    if r.get("kernel") == kernel and r.get("workload") == workload_label]
        if not recs:
            return None
        rec = recs[0]
        h = hashlib.sha256()
        for src in rec["sources"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        if h.hexdigest()[:16] != rec["source_sha256_16"]:
            return None
        return {"bytes": int(rec["dram_read_bytes"]) + int(rec["dram_write_bytes"]),
                "note": rec.get("note", "") + f" ({rec.get('profile', '')})"}
    except (OSError, ValueError, KeyError):
        return None


def algorithmic_work(M: int, K: int, N: int, rank: int, center: bool, lut: bool = False,
                     out_bf16: bool = True):
    """Roofline numerators of one step: the GEMM's flops (the 4-bit product, the rank-r
    branch and the rank-1 restore), the GEMM's bytes (every operand read once, Y written
    once) and the quantize phase's bytes (X read once; codes, scales, means and U written
    once). The low-rank operands are stored 64 wide whatever the rank."""
    rp = 64 if rank else 0
    gemm_flops = 2.0 * M * N * K + 2.0 * M * N * rank + (M * N if center else 0)
    ybytes = M * N * (2 if out_bf16 else 4)
    if lut:   # fp16 operand and fp16 residual, no block scales
        gemm_bytes = M * K * 2 + N * K * 2 + M * rp * 2 + N * rp * 2 + N * 4 + \
            (M * 4 if center else 0) + ybytes
        q_bytes = M * K * 2 + M * K * 2 + M * 8 + M * rp * 2
    else:
        gemm_bytes = M * K / 2 + N * K / 2 + (M + N) * K / 32 + M * rp * 2 + N * rp * 2 + N * 4 + \
            (M * 4 if center else 0) + ybytes
        q_bytes = M * K * 2 + M * K / 2 + M * K / 32 + M * 4 + M * rp * 2
    return gemm_flops, gemm_bytes, q_bytes


# nominal dense ratio FP4 : BF16 on B200 (9 : 2.25 PFLOP/s), and the nominal dense peaks
FP4_OVER_BF16 = 4.0
NOMINAL_FP4_TFLOPS = 9000.0
NOMINAL_FP16_TFLOPS = 2250.0


class Clocks:
    """nvidia-smi sampler for the SM clock and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sms, maxs, reasons = [], [], set()
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, mx = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            sms.append(sm)
            maxs.append(mx)
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sms:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxs),
                "reasons": sorted(reasons), "samples": len(sms)}


def oracle_tokens_per_s(w, inp, prep, budget_s: float, max_rows: int | None = None, ln=None,
                        lut: bool = False):
    """Time the CPU oracle's online path (LayerNorm front-end when on, centre, transform,
    encode, fp64 contraction with both branches) on the first rows of the batch, in
    4096-token pieces, for about budget_s seconds of work."""
    from oracle import layer as olayer
    X = inp["X"]
    if ln is not None:
        from oracle import layernorm as oln

        def linear(Xs, T, c, p):
            Y = oln.layernorm(Xs.double().numpy(), ln["gamma"], ln["beta"], ln["eps"])
            return olayer.linear(Y, T, c, p)
    elif lut:
        from oracle import lloydmax as olm

        def linear(Xs, T, c, p):
            return olm.linear(Xs.double().numpy(), T, c, p)
    else:
        linear = olayer.linear
    linear(X[:8], inp["T"], w.center, prep)                   # warm caches
    rows = int(max_rows or w.M)
    t0 = time.perf_counter()
    done = 0
    # 4096-token pieces (the oracle's matrix products stay as efficient as on a whole batch)
    # until about budget_s of work has run, or every token is done
    while done < rows and time.perf_counter() - t0 < budget_s:
        n = min(4096, rows - done)
        linear(X[done:done + n], inp["T"], w.center, prep)
        done += n
    dt = time.perf_counter() - t0
    return done / dt, done, dt


def oracle_stage_seconds(w, inp, prep, rows: int = 256) -> dict:
    """Wall time of the oracle's steps on the first `rows` tokens, per 1000 tokens: centring
    and block transform, MXFP4 encode (with the float32 rounding of its input), the low-rank
    input U, and the fp64 contraction (decode and the three terms)."""
    from oracle import bf16 as obf16
    from oracle import layer as olayer
    from oracle import mxfp4 as omx
    from oracle import transforms as otr
    X = inp["X"][:rows].double().numpy()
    out = {}
    t0 = time.perf_counter()
    mu, Xc = olayer.center(X, w.center)
    Xt = otr.apply(Xc, inp["T"])
    t1 = time.perf_counter()
    codes, scales = omx.encode(obf16.round_f32(Xt))
    t2 = time.perf_counter()
    U = Xt @ prep["L1"]
    t3 = time.perf_counter()
    olayer.linear_from_parts({"codes": codes, "scales": scales, "U": U, "mu": mu}, prep)
    t4 = time.perf_counter()
    k = 1000.0 / rows
    out["transform"] = (t1 - t0) * k
    out["encode"] = (t2 - t1) * k
    out["lowrank_input"] = (t3 - t2) * k
    out["contraction"] = (t4 - t3) * k
    return out


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def run_reference(args, w):
    """The oracle on the host cores, same workload/metric/unit (bounded sample per step)."""
    from oracle import layer as olayer
    from synthetic import make_inputs
    inp = make_inputs(w)
    prep = olayer.prepare(inp["W"], inp["T"], w.rank)
    X = inp["X"]
    t0 = time.perf_counter()
    olayer.linear(X[:32], inp["T"], w.center, prep)
    per_row = max((time.perf_counter() - t0) / 32, 1e-6)
    total_steps = max(1, args.steps + args.warmup)
    rows = int(np.clip(120.0 / total_steps / per_row, 1, w.M))
    for i in range(args.warmup):
        olayer.linear(X[:rows], inp["T"], w.center, prep)
    t0 = time.perf_counter()
    for i in range(args.steps):
        olayer.linear(X[:rows], inp["T"], w.center, prep)
    dt = time.perf_counter() - t0
    value = rows * args.steps / dt
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.label, "tokens_per_step": rows, "global_batch": w.M},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"first {rows} of {w.M} tokens per step, {args.steps} steps"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50000)
    ap.add_argument("--warmup", type=int, default=30)
    ap.add_argument("--workload", type=int, default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", choices=["kq", "reference"], default="kq")
    ap.add_argument("--out", choices=["bf16", "f32"], default="bf16")
    ap.add_argument("--sets", type=int, default=0, help="rotating buffer sets (0 = auto)")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-comparator", action="store_true",
                    help="skip the KroQuant-vs-SmoothQuant quantize-kernel timing")
    ap.add_argument("--center", action="store_true",
                    help="force per-token centring on (the workload's own setting otherwise)")
    ap.add_argument("--codebook", choices=["mxfp4", "lloydmax"], default="mxfp4",
                    help="activation format: MXFP4 (FP4 tensor cores) or the Lloyd-Max codebook "
                         "with a per-token sigma (fp16 tensor cores; RPBH workloads)")
    ap.add_argument("--layernorm", action="store_true",
                    help="fuse a LayerNorm front-end (seeded gamma, beta) into the layer; "
                         "implies --center")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    from synthetic import workload
    w = workload(args.workload, **({"center": True} if args.center or args.layernorm else {}))

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            run_reference(args, w)
        return

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    import w4a4_post_quantization_token_b200 as kq
    from synthetic import make_inputs

    inp = make_inputs(w)
    ln = None
    if args.layernorm:
        from synthetic import make_layernorm
        ln = make_layernorm(w)
    L = kq.Layer(w.K, w.N, w.rank, w.center, inp["T"], layernorm=ln, codebook=args.codebook)
    lut = args.codebook == "lloydmax"
    out_bf16 = args.out == "bf16"
    ydt = torch.bfloat16 if out_bf16 else torch.float32
    odt = kq.OUT_BF16 if out_bf16 else kq.OUT_F32

    # offline preparation on the GPU (timed separately)
    W = inp["W"].to(dev)
    wbuf0 = torch.empty(kq.weights_bytes(L), dtype=torch.uint8, device=dev)
    ws = torch.empty(kq.prepare_ws_bytes(L), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    kq.prepare_weights(L, W, wbuf0, ws)
    torch.cuda.synchronize()
    prepare_ms = (time.perf_counter() - t0) * 1e3
    del ws, W

    # rotating buffer sets
    X0 = inp["X"].to(dev)
    abytes = kq.act_bytes(L, w.M)
    set_bytes = X0.numel() * 2 + abytes + w.M * w.N * (2 if out_bf16 else 4) + wbuf0.numel()
    R = args.sets or max(2, int(np.ceil(2 * 126e6 / set_bytes)) + 1)
    sets = []
    for j in range(R):
        Xj = X0 if j == 0 else X0.clone()
        wj = wbuf0 if j == 0 else wbuf0.clone()
        sets.append({"X": Xj, "w": wj,
                     "act": torch.empty(abytes, dtype=torch.uint8, device=dev),
                     "Y": torch.empty((w.M, w.N), dtype=ydt, device=dev)})
    stream = torch.cuda.current_stream()

    def step(j):
        s = sets[j]
        kq.quantize_act(L, s["w"], s["X"], s["act"])
        kq.gemm(L, s["w"], s["act"], w.M, s["Y"], odt)

    for i in range(args.warmup):
        step(i % R)
    torch.cuda.synchronize()
    for s in sets:
        assert kq.last_device_error(L, s["act"], w.M) == 0

    # CUDA graphs: one rotation (R steps) of the whole path, and phase-isolated rotations
    # (quantize only, GEMM only) used to attribute the step time to kernels
    graph = gq = gg = None
    if not args.no_graph:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, capture_error_mode="relaxed"):
                for j in range(R):
                    step(j)
            gq = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gq, capture_error_mode="relaxed"):
                for j in range(R):
                    kq.quantize_act(L, sets[j]["w"], sets[j]["X"], sets[j]["act"])
            gg = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gg, capture_error_mode="relaxed"):
                for j in range(R):
                    kq.gemm(L, sets[j]["w"], sets[j]["act"], w.M, sets[j]["Y"], odt)
            graph.replay()
            gq.replay()
            gg.replay()
            torch.cuda.synchronize()
        except Exception as e:  # pragma: no cover - fall back to eager launches
            print(f"# graph capture failed ({e}); timing eager launches", file=sys.stderr)
            graph = gq = gg = None
    stream = torch.cuda.current_stream()

    def timed(fn, n):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    clocks = Clocks(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    if graph is not None:
        full, rem = divmod(args.steps, R)
        for _ in range(full):
            graph.replay()
        for j in range(rem):
            step(j)
    else:
        for i in range(args.steps):
            step(i % R)
    t_end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), dist if world > 1 else None, dev)
    if world > 1:
        dist.barrier()

    # per-kernel attribution: the same launches, one phase at a time, each replayed for at
    # least PHASE_MIN_S of device time whatever --steps is
    if gq is not None:
        q_fn, g_fn = gq.replay, gg.replay
    else:
        def q_fn():
            for s in sets:
                kq.quantize_act(L, s["w"], s["X"], s["act"])

        def g_fn():
            for s in sets:
                kq.gemm(L, s["w"], s["act"], w.M, s["Y"], odt)

    def phase_ms(fn):
        once = max(timed(fn, 1), 1e-3)
        reps = max(3, int(np.ceil(PHASE_MIN_S * 1e3 / once)))
        return timed(fn, reps) / (reps * R), reps

    q_ms, q_reps = phase_ms(q_fn)
    g_ms, g_reps = phase_ms(g_fn)
    for s in sets:
        assert kq.last_device_error(L, s["act"], w.M) == 0

    ms_per_step = elapsed_ms / args.steps
    tokens_per_s = w.M * world * args.steps / (elapsed_ms / 1e3)

    # roofline of the dominant kernel (algorithmic work per launch / event-timed duration).
    # Each phase is timed alone (graph replays of that phase only), so the denominators are
    # the burst figures: FP4 = 4 x the measured burst bf16 rate (the nominal 9 : 2.25 dense
    # ratio), fp16 = the burst bf16 rate, HBM = the measured copy rate.
    peaks = _peaks()
    M, K, N = w.M, w.K, w.N
    gemm_flops, gemm_bytes, q_bytes = algorithmic_work(M, K, N, w.rank, w.center, lut, out_bf16)
    tensor_peak = peaks["bf16"] * (1.0 if lut else FP4_OVER_BF16)
    nominal_peak = NOMINAL_FP16_TFLOPS if lut else NOMINAL_FP4_TFLOPS
    t_tensor = gemm_flops / (tensor_peak * 1e12)
    t_hbm = gemm_bytes / (peaks["hbm_gbs"] * 1e9)
    gname = "k_gemm_mxf4"
    if t_tensor >= t_hbm:
        ach = gemm_flops / (g_ms * 1e-3) / 1e12
        roof_g = {"kernel": gname, "bound": "tensor", "achieved": ach, "peak": tensor_peak,
                  "unit": "TFLOP/s", "frac": ach / tensor_peak,
                  "frac_of_nominal": ach / nominal_peak, "nominal_peak": nominal_peak,
                  # context: the same rate against the power-capped (sustained) measurement
                  "frac_of_sustained": ach / (peaks["bf16_sustained"] * (1.0 if lut else FP4_OVER_BF16)),
                  "peak_source": peaks["source"] + (" burst bf16 (fp16 rate)" if lut else
                                                    " burst bf16 x 4 (FP4 rate)")}
    else:
        ach = gemm_bytes / (g_ms * 1e-3) / 1e9
        roof_g = {"kernel": gname, "bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"],
                  "unit": "GB/s", "frac": ach / peaks["hbm_gbs"],
                  "peak_source": peaks["source"] + " copy bandwidth"}
    roof_g["algorithmic_per_launch"] = gemm_flops if roof_g["unit"] == "TFLOP/s" else gemm_bytes
    q_ach = q_bytes / (q_ms * 1e-3) / 1e9
    # Kronecker (or no) transform without the front-end or the codebook: the statistics +
    # low-rank kernel, then the streaming quantizer; otherwise the row-staged quantizer
    streaming = w.transform in ("kron", "none") and ln is None and not lut
    if streaming:
        qname = "k_lowrank_u+k_quantize_chunks" if (w.rank or w.center) else "k_quantize_chunks"
    else:
        qname = "k_quantize_rows+k_lowrank_u" if w.rank else "k_quantize_rows"
    roof_q = {"kernel": qname, "bound": "hbm", "achieved": q_ach, "peak": peaks["hbm_gbs"],
              "unit": "GB/s", "frac": q_ach / peaks["hbm_gbs"],
              "peak_source": peaks["source"] + " copy bandwidth", "algorithmic_per_launch": q_bytes}
    for r_ in (roof_g, roof_q):
        tr = measured_traffic(r_["kernel"], w.label)
        r_["traffic"] = tr["bytes"] if tr else None
        if tr:
            r_["traffic_note"] = tr["note"]
    roof = roof_g if g_ms >= q_ms else roof_q

    # end-to-end through the host-buffer entry point (pinned memory, copies timed)
    e2e = None
    if args.e2e_steps > 0:
        Xh = inp["X"].pin_memory()
        Yh = torch.empty((w.M, w.N), dtype=ydt).pin_memory()
        s0 = sets[0]
        for _ in range(2):
            kq.linear_host(L, s0["w"], Xh, s0["X"], Yh, s0["Y"], s0["act"], odt)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        e0.record()
        for _ in range(args.e2e_steps):
            kq.linear_host(L, s0["w"], Xh, s0["X"], Yh, s0["Y"], s0["act"], odt)
        e1.record()
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist if world > 1 else None, dev)
        e2e = {"value": w.M * world * args.e2e_steps / (e2e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": int(w.M * w.K * 2),
               "d2h_bytes_per_step": int(w.M * w.N * (2 if out_bf16 else 4)),
               "steps": args.e2e_steps, "api": "kq_linear_host"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import layer as olayer
        prep = olayer.prepare(inp["W"], inp["T"], w.rank)
        v, rows, dt = oracle_tokens_per_s(w, inp, prep, budget_s=12.0, ln=ln, lut=lut)
        cpu = {"value": v, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"first {rows} of {w.M} tokens ({dt:.1f} s, fp64 NumPy, weights "
                         f"prepared beforehand)"}
        if ln is None and not lut:
            cpu["stage_seconds_per_1k_tokens"] = oracle_stage_seconds(w, inp, prep)

    comparator = None
    if not args.no_comparator:
        comparator = quantize_comparator(kq, torch, args, w, inp, sets, R, dev)

    # launches per step: the streaming path (Kronecker or none) runs the statistics kernel
    # (when the layer centres or has a low-rank branch) and the quantizer, the row-staged
    # path the quantizer and the low-rank kernel; then the GEMM
    if streaming:
        launches_per_step = (2 if (w.rank or w.center) else 1) + 1
    else:
        launches_per_step = 2 + (1 if w.rank else 0)
    line = {
        "metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp16" if lut else "mxfp4",
        "data": "synthetic",
        "config": {"workload": w.label, "global_batch": w.M * world, "tokens_per_gpu": w.M,
                   "K": K, "N": N, "transform": w.transform, "center": w.center, "rank": w.rank,
                   "layernorm": ln is not None, "codebook": args.codebook, "out_dtype": args.out, "parallelism": f"replicas x{world} (token-sharded)",
                   "l2": f"{R} rotating buffer sets of {set_bytes / 1e6:.0f} MB (> L2)",
                   "graph": graph is not None},
        "phases_ms": {"quantize": q_ms, "gemm": g_ms,
                      "how": f"phase-isolated "
                             f"{'CUDA-graph replays' if gq is not None else 'eager launches'} "
                             f"over the same buffer sets, "
                             f"each >= {PHASE_MIN_S * 1e3:.0f} ms ({q_reps} and {g_reps} "
                             f"replays of {R} launches)"},
        "quantize_gbs": q_bytes / (q_ms * 1e-3) / 1e9,
        "gemm_tflops": gemm_flops / (g_ms * 1e-3) / 1e12,
        "roofline": roof,
        "roofline_gemm": roof_g,
        "roofline_quantize": roof_q,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
        "prepare_ms": prepare_ms,
        "comparator": comparator,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        del graph
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
