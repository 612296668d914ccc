"""Benchmark of the MoE layer forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload 131k_skewed|20b_decode|20b_prefill|120b_sweep|tiny|...] [--T n]

One step = one moe_forward call (router, top-k, histogram/scan/permutation, gate/up + SwiGLU,
down + weighted combine) over one batch of seeded synthetic tokens of the named workload.
Default: the largest configuration that fits one GPU -- a packed 131,072-token sequence
through the gpt-oss-20b-shaped layer (H = I = 2880, 32 experts, top-4) with Zipf-skewed
routing (max/mean expert load 4).  Inputs are resident in HBM before the timed region; every
step reads 0.75 GB of tokens and 1.6 GB of expert weights and writes 1.5 GB of output, far
more than the 126 MB L2.  Without --steps, K is chosen from the warm-up timing so that the
timed region lasts at least a second.

Prints one JSON line.  With N > 1 (torchrun, one process per GPU) every rank runs its own
replica on its own tokens (the layer is token-wise, so there is no data-path collective);
`value` is the tokens all ranks processed divided by the slowest rank's time.

--impl reference times the fp64 CPU oracle (the deliberately slow reference) on the host cores
on a bounded token sample of the same workload; only rank 0 works.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402

METRIC = "MoE layer tokens/s and µs/layer at 1 GPU; % of HBM or bf16 tensor roofline"
UNIT = "tokens/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0


# ----------------------------------------------------------------------------------------
# host-side helpers (CPU-testable)
# ----------------------------------------------------------------------------------------
def dist_env() -> tuple[int, int, int]:
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def reduce_max(value: float, world: int) -> float:
    """Max of a float over all ranks (identity for one rank)."""
    if world == 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(tokens_per_rank: int, world: int, max_seconds: float, steps: int) -> dict:
    """Whole-job throughput: all ranks' tokens over the slowest rank's timed seconds."""
    total = tokens_per_rank * world * steps
    return dict(value=total / max_seconds, ms_per_step=1e3 * max_seconds / steps)


def measured_peaks() -> tuple[float, float, float, str]:
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def peak_label(source: str, key: str) -> str:
    """Where a roofline denominator comes from, for the JSON line."""
    if source == "measured":
        return f"measured {key} (MEASURED_PEAKS.json)"
    return f"fallback {key} (no MEASURED_PEAKS.json: 6650 GB/s, 1590 TFLOP/s burst, 1400 sustained)"


def source_digest(paths) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key: str, workload: str, T: int) -> float | None:
    """DRAM bytes per launch of a kernel on a workload and token count, from the committed ncu
    summaries (profiles/traffic.json), if the kernel's sources are unchanged since."""
    try:
        with open(TRAFFIC_FILE) as f:
            entries = json.load(f)[kernel_key]
    except (OSError, KeyError, ValueError):
        return None
    for t in entries:
        if (t.get("workload") == workload and t.get("T") == T
                and t.get("sources_sha") == source_digest(t["sources"])):
            return float(t["dram_bytes_per_launch"])
    return None


def parse_clocks(csv_text: str) -> dict:
    """Median SM clock under load, max clock and the throttle reasons seen, from nvidia-smi CSV."""
    rows = [r.split(",") for r in csv_text.strip().splitlines()[1:] if r.strip()]
    sm, mx, reasons = [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for r in rows:
        r = [c.strip() for c in r]
        try:
            s, m, pw = float(r[1].split()[0]), float(r[2].split()[0]), float(r[3].split()[0])
        except (ValueError, IndexError):
            continue
        if pw > 200.0:  # under load
            sm.append(s)
        mx.append(m)
        for n, v in zip(names, r[5:9]):
            if v.lower() == "active":
                reasons.add(n)
    return dict(sm_mhz=statistics.median(sm) if sm else None, sm_max_mhz=max(mx) if mx else None,
                reasons=sorted(reasons), samples=len(rows), samples_under_load=len(sm))


class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index, self.proc, self.path = index, None, None

    def __enter__(self):
        self.path = f"/tmp/moe_bench_clocks_{os.getpid()}.csv"
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv", "-lms", "50"], stdout=open(self.path, "w"),
                stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def result(self) -> dict:
        if self.proc is None:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["nvidia-smi unavailable"])
        with open(self.path) as f:
            return parse_clocks(f.read())


# ----------------------------------------------------------------------------------------
# algorithmic work (what the method must touch)
# ----------------------------------------------------------------------------------------
def algorithmic(T: int, H: int, E: int, k: int, I: int, counts, weights: str = "bf16") -> dict:
    touched = int(sum(1 for c in counts if c > 0))
    R = T * k
    if weights == "mxfp4":   # 4-bit codes + one scale byte per 32 elements
        w_gate_up = touched * (H * 2 * I // 2 + H // 32 * 2 * I)
        w_down = touched * (I * H // 2 + I // 32 * H)
    else:
        w_gate_up = touched * H * 2 * I * 2
        w_down = touched * I * H * 2
    gate_up_bytes = w_gate_up + T * H * 2 + R * I * 2          # weights + x read + h write
    down_bytes = w_down + R * I * 2 + T * H * 4                 # weights + h read + out write
    layer_bytes = w_gate_up + w_down + H * E * 2 + T * H * 2 + T * H * 4
    gate_up_flops = 2 * R * H * 2 * I
    down_flops = 2 * R * I * H
    flops = gate_up_flops + down_flops + 2 * T * H * E
    return dict(touched=touched, gate_up_bytes=gate_up_bytes, down_bytes=down_bytes,
                layer_bytes=layer_bytes, flops=flops, gate_up_flops=gate_up_flops,
                down_flops=down_flops)


FAMILIES = ("stream", "tile", "gemm")
KERNEL_NAMES = {  # the gate/up kernel of each family, as ncu lists it
    "stream": "stream_gate_up_kernel", "tile": "expert_tile_kernel<0>",
    "gemm": "grouped_gemm_kernel<gate_up>"}


MX_STREAM_T = 176   # MXFP4 layers stream in calls of at most this many tokens


def split_families(counts, path: str, T: int, stream_T: int, stream_rows: int, tile_rows: int,
                   weights: str = "bf16", per_expert: bool = False) -> dict:
    """Row counts of the experts each kernel family multiplies, as the library dispatches them
    (moe_path in include/moe.h): with "auto", in calls of at most stream_T tokens an expert with
    c <= stream_rows rows streams; the others take expert tiles up to tile_rows (unless the mean
    load is at least 8 * tile_rows) and row tiles above, and a side of a boundary that the call's
    counts barely populate joins its neighbour (the library's snap rule).  Without per_expert,
    the experts of expert tiles and row tiles then all go to one of the two, row tiles if their
    mean count is at least tile_rows.  `counts` is the call's full histogram (one entry per
    expert)."""
    out = {f: [] for f in FAMILIES}
    cs = [int(c) for c in counts if c > 0]
    if weights == "mxfp4":
        f = "stream" if path == "stream" or (path == "auto" and T <= MX_STREAM_T) else "tile"
        out[f] = cs
        return out
    if path in FAMILIES:
        out[path] = cs
        return out
    s_on = T <= stream_T and stream_rows > 0
    lists = []                                   # (family, upper bound), launched families only
    lo = stream_rows if s_on else 0
    mean = sum(int(c) for c in counts) // max(1, len(counts))   # T * k / E for a full histogram
    if s_on:
        lists.append(["stream", stream_rows])
    if T > lo and tile_rows > lo and mean < 8 * tile_rows:
        lists.append(["tile", tile_rows])
    if T > max(lo, tile_rows):
        lists.append(["gemm", None])
    lists[-1][1] = None                          # the last family takes everything above
    fam = {}
    for i, c in enumerate(cs):
        for f, ub in lists:
            if ub is None or c <= ub:
                fam[i] = f
                break
    for l in range(len(lists) - 1):
        b = lists[l][1]
        lo_f, hi_f = lists[l][0], lists[l + 1][0]
        lo_c = [cs[i] for i in fam if fam[i] == lo_f]
        hi_c = [cs[i] for i in fam if fam[i] == hi_f]
        if lo_c and hi_c:
            if len(hi_c) <= len(lo_c) and max(hi_c) <= 2 * b:
                src, dst = hi_f, lo_f
            elif len(lo_c) < len(hi_c) and min(lo_c) > b // 2:
                src, dst = lo_f, hi_f
            else:
                continue
            for i in fam:
                if fam[i] == src:
                    fam[i] = dst
    names = [f for f, _ in lists]
    if not per_expert and "tile" in names and "gemm" in names:
        both = [i for i in fam if fam[i] in ("tile", "gemm")]
        rows = sum(cs[i] for i in both)
        dst = "gemm" if rows >= tile_rows * len(both) else "tile"
        for i in both:
            fam[i] = dst
    for i, f in fam.items():
        out[f].append(cs[i])
    return out


def family_work(counts, H: int, I: int, weights: str = "bf16") -> dict:
    """Algorithmic work of one projection pair over the given experts (their row counts): the
    touched experts' weights, the rows read and written, and the MMA FLOPs."""
    n, rows = len(counts), int(sum(counts))
    per_gu = H * 2 * I // 2 + H // 32 * 2 * I if weights == "mxfp4" else H * 2 * I * 2
    per_dn = I * H // 2 + I // 32 * H if weights == "mxfp4" else I * H * 2
    return dict(experts=n, rows=rows,
                gate_up_bytes=n * per_gu + rows * H * 2 + rows * I * 2,
                down_bytes=n * per_dn + rows * I * 2 + rows * H * 4,
                gate_up_flops=2 * rows * H * 2 * I, down_flops=2 * rows * I * H)


def dominant_roofline(work: dict, gate_up_ms: dict, hbm: float, bf16: float, bf16_sus: float,
                      peak_src: str) -> dict:
    """Roofline of the dominant kernel: the gate/up kernel of the family that spent the most
    time per call.  Its bound is its own: weight bytes over HBM bandwidth, or FLOPs over the
    tensor peak, whichever takes longer.  gate_up_ms: family -> ms per call (profiled)."""
    fam = max((f for f in FAMILIES if gate_up_ms.get(f, 0) > 0), key=lambda f: gate_up_ms[f])
    wk, secs = work[fam], gate_up_ms[fam] / 1e3
    t_hbm = wk["gate_up_bytes"] / (hbm * 1e9)
    t_tc = wk["gate_up_flops"] / (bf16 * 1e12)
    base = dict(kernel=KERNEL_NAMES[fam], family=fam, experts=wk["experts"], rows=wk["rows"],
                avg_launch_ms=gate_up_ms[fam])
    if t_hbm >= t_tc:
        ach = wk["gate_up_bytes"] / secs / 1e9
        return dict(bound="hbm", achieved=ach, peak=hbm, unit="GB/s", frac=ach / hbm,
                    alg_bytes_per_launch=wk["gate_up_bytes"],
                    peak_source=peak_label(peak_src, "hbm_gbs"), **base)
    # a launch well under a second is timed alone: the burst tensor peak applies
    ach = wk["gate_up_flops"] / secs / 1e12
    return dict(bound="tensor", achieved=ach, peak=bf16, unit="TFLOP/s", frac=ach / bf16,
                alg_flops_per_launch=wk["gate_up_flops"],
                peak_source=peak_label(peak_src, "bf16_tflops (burst)"),
                frac_of_sustained=ach / bf16_sus, frac_of_nominal_2250=ach / 2250.0, **base)


# ----------------------------------------------------------------------------------------
# the CPU oracle as a baseline (rank 0, N = 1 only; and the reference arm)
# ----------------------------------------------------------------------------------------
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_time(h: dict, k: int, tokens, reps: int) -> float:
    """Seconds for `reps` oracle calls of the layer on the given token rows (the layer is
    token-wise, so a subset of tokens gives the same rows as the whole batch)."""
    import oracle
    x = h["x"][np.asarray(tokens)]
    t0 = time.perf_counter()
    for _ in range(reps):
        if "gu_codes" in h:
            oracle.moe_forward_mxfp4_ref(x, h["W_router"], h["b_router"], h["gu_codes"],
                                         h["gu_scales"], h["dn_codes"], h["dn_scales"], k)
        else:
            oracle.moe_forward_ref(x, h["W_router"], h["b_router"], h["W_gate_up"], h["W_down"],
                                   k)
    return time.perf_counter() - t0


def baseline_tokens(w: mi.Workload, T: int) -> np.ndarray:
    """Tokens the oracle baseline runs on: the workload's seeded sample, else all T."""
    return mi.sample_tokens(T, w.oracle_sample, w.seed) if w.oracle_sample else np.arange(T)


def cpu_baseline(h: dict, w: mi.Workload, T: int, budget_s: float = 20.0) -> dict:
    toks = baseline_tokens(w, T)
    t1 = oracle_time(h, w.k, toks, 1)       # one call, also the warm-up
    reps = max(1, int(budget_s / max(t1, 1e-3)))
    secs = oracle_time(h, w.k, toks, reps)
    what = (f"a seeded {toks.size}-token sample of the {w.name} layer (T={T})"
            if toks.size < T else f"the {w.name} layer at T={T}")
    return dict(value=reps * toks.size / secs, unit=UNIT, cores=blas_threads(), kind="oracle",
                sample=f"{reps} oracle calls on {what}; numpy float64, "
                       f"{blas_threads()} BLAS threads on {os.cpu_count()} host cores")


def run_reference(args, w: mi.Workload, T: int) -> None:
    rank, world, _ = dist_env()
    if rank != 0:
        return
    h = mi.host_inputs(mi.make_inputs(T, w.H, w.E, w.k, w.I, w.seed, "cpu", zipf=w.zipf,
                                      weights=w.weights))
    steps = args.steps or 10
    budget = 150.0 / (steps + args.warmup)               # whole run within a few minutes
    pool = baseline_tokens(w, T) if w.oracle_sample else mi.sample_tokens(T, T, w.seed)
    t1 = oracle_time(h, w.k, pool[:1], 1)
    n = max(1, min(pool.size, int(budget / max(t1, 1e-3))))
    toks = np.sort(pool[:n]) if n < pool.size else pool
    for _ in range(args.warmup):
        oracle_time(h, w.k, toks, 1)
    secs = oracle_time(h, w.k, toks, steps)
    value = steps * n / secs
    line = dict(metric=METRIC, value=value, unit=UNIT, n_gpus=args.gpus, steps=steps,
                warmup=args.warmup, ms_per_step=1e3 * secs / steps, higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="f64", data="synthetic",
                impl="reference",
                config=dict(workload=w.name, T=T, H=w.H, E=w.E, k=w.k, I=w.I, sample_tokens=n),
                cpu_baseline=dict(value=value, unit=UNIT, cores=blas_threads(), kind="oracle",
                                  sample=f"{n} seeded tokens of {T} per step, full layer"),
                e2e=dict(value=value, unit=UNIT, h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------------------
MIN_TIMED_S = 1.2   # the timed region lasts at least this long (the clock sampler sees it)


def steps_for(step_s: float, min_s: float = MIN_TIMED_S, lo: int = 10, hi: int = 200000) -> int:
    """Steps that make the timed region last at least min_s, given one step's seconds."""
    return int(min(hi, max(lo, -(-min_s // max(step_s, 1e-7)))))


def default_steps(step, stream, world: int) -> int:
    """K from three timed extra warm-up steps (same K on every rank: the max)."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(3):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    k = steps_for(e0.elapsed_time(e1) / 3e3)
    return int(reduce_max(float(k), world))


def graph_timing(step, steps: int, world: int, per_graph: int = 1) -> dict:
    """The same calls captured once in a CUDA graph (per_graph consecutive steps: one per input
    batch) and replayed: no host launch work in the timed region, so the difference from
    `us_per_layer` is what launching from the host costs (it matters only at a few tokens)."""
    g = torch.cuda.CUDAGraph()
    try:
        with torch.cuda.graph(g):
            for _ in range(per_graph):
                step()
    except RuntimeError as e:      # capture refused: report it, the eager numbers stand
        return dict(error=str(e).splitlines()[0][:200])
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    replays = max(1, steps // per_graph)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    e0.record(stream)
    for _ in range(replays):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    secs = reduce_max(e0.elapsed_time(e1) / 1e3, world)
    del g
    return dict(us_per_layer=secs / (replays * per_graph) * 1e6, steps=replays * per_graph)


# A step whose touched expert weights are less than this many L2 sizes would keep part of them in
# L2 for the next step if every step routed the same tokens; such workloads cycle through
# ROTATE_BATCHES seeded token batches instead, so that consecutive steps touch other experts.
ROTATE_L2_FACTOR = 4
ROTATE_BATCHES = 16


def mean_dicts(ds: list) -> dict:
    """Field-wise mean of dicts with the same numeric fields."""
    return {k_: sum(d_[k_] for d_ in ds) / len(ds) for k_ in ds[0]}


def run_ours(args, w: mi.Workload, T: int) -> None:
    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    import mixture_experts_layer_48_b200 as moe

    seed = w.seed + 7919 * rank          # every rank its own tokens (weights identical)
    d = mi.make_inputs(T, w.H, w.E, w.k, w.I, w.seed, "cuda", zipf=w.zipf, weights=w.weights)
    if rank:
        d["x"] = mi.draw_x(T, w.H, seed, "cuda")
    layer = moe.Moe(w.E, w.H, w.I, w.k)
    layer.set_path({"auto": moe.MOE_PATH_AUTO, "stream": moe.MOE_PATH_STREAM,
                    "tile": moe.MOE_PATH_TILE, "gemm": moe.MOE_PATH_GEMM}[args.path])
    def route_counts(x):
        r = layer.route(x, d["W_router"], d["b_router"])
        return torch.diff(r["expert_offsets"]).cpu().tolist()

    counts = route_counts(d["x"])
    alg = algorithmic(T, w.H, w.E, w.k, w.I, counts, w.weights)
    xs = [d["x"]]
    l2_bytes = torch.cuda.get_device_properties(local).L2_cache_size
    rotate = alg["layer_bytes"] < ROTATE_L2_FACTOR * l2_bytes
    if rotate:
        xs += [mi.draw_x(T, w.H, seed + 104729 * j, "cuda") for j in range(1, ROTATE_BATCHES)]
    counts_all = [counts] + [route_counts(x) for x in xs[1:]]
    alg = mean_dicts([algorithmic(T, w.H, w.E, w.k, w.I, c_, w.weights) for c_ in counts_all])
    out = torch.empty((T, w.H), dtype=torch.float32, device="cuda")
    mx = w.weights == "mxfp4"
    if mx:
        fwd = layer.forward_mxfp4
        ws = torch.empty(layer.workspace_bytes_mxfp4(T), dtype=torch.uint8, device="cuda")
        args_fwd = (d["x"], d["W_router"], d["b_router"], d["gu_codes"], d["gu_scales"],
                    d["dn_codes"], d["dn_scales"])
    else:
        fwd = layer.forward
        ws = torch.empty(layer.workspace_bytes(T), dtype=torch.uint8, device="cuda")
        args_fwd = (d["x"], d["W_router"], d["b_router"], d["W_gate_up"], d["W_down"])
    stream = torch.cuda.current_stream()

    cur = [0]

    def step():  # one layer call on the next input batch
        x = xs[cur[0] % len(xs)]
        cur[0] += 1
        fwd(x, *args_fwd[1:], out=out, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert layer.sync_status() == moe.MOE_OK
    steps = args.steps or default_steps(step, stream, world)

    # ---- timed region: K calls between device events on the launching stream ----
    n_launch0 = layer.launch_count()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
    gpu_launches = layer.launch_count() - n_launch0
    secs = reduce_max(ev0.elapsed_time(ev1) / 1e3, world)
    assert layer.sync_status() == moe.MOE_OK
    agg = aggregate(T, world, secs, steps)

    # ---- second timed region: the same K calls with CUDA events around every kernel (on the
    # launching stream); these per-kernel times give the roofline.  The events stop successive
    # kernels from overlapping, so this pass is kept apart from the one that gives `value`.
    prof_steps = min(steps, 200)
    layer.profile_begin(prof_steps)
    for _ in range(prof_steps):
        step()
    prof = layer.profile_end()
    assert layer.sync_status() == moe.MOE_OK
    # ---- e2e: the same call with host buffers, copies inside the timed region ----
    x_hosts = [x.cpu().pin_memory() for x in xs]
    out_host = torch.empty((T, w.H), dtype=torch.float32).pin_memory()
    x_dev = torch.empty_like(d["x"])
    cur_e = [0]

    def e2e_step():
        x_dev.copy_(x_hosts[cur_e[0] % len(x_hosts)], non_blocking=True)
        cur_e[0] += 1
        fwd(x_dev, *args_fwd[1:], out=out, workspace=ws)
        out_host.copy_(out, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_secs = reduce_max(e0.elapsed_time(e1) / 1e3, world)
    graph = graph_timing(step, steps, world, per_graph=len(xs))
    assert layer.sync_status() == moe.MOE_OK

    # ---- roofline of the dominant kernel: the gate/up projection (2/3 of bytes and FLOPs) of
    # the kernel family that spent the most time ----
    hbm, bf16, bf16_sus, peak_src = measured_peaks()
    path_setting, stream_T = layer.get_path()
    stream_rows, tile_rows, per_expert = layer.get_dispatch()
    path = {moe.MOE_PATH_STREAM: "stream", moe.MOE_PATH_GEMM: "gemm",
            moe.MOE_PATH_TILE: "tile"}.get(path_setting, "auto")
    fams_all = [split_families(c_, path, T, stream_T, stream_rows, tile_rows, w.weights,
                               per_expert) for c_ in counts_all]
    fams = fams_all[0]
    work = {f: mean_dicts([family_work(fa[f], w.H, w.I, w.weights) for fa in fams_all])
            for f in FAMILIES}
    n_prof = prof_steps
    gu_ms = {f: prof["gate_up_" + f][0] / n_prof for f in FAMILIES}
    dn_ms = {f: prof["down_" + f][0] / n_prof for f in FAMILIES}
    layer_roof_s = max(alg["layer_bytes"] / (hbm * 1e9), alg["flops"] / (bf16 * 1e12))
    kernels_ms = {k_: round(v[0] / n_prof, 4) for k_, v in prof.items() if v[1]}
    roof = dominant_roofline(work, gu_ms, hbm, bf16, bf16_sus, peak_src)
    if mx:
        roof["kernel"] = {"stream": "stream_gate_up_mx_kernel",
                          "tile": "expert_tile_mx_kernel<0>"}.get(roof["family"], roof["kernel"])
    roof["traffic"] = ncu_traffic(roof["kernel"], w.name, T)
    down_rate = {f"down_{f}_ms": round(dn_ms[f], 4) for f in FAMILIES if dn_ms[f] > 0}
    dispatch = dict(stream_T=stream_T, stream_rows=stream_rows, tile_rows=tile_rows,
                    per_expert=per_expert,
                    experts={f: round(sum(len(fa[f]) for fa in fams_all) / len(fams_all), 2)
                             for f in FAMILIES},
                    rows={f: round(sum(sum(fa[f]) for fa in fams_all) / len(fams_all), 1)
                          for f in FAMILIES})

    line = dict(
        metric=METRIC, value=agg["value"], unit=UNIT, n_gpus=world, steps=steps,
        warmup=args.warmup, ms_per_step=agg["ms_per_step"], us_per_layer=agg["ms_per_step"] * 1e3,
        higher_is_better=True, scaling="weak", vs_baseline=None,
        dtype="mxfp4 weights, bf16 activations" if mx else "bf16",
        data="synthetic (seeded N(0,1) tokens, N(0,1/fan_in) bf16 weights; no trained weights)",
        config=dict(workload=w.name, T=T, H=w.H, E=w.E, k=w.k, I=w.I, path=path,
                    weights=w.weights, dispatch=dispatch,
                    parallelism=f"replicas{world}" if world > 1 else "single",
                    l2=("steps cycle through %d seeded token batches, so consecutive steps "
                        "touch other experts (%.2f GB of touched expert weights and tokens per "
                        "step vs %d MB L2)" % (len(xs), alg["layer_bytes"] / 1e9, l2_bytes >> 20))
                    if rotate else
                    ("inputs larger than L2: %.2f GB of touched expert weights and tokens per "
                     "step vs %d MB L2" % (alg["layer_bytes"] / 1e9, l2_bytes >> 20))),
        roofline=roof,
        layer_roofline=dict(touched_experts=alg["touched"], alg_bytes=alg["layer_bytes"],
                            alg_flops=alg["flops"], roofline_us=layer_roof_s * 1e6,
                            frac=layer_roof_s / (secs / steps), **down_rate),
        kernel_avg_ms=kernels_ms,
        kernel_timing="per-kernel CUDA events over a second timed pass of min(K, 200) of the same "
                      "calls (ms per call)",
        e2e=dict(value=T * world * steps / e2e_secs, unit=UNIT,
                 h2d_bytes_per_step=T * w.H * 2, d2h_bytes_per_step=T * w.H * 4),
        gpu_launches=gpu_launches,
        clocks=clk.result(),
        graph=graph,
    )
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        h = mi.host_inputs(d)
        line["cpu_baseline"] = cpu_baseline(h, w, T)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: enough for a timed region of >= 1.2 s)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="131k_skewed", choices=sorted(mi.WORKLOADS))
    ap.add_argument("--T", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--path", default="auto", choices=["auto", "stream", "tile", "gemm"],
                    help="kernel family for every expert (default: chosen from the call's counts)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = mi.WORKLOADS[args.workload]
    T = args.T or w.T
    if args.impl == "reference":
        run_reference(args, w, T)
    else:
        run_ours(args, w, T)


if __name__ == "__main__":
    main()
