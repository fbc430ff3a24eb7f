"""Benchmark of the sparse MLA prefill attend block on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 1] [--impl ours|reference]

One step = one mla_prefill call (W_kvb up-projection, top-k bitmap,
sparse-causal attention, W_o) over one batch of seeded synthetic inputs of
the chosen workload (default: DeepSeek-V3.2-Exp-shaped sparse prefill,
B=1, T=4096, H=128, top-k 2048). With N > 1 (torchrun, one rank per GPU)
every rank runs its own independent instance: the work shards by sequence
with no collective on the data path ("weak" scaling); the time is the max
over ranks.

Metric: algorithmic TFLOP/s (the method's own work: up-projection, the
selected causal (query, key) pairs only, output projection), plus
queries/s and the fraction of the measured bf16 tensor peak. Rank 0 prints
one JSON line. ``--impl reference`` times the fp64 CPU oracle on the host
cores instead (the reference arm; a deliberately slow program).
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "sparse MLA prefill TFLOP/s and queries/s (T=4096,H=128,top-k 2048); % of bf16 peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ("ptx.cuh", "gemm2.cuh", "gemm8.cuh", "gemm_w8t.cuh", "gemm_m64.cuh", "quant.cuh", "attn.cuh", "attn_abs.cuh",
                  "prepass.cuh",
                  "dequant.cuh", "mla_api.cu")


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=None,
                   help="timed steps (default 200; 2000 for the decode step, so that its timed region lasts "
                        "long enough for the clock samples)")
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--config", type=int, default=1)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--mode", choices=["prefill", "decode"], default="prefill",
                   help="decode: one new position per sequence against a cache (B=64, T=32768 unless overridden)")
    p.add_argument("--e2e-steps", type=int, default=None, help="steps of the host-buffer run (default: --steps)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU-baseline sample budget")
    p.add_argument("--B", type=int, default=None, help="override the workload's batch (profiling runs)")
    p.add_argument("--T", type=int, default=None, help="override the workload's sequence length")
    p.add_argument("--H", type=int, default=None, help="override the workload's head count")
    p.add_argument("--topk", type=int, default=None, help="override the workload's top-k")
    p.add_argument("--parallel", choices=["sequences", "heads"], default="sequences",
                   help="N > 1: independent sequences per rank (weak scaling) or one problem with its heads "
                        "split over the ranks and the partial outputs all-reduced (strong scaling)")
    p.add_argument("--selections", type=int, default=1,
                   help="decode: rotate through this many different top-k selections, one per step (a device "
                        "copy of the next selection precedes every timed step); 1 repeats the same selection")
    p.add_argument("--path", choices=["auto", "dense", "absorbed"], default="auto",
                   help="attention path: the library's per-group choice (auto), every row block-dense, or every "
                        "row absorbed (needs top-k indices)")
    p.add_argument("--act", choices=["bf16", "e4m3"], default="bf16",
                   help="activations entering the projections (e4m3: dynamic per-token, needs e4m3 weights)")
    p.add_argument("--e4m3-weights", choices=["dequant", "onchip"], default="dequant",
                   help="e4m3 weights with bf16 activations: a dequantised bf16 copy per call (default), or "
                        "converted on chip inside the projection GEMMs")
    args = p.parse_args(argv)
    if args.steps is None:
        args.steps = 2000 if args.mode == "decode" and args.impl == "ours" else 200
    return args


def workload(args):
    """(name, inputs) of the chosen config with any size overrides applied."""
    cfg = dict(synth.CONFIGS[args.config])
    over = {k: getattr(args, k) for k in ("B", "T", "H", "topk") if getattr(args, k) is not None}
    name = cfg["name"]
    if over:
        name += "_" + "_".join(f"{k}{v}" for k, v in over.items())
    return name, synth.make_inputs(args.config, **over)


# ------------------------------------------------------------------ work model

def selected_pairs(x) -> int:
    """Sum over queries of |A_s| = |{t in topk_idx[b,s,:] : 0 <= t <= s}| (distinct)."""
    if x.topk_idx is None:
        return x.B * x.T * (x.T + 1) // 2
    total = 0
    s = torch.arange(x.T, dtype=torch.int64)[:, None]
    for b in range(x.B):
        for lo in range(0, x.T, 512):
            tk = x.topk_idx[b, lo:lo + 512].to(torch.int64)
            ok = (tk >= 0) & (tk <= s[lo:lo + 512])
            v = torch.where(ok, tk, torch.full_like(tk, -1)).sort(dim=1).values
            distinct = (v[:, 1:] != v[:, :-1]) & (v[:, 1:] >= 0)
            total += int(distinct.sum()) + int((v[:, 0] >= 0).sum())
    return total


def work_model(x):
    M, H = x.B * x.T, x.H
    pairs = selected_pairs(x)
    f_kvb = 2.0 * M * 512 * H * 256
    f_attn = float(pairs) * H * (2 * 192 + 2 * 128)
    f_wo = 2.0 * M * H * 128 * 7168
    wbytes = 1 if x.fp8 else 2
    comp = (x.q.numel() * 2 + x.kv_latent.numel() * 2 + x.k_pe.numel() * 2
            + x.W_kvb.numel() * wbytes + x.W_o.numel() * wbytes
            + (x.W_kvb_scale.numel() * 4 + x.W_o_scale.numel() * 4 if x.fp8 else 0)
            + (x.topk_idx.numel() * 4 if x.topk_idx is not None else 0) + M * 7168 * 2)
    return dict(pairs=pairs, flops_kvb=f_kvb, flops_attn=f_attn, flops_wo=f_wo,
                flops=f_kvb + f_attn + f_wo, compulsory_bytes=comp)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "sparse_head_latent_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    src = kernel_source_hash()
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel and parts[1] == workload \
                    and parts[3] == src:
                return float(parts[2])
    return None


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 20):
        self.gpu, self.period = gpu_index, period_ms
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 f"-lms={self.period}", f"--id={self.gpu}"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return self
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0: float, t1: float):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, line in self.lines:
            if not (t0 <= ts <= t1):
                continue
            f = [v.strip() for v in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle sampling

def host_info() -> dict:
    """The host's core count and CPU model (for the CPU-baseline fields)."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count() or 1, "cpu_model": model}


def selected_sets(x, rows):
    """A_s of each flattened row b*T + s: the distinct selected keys t <= s."""
    out = []
    for r in rows:
        b, s = divmod(int(r), x.T)
        if x.topk_idx is None:
            out.append(torch.arange(s + 1))
        else:
            tk = x.topk_idx[b, s].to(torch.int64)
            out.append(torch.unique(tk[(tk >= 0) & (tk <= s)]))
    return out


def oracle_sample(x, rows, act_e4m3: bool = False, threads: int = 1):
    """The oracle's whole block on a sample of query rows: the attention of
    every head (the fp64 up-projection of the keys these rows select, the
    masked softmax and the value mix) and then W_o on the full rows, with the
    heads spread over `threads` host threads (oracle.prefill_rows_threaded).
    Returns (seconds, algorithmic flops credited).

    The credit follows the GPU line's work model restricted to what the sample
    computes: every key the sample's rows select is up-projected once per
    head (2*512*256 FLOP; the full problem up-projects each of its B*T keys
    once, so the per-key cost is the same), each selected (row, key) pair
    costs H*(2*192 + 2*128) FLOP, and each row's output projection
    2*H*128*7168 FLOP."""
    import oracle
    sets = selected_sets(x, rows)
    keys = 0
    for b in sorted({int(r) // x.T for r in rows}):
        mine = [a for r, a in zip(rows, sets) if int(r) // x.T == b and a.numel()]
        if mine:
            keys += int(torch.unique(torch.cat(mine)).numel())
    pairs = sum(int(a.numel()) for a in sets)
    flops = (keys * x.H * 2.0 * 512 * 256 + pairs * x.H * (2 * 192 + 2 * 128)
             + len(rows) * 2.0 * x.H * 128 * 7168)
    t0 = time.perf_counter()
    oracle.prefill_rows_threaded(x, rows, act_e4m3=act_e4m3, n_threads=threads)
    return time.perf_counter() - t0, flops


def sample_rows_cpu(x, rng, n: int):
    """n random flattened rows (b*T + s) for one CPU sample pass."""
    return sorted({int(rng.integers(0, x.B)) * x.T + int(rng.integers(0, x.T)) for _ in range(n)})


def cpu_baseline(x, budget_s: float, total_flops: float, seed: int = 7, act_e4m3: bool = False):
    """The oracle timed on the host cores: passes over fresh random rows
    (4 rows, every head, then W_o) until `budget_s` is spent."""
    import oracle
    rng = np.random.default_rng(seed)
    threads = oracle.host_threads()
    tot_t, tot_f, n_rows, passes = 0.0, 0.0, 0, 0
    while tot_t < budget_s and passes < 1000:
        rows = sample_rows_cpu(x, rng, 4)
        dt, fl = oracle_sample(x, rows, act_e4m3, threads)
        tot_t += dt
        tot_f += fl
        n_rows += len(rows)
        passes += 1
    rate = tot_f / tot_t
    return {"value": rate / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{passes} passes over 4 random query rows of {x.name} ({n_rows} rows): the fp64 oracle's "
                      f"whole block for those rows (up-projection of the keys they select, attention of all "
                      f"{x.H} heads, W_o), heads spread over {threads} host threads; {tot_t:.1f} s",
            "gflops": round(rate / 1e9, 3), **host_info(),
            "extrapolated_full_step_s": round(total_flops / rate, 1),
            "extrapolation": "extrapolated: the workload's algorithmic FLOPs per step over the sample's rate",
            "seconds": tot_t}


DECODE_METRIC = "sparse MLA decode tokens/s (one new position per sequence, absorbed form)"


def decode_unit_problem(q_row, lat_b, kpe_b, W_kvb, W_o, sel, h, scale):
    """The oracle's problem for one (sequence, head) of a decode step: the
    head's query row attending its selected cache positions `sel` (ascending),
    laid out as a causal prefill of n = len(sel) positions whose last row is
    the query, so that it attends exactly those keys in the same ascending
    order; the head's W_kvb rows and W_o rows. Its output row is the head's
    share of the decode output (the shares sum over heads)."""
    from types import SimpleNamespace
    n = int(sel.numel())
    q = torch.zeros(1, n, 1, q_row.shape[-1], dtype=q_row.dtype)
    q[0, n - 1, 0] = q_row
    return SimpleNamespace(B=1, T=n, H=1, fp8=False, scale=scale, topk_idx=None, q=q,
                           kv_latent=lat_b[sel].unsqueeze(0).contiguous(),
                           k_pe=kpe_b[sel].unsqueeze(0).contiguous(),
                           W_kvb=W_kvb[h * 256:(h + 1) * 256], W_kvb_scale=None,
                           W_o=W_o[h * 128:(h + 1) * 128], W_o_scale=None)


def oracle_decode_unit(x, rng):
    """One sampled unit of the decode workload for the CPU oracle: a random
    (sequence, head): the fp64 up-projection of its selected cache rows for
    that head, the masked softmax, the value mix and the head's slice of
    W_o. Returns seconds."""
    import oracle
    b = int(rng.integers(0, x.B))
    h = int(rng.integers(0, x.H))
    if x.topk_idx is None:
        sel = torch.arange(x.T)
    else:
        tk = x.topk_idx[b]
        sel = torch.unique(tk[(tk >= 0) & (tk < x.T)])
    y = decode_unit_problem(x.q[b, h], x.kv_latent[b], x.k_pe[b], x.W_kvb, x.W_o, sel, h, x.scale)
    t0 = time.perf_counter()
    oracle.prefill_rows(y, [y.T - 1])
    return time.perf_counter() - t0


# ------------------------------------------------------------------ distributed plumbing

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, world: int) -> float:
    """Max of a per-rank scalar over all ranks (a no-op on one rank)."""
    if world <= 1:
        return value
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ our arm

def run_ours(args, rank, world, local):
    import sparse_head_latent_b200 as mla

    name, x = workload(args)
    wm = work_model(x)
    dev = torch.device("cuda", local)
    g = {k: v.to(dev) for k, v in x.tensors().items()}
    act = mla.MLA_ACT_E4M3_DYNAMIC if args.act == "e4m3" else mla.MLA_ACT_BF16
    if act and not x.fp8:
        raise SystemExit("--act e4m3 needs a workload with e4m3 weights (--config 4)")
    path = {"auto": mla.MLA_PATH_AUTO, "dense": mla.MLA_PATH_BLOCK_DENSE, "absorbed": mla.MLA_PATH_ABSORBED}[args.path]
    mla.mla_set_e4m3_weight_conversion(args.e4m3_weights == "onchip")
    dims = mla.make_dims(x.B, x.T, x.H, x.topk_idx.shape[-1] if x.topk_idx is not None else 0, x.fp8, path=path,
                         act=act)
    ws_bytes = mla.mla_workspace_bytes(dims, mla.MLA_ENTRY_PREFILL, x.topk_idx is not None)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    out = torch.empty(x.B, x.T, 7168, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(st=None):
        mla.mla_prefill(g["q"], g["kv_latent"], g["k_pe"], g["W_kvb"], g["W_o"], g.get("W_kvb_scale"),
                        g.get("W_o_scale"), topk_idx=g.get("topk_idx"), scale=x.scale, out=out,
                        workspace=ws, stream=st or stream, path=path, act=act)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    if mla.mla_device_status(stream) != 0:
        raise RuntimeError("device error during warm-up")
    # ---- per-kernel times: a short eager pass (up to 20 steps; it runs before
    # the timed region and should not heat the GPU for it) with an event pair
    # around every launch
    prof_steps = min(args.steps, 20)
    mla.mla_profile_begin()
    for _ in range(prof_steps):
        step()
    torch.cuda.synchronize(dev)
    prof = mla.mla_profile_end()
    # ---- device-resident timing: the step captured once as a CUDA graph (the
    # library only enqueues kernels on the given stream) and replayed, so the
    # number is the kernels' and not the host's launch gaps
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(torch.cuda.current_stream(dev))
    for _ in range(max(3, args.warmup)):
        graph.replay()
    torch.cuda.synchronize(dev)

    clocks = ClockSampler(local).start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    barrier(world)
    ms_local = e0.elapsed_time(e1) / args.steps
    del graph
    if mla.mla_device_status(stream) != 0:
        raise RuntimeError("device error in the timed region")

    # ---- end to end through the public API with host buffers: each step copies
    # its inputs from pinned host memory and its output back (PrefillPipeline
    # overlaps those copies with the previous/next step's kernels).
    e2e_steps = args.e2e_steps or args.steps
    host_in = {k: g[k].cpu().pin_memory() for k in ("q", "kv_latent", "k_pe", "topk_idx") if g.get(k) is not None}
    host_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = host_out.numel() * host_out.element_size()
    pipe = mla.PrefillPipeline(x.B, x.T, x.H, g["W_kvb"], g["W_o"], g.get("W_kvb_scale"), g.get("W_o_scale"),
                               topk=x.topk_idx.shape[-1] if x.topk_idx is not None else None, scale=x.scale,
                               device=dev, path=path, act=act)
    for _ in range(3):
        pipe.submit(host_in, host_out)
    pipe.synchronize()
    barrier(world)
    torch.cuda.synchronize(dev)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(pipe.h2d)
    for _ in range(e2e_steps):
        pipe.submit(host_in, host_out)
    f1.record(pipe.d2h)
    pipe.synchronize()
    torch.cuda.synchronize(dev)
    t_wall2 = time.time()
    barrier(world)
    e2e_ms_local = f0.elapsed_time(f1) / e2e_steps
    time.sleep(0.2)
    clocks.stop()

    ms = max_over_ranks(ms_local, world)
    e2e_ms = max_over_ranks(e2e_ms_local, world)
    if rank != 0:
        return None

    peaks, peak_src = load_peaks()
    tflops = wm["flops"] * world / (ms * 1e-3) / 1e12
    qps = x.B * x.T * world / (ms * 1e-3)
    e2e_tflops = wm["flops"] * world / (e2e_ms * 1e-3) / 1e12
    # Per-kernel algorithmic work per launch.
    kflops = {"gemm_kvb": wm["flops_kvb"], "attention": wm["flops_attn"], "gemm_wo": wm["flops_wo"]}
    per_kernel = {}
    for kname, (tot_ms, n) in prof.items():
        if n == 0:
            continue
        avg = tot_ms / n
        d = {"launches": n, "avg_ms": round(avg, 5)}
        if kname in kflops:
            d["tflops"] = round(kflops[kname] / (avg * 1e-3) / 1e12, 1)
        per_kernel[kname] = d
    if "gemm_wo" in per_kernel and "gemm_wo_split_sum" in per_kernel:
        # the K-split last wave's partial tiles are summed by a second kernel
        wo_ms = (prof["gemm_wo"][0] + prof["gemm_wo_split_sum"][0]) / prof["gemm_wo"][1]
        per_kernel["gemm_wo"]["tflops_with_split_sum"] = round(kflops["gemm_wo"] / (wo_ms * 1e-3) / 1e12, 1)
    dom = max((k for k in per_kernel if k in kflops), key=lambda k: prof[k][0])
    dom_avg_ms = prof[dom][0] / prof[dom][1]
    achieved = kflops[dom] / (dom_avg_ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    # With e4m3 activations the projections are e4m3 x e4m3 contractions: their
    # peak is the measured bf16 peak times the nominal fp8 / bf16 ratio (2).
    dom_fp8 = act and dom in ("gemm_kvb", "gemm_wo")
    dom_peak = 2 * peak if dom_fp8 else peak
    roof_t = max(wm["flops"] / (peak * 1e12), wm["compulsory_bytes"] / (peaks["hbm_gbs"] * 1e9))
    clk = clocks.summary(t_wall0, t_wall2)
    result = {
        "metric": METRIC, "value": round(tflops, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 x e4m3 projections, bf16 attention" if act else "bf16",
        "data": "synthetic (seeded; shapes and distributions of the workload; no checkpoint)",
        "config": {"workload": name, "B": x.B, "T": x.T, "H": x.H, "topk": x.topk,
                   "weights": "e4m3 block-128" if x.fp8 else "bf16",
                   "activations": "e4m3 dynamic 1x128" if act else "bf16",
                   **({"e4m3_weights": "converted on chip" if args.e4m3_weights == "onchip" else "dequantised copy"}
                      if x.fp8 and not act else {}),
                   "path": args.path,
                   "parallelism": f"independent sequences x{world}",
                   "l2": "no flush: every step reads > 600 MB, inputs larger than the 126 MB L2"},
        "queries_per_s": round(qps, 1),
        "frac_of_bf16_peak": round(tflops / world / peak, 4),
        "frac_of_roofline": round(roof_t / (ms * 1e-3), 4),
        "algorithmic_gflop_per_step": round(wm["flops"] / 1e9, 2),
        "selected_pairs": wm["pairs"],
        "per_kernel": per_kernel,
        "per_kernel_source": f"eager pass of {prof_steps} steps with an event pair around every launch",
        "timing": "CUDA graph replay of the whole step (inputs resident, larger than L2)",
        "roofline": {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 1), "peak": dom_peak,
                     "unit": "TFLOP/s", "frac": round(achieved / dom_peak, 4),
                     "traffic": ncu_traffic(dom, name + ("_act8" if act else "")),
                     "peak_source": (f"{peak_src} bf16 dense (burst) x 2 (nominal e4m3/bf16 ratio), MEASURED_PEAKS.json"
                                     if dom_fp8 else f"{peak_src} bf16 dense (burst), MEASURED_PEAKS.json")},
        "e2e": {"value": round(e2e_tflops, 2), "unit": UNIT, "h2d_bytes_per_step": h2d * world,
                "d2h_bytes_per_step": d2h * world, "ms_per_step": round(e2e_ms, 4)},
        # this rank's launches in the timed region: per step as counted in the
        # profiled pass, times the timed steps (graph replays launch the same kernels)
        "gpu_launches": int(round(sum(n for _, n in prof.values()) / prof_steps * args.steps)),
        "clocks": clk,
        "pages_note": "the source pages give only shapes and parameter counts: no throughput numbers or hardware",
    }
    if world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = {k: v for k, v in cpu_baseline(x, args.cpu_seconds, wm["flops"],
                                                                 act_e4m3=bool(act)).items() if k != "seconds"}
    return result


def run_heads(args, rank, world, local):
    """One problem of the workload with its heads split over the ranks
    (sparse_head_latent_b200.tp.HeadShardedPrefill): per step every rank runs
    its heads' attention and W_o rows and the partial outputs are all-reduced
    in row chunks overlapped with the projection. `value` is the problem's
    algorithmic FLOPs over the max-over-ranks step time (strong scaling)."""
    import sparse_head_latent_b200 as mla
    from sparse_head_latent_b200.tp import HeadShardedPrefill

    name, x = workload(args)
    wm = work_model(x)
    dev = torch.device("cuda", local)
    act = mla.MLA_ACT_E4M3_DYNAMIC if args.act == "e4m3" else mla.MLA_ACT_BF16
    tk = x.topk_idx.shape[-1] if x.topk_idx is not None else None
    g = {k: v.to(dev) for k, v in x.tensors().items() if k not in ("q",)}
    tp = HeadShardedPrefill(x.B, x.T, x.H, g["W_kvb"], g["W_o"], g.get("W_kvb_scale"), g.get("W_o_scale"), topk=tk,
                            scale=x.scale, act=act, device=dev)
    q_local = x.q[:, :, tp.h0:tp.h1].contiguous().to(dev)
    out = torch.empty(x.B, x.T, 7168, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        tp(q_local, g["kv_latent"], g["k_pe"], g.get("topk_idx"), out=out)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local).start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    mla.mla_profile_begin()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    prof = mla.mla_profile_end()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    # End to end: the rank's inputs from pinned host memory and the output back, every step.
    host = {"q": q_local.cpu().pin_memory(), "kv_latent": g["kv_latent"].cpu().pin_memory(),
            "k_pe": g["k_pe"].cpu().pin_memory()}
    if g.get("topk_idx") is not None:
        host["topk_idx"] = g["topk_idx"].cpu().pin_memory()
    dev_in = {k: torch.empty_like(v, device=dev) for k, v in host.items()}
    host_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = host_out.numel() * host_out.element_size()
    barrier(world)
    torch.cuda.synchronize(dev)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = args.e2e_steps or args.steps
    f0.record(stream)
    for _ in range(e2e_steps):
        for k, v in host.items():
            dev_in[k].copy_(v, non_blocking=True)
        tp(dev_in["q"], dev_in["kv_latent"], dev_in["k_pe"], dev_in.get("topk_idx"), out=out)
        host_out.copy_(out, non_blocking=True)
    f1.record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    barrier(world)
    e2e_ms = max_over_ranks(f0.elapsed_time(f1) / e2e_steps, world)
    clocks.stop()
    if mla.mla_device_status(stream) != 0:
        raise RuntimeError("device error in the timed region")
    if rank != 0:
        return None
    peaks, peak_src = load_peaks()
    tflops = wm["flops"] / (ms * 1e-3) / 1e12
    kflops = {"gemm_kvb": wm["flops_kvb"] / world, "attention": wm["flops_attn"] / world,
              "gemm_wo": wm["flops_wo"] / world}
    # Work per step of each kernel class on this rank (W_o runs once per row
    # chunk, so rates are per step, not per launch).
    per_kernel = {}
    for kname, (tot_ms, n) in prof.items():
        if n:
            per_kernel[kname] = {"launches": n, "avg_ms": round(tot_ms / n, 5)}
            if kname in kflops:
                per_kernel[kname]["tflops"] = round(kflops[kname] / (tot_ms / args.steps * 1e-3) / 1e12, 1)
    dom = max((k for k in per_kernel if k in kflops), key=lambda k: prof[k][0])
    achieved = kflops[dom] / (prof[dom][0] / args.steps * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    return {
        "metric": METRIC, "value": round(tflops, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "e4m3 x e4m3 projections, bf16 attention" if act else "bf16",
        "data": "synthetic (seeded; shapes and distributions of the workload; no checkpoint)",
        "config": {"workload": name, "B": x.B, "T": x.T, "H": x.H, "topk": x.topk,
                   "weights": "e4m3 block-128" if x.fp8 else "bf16",
                   "activations": "e4m3 dynamic 1x128" if act else "bf16",
                   "parallelism": f"heads split over {world} ranks, partial outputs all-reduced (NCCL)",
                   "l2": "no flush: every step reads more than the 126 MB L2"},
        "queries_per_s": round(x.B * x.T / (ms * 1e-3), 1),
        "per_kernel": per_kernel,
        "roofline": {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": None,
                     "peak_source": f"{peak_src} bf16 dense (burst), MEASURED_PEAKS.json"},
        "e2e": {"value": round(wm["flops"] / (e2e_ms * 1e-3) / 1e12, 2), "unit": UNIT,
                "h2d_bytes_per_step": h2d * world, "d2h_bytes_per_step": d2h * world, "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": int(sum(n for _, n in prof.values())),
        "clocks": clocks.summary(t_wall0, t_wall1),
    }


# ------------------------------------------------------------------ reference arm (CPU oracle)

def run_decode(args, local):
    """Decode throughput: B sequences, one new position each, against a cache
    of T positions (the new one last), top-k selected positions per query.
    Bound by HBM: the weights plus the gathered latent rows."""
    import sparse_head_latent_b200 as mla

    B, T = args.B or 64, args.T or 32768
    H, k = args.H or 128, args.topk or 2048
    x = synth.make_decode_inputs(B, T, H, k, seed=11)
    dev = torch.device("cuda", local)
    g = {n: v.to(dev) for n, v in x.tensors().items()}
    # Selections to rotate through (set 0 is the inputs' own): with a single
    # repeated selection the gathered latent rows of one step can still be in
    # L2 at the next.
    nsel = max(1, args.selections)
    sel_sets = torch.stack([x.topk_idx] + [synth.decode_topk(B, T, k, 11 + r) for r in range(1, nsel)]).to(dev)
    dims = mla.make_dims(B, T, H, k, False)
    ws = torch.empty(mla.mla_workspace_bytes(dims, mla.MLA_ENTRY_DECODE, True), dtype=torch.uint8, device=dev)
    out = torch.empty(B, 7168, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(st=None):
        mla.mla_decode(g["q"], g["kv_latent"], g["k_pe"], g["W_kvb"], g["W_o"], topk_idx=g["topk_idx"],
                       scale=x.scale, out=out, workspace=ws, stream=st or stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    # Per-kernel times from an eager, profiled run of a few of the steps.
    prof_steps = min(args.steps, 50)
    mla.mla_profile_begin()
    for _ in range(prof_steps):
        step()
    torch.cuda.synchronize(dev)
    prof = mla.mla_profile_end()
    # The step is a handful of short kernels, so it is timed as a CUDA graph
    # replay (the host's launch gaps would otherwise dominate).
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(torch.cuda.current_stream(dev))
    for _ in range(max(3, args.warmup)):
        graph.replay()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local).start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    e0.record(stream)
    for i in range(args.steps):
        if nsel > 1:
            g["topk_idx"].copy_(sel_sets[i % nsel], non_blocking=True)
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    clocks.stop()
    if mla.mla_device_status(stream) != 0:
        raise RuntimeError("device error in the timed region")
    ms = e0.elapsed_time(e1) / args.steps
    g["topk_idx"].copy_(sel_sets[0])
    # End to end: every step copies its new inputs from pinned host memory --
    # the queries, the selections and the new position's latent and rope rows
    # (the cache itself stays resident) -- replays the step and copies the
    # output back.
    h_q, h_tk = g["q"].cpu().pin_memory(), g["topk_idx"].cpu().pin_memory()
    h_lat, h_pe = g["kv_latent"][:, T - 1].cpu().pin_memory(), g["k_pe"][:, T - 1].cpu().pin_memory()
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (h_q, h_tk, h_lat, h_pe))
    d2h = h_out.numel() * h_out.element_size()
    e2e_steps = args.e2e_steps or args.steps
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(e2e_steps):
        g["q"].copy_(h_q, non_blocking=True)
        g["topk_idx"].copy_(h_tk, non_blocking=True)
        g["kv_latent"][:, T - 1].copy_(h_lat, non_blocking=True)
        g["k_pe"][:, T - 1].copy_(h_pe, non_blocking=True)
        graph.replay()
        h_out.copy_(out, non_blocking=True)
    f1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = f0.elapsed_time(f1) / e2e_steps
    del graph
    sel = min(k, T)
    compulsory = (H * 256 * 512 * 2 + H * 128 * 7168 * 2        # W_kvb, W_o
                  + B * sel * (512 + 64) * 2                      # gathered latent and rope rows
                  + B * H * 192 * 2 + B * k * 4 + B * 7168 * 2)  # q, top-k, out
    flops = B * (2.0 * H * 128 * 512 * 2 + sel * H * 2 * (576 + 512) + 2.0 * H * 128 * 7168)
    peaks, src = load_peaks()
    gbs = compulsory / (ms * 1e-3) / 1e9
    per = {n: {"launches": c, "avg_ms": round(t / max(c, 1), 5)} for n, (t, c) in prof.items() if c}
    return {
        "metric": DECODE_METRIC,
        "value": round(B / (ms * 1e-3), 1), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; no checkpoint)",
        "config": {"workload": f"decode_B{B}_T{T}", "B": B, "T": T, "H": H, "topk": k, "weights": "bf16",
                   "selections": nsel,
                   "l2": "no flush: W_o alone (235 MB) exceeds the 126 MB L2; "
                         + ("the same selection every step (its gathered rows can stay in L2)" if nsel == 1 else
                            f"{nsel} selections in rotation, a device copy of the next one inside each timed step")},
        "algorithmic_gflop_per_step": round(flops / 1e9, 3),
        "roofline": {"kernel": "whole decode step", "bound": "hbm", "achieved": round(gbs, 1),
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                     "traffic": None, "peak_source": f"{src} HBM copy bandwidth",
                     "bytes_per_step": compulsory},
        "per_kernel": per, "per_kernel_source": f"eager profiled run of {prof_steps} of the steps",
        "timing": "CUDA graph replay of the whole decode step",
        "gpu_launches": int(round(sum(c for _, c in prof.values()) / prof_steps * args.steps)),
        "e2e": {"value": round(B / (e2e_ms * 1e-3), 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 5)},
        "clocks": clocks.summary(t_wall0, t_wall1),
    }


def run_reference_decode(args):
    """The oracle on decode units: each step is one (sequence, head) unit;
    a token needs H of them, so tokens/s = 1 / (H x mean unit time)."""
    B, T = args.B or 64, args.T or 32768
    H, k = args.H or 128, args.topk or 2048
    x = synth.make_decode_inputs(B, T, H, k, seed=11)
    rng = np.random.default_rng(11)
    for _ in range(args.warmup):
        oracle_decode_unit(x, rng)
    tot = sum(oracle_decode_unit(x, rng) for _ in range(args.steps))
    v = args.steps / (tot * H)
    sample = (f"{args.steps} random (sequence, head) units of decode_B{B}_T{T} (fp64 oracle, 1 host thread); "
              f"a token is H = {H} units")
    return {"impl": "reference", "metric": DECODE_METRIC, "value": v, "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)",
            "config": {"workload": f"decode_B{B}_T{T}", "B": B, "T": T, "H": H, "topk": k, "weights": "bf16"},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    if args.mode == "decode":
        return run_reference_decode(args)
    import oracle
    name, x = workload(args)
    wm = work_model(x)
    rng = np.random.default_rng(11)
    threads = oracle.host_threads()
    # Each step is one sample pass: 2 random query rows, the oracle's whole
    # block for them (every head, then W_o), heads spread over the host
    # threads; a few seconds each at this workload, so a default run stays
    # within a few minutes.
    act8 = args.act == "e4m3"
    for _ in range(args.warmup):
        oracle_sample(x, sample_rows_cpu(x, rng, 2), act8, threads)
    tot_t, tot_f = 0.0, 0.0
    for _ in range(args.steps):
        dt, fl = oracle_sample(x, sample_rows_cpu(x, rng, 2), act8, threads)
        tot_t += dt
        tot_f += fl
    v = tot_f / tot_t / 1e12
    sample = (f"{args.steps} passes over 2 random query rows of {name}: the fp64 oracle's whole block for those "
              f"rows (up-projection of the keys they select, attention of all {x.H} heads, W_o), heads spread "
              f"over {threads} host threads" + (", dynamic e4m3 activations" if act8 else ""))
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
            "higher_is_better": True, "scaling": "strong" if args.parallel == "heads" else "weak",
            "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "config": {"workload": name, "B": x.B, "T": x.T, "H": x.H,
                                                    "topk": x.topk,
                                                    "weights": "e4m3 block-128" if x.fp8 else "bf16",
                                                    "activations": "e4m3 dynamic 1x128" if act8 else "bf16"},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample,
                             "gflops": round(v * 1e3, 3), **host_info(),
                             "extrapolated_full_step_s": round(wm["flops"] / (v * 1e12), 1),
                             "extrapolation": "extrapolated: the workload's algorithmic FLOPs per step over the "
                                              "sample's rate"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        res = run_reference(args, rank, int(os.environ.get("WORLD_SIZE", "1")))
    else:
        rank, world, local = dist_setup()
        try:
            if args.mode == "decode":
                res = run_decode(args, local)
            elif args.parallel == "heads":
                res = run_heads(args, rank, world, local)
            else:
                res = run_ours(args, rank, world, local)
        finally:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
