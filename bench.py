"""Benchmark of the MoE-layer forward on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                [--workload mixtral_bf16]

One step = one whole layer forward (route -> permute -> gate/up GEMM with fused gather and
SwiGLU -> down GEMM -> combine) over one batch of seeded synthetic input, through
moe_forward. Default workload: Mixtral-like, T=4096 d=4096 E=8 K=2 n=14336 bf16.
For N > 1 (torchrun, one rank per GPU) every rank runs an independent replica: the layer
shards by tokens with replicated weights and needs no collective; timing is the max over
ranks and `value` counts the tokens of all ranks (weak scaling).

--impl reference times the CPU oracle (numpy, fp64) as it stands on this host's cores, each
step a bounded sample of the same workload (a few tokens through the whole layer); rank 0
only.
"""
from __future__ import annotations

import argparse
import ctypes
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

METRIC = "MoE layer fwd tokens/s at 1 B200; dispatch+combine GB/s and GEMM % of peak"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
RECORDS_FILE = os.path.join(ROOT, "profiles", "records.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mixtral_bf16")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-tokens", type=int, default=0,
                    help="tokens in the CPU oracle sample (0: the workload's whole batch)")
    ap.add_argument("--ref-tokens", type=int, default=64,
                    help="tokens per step of the reference arm (the CPU oracle)")
    ap.add_argument("--ffn-variant", type=int, default=0, choices=[0, 1, 2, 3],
                    help="grouped-GEMM tile variant (moe_shape.ffn_variant): 0 automatic, 1 "
                         "single-CTA, 2 CTA pairs, 3 CTA pairs with the rows gathered first")
    ap.add_argument("--no-secondary", action="store_true",
                    help="only the layer forward, its roofline, dispatch + combine and e2e (no "
                         "decode, rounding, backward, atomic-expert or other-workload figures)")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the fine-grained and skewed workload figures")
    ap.add_argument("--only", choices=["atomic_experts", "backward", "dispatch", "decode",
                                       "rounding"],
                    default=None,
                    help="run one secondary figure alone and print it (for profiling)")
    return ap.parse_args()


# ------------------------------------------------------------------ distributed plumbing
def dist_init(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return rank, world, local  # rank 0 alone times the oracle; no process group
    if world > 1:
        import datetime
        backend = "nccl" if args.impl == "ours" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif args.impl == "ours":
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """The slowest rank's time: every rank's device-timed value, reduced with MAX."""
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64,
                     device="cuda" if torch.distributed.get_backend() == "nccl" else "cpu")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(tokens_per_rank: int, world: int, steps: int, ms_max: float) -> float:
    """Whole-job tokens/s: every rank processes its own batch of `tokens_per_rank` tokens per
    step (independent replicas), timed by the slowest rank."""
    return tokens_per_rank * world * steps / (ms_max / 1e3)


# ------------------------------------------------------------------ measurement helpers
def load_peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# Source file of each kernel a profiles/ record may describe; the shared headers count too
# (kernel_ids.h, the profiler's host-side kernel numbering, holds no device code).
KERNEL_SOURCES = {"gateup_tc": "ffn_tc.cu", "down_tc": "ffn_tc.cu", "gateup_tc2": "ffn_tc2.cu",
                  "down_tc2": "ffn_tc2.cu", "route_tc": "route_tc.cu", "combine": "combine.cu",
                  "gather_rows": "permute.cu", "permute_cluster": "permute.cu"}
KERNEL_HEADERS = ("common.cuh", "tc_ptx.cuh", "ffn_args.cuh")


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for name in (KERNEL_SOURCES.get(kernel, "ffn_tc.cu"),) + KERNEL_HEADERS:
        with open(os.path.join(ROOT, "token_dispatch_router_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """ncu DRAM bytes per launch for `kernel` from profiles/records.json, reported only if the
    record was taken on the current kernel source."""
    try:
        with open(RECORDS_FILE) as f:
            recs = json.load(f)["records"]
    except (OSError, ValueError, KeyError):
        return None
    want = kernel_source_hash(kernel)
    for r in recs:
        if r.get("workload") == workload and r.get("kernel") == kernel and \
                r.get("source_hash") == want:
            return int(r["bytes_per_launch"])
    return None


# ------------------------------------------------------------------ CPU oracle leg
def cpu_oracle_tokens_per_s(inp, n_tokens: int, start: int = 0, wide=None):
    """The oracle on a bounded sample: n_tokens tokens through the whole layer (router
    logits, softmax/top-k, counts/scan/permutation of the sample, expert FFNs, combine).
    Expert weights are widened to fp64 once (outside the timing) in `wide`."""
    from oracle import moe_oracle as orc
    cfg = inp.cfg
    if wide is None:
        wide = {}
    tok = (start + np.arange(n_tokens)) % cfg.T
    x = orc.as_f64(inp.x[torch.from_numpy(tok)])
    # widen the weights of the experts this sample uses, untimed
    lg0 = orc.router_logits(x, inp.w_r, None if inp.bias is None else inp.bias.numpy())
    for e in np.unique(orc.topk_ids(lg0, cfg.K)):
        if int(e) not in wide:
            wide[int(e)] = tuple(orc.as_f64(w[int(e)]) for w in (inp.w_gate, inp.w_up, inp.w_down))
    t0 = time.perf_counter()
    lg = orc.router_logits(x, inp.w_r, None if inp.bias is None else inp.bias.numpy())
    ids, w = orc.route(lg, cfg.K)
    C = orc.capacity(cfg.capacity_factor, n_tokens, cfg.K, cfg.E)
    _, offsets, a2p, p2a = orc.permute(ids, cfg.E, C)
    E = cfg.E
    wg = [wide.get(e, (None,) * 3)[0] for e in range(E)]
    wu = [wide.get(e, (None,) * 3)[1] for e in range(E)]
    wd = [wide.get(e, (None,) * 3)[2] for e in range(E)]
    off = np.asarray(offsets)
    y = np.zeros((int(off[-1]), cfg.d))
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi > lo:
            rows = x[np.asarray(p2a[lo:hi]) // cfg.K]
            y[lo:hi] = orc.expert_ffn(rows, wg[e], wu[e], wd[e])
    orc.combine(y, a2p, w, n_tokens, cfg.K)
    dt = time.perf_counter() - t0
    return n_tokens / dt, dt, wide


def cpu_oracle_figures(inp, wide, R: int = 128, n_tok: int = 256, n_omni: int = 16) -> dict:
    """The oracle, as it stands, on bounded samples of each secondary figure's work (timed on
    the host beside the GPU figures): the token-rounded layer and the layer's backward on an
    n_tok-token batch of the bench workload, the dispatch/combine-only pipeline at its decode
    sizes, and n_omni tokens of the atomic-expert layer. Expert weights are the fp64 copies
    the CPU baseline made (untimed)."""
    from oracle import moe_oracle as orc
    from oracle import omni_oracle as oo
    cfg = inp.cfg
    res = {}
    E = cfg.E
    class _Experts:  # the per-expert fp64 matrices, indexable like the stacked tensor
        def __init__(self, mats):
            self.mats = mats
            self.shape = (len(mats),) + tuple(mats[0].shape)

        def __getitem__(self, e):
            return self.mats[e]

    wg = _Experts([wide[e][0] if e in wide else orc.as_f64(inp.w_gate[e]) for e in range(E)])
    wu = _Experts([wide[e][1] if e in wide else orc.as_f64(inp.w_up[e]) for e in range(E)])
    wd = _Experts([wide[e][2] if e in wide else orc.as_f64(inp.w_down[e]) for e in range(E)])
    x = orc.as_f64(inp.x[:n_tok])
    bias = None if inp.bias is None else inp.bias.numpy()
    if cfg.capacity_factor <= 0:
        t0 = time.perf_counter()
        orc.forward(x, inp.w_r, wg, wu, wd, cfg.K, bias=bias, tile_round=R)
        dt = time.perf_counter() - t0
        res["token_rounding"] = {"tokens_per_s": n_tok / dt, "sample": f"{n_tok} tokens, R={R}"}
    # backward: forward pieces untimed, then the oracle's backward of the expert half + router
    f = orc.forward(x, inp.w_r, wg, wu, wd, cfg.K, capacity_factor=cfg.capacity_factor, bias=bias)
    g, u = orc.gate_up_preact(x, f["perm_to_assign"], f["offsets"], cfg.K, wg, wu)
    d_out = np.random.default_rng(0).standard_normal((n_tok, cfg.d))
    t0 = time.perf_counter()
    dG, dU, d_w = orc.backward_act(d_out, f["topk_w"], f["assign_to_perm"], f["perm_to_assign"],
                                   f["offsets"], cfg.K, wd, g, u)
    orc.backward_dx(dG, dU, f["assign_to_perm"], f["perm_to_assign"], f["offsets"], cfg.K, n_tok,
                    wg, wu)
    orc.backward_router(d_w, f["topk_ids"], f["logits"], x, inp.w_r)
    dt = time.perf_counter() - t0
    res["backward_act"] = {"tokens_per_s": n_tok / dt, "sample": f"{n_tok} tokens"}
    # dispatch / combine only (given logits, identity experts), the decode sizes
    dcfg = mi.DISPATCH_COMBINE
    dd = {}
    for T in (64, 1024):
        di = mi.make_inputs(dcfg.with_T(T))
        lg = di.logits.numpy()
        xd = orc.as_f64(di.x)
        t0 = time.perf_counter()
        ids, w = orc.route(lg, dcfg.K)
        _, offs, a2p, p2a = orc.permute(ids, dcfg.E)
        xp = orc.gather_rows(xd, p2a, offs, dcfg.K)
        orc.combine(xp, a2p, w, T, dcfg.K)
        dd[f"T={T}"] = round((time.perf_counter() - t0) * 1e6, 1)
    res["decode_dispatch"] = {"us": dd, "sample": "route + permute + gather + combine"}
    # atomic experts: routing over the whole grid and the outputs of n_omni tokens
    oc = mi.OMNI_102K
    oi = mi.make_omni_inputs(oc)
    toks = np.arange(n_omni)
    t0 = time.perf_counter()
    lg = oo.cartesian_logits(oi.x[:n_omni], oi.w_row, oi.w_col)
    ids, w = oo.cartesian_route(lg, oc.n_rows, oc.K)
    oo.token_outputs(oi.x[:n_omni], oi.w_in, oi.w_out, ids, w)
    dt = time.perf_counter() - t0
    res["atomic_experts"] = {"tokens_per_s": n_omni / dt, "sample": f"{n_omni} tokens of omni_102k"}
    res["cores"] = cpu_cores()
    return res


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ------------------------------------------------------------------ reference arm
def run_reference(args, rank, world):
    if rank != 0:
        return
    cfg = mi.CONFIGS[args.workload]
    inp = mi.make_inputs(cfg)
    wide = {}
    per_step = max(1, args.ref_tokens)
    for i in range(args.warmup):
        cpu_oracle_tokens_per_s(inp, per_step, start=i * per_step, wide=wide)
    total_t, total_tok = 0.0, 0
    for i in range(args.steps):
        _, dt, wide = cpu_oracle_tokens_per_s(inp, per_step, start=(args.warmup + i) * per_step,
                                              wide=wide)
        total_t += dt
        total_tok += per_step
    value = total_tok / total_t
    sample = f"{per_step} tokens per step through the whole layer (oracle, fp64)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_t / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "T": cfg.T, "d": cfg.d, "E": cfg.E, "K": cfg.K,
                   "n": cfg.n},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_cores(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ dispatch + combine
def hold_gpu(us: float = 200.0):
    """Keep the GPU busy for `us` microseconds so that the host has queued the next timed
    sequence before the GPU reaches it (the timed region then holds no host time)."""
    sleep = getattr(torch.cuda, "_sleep", None)
    if sleep is not None:
        sleep(int(us * 2000))  # cycles at about 2 GHz


def dispatch_combine_bytes(cfg) -> int:
    """Algorithmic bytes of route + permute (gathered rows materialised) + combine:
    route reads x and writes logits, ids and weights; permute reads ids and writes both
    index maps, reads x and writes x_perm; combine reads x_perm, ids/weights and writes out."""
    b = 2 if cfg.dtype == "bf16" else 4
    T, d, E, K = cfg.T, cfg.d, cfg.E, cfg.K
    A = T * K
    route = T * d * b + d * E * b + T * E * 4 + T * K * 8
    permute = A * 4 + A * 8 + E * 8 + T * d * b + A * d * b
    combine = A * d * b + A * 8 + T * d * b
    return route + permute + combine


def dispatch_combine(tdr, s, cfg, x, w_r, bias, steps, world, peaks):
    """Time route -> permute (x_perm) -> combine(x_perm) at the layer's shape."""
    dev = x.device
    T, d, E, K = cfg.T, cfg.d, cfg.E, cfg.K
    ids = torch.empty(T, K, dtype=torch.int32, device=dev)
    w = torch.empty(T, K, dtype=torch.float32, device=dev)
    lo = torch.empty(T, E, dtype=torch.float32, device=dev)
    pws = torch.empty(max(tdr.permute_workspace_size(s), 256), dtype=torch.uint8, device=dev)
    out = torch.empty(T, d, dtype=x.dtype, device=dev)

    def once():
        tdr.route(s, x, w_r, bias=bias, logits_out=lo, topk_ids=ids, topk_w=w)
        p = tdr.permute(s, ids, x=x, materialize=True, workspace=pws)
        tdr.combine(s, p["x_perm"], p["assign_to_perm"], w, out=out)

    # L2 flush by reading 512 MB (> 126 MB of L2): leaves only clean lines, so no write-back
    # of the flush itself lands in the timed sequence, and gives the host time to queue the
    # sequence's launches before the GPU reaches them
    flush = torch.ones(64 << 20, dtype=torch.int64, device=dev)
    for _ in range(3):
        once()
    torch.cuda.synchronize()
    n = max(10, min(steps, 100))
    # one sequence per flushed iteration, CUDA events around it (device launch gaps included)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n)]
    for a, b in ev:
        flush.sum()
        hold_gpu()
        a.record()
        once()
        b.record()
    torch.cuda.synchronize()
    seq = sorted(a.elapsed_time(b) for a, b in ev)
    ms = max_over_ranks(sum(seq) / n, world)  # the mean is the headline figure
    ms_median = max_over_ranks(statistics.median(seq), world)
    ms_min = max_over_ranks(seq[0], world)
    # the same sequence back to back with warm L2 (reported beside it)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n):
        once()
    e1.record()
    torch.cuda.synchronize()
    ms_warm = max_over_ranks(e0.elapsed_time(e1) / n, world)
    del flush
    # per-kernel breakdown from a separate pass with the library's event profiler
    prof = tdr.Profiler()
    with prof:
        for _ in range(n):
            once()
        torch.cuda.synchronize()
    kern = {k: round(v[1] / n, 4) for k, v in prof.results().items()}
    nbytes = dispatch_combine_bytes(cfg)
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"bytes": nbytes, "ms": round(ms, 4), "achieved_gbs": round(gbs, 1), "peak_gbs": peak,
            "frac": round(gbs / peak, 4), "ms_median": round(ms_median, 4),
            "ms_min": round(ms_min, 4), "ms_back_to_back": round(ms_warm, 4),
            "kernels_ms_with_events": kern,
            "note": "route + permute with x_perm materialised + combine(x_perm) at the layer's "
                    "shape; GB/s = algorithmic bytes over the device time of one sequence after "
                    "an L2 flush (launch gaps inside the sequence included)"}


def decode_dispatch(tdr, world, Ts=(64, 256, 512, 1024)):
    """Dispatch workload (given N(0,1) logits, E=64 K=6 d=4096 bf16) in the decode regime:
    route + permute with x_perm materialised + combine of those rows, per L2-flushed
    sequence with CUDA events around it, through the two calls (moe_route, moe_permute) and
    through moe_dispatch (the same kernels from one call) with either top-K form."""
    base = mi.CONFIGS["dispatch_combine"]
    dev = torch.device("cuda", torch.cuda.current_device())
    flush = torch.ones(64 << 20, dtype=torch.int64, device=dev)
    res = {}
    for T in Ts:
        cfg = base.with_T(T)
        inp = mi.make_inputs(cfg)
        x, lg = inp.x.to(dev), inp.logits.to(dev)
        shapes = {f: tdr.make_shape(T, cfg.d, cfg.E, cfg.K, 64, 0.0, True, torch.bfloat16,
                                    route_topk=f) for f in (1, 2)}
        s = shapes[1]
        pws = torch.empty(max(tdr.permute_workspace_size(s), 256), dtype=torch.uint8, device=dev)
        out = torch.empty(T, cfg.d, dtype=x.dtype, device=dev)
        bufs = {}

        def two_calls():
            ids, w, _ = tdr.route(s, logits_in=lg)
            p = tdr.permute(s, ids, x=x, materialize=True, workspace=pws)
            tdr.combine(s, p["x_perm"], p["assign_to_perm"], w, out=out)

        def one_call(form):
            def fn():
                r = tdr.dispatch(shapes[form], x=x, logits_in=lg, materialize=True,
                                 workspace=pws, out=bufs)
                bufs.update(r)
                tdr.combine(s, r["x_perm"], r["assign_to_perm"], r["topk_w"], out=out)
            return fn

        variants = (("two_calls_us", two_calls), ("dispatch_rounds_us", one_call(1)),
                    ("dispatch_bitonic_us", one_call(2)))
        for _, fn in variants:
            for _ in range(3):
                fn()
        torch.cuda.synchronize()
        # blocks of 10 flushed sequences, the variants interleaved block by block (the clock
        # drifts), the median of every variant's sequences
        times = {name: [] for name, _ in variants}
        for _ in range(5):
            for name, fn in variants:
                ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                      for _ in range(10)]
                for a, b in ev:
                    flush.sum()
                    hold_gpu()
                    a.record()
                    fn()
                    b.record()
                torch.cuda.synchronize()
                times[name] += [a.elapsed_time(b) for a, b in ev]
        row = {name: round(1e3 * max_over_ranks(statistics.median(v), world), 2)
               for name, v in times.items()}
        res[f"T={T}"] = row
    del flush
    # route + permute with x_perm + combine, one sequence per L2-flushed iteration, CUDA
    # events, launch gaps included; moe_dispatch with either top-K form of the router
    return {"workload": "dispatch_combine (E=64 K=6 d=4096 bf16, given logits)", "latency": res}


def token_rounding_figure(tdr, cfg, x, w_r, wg, wu, wd, bias, world, R=128, rounds=5, per=10):
    """The layer with tile-aware token rounding to whole R-row tiles, in each direction (down:
    an expert's weakest assignments dropped; up: the strongest tokens that did not route to it
    added; nearest: whichever is closer), against the plain layer: blocks of `per` steps
    alternate between the four `rounds` times (the power-capped clock drifts), CUDA events;
    reports each step time, the rows each expert-major list holds (kept plus added) and the
    128-row tile rows the gate/up GEMM computes in each case."""
    if cfg.capacity_factor > 0:
        return None
    dev = x.device
    dt = x.dtype
    out = torch.empty(cfg.T, cfg.d, dtype=dt, device=dev)
    shapes = {"plain": tdr.make_shape(cfg.T, cfg.d, cfg.E, cfg.K, cfg.n, 0.0, True, dt),
              "down": tdr.make_shape(cfg.T, cfg.d, cfg.E, cfg.K, cfg.n, 0.0, True, dt,
                                     tile_round=R),
              "up": tdr.make_shape(cfg.T, cfg.d, cfg.E, cfg.K, cfg.n, 0.0, True, dt,
                                   tile_round=R, tile_round_mode=1),
              "nearest": tdr.make_shape(cfg.T, cfg.d, cfg.E, cfg.K, cfg.n, 0.0, True, dt,
                                        tile_round=R, tile_round_mode=2)}
    wss = {k: torch.empty(tdr.forward_workspace_size(v), dtype=torch.uint8, device=dev)
           for k, v in shapes.items()}
    ms = {k: 0.0 for k in shapes}
    for k in shapes:
        for _ in range(3):
            tdr.forward(shapes[k], x, w_r, wg, wu, wd, bias=bias, out=out, workspace=wss[k])
    torch.cuda.synchronize()
    for _ in range(rounds):
        for k in shapes:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(per):
                tdr.forward(shapes[k], x, w_r, wg, wu, wd, bias=bias, out=out, workspace=wss[k])
            e1.record()
            torch.cuda.synchronize()
            ms[k] += e0.elapsed_time(e1)
    kern = {}
    for k in shapes:  # per-kernel device time, a separate pass under the event profiler
        prof = tdr.Profiler()
        with prof:
            for _ in range(per):
                tdr.forward(shapes[k], x, w_r, wg, wu, wd, bias=bias, out=out, workspace=wss[k])
            torch.cuda.synchronize()
        kern[k] = {n: round(v[1] / per * 1e3, 1) for n, v in prof.results().items()}
    if tdr.device_status() != 0:
        raise RuntimeError("device status set during the token-rounding runs")
    res = {}
    for k in shapes:
        step = max_over_ranks(ms[k] / (rounds * per), world)
        offs = tdr.workspace_views(shapes[k], wss[k])["offsets"].cpu().numpy()
        kept = np.diff(offs)
        res[k] = {"ms_per_step": round(step, 4),
                  "tokens_per_s": cfg.T * world / (step / 1e3),
                  "kept_assignments": int(offs[-1]),
                  "gemm_tile_rows": int(sum(-(-int(c) // 128) * 128 for c in kept)),
                  "kernels_us": kern[k]}
    res["R"] = R
    for k in ("down", "up", "nearest"):
        res[k]["row_share"] = round(res[k]["kept_assignments"] / (cfg.T * cfg.K), 4)
        res[k]["speedup"] = round(res["plain"]["ms_per_step"] / res[k]["ms_per_step"], 4)
    res["note"] = ("each a different layer output: dropped assignments add nothing, added ones "
                   "add their weighted expert output; same weights, inputs and kernels otherwise")
    return res


def backward_figure(tdr, cfg, s, x, w_r, wg, wu, wd, bias, world, peak_t, steps=20):
    """The layer's backward at its shape, after a moe_forward_h: moe_backward with the input
    gradient, then moe_backward_router (its term added to d_x); CUDA events over `steps`
    calls, per-kernel times from the library's event profiler."""
    if cfg.dtype != "bf16":
        return None
    dev = x.device
    out, ws, h = tdr.forward_h(s, x, w_r, wg, wu, wd, bias=bias)
    v = tdr.workspace_views(s, ws)
    d_out = torch.randn(cfg.T, cfg.d, dtype=torch.bfloat16, device=dev,
                        generator=torch.Generator(device=dev).manual_seed(0))
    d_h = torch.empty_like(h)
    d_w = torch.empty(cfg.T, cfg.K, dtype=torch.float32, device=dev)
    bws = torch.empty(max(int(tdr.load_library().moe_backward_workspace_size(
        ctypes.byref(s))), 256), dtype=torch.uint8, device=dev)

    d_x = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16, device=dev)

    def call():
        tdr.backward(s, d_out, v["topk_w"], v["offsets"], v["perm_to_assign"],
                     v["assign_to_perm"], wd, h, w_gate=wg, w_up=wu, d_h=d_h, d_w=d_w, d_x=d_x,
                     input_grad=True, workspace=bws)

    def call_all():
        call()
        tdr.backward_router(s, x, w_r, v["topk_ids"], v["topk_w"], d_w, logits=v["logits"],
                            d_x=d_x, with_bias=bias is not None)

    for _ in range(3):
        call_all()
    torch.cuda.synchronize()
    prof = tdr.Profiler()
    with prof:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            call_all()
        e1.record()
        torch.cuda.synchronize()
    if tdr.device_status() != 0:
        raise RuntimeError("device status set during the backward runs")
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    k = prof.results()
    a_kept = int(v["offsets"][cfg.E].item())
    flops = 2.0 * cfg.d * cfg.n * a_kept
    def avg(name):
        c, t = k.get(name, (0, 0.0))
        return t / max(c, 1)

    act_ms, dx_ms = avg("bwd_act"), avg("bwd_dx")
    tf_act = flops / (act_ms / 1e3) / 1e12 if act_ms > 0 else 0.0
    tf_dx = 2 * flops / (dx_ms / 1e3) / 1e12 if dx_ms > 0 else 0.0
    return {"ms_per_call": round(ms, 4),
            "dact_gemm_ms": round(act_ms, 4), "dact_tflops": round(tf_act, 2),
            "dact_frac_of_sustained_peak": round(tf_act / peak_t, 4),
            "dx_gemm_ms": round(dx_ms, 4), "dx_tflops": round(tf_dx, 2),
            "dx_frac_of_sustained_peak": round(tf_dx / peak_t, 4),
            "dw_ms": round(avg("bwd_dw"), 4), "scatter_add_ms": round(avg("combine"), 4),
            "router_ms": {"d_logits": round(avg("router_dlogits"), 4),
                          "d_w_r_and_bias": round(avg("router_dwr"), 4),
                          "d_x_term": round(avg("router_dx"), 4)},
            "note": "dA' = dO W_down^T (dO rows by token: copied expert-major first when "
                    "n >= 4096, else gathered in the GEMM; dS and the SwiGLU backward in the "
                    "epilogue: reads h, writes d_h), d_w reduction, dX_perm = (dG|dU) "
                    "(W_gate|W_up)^T, scatter-add to tokens, router backward (d_logits, "
                    "d_W_r, d_bias, its d_x term); TFLOP/s on 2*d*n (dA') and 4*d*n (dX) per "
                    "kept slot"}


def workload_figure(tdr, name, world, peak_t, steps=20):
    """The layer forward at one of the other bf16 workloads (fine-grained: 128 small uneven
    experts; skewed: Zipf-biased routing with a capacity limit): `steps` forwards back to back
    (their weights, 1.2-1.6 GB, stream from HBM every step), CUDA events, per-kernel times from
    the library's event profiler. Reports the grouped GEMMs against the sustained bf16 peak on
    algorithmic FLOPs (kept rows only), the share of gate/up tile rows that is padding, and
    the share of the step spent routing and permuting."""
    cfg = mi.CONFIGS[name]
    inp = mi.make_inputs(cfg)
    dev = torch.device("cuda", torch.cuda.current_device())
    x, w_r = inp.x.to(dev), inp.w_r.to(dev)
    wg, wu, wd = inp.w_gate.to(dev), inp.w_up.to(dev), inp.w_down.to(dev)
    bias = None if inp.bias is None else inp.bias.to(dev)
    del inp
    s = tdr.make_shape(cfg.T, cfg.d, cfg.E, cfg.K, cfg.n, cfg.capacity_factor, True,
                       torch.bfloat16)
    ws = torch.empty(tdr.forward_workspace_size(s), dtype=torch.uint8, device=dev)
    out = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16, device=dev)

    def step():
        tdr.forward(s, x, w_r, wg, wu, wd, bias=bias, out=out, workspace=ws)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    prof = tdr.Profiler()
    with prof:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            step()
        e1.record()
        torch.cuda.synchronize()
    if tdr.device_status() != 0:
        raise RuntimeError(f"device status set during the {name} runs")
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    kern = prof.results()
    offs = tdr.workspace_views(s, ws)["offsets"].cpu().numpy()
    kept = np.diff(offs)
    a_kept = int(offs[-1])
    tile_rows = int(sum(-(-int(c) // 128) * 128 for c in kept))

    def avg(*names):
        return sum(kern.get(k, (0, 0.0))[1] for k in names) / steps

    g_ms = avg("gateup_tc", "gateup_tc2")
    d_ms = avg("down_tc", "down_tc2")
    fg, fd = 4.0 * cfg.d * cfg.n * a_kept, 2.0 * cfg.d * cfg.n * a_kept
    tg = fg / (g_ms / 1e3) / 1e12 if g_ms > 0 else 0.0
    td = fd / (d_ms / 1e3) / 1e12 if d_ms > 0 else 0.0
    rp = avg("route_tc", "route", "permute_small", "permute_cluster", "hist", "scan", "scatter")
    del x, wg, wu, wd, ws
    torch.cuda.empty_cache()
    return {"ms": round(ms, 4), "tok_s": round(cfg.T * world / (ms / 1e3)),
            "gateup_ms": round(g_ms, 4), "gateup_tflops": round(tg, 1),
            "gateup_frac": round(tg / peak_t, 4), "down_ms": round(d_ms, 4),
            "down_tflops": round(td, 1), "down_frac": round(td / peak_t, 4),
            "kept": a_kept, "pad_share": round(1.0 - a_kept / max(tile_rows, 1), 4),
            "route_ms": round(avg("route_tc", "route"), 4),
            "route_permute_share": round(rp / ms, 4), "combine_ms": round(avg("combine"), 4)}


# ------------------------------------------------------------------ our arm
def atomic_experts_bytes(c) -> dict:
    """Algorithmic HBM bytes of one atomic-expert forward (each tensor read or written once)
    and the row gathers its two expert kernels make (one d-row per task and side)."""
    T, d, K, N, P = c.T, c.d, c.K, c.N, c.n_rows + c.n_cols
    M = T * K
    hbm = (T * d * 2 + d * P * 2          # x, the two router tables
           + 2 * T * P * 4                # logits written, read by the top-K
           + 2 * M * 4 + 2 * M * 4        # ids and weights written; ids read by the schedule
           + N * 4 * 2 + (N + 1) * 4 + 2 * M * 4  # counts, offsets, both task maps
           + N * d * 2 + M * 4 * 3        # w_in once; task map, weights, scalars (act)
           + N * d * 2 + M * 8 + T * d * 2)  # w_out once, ids and scalars, out (gather)
    return {"hbm_bytes": int(hbm), "row_gather_bytes": int(2 * M * d * 2)}


def atomic_experts_figure(tdr, world, peaks, n=10):
    """Fine-grained (rank-1) experts behind a Cartesian-product router: the 4096-token layer
    with 320 x 320 = 102,400 experts, K = 512, d = 1024, through moe_omni_forward. One
    forward per L2 flush, CUDA events; per-kernel times from the library's event profiler."""
    c = mi.OMNI_102K
    inp = mi.make_omni_inputs(c)
    s = tdr.make_omni_shape(c.T, c.d, c.n_rows, c.n_cols, c.K, c.renormalize)
    x, wr, wc, wi, wo = (t.cuda() for t in (inp.x, inp.w_row, inp.w_col, inp.w_in, inp.w_out))
    ws = torch.empty(tdr.omni_workspace_size(s), dtype=torch.uint8, device=x.device)
    out = torch.empty(c.T, c.d, dtype=torch.bfloat16, device=x.device)

    def once():
        tdr.omni_forward(s, x, wr, wc, wi, wo, out=out, workspace=ws)

    flush = torch.ones(64 << 20, dtype=torch.int64, device=x.device)
    for _ in range(3):
        once()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n)]
    for a, b in ev:
        flush.sum()
        hold_gpu()
        a.record()
        once()
        b.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev) / n, world)
    del flush
    prof = tdr.Profiler()
    with prof:
        for _ in range(n):
            once()
        torch.cuda.synchronize()
    if tdr.device_status() != 0:
        raise RuntimeError("device status set during the atomic-expert runs")
    kern = {k: round(v[1] / n * 1e3, 1) for k, v in prof.results().items()}
    # the page's output side for comparison: expert-centric scatter-add (atomic fp32 rows)
    s_sc = tdr.make_omni_shape(c.T, c.d, c.n_rows, c.n_cols, c.K, c.renormalize, output_mode=1)

    def once_scatter():
        tdr.omni_forward(s_sc, x, wr, wc, wi, wo, out=out, workspace=ws)

    for _ in range(2):
        once_scatter()
    torch.cuda.synchronize()
    prof2 = tdr.Profiler()
    with prof2:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            once_scatter()
        e1.record()
        torch.cuda.synchronize()
    scatter = {"ms_back_to_back": round(max_over_ranks(e0.elapsed_time(e1) / n, world), 4),
               "output_us": round(prof2.results()["omni_out"][1] / n * 1e3, 1)}
    counts = tdr.omni_workspace_views(s, ws)["counts"]
    active = int((counts > 0).sum().item())
    nb = atomic_experts_bytes(c)
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    gbs = nb["hbm_bytes"] / (ms / 1e3) / 1e9
    half = nb["row_gather_bytes"] / 2
    gather = {k: round(half / (kern[k] / 1e6) / 1e12, 2) for k in ("omni_act", "omni_out")
              if k in kern}
    return {"workload": c.name, "T": c.T, "d": c.d, "grid": [c.n_rows, c.n_cols], "N": c.N,
            "K": c.K, "ms": round(ms, 4), "tokens_per_s": c.T * world / (ms / 1e3),
            "kernels_us": kern, "hbm_bytes": nb["hbm_bytes"], "hbm_gbs": round(gbs, 1),
            "hbm_frac": round(gbs / peak, 4), "row_gather_bytes": nb["row_gather_bytes"],
            "row_gather_tbs": gather, "scatter_add_output": scatter, "active_experts": active,
            "reuse_tasks_per_active_expert": round(c.T * c.K / max(active, 1), 2),
            "note": "one forward per L2 flush (expert tables 420 MB > L2); hbm_frac counts each "
                    "tensor once; the expert kernels are bound by 2 KB row gathers "
                    "(row_gather_tbs: TB/s of rows moved per kernel); scatter_add_output: the "
                    "same forward with the expert-centric scatter-add on the output side "
                    "(zero, atomic fp32 rows, bf16 rounding), back to back"}


def run_ours(args, rank, world, local):
    import token_dispatch_router_b200 as tdr
    tdr.load_library()  # fails loudly if the CUDA library is missing
    if args.only == "atomic_experts":
        fig = atomic_experts_figure(tdr, world, load_peaks()[0], n=max(1, args.steps))
        if rank == 0:
            print(json.dumps({"atomic_experts": fig}), flush=True)
        return
    cfg = mi.CONFIGS[args.workload]
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    if args.only == "decode":  # the decode-regime dispatch latencies alone
        a = torch.randn(4096, 4096, device="cuda", dtype=torch.bfloat16)
        t_end = time.time() + 0.5  # bring the clocks up first
        while time.time() < t_end:
            a @ a
        torch.cuda.synchronize()
        del a
        dd = decode_dispatch(tdr, world)
        if rank == 0:
            print(json.dumps({"decode_dispatch": dd}), flush=True)
        return
    if args.only == "dispatch":  # the dispatch + combine sequence alone (no expert weights)
        inp = mi.make_inputs(cfg, with_experts=False)
        dev = torch.device("cuda", torch.cuda.current_device())
        x, w_r = inp.x.to(dev), inp.w_r.to(dev)
        bias = None if inp.bias is None else inp.bias.to(dev)
        s = tdr.make_shape(cfg.T, cfg.d, cfg.E, cfg.K, cfg.n, cfg.capacity_factor, True, dt)
        with ClockSampler(local) as dc_clocks:
            dc = dispatch_combine(tdr, s, cfg, x, w_r, bias, args.steps, world, load_peaks()[0])
        dc["clocks"] = dc_clocks.summary()
        if rank == 0:
            print(json.dumps({"dispatch_combine": dc}), flush=True)
        return
    inp = mi.make_inputs(cfg)
    dev = torch.device("cuda", torch.cuda.current_device())
    x = inp.x.to(dev)
    w_r = inp.w_r.to(dev)
    wg, wu, wd = inp.w_gate.to(dev), inp.w_up.to(dev), inp.w_down.to(dev)
    bias = None if inp.bias is None else inp.bias.to(dev)
    s = tdr.make_shape(cfg.T, cfg.d, cfg.E, cfg.K, cfg.n, cfg.capacity_factor, True, dt,
                       ffn_variant=args.ffn_variant)
    ws = torch.empty(tdr.forward_workspace_size(s), dtype=torch.uint8, device=dev)
    out = torch.empty(cfg.T, cfg.d, dtype=dt, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        tdr.forward(s, x, w_r, wg, wu, wd, bias=bias, out=out, workspace=ws)

    if args.only == "rounding":
        fig = token_rounding_figure(tdr, cfg, x, w_r, wg, wu, wd, bias, world)
        if rank == 0:
            print(json.dumps({"token_rounding": fig}), flush=True)
        return
    if args.only == "backward":
        peaks = load_peaks()[0]
        peak_t = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
        fig = backward_figure(tdr, cfg, s, x, w_r, wg, wu, wd, bias, world, peak_t,
                              steps=max(1, args.steps))
        if rank == 0:
            print(json.dumps({"backward_act": fig}), flush=True)
        return

    # ---- dispatch + combine byte stream at the layer's shape (route, permute with the
    # gathered rows materialised, combine of those rows as identity experts): measured first,
    # on its own, before the GEMM-bound steps heat the GPU into its power cap, with its own
    # clock record
    peaks = load_peaks()[0]
    with ClockSampler(local) as dc_clocks:
        dc = dispatch_combine(tdr, s, cfg, x, w_r, bias, args.steps, world, peaks)
    dc["clocks"] = dc_clocks.summary()

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if tdr.device_status() != 0:
        raise RuntimeError("device status set during warm-up")

    # ---- timed region: K whole-layer steps, per-kernel events recorded by the library
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = tdr.launch_count()
    prof = tdr.Profiler()
    with ClockSampler(local) as clocks:
        barrier(world)
        torch.cuda.synchronize()
        with prof:
            ev0.record(stream)
            for _ in range(args.steps):
                step()
            ev1.record(stream)
            torch.cuda.synchronize()
        barrier(world)
    launches = tdr.launch_count() - launches0
    ms_total = ev0.elapsed_time(ev1)
    ms_total = max_over_ranks(ms_total, world)
    ms_step = ms_total / args.steps
    value = weak_scaling_value(cfg.T, world, args.steps, ms_total)
    kern = prof.results()
    if tdr.device_status() != 0:
        raise RuntimeError("device status set during the timed region")

    # ---- roofline of the dominant kernel (gate/up grouped GEMM, tensor cores)
    v = tdr.workspace_views(s, ws)
    a_kept = int(v["offsets"][cfg.E].item())
    peaks, peak_src = load_peaks()
    flops_gateup = 4.0 * cfg.d * cfg.n * a_kept
    flops_down = 2.0 * cfg.d * cfg.n * a_kept
    # the grouped GEMMs run as single-CTA (`*_tc`) or CTA-pair (`*_tc2`) kernels
    g_name = "gateup_tc2" if "gateup_tc2" in kern else "gateup_tc"
    d_name = "down_tc2" if "down_tc2" in kern else "down_tc"
    n_g, ms_g = kern.get(g_name, (0, 0.0))
    n_d, ms_d = kern.get(d_name, (0, 0.0))
    avg_g = ms_g / max(n_g, 1)
    avg_d = ms_d / max(n_d, 1)
    peak_t = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    ach_g = flops_gateup / (avg_g / 1e3) / 1e12 if avg_g > 0 else 0.0
    ach_d = flops_down / (avg_d / 1e3) / 1e12 if avg_d > 0 else 0.0
    ach_gemm = (flops_gateup + flops_down) / ((avg_g + avg_d) / 1e3) / 1e12 if avg_g > 0 else 0.0
    roofline = {"bound": "tensor", "kernel": g_name, "achieved": round(ach_g, 2),
                "peak": peak_t, "unit": "TFLOP/s", "frac": round(ach_g / peak_t, 4),
                "traffic": traffic_for(g_name, cfg.name),
                "peak_source": f"{peak_src} sustained bf16",
                "flop_per_launch": flops_gateup, "avg_launch_ms": round(avg_g, 4)}

    # ---- end to end through the public API with host buffers: every step uploads its input
    # from pinned host memory and downloads its output. Uploads and downloads run on their
    # own streams, double-buffered, so step i+1's upload and step i-1's download overlap
    # step i's layer forward (the way a serving loop would drive the library).
    e2e_steps = max(3, min(args.steps, 50))
    x_host = inp.x.pin_memory()
    out_host = [torch.empty(cfg.T, cfg.d, dtype=dt).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(x) for _ in range(2)]
    o_dev = [torch.empty_like(out) for _ in range(2)]
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    free = [torch.cuda.Event() for _ in range(2)]   # buffers b reusable
    up = [torch.cuda.Event() for _ in range(2)]     # input b uploaded
    done = [torch.cuda.Event() for _ in range(2)]   # output b computed
    for b in range(2):
        free[b].record(stream)

    def e2e_run(n):
        for i in range(n):
            b = i % 2
            h2d.wait_event(free[b])
            with torch.cuda.stream(h2d):
                x_dev[b].copy_(x_host, non_blocking=True)
                up[b].record(h2d)
            stream.wait_event(up[b])
            tdr.forward(s, x_dev[b], w_r, wg, wu, wd, bias=bias, out=o_dev[b], workspace=ws)
            done[b].record(stream)
            d2h.wait_event(done[b])
            with torch.cuda.stream(d2h):
                out_host[b].copy_(o_dev[b], non_blocking=True)
                free[b].record(d2h)
        stream.wait_stream(d2h)

    e2e_run(2)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d.wait_stream(stream)
    d2h.wait_stream(stream)
    e2e_run(e2e_steps)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    assert torch.equal(out_host[(e2e_steps - 1) % 2], out.cpu()), "e2e output differs"
    elem = 2 if dt == torch.bfloat16 else 4
    # public API (token_dispatch_router_b200.forward); pinned host input uploaded and output
    # downloaded every step on separate streams, double-buffered
    e2e = {"value": round(cfg.T * world * e2e_steps / (e2e_ms / 1e3), 1), "unit": "tokens/s",
           "h2d_bytes_per_step": cfg.T * cfg.d * elem, "d2h_bytes_per_step": cfg.T * cfg.d * elem,
           "steps": e2e_steps}

    # ---- dispatch + combine byte stream at the same shape (route, permute with the gathered
    # rows materialised, combine of those rows as identity experts): the unfused traffic
    dd = tr = bw = ae = None
    if not args.no_secondary:
        dd = decode_dispatch(tdr, world)
        tr = token_rounding_figure(tdr, cfg, x, w_r, wg, wu, wd, bias, world)
        bw = backward_figure(tdr, cfg, s, x, w_r, wg, wu, wd, bias, world, peak_t)
        ae = atomic_experts_figure(tdr, world, peaks)

    wl = {}
    if cfg.name == "mixtral_bf16" and not (args.no_workloads or args.no_secondary):
        for other in ("fine_grained_bf16", "skewed_capacity_bf16"):
            wl[other] = workload_figure(tdr, other, world, peak_t)

    weights_gb = 3 * cfg.E * cfg.d * cfg.n * (2 if dt == torch.bfloat16 else 4) / 1e9
    per_kernel = {k: round(ms / args.steps, 4) for k, (n, ms) in kern.items()}
    # One compact JSON line (no spaces, short keys, no prose): the driver keeps the last few
    # thousand characters of the output, so the headline figures come last.
    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16"
        if dt == torch.bfloat16 else "f32", "data": "synthetic",
        "config": {"workload": cfg.name, "T": cfg.T, "d": cfg.d, "E": cfg.E, "K": cfg.K,
                   "n": cfg.n, "global_batch": cfg.T * world, "parallelism": f"replicas{world}",
                   "ffn_variant": args.ffn_variant,
                   "l2": f"{weights_gb:.2f} GB of weights stream each step (> L2)"},
    }
    if bw:
        result["backward"] = {"ms": bw["ms_per_call"], "dact_ms": bw["dact_gemm_ms"],
                              "dact_frac": bw["dact_frac_of_sustained_peak"],
                              "dx_ms": bw["dx_gemm_ms"], "dx_frac": bw["dx_frac_of_sustained_peak"],
                              "router_ms": round(sum(bw["router_ms"].values()), 4)}
    if ae:
        ku = ae["kernels_us"]
        result["atomic_experts"] = {"workload": ae["workload"], "ms": ae["ms"],
                                    "tok_s": round(ae["tokens_per_s"]), "hbm_frac": ae["hbm_frac"],
                                    "topk_us": ku.get("omni_topk"), "act_us": ku.get("omni_act"),
                                    "out_us": ku.get("omni_out"),
                                    "scatter_out_us": ae["scatter_add_output"]["output_us"]}
    if tr:
        result["token_rounding"] = {"R": tr["R"], "plain_ms": tr["plain"]["ms_per_step"],
                                    **{f"{k}_ms": tr[k]["ms_per_step"]
                                       for k in ("down", "up", "nearest")},
                                    **{f"{k}_rows": tr[k]["row_share"]
                                       for k in ("down", "up", "nearest")}}
    if dd:
        result["decode_dispatch_us"] = {"cols": "two_calls,dispatch_rounds,dispatch_bitonic",
                                        **{k.split("=")[1]: [v["two_calls_us"],
                                                             v["dispatch_rounds_us"],
                                                             v["dispatch_bitonic_us"]]
                                           for k, v in dd["latency"].items()}}
    # ---- CPU oracle baseline (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ntok = args.cpu_tokens if args.cpu_tokens > 0 else cfg.T
        v_cpu, dt_cpu, wide = cpu_oracle_tokens_per_s(inp, ntok)
        cpu = {"value": round(v_cpu, 1), "unit": "tokens/s", "cores": cpu_cores(),
               "kind": "oracle",
               "sample": f"{ntok} tokens, whole layer, numpy fp64, {dt_cpu:.1f} s"}
        if cfg.dtype == "bf16" and not args.no_secondary:
            cf = cpu_oracle_figures(inp, wide)
            result["cpu_oracle_figures"] = {
                "token_rounding_tok_s": round(cf["token_rounding"]["tokens_per_s"], 1)
                if "token_rounding" in cf else None,
                "backward_tok_s": round(cf["backward_act"]["tokens_per_s"], 1),
                "decode_us": cf["decode_dispatch"]["us"],
                "atomic_tok_s": round(cf["atomic_experts"]["tokens_per_s"], 1)}
    result["kernel_ms_per_step"] = per_kernel
    if wl:
        result["workloads"] = wl
    result["gemm"] = {"tflops": round(ach_gemm, 1), "frac": round(ach_gemm / peak_t, 4),
                      "gateup_tflops": round(ach_g, 1), "gateup_frac": round(ach_g / peak_t, 4),
                      "down_tflops": round(ach_d, 1), "down_frac": round(ach_d / peak_t, 4)}
    kd = dc["kernels_ms_with_events"]
    result["dispatch_combine"] = {"bytes": dc["bytes"], "ms": dc["ms"],
                                  "gbs": dc["achieved_gbs"], "frac": dc["frac"],
                                  "peak_gbs": dc["peak_gbs"], "ms_median": dc["ms_median"],
                                  "ms_min": dc["ms_min"], "ms_warm": dc["ms_back_to_back"],
                                  "route_ms": kd.get("route_tc", kd.get("route")),
                                  "permute_ms": round(sum(v for k, v in kd.items() if k in (
                                      "permute_small", "permute_cluster", "hist", "scan",
                                      "scatter")), 4),
                                  "gather_ms": kd.get("gather_rows"), "combine_ms": kd.get("combine"),
                                  "sm_mhz": dc["clocks"]["sm_mhz"],
                                  "clock_reasons": dc["clocks"]["reasons"]}
    result["roofline"] = roofline
    result["e2e"] = e2e
    result["clocks"] = clocks.summary()
    if cpu is not None:
        result["cpu_baseline"] = cpu
    result["gpu_launches"] = int(launches)
    if rank == 0:
        print(json.dumps(result, separators=(",", ":")), flush=True)


def main():
    args = parse()
    rank, world, local = dist_init(args)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
