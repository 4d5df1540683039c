#!/usr/bin/env python
"""Benchmark of the routed MXFP4 MoE layer on B200.

One step = one call of the whole layer (route, top-k, bucket, expert SwiGLU
FFNs, combine) on one batch of T tokens.  Weights are kept cold in L2 by
cycling over NL independent copies of the layer (inputs larger than L2).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--T T] [--sweep]

Prints one JSON line (rank 0).  The headline is the decode/verify layer
(H 4096, I 1408, 64 experts, top-2, T = 5); the line's "extra" object holds
every other workload of the benchmark with its own roofline: the same layer at
T = 1, the fine-grained layer (256 experts, top-8, shared expert) at T = 1 and
5, the prefill chunk at T = 2048 and 4096 on the tensor-core path, and the
crossover of the multi-layer batch sweep.  With N > 1 (torchrun) every rank
runs its own batches (independent decode streams, no collective on the data
path): weak scaling, value = tokens of all ranks / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/s; decode HBM GB/s and prefill FP4 TFLOPS as % of roofline"
DEFAULT_WORKLOAD = "decode_h4096_i1408_e64_k2"
DEFAULT_T = 5
FIELDS = ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s")


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--T", type=int, default=DEFAULT_T)
    ap.add_argument("--layers", type=int, default=8)
    ap.add_argument("--precision", choices=["exact", "mxfp4"], default="exact",
                    help="activation precision of the expert projections")
    ap.add_argument("--path", choices=["auto", "gemv", "gemm"], default="auto")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--extra-steps", type=int, default=200,
                    help="timed steps of each extra workload (prefill: a quarter)")
    ap.add_argument("--sweep", action="store_true",
                    help="the multi-layer cold-cache batch sweep with more repetitions "
                         "(prints its own JSON line)")
    a = ap.parse_args(argv)
    a.warmup = max(3, a.warmup)
    return a


def _consts(args):
    from routed_expert_ffn_fp32_b200 import moe
    prec = moe.MOE_ACT_MXFP4 if args.precision == "mxfp4" else moe.MOE_ACT_EXACT
    path = {"auto": moe.MOE_PATH_AUTO, "gemv": moe.MOE_PATH_GEMV, "gemm": moe.MOE_PATH_GEMM}[args.path]
    return prec, path


# ---------------------------------------------------------------- clocks ---
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, index: int, period: float = 0.002):
        self.samples = []
        self.ok = False
        self.period = period
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self, t0: float, t1: float) -> dict:
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside and self.samples:   # region shorter than one period: nearest samples
            inside = sorted(self.samples, key=lambda s: abs(s[0] - (t0 + t1) / 2))[:3]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mask = 0
        for s in inside:
            mask |= s[2]
        reasons = [n for n, b in self.REASONS.items() if mask & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(s[1] for s in inside), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(inside)}


# ------------------------------------------------------------ ranks -------
def max_over_ranks(value: float, dist, device) -> float:
    """The largest value over all ranks (step time is max over ranks); dist is
    torch.distributed or None for one process."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(tokens_per_rank: int, world: int, ms: float) -> float:
    """Whole-job tokens/s: every rank runs its own batches of the same size."""
    return world * tokens_per_rank / (ms / 1e3)


# ------------------------------------------------------------- workload ----
def workload(name: str, T: int):
    from routed_expert_ffn_fp32_b200 import synth
    return synth.CONFIGS[name].with_T(T)


def expert_bytes(cfg) -> int:
    """Algorithmic bytes of one MXFP4 expert: codes + scales of its three matrices."""
    return 3 * (cfg.H * cfg.I // 2 + cfg.H * cfg.I // 32)


def activated_bytes(cfg, counts: np.ndarray) -> int:
    """Algorithmic bytes of one call: codes + scales of every activated expert."""
    n = int((np.asarray(counts) > 0).sum()) + (1 if cfg.shared else 0)
    return n * expert_bytes(cfg)


def ffn_flops(cfg, T: int) -> float:
    """FLOPs of the expert FFNs of one call: 3 projections x 2 H I per row."""
    return 6.0 * cfg.H * cfg.I * T * (cfg.k + (1 if cfg.shared else 0))


def workload_config(cfg, T, prec_name, path_name, NL) -> dict:
    return {"workload": cfg.name, "T": T, "H": cfg.H, "I": cfg.I, "E": cfg.E, "k": cfg.k,
            "shared": cfg.shared, "weights": "MXFP4 (E2M1 + E8M0 per 32)",
            "activations": "bf16" if prec_name == "exact" else "MXFP4 (quantised)",
            "accumulate": "f32", "path": path_name, "layer_copies": NL,
            "l2": f"inputs larger than L2: {NL} layer copies "
                  f"({NL * (cfg.E + cfg.shared) * expert_bytes(cfg) / 1e9:.2f} GB) cycled"}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "source": "measured (MEASURED_PEAKS.json: STREAM-style copy, cuBLAS bf16 burst)"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


def measured_traffic(record: str, bytes_per_launch: float):
    """DRAM bytes per FFN call from a committed ncu record (profiles/<record>),
    scaled by the activated bytes of this workload (traffic grows with them);
    None once the kernel source differs from the one the counters were taken
    on, or when there is no record."""
    import hashlib
    rec = os.path.join(ROOT, "profiles", record)
    if not os.path.exists(rec):
        return None
    d = json.load(open(rec))
    src = os.path.join(ROOT, d["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != d["source_sha256"]:
        return None
    return int(d["dram_bytes_per_call"] / d["algorithmic_bytes_per_call"] * bytes_per_launch)


# ---------------------------------------------------------- device layers ---
class LayerSet:
    """NL independent device copies of one layer's expert weights (every call
    of a cycle reads cold weights) and any number of routers over them."""

    def __init__(self, cfg, NL, dev, seed=0):
        import torch  # noqa: F401
        from routed_expert_ffn_fp32_b200 import moe, synth
        self.cfg = cfg
        L = synth.layer(cfg, seed=seed, T=1)
        ex0 = moe.Experts.from_numpy(L["experts"], dev)
        sh0 = moe.Experts.from_numpy(L["shared"], dev) if cfg.shared else None
        self.layers = [(ex0, sh0)]
        for _ in range(NL - 1):
            ex = moe.Experts(**{f: getattr(ex0, f).clone() for f in FIELDS})
            sh = None if sh0 is None else moe.Experts(**{f: getattr(sh0, f).clone() for f in FIELDS})
            self.layers.append((ex, sh))
        self.host = L      # host copy (router, first layer's weights) for the oracle baseline
        self.dev = dev

    def router(self, rcfg, seed=0):
        import torch
        from routed_expert_ffn_fp32_b200 import synth
        W_r, bias = synth.router(rcfg, seed)
        return (torch.from_numpy(W_r).to(self.dev),
                None if bias is None else torch.from_numpy(bias).to(self.dev))


def measure(ls, router, rcfg, T, path, prec, steps, warmup, stream, NX=8, seed0=0,
            ffn=True, sampler=None, dist=None):
    """Time NL-cycled whole-layer calls (CUDA graphs, one per layer copy and
    batch) and, with ffn, the expert-FFN call alone on the same routed batches.
    Returns timings (ms per call), realised activated bytes and the graphs."""
    import torch
    from routed_expert_ffn_fp32_b200 import moe, synth
    dev = ls.dev
    cfg = rcfg.with_T(T)
    Wd, bd = router
    NL = len(ls.layers)
    xs_np = [synth.activations(cfg, seed=seed0 + i, T=T) for i in range(NX)]
    xs = [torch.from_numpy(a.view(np.int16)).to(dev) for a in xs_np]
    shape = moe.shape_of(T, cfg.H, cfg.I, cfg.E, cfg.k)
    ws = moe.make_workspace(shape, path, prec, cfg.shared, dev, stream)
    y = torch.empty((T, cfg.H), dtype=torch.int16, device=dev)
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device=dev)
    wts = torch.empty((T, cfg.k), dtype=torch.float32, device=dev)
    ncyc = int(np.lcm(NL, NX))

    def call(i, st):
        ex, sh = ls.layers[i % NL]
        moe.moe_layer_forward(xs[i % NX], Wd, bd, ex, sh, shape, y, ws, path, prec, idx, wts,
                              stream=st)

    nbytes = []
    with torch.cuda.stream(stream):
        for i in range(NX):
            call(i, stream)
            stream.synchronize()
            nbytes.append(activated_bytes(cfg, np.bincount(idx.cpu().numpy().reshape(-1),
                                                           minlength=cfg.E)))
        graphs = []
        for i in range(ncyc):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                call(i, stream)
            graphs.append(g)
        for i in range(warmup):
            graphs[i % ncyc].replay()
        stream.synchronize()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        h0 = time.perf_counter()
        if sampler is not None:
            sampler.start()
        e0.record(stream)
        for i in range(steps):
            graphs[i % ncyc].replay()
        e1.record(stream)
        stream.synchronize()
        h1 = time.perf_counter()
        if sampler is not None:
            sampler.stop()
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()
    st = moe.moe_get_error(ws, stream)
    assert st == 0, f"device status {st}"
    out = {"ms_layer": e0.elapsed_time(e1) / steps, "bytes_layer": float(np.mean(nbytes)),
           "graphs": graphs, "ncyc": ncyc, "h0": h0, "h1": h1, "xs_np": xs_np, "xs": xs,
           "ws": ws, "shape": shape, "y": y}
    if not ffn:
        return out
    # the expert-FFN call alone (plan, scaled f16 token rows or the MXFP4
    # gather, gate/up + SwiGLU, down) over the same routed batches
    offs = torch.empty(cfg.E + 1, dtype=torch.int32, device=dev)
    cnts = torch.empty(cfg.E, dtype=torch.int32, device=dev)
    ents = torch.empty(T * cfg.k, dtype=torch.int32, device=dev)
    rows = T * cfg.k + (T if cfg.shared else 0)
    partial = torch.empty((rows, cfg.H), dtype=torch.float32, device=dev)
    fgraphs, fbytes, keep = [], [], []
    with torch.cuda.stream(stream):
        for i in range(ncyc):
            ex, sh = ls.layers[i % NL]
            moe.moe_route_topk(xs[i % NX], Wd, bd, shape, idx, wts, ws, stream=stream)
            moe.moe_bucket(idx, shape, cnts, offs, ents, ws, stream=stream)
            stream.synchronize()
            fbytes.append(activated_bytes(cfg, cnts.cpu().numpy()))
            o_i, e_i = offs.clone(), ents.clone()   # each graph keeps its own routing
            keep.append((o_i, e_i))
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                moe.moe_expert_ffn_mxfp4(ex, sh, xs[i % NX], o_i, e_i, shape, partial, ws, path,
                                         prec, stream=stream)
            fgraphs.append(g)
        for i in range(warmup):
            fgraphs[i % ncyc].replay()
        stream.synchronize()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        nrep = max(steps, ncyc)
        f0.record(stream)
        for i in range(nrep):
            fgraphs[i % ncyc].replay()
        f1.record(stream)
        stream.synchronize()
    assert moe.moe_get_error(ws, stream) == 0
    out["ms_ffn"] = f0.elapsed_time(f1) / nrep
    out["bytes_ffn"] = float(np.mean([fbytes[i % ncyc] for i in range(nrep)]))
    return out


def roofline_of(cfg, T, r, peaks, uses_tc, record=None) -> dict:
    """Roofline of the expert-FFN call: algorithmic bytes (activated experts) /
    its measured time against the measured HBM copy peak; on the tensor-core
    path also FP4 TFLOP/s against the FP4 peak and the attainable fraction."""
    ms, b = r["ms_ffn"], r["bytes_ffn"]
    achieved = b / (ms / 1e3) / 1e9
    out = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
           "frac": round(achieved / peaks["hbm_gbs"], 4),
           "traffic": measured_traffic(record, b) if record else None,
           **({"traffic_source": f"ncu dram__bytes_read.sum + dram__bytes_write.sum of both phases "
                                 f"(profiles/{record}), scaled by activated bytes"}
              if record and measured_traffic(record, b) is not None else {}),
           "kernel": "expert FFN call (plan, scaled f16 token rows, gate/up + SwiGLU, down)",
           "peak_source": peaks["source"], "bytes_per_launch": int(b), "launch_ms": round(ms, 5)}
    if uses_tc:
        flops = ffn_flops(cfg, T)
        fp4_peak = peaks["bf16_tflops"] * 4.0  # dense FP4 = 4 x dense bf16 (nominal ratio)
        t_hbm = b / (peaks["hbm_gbs"] * 1e9)
        t_tc = flops / (fp4_peak * 1e12)
        tflops = flops / (ms / 1e3) / 1e12
        out["kernel"] = "expert FFN on tcgen05 kind::mxf4 (MXFP4 gather, gate/up + SwiGLU + requant, down)"
        out["tensor"] = {"achieved_tflops": round(tflops, 1), "fp4_peak_tflops": round(fp4_peak, 1),
                         "frac_of_fp4_peak": round(tflops / fp4_peak, 4),
                         "fp4_peak_source": "measured bf16 burst x 4 (nominal dense FP4/bf16 ratio)",
                         "flops_per_launch": flops,
                         "attainable_frac": round(max(t_hbm, t_tc) / (ms / 1e3), 4),
                         "bound_by": "hbm" if t_hbm >= t_tc else "tensor"}
    return out


def step_percentiles(graphs, ncyc, stream, steps, n=200):
    """p10 / median / p90 of single-step times (ms) from a separate pass of n
    replays, one event pair per step (after the timed region, so the headline
    timing carries no per-step events).  None if anything goes wrong."""
    try:
        import torch
        n = min(n, steps)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n)]
        with torch.cuda.stream(stream):
            for i in range(n):
                ev[i][0].record(stream)
                graphs[i % ncyc].replay()
                ev[i][1].record(stream)
            stream.synchronize()
        t = np.array([a.elapsed_time(b) for a, b in ev])
        return {"p10": round(float(np.percentile(t, 10)), 5),
                "median": round(float(np.median(t)), 5),
                "p90": round(float(np.percentile(t, 90)), 5), "steps": n}
    except Exception:
        return None


def e2e_measure(ls, router, cfg, T, path, prec, r, steps, warmup, stream):
    """The same metric end to end through the public API: every step copies
    its batch from pinned host memory, calls moe_layer_forward eagerly and
    reads the bf16 output back into pinned host memory."""
    import torch
    from routed_expert_ffn_fp32_b200 import moe
    Wd, bd = router
    NL = len(ls.layers)
    xh = [torch.from_numpy(a.view(np.int16)).pin_memory() for a in r["xs_np"]]
    NX = len(xh)
    yh = torch.empty((T, cfg.H), dtype=torch.int16).pin_memory()
    xd = torch.empty_like(r["xs"][0])
    y, ws, shape = r["y"], r["ws"], r["shape"]
    n = min(steps, 2000)
    with torch.cuda.stream(stream):
        for i in range(warmup):
            xd.copy_(xh[i % NX], non_blocking=True)
            ex, sh = ls.layers[i % NL]
            moe.moe_layer_forward(xd, Wd, bd, ex, sh, shape, y, ws, path, prec, stream=stream)
            yh.copy_(y, non_blocking=True)
        stream.synchronize()
        g0 = torch.cuda.Event(enable_timing=True)
        g1 = torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for i in range(n):
            xd.copy_(xh[i % NX], non_blocking=True)
            ex, sh = ls.layers[i % NL]
            moe.moe_layer_forward(xd, Wd, bd, ex, sh, shape, y, ws, path, prec, stream=stream)
            yh.copy_(y, non_blocking=True)
        g1.record(stream)
        stream.synchronize()
    ms = g0.elapsed_time(g1) / n
    return {"value": round(T / (ms / 1e3), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": T * cfg.H * 2, "d2h_bytes_per_step": T * cfg.H * 2,
            "ms_per_step": round(ms, 5), "api": "moe_layer_forward (eager, ctypes)"}


# ------------------------------------------------------------ our arm ------
def run_ours(args, rank, world, local_rank):
    import torch
    from routed_expert_ffn_fp32_b200 import build, moe, synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    build.build()
    moe.load_library()
    cfg = workload(args.workload, args.T)
    T, NL = cfg.T, args.layers
    PREC, PATH = _consts(args)
    peaks = load_peaks()
    stream = torch.cuda.Stream(dev)
    ls = LayerSet(cfg, NL, dev)
    router = ls.router(cfg)
    dist = None
    if world > 1:
        import torch.distributed as dist  # noqa: F811

    sampler = ClockSampler(local_rank)
    r = measure(ls, router, cfg, T, PATH, PREC, args.steps, args.warmup, stream,
                NX=16, seed0=1000 * rank, sampler=sampler, dist=dist)
    ms = max_over_ranks(r["ms_layer"], dist, dev)
    value = weak_scaling_value(T, world, ms)
    uses_tc = PREC == moe.MOE_ACT_MXFP4 and PATH in (moe.MOE_PATH_GEMM, moe.MOE_PATH_AUTO)
    if not uses_tc:
        record = "k_ffn_mma_decode64_t5.json"
    else:
        record = "k_ffn_gemm_prefill_t2048.json" if cfg.name == synth.PREFILL.name and T == 2048 else None
    roof = roofline_of(cfg, T, r, peaks, uses_tc, record)
    e2e = e2e_measure(ls, router, cfg, T, PATH, PREC, r, args.steps, args.warmup, stream)
    # route (fused for T <= 32) + gate/up + down + combine; the tensor-core
    # path adds the activation gather and the work-item plan
    launches_per_step = (4 if T <= 32 else 7) + (2 if uses_tc else 0)
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32" if PREC == moe.MOE_ACT_EXACT else "mxfp4 x mxfp4 -> f32",
        "data": "synthetic",
        "config": dict(workload_config(cfg, T, args.precision, args.path, NL),
                       parallelism=f"independent streams x{world}"),
        "layer_hbm_gbs": round(r["bytes_layer"] / (r["ms_layer"] / 1e3) / 1e9, 1),
        "activated_bytes_per_call": int(r["bytes_layer"]),
        "roofline": roof, "clocks": sampler.summary(r["h0"], r["h1"]), "e2e": e2e,
        "step_ms_pctl": step_percentiles(r["graphs"], r["ncyc"], stream, args.steps),
        "gpu_launches": launches_per_step * args.steps,
    }
    del r
    if not args.no_extra and args.workload == DEFAULT_WORKLOAD and rank == 0:
        out["extra"] = run_extra(ls, router, args, stream, dev, peaks)
    ctx = {"L": ls.host, "cfg": cfg}
    return out, ctx


def run_extra(ls64, router64, args, stream, dev, peaks):
    """Every other workload of the benchmark, each with its own roofline."""
    from routed_expert_ffn_fp32_b200 import moe, synth
    ex = {}
    steps = max(10, args.extra_steps)
    E, G, A, M = moe.MOE_ACT_EXACT, moe.MOE_PATH_GEMV, moe.MOE_PATH_AUTO, moe.MOE_ACT_MXFP4

    def entry(ls, router, rcfg, T, path, prec, n, record=None, uses_tc=False):
        r = measure(ls, router, rcfg, T, path, prec, n, max(3, min(args.warmup, 20)), stream,
                    seed0=7000)
        cfg = rcfg.with_T(T)
        e = {"tokens_per_s": round(T / (r["ms_layer"] / 1e3), 1),
             "ms_per_step": round(r["ms_layer"], 5),
             "layer_hbm_gbs": round(r["bytes_layer"] / (r["ms_layer"] / 1e3) / 1e9, 1),
             "activated_bytes_per_call": int(r["bytes_layer"]),
             "roofline": roofline_of(cfg, T, r, peaks, uses_tc, record),
             "config": workload_config(cfg, T, "mxfp4" if prec == M else "exact",
                                       "auto" if path == A else "gemv", len(ls.layers))}
        return e

    # a single token takes the K-split GEMV: no ncu record of that kernel here
    ex["decode64_T1"] = entry(ls64, router64, synth.DECODE64, 1, A, E, steps)
    fg = synth.FINEGRAINED
    lsf = LayerSet(fg.with_T(1), len(ls64.layers), dev)
    rf = lsf.router(fg)
    ex["finegrained_T1"] = entry(lsf, rf, fg, 1, A, E, steps)
    ex["finegrained_T5"] = entry(lsf, rf, fg, 5, A, E, steps)
    pre = synth.PREFILL
    rp = lsf.router(pre)
    for T in (2048, 4096):
        ex[f"prefill_T{T}"] = entry(lsf, rp, pre, T, A, M, max(10, steps // 4), uses_tc=True,
                                    record="k_ffn_gemm_prefill_t2048.json" if T == 2048 else None)
    ex["sweep"] = sweep_rows(lsf, rp, synth.SWEEP, stream, reps=max(10, steps // 10),
                             variants=("gemv_mxfp4", "gemm_mxfp4"))
    ex["banked_decode64_T5"] = banked_entry(ls64, router64, synth.DECODE64, 5, 32,
                                            max(20, steps // 2), stream, dev)
    return ex


def banked_entry(ls, router, cfg, T, n_slots, steps, stream, dev):
    """The decode layer with its routed experts in pinned host memory and
    n_slots of them in a device slot bank (least recently used first): eager
    banked calls (each reads the chosen experts back to the host once), timed
    with CUDA events on the stream; hit rate and host-to-device traffic of the
    paging."""
    import torch
    from routed_expert_ffn_fp32_b200 import moe, synth
    L = ls.host
    host = moe.Experts(**{f: torch.from_numpy(L["experts"][f]) for f in FIELDS})
    bank = moe.SlotBank(host, cfg.H, cfg.I, n_slots, device=dev)
    Wd, bd = router
    xs = [torch.from_numpy(synth.activations(cfg, 8000 + i, T).view(np.int16)).to(dev)
          for i in range(16)]
    shape = moe.shape_of(T, cfg.H, cfg.I, cfg.E, cfg.k)
    ws = moe.banked_workspace(shape, n_slots, device=dev, stream=stream)
    y = torch.empty((T, cfg.H), dtype=torch.int16, device=dev)
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device=dev)
    w = torch.empty((T, cfg.k), dtype=torch.float32, device=dev)
    with torch.cuda.stream(stream):
        for i in range(5):
            moe.moe_layer_forward_banked(xs[i % 16], Wd, bd, bank, None, shape, y, ws, idx, w,
                                         stream=stream)
        stream.synchronize()
        h0, m0, e0 = bank.stats()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(steps):
            moe.moe_layer_forward_banked(xs[i % 16], Wd, bd, bank, None, shape, y, ws, idx, w,
                                         stream=stream)
        b.record(stream)
        stream.synchronize()
    assert moe.moe_get_error(ws, stream) == 0
    ms = a.elapsed_time(b) / steps
    h, m, e = (v - v0 for v, v0 in zip(bank.stats(), (h0, m0, e0)))
    bank.close()
    h2d = m * expert_bytes(cfg) / steps
    return {"tokens_per_s": round(T / (ms / 1e3), 1), "ms_per_step": round(ms, 5),
            "slots": n_slots, "experts": cfg.E, "hit_rate": round(h / max(1, h + m), 4),
            "h2d_bytes_per_step": int(h2d), "h2d_gbs": round(h2d / (ms / 1e3) / 1e9, 1),
            "config": dict(workload_config(cfg.with_T(T), T, "exact", "auto", 1),
                           l2=f"{cfg.E} experts in pinned host memory, {n_slots} device slots "
                              f"({n_slots * expert_bytes(cfg) / 1e9:.2f} GB, larger than L2)"),
            "api": "moe_layer_forward_banked (eager: one host read of the routing per call)"}


# ----------------------------------------------------- batch-size sweep ----
SWEEP_VARIANTS = {"gemv_exact": ("gemv", "exact"), "gemv_mxfp4": ("gemv", "mxfp4"),
                  "gemm_mxfp4": ("gemm", "mxfp4")}


def sweep_rows(ls, router, base, stream, reps, variants):
    """Eight cold copies of the fine-grained layer, Zipf 1.2 routing: for each
    batch size of the sweep, whole-layer tokens/s of each path, and the
    crossover (the smallest batch at which the tensor-core path beats the
    CUDA-core path at the same MXFP4 activations)."""
    from routed_expert_ffn_fp32_b200 import moe, synth
    rows = []
    for T in synth.SWEEP_T:
        row = {"T": T}
        for name in variants:
            path_n, prec_n = SWEEP_VARIANTS[name]
            path = moe.MOE_PATH_GEMM if path_n == "gemm" else moe.MOE_PATH_GEMV
            prec = moe.MOE_ACT_MXFP4 if prec_n == "mxfp4" else moe.MOE_ACT_EXACT
            r = measure(ls, router, base, T, path, prec, max(len(ls.layers), reps), 3, stream,
                        NX=4, seed0=9000, ffn=False)
            row[name] = {"tokens_per_s": round(T / (r["ms_layer"] / 1e3), 1),
                         "ms_per_step": round(r["ms_layer"], 5),
                         "hbm_gbs": round(r["bytes_layer"] / (r["ms_layer"] / 1e3) / 1e9, 1)}
            row["activated_bytes_per_call"] = int(r["bytes_layer"])
            del r
        rows.append(row)
    cross = None
    if "gemv_mxfp4" in variants and "gemm_mxfp4" in variants:
        cross = next((r["T"] for r in rows
                      if r["gemm_mxfp4"]["tokens_per_s"] > r["gemv_mxfp4"]["tokens_per_s"]), None)
    return {"workload": base.name, "layers": len(ls.layers), "rows": rows,
            "crossover_T_gemm_over_gemv_mxfp4": cross}


def run_sweep(args, local_rank):
    import torch
    from routed_expert_ffn_fp32_b200 import build, moe, synth
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    build.build()
    moe.load_library()
    base = synth.SWEEP
    ls = LayerSet(base.with_T(1), synth.SWEEP_LAYERS, dev)
    stream = torch.cuda.Stream(dev)
    res = sweep_rows(ls, ls.router(base), base, stream, reps=200,
                     variants=("gemv_exact", "gemv_mxfp4", "gemm_mxfp4"))
    peaks = load_peaks()
    return {"metric": "MoE layer tokens/s over the batch sweep (cold weights, 8 layers)",
            "unit": "tokens/s", "n_gpus": 1, "data": "synthetic", "hbm_peak_gbs": peaks["hbm_gbs"],
            "config": {"workload": base.name, "layers": synth.SWEEP_LAYERS,
                       "T": list(synth.SWEEP_T)}, **res}


# ------------------------------------------------------- oracle on the CPU ---
def oracle_sample(cfg, L, x_bits, budget_s: float):
    """Time the fp64 oracle on whole tokens of the workload until budget_s."""
    import oracle as O
    t0 = time.perf_counter()
    tokens = 0
    while True:
        row = x_bits[tokens % x_bits.shape[0]: tokens % x_bits.shape[0] + 1]
        O.layer_forward(row, L["W_r"], L["bias"], L["experts"], L["shared"], cfg.k)
        tokens += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return tokens / dt, tokens, dt


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def cpu_baseline(ctx, budget_s=15.0):
    from routed_expert_ffn_fp32_b200 import synth
    cfg = ctx["cfg"]
    x = synth.activations(cfg, seed=0, T=cfg.T)
    v, n, dt = oracle_sample(cfg, ctx["L"], x, budget_s)
    return {"value": round(v, 3), "unit": "tokens/s", "cores": blas_threads(),
            "host_cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{n} tokens of {cfg.name} (one token per oracle call, fp64 numpy on "
                      f"{blas_threads()} BLAS threads of {os.cpu_count()} host cores; {dt:.1f} s)"}


def run_reference(args, rank, world):
    """The oracle as the reference arm: rank 0 only, one token per step."""
    if rank != 0:
        return None
    from routed_expert_ffn_fp32_b200 import synth
    cfg = workload(args.workload, args.T)
    L = synth.layer(cfg, seed=0)
    x = synth.activations(cfg, seed=0, T=cfg.T)
    import oracle as O
    for i in range(args.warmup):
        O.layer_forward(x[i % cfg.T:i % cfg.T + 1], L["W_r"], L["bias"], L["experts"],
                        L["shared"], cfg.k)
    t0 = time.perf_counter()
    for i in range(args.steps):
        O.layer_forward(x[i % cfg.T:i % cfg.T + 1], L["W_r"], L["bias"], L["experts"],
                        L["shared"], cfg.k)
    dt = time.perf_counter() - t0
    v = args.steps / dt
    cores = blas_threads()
    return {"impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(workload_config(cfg, cfg.T, args.precision, args.path, args.layers),
                           parallelism=f"independent streams x{world}"),
            "cpu_baseline": {"value": round(v, 3), "unit": "tokens/s", "cores": cores,
                             "host_cores": os.cpu_count(), "kind": "oracle",
                             "sample": "one token of the batch per step, fp64 numpy oracle"},
            "e2e": {"value": round(v, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.sweep:
        if rank == 0:
            print(json.dumps(run_sweep(args, local_rank)), flush=True)
        return
    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    out, ctx = run_ours(args, rank, world, local_rank)
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        out["cpu_baseline"] = cpu_baseline(ctx)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
