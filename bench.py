#!/usr/bin/env python
"""Benchmark of the routed MXFP4 MoE layer on B200.

One step = one call of the whole layer (route, top-k, bucket, expert SwiGLU
FFNs, combine) on one batch of T tokens.  Weights are kept cold in L2 by
cycling over NL independent copies of the layer (inputs larger than L2).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--T T]

Prints one JSON line (rank 0).  With N > 1 (torchrun) every rank runs its own
batches (independent decode streams, no collective on the data path): weak
scaling, value = tokens of all ranks / max-over-ranks time.
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


def parse():
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
    ap.add_argument("--sweep", action="store_true",
                    help="the multi-layer cold-cache batch sweep: GEMV and GEMM paths per T, "
                         "and the crossover (prints its own JSON line)")
    a = ap.parse_args()
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
    cfg = synth.CONFIGS[name]
    return cfg.with_T(T)


def activated_bytes(cfg, counts: np.ndarray) -> int:
    """Algorithmic bytes of one call: codes + scales of every activated expert."""
    per = 3 * (cfg.H * cfg.I // 2 + cfg.H * cfg.I // 32)
    n = int((counts > 0).sum()) + (1 if cfg.shared else 0)
    return n * per


def expert_bytes(cfg) -> int:
    return 3 * (cfg.H * cfg.I // 2 + cfg.H * cfg.I // 32)


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
    L = synth.layer(cfg, seed=0)
    W_r, bias = L["W_r"], L["bias"]
    ex0 = moe.Experts.from_numpy(L["experts"], dev)
    sh0 = moe.Experts.from_numpy(L["shared"], dev) if cfg.shared else None
    layers = [(ex0, sh0)]
    for _ in range(NL - 1):   # independent copies: every call reads cold weights
        ex = moe.Experts(**{f: getattr(ex0, f).clone() for f in
                            ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s")})
        sh = None if sh0 is None else moe.Experts(**{f: getattr(sh0, f).clone() for f in
                                                     ("gate_q", "gate_s", "up_q", "up_s",
                                                      "down_q", "down_s")})
        layers.append((ex, sh))
    Wd = torch.from_numpy(W_r).to(dev)
    bd = None if bias is None else torch.from_numpy(bias).to(dev)
    NX = 16
    xs_np = [synth.activations(cfg, seed=1000 * rank + i, T=T) for i in range(NX)]
    xs = [torch.from_numpy(a.view(np.int16)).to(dev) for a in xs_np]
    shape = moe.shape_of(T, cfg.H, cfg.I, cfg.E, cfg.k)
    stream = torch.cuda.Stream(dev)
    ws = moe.make_workspace(shape, PATH, PREC, cfg.shared, dev, stream)
    y = torch.empty((T, cfg.H), dtype=torch.int16, device=dev)
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device=dev)
    wts = torch.empty((T, cfg.k), dtype=torch.float32, device=dev)

    def call(i, st):
        ex, sh = layers[i % NL]
        moe.moe_layer_forward(xs[i % NX], Wd, bd, ex, sh, shape, y, ws, PATH, PREC, idx, wts,
                              stream=st)

    # one graph per (layer copy, batch) pair in the cycle
    ncyc = int(np.lcm(NL, NX))
    with torch.cuda.stream(stream):
        for i in range(min(ncyc, 4)):
            call(i, stream)
        stream.synchronize()
        graphs = []
        for i in range(ncyc):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                call(i, stream)
            graphs.append(g)
    assert moe.moe_get_error(ws, stream) == 0

    # routed activated bytes per call (the bench reports the realised mean)
    act_bytes = []
    with torch.cuda.stream(stream):
        for i in range(NX):
            call(i, stream)
            stream.synchronize()
            counts = np.bincount(idx.cpu().numpy().reshape(-1), minlength=cfg.E)
            act_bytes.append(activated_bytes(cfg, counts))
    bytes_per_call = float(np.mean(act_bytes))

    dist = None
    if world > 1:
        import torch.distributed as dist  # noqa: F811

    def barrier():
        if dist is not None:
            dist.barrier()

    sampler = ClockSampler(local_rank)
    sampler.start()
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            graphs[i % ncyc].replay()
        stream.synchronize()
        barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        h0 = time.perf_counter()
        e0.record(stream)
        for i in range(args.steps):
            graphs[i % ncyc].replay()
        e1.record(stream)
        stream.synchronize()
        h1 = time.perf_counter()
        torch.cuda.synchronize(dev)
        barrier()
    sampler.stop()
    ms_local = e0.elapsed_time(e1) / args.steps
    ms = max_over_ranks(ms_local, dist, dev)
    step_pctl = step_percentiles(graphs, ncyc, stream, args.steps)
    assert moe.moe_get_error(ws, stream) == 0
    value = weak_scaling_value(T, world, ms)

    # ---- dominant kernels: expert FFN (gate/up + down) timed alone -------------
    offs = torch.empty(cfg.E + 1, dtype=torch.int32, device=dev)
    cnts = torch.empty(cfg.E, dtype=torch.int32, device=dev)
    ents = torch.empty(T * cfg.k, dtype=torch.int32, device=dev)
    rows = T * cfg.k + (T if cfg.shared else 0)
    partial = torch.empty((rows, cfg.H), dtype=torch.float32, device=dev)
    ffn_graphs, ffn_bytes = [], []
    with torch.cuda.stream(stream):
        for i in range(ncyc):
            ex, sh = layers[i % NL]
            moe.moe_route_topk(xs[i % NX], Wd, bd, shape, idx, wts, ws, stream=stream)
            moe.moe_bucket(idx, shape, cnts, offs, ents, ws, stream=stream)
            stream.synchronize()
            counts = cnts.cpu().numpy()
            ffn_bytes.append(activated_bytes(cfg, counts))
            # each graph keeps its own routing in its own buffers
            o_i, e_i = offs.clone(), ents.clone()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                moe.moe_expert_ffn_mxfp4(ex, sh, xs[i % NX], o_i, e_i, shape, partial, ws,
                                         PATH, PREC, stream=stream)
            ffn_graphs.append((g, o_i, e_i))
        for i in range(args.warmup):
            ffn_graphs[i % ncyc][0].replay()
        stream.synchronize()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        nrep = max(args.steps, ncyc)
        f0.record(stream)
        for i in range(nrep):
            ffn_graphs[i % ncyc][0].replay()
        f1.record(stream)
        stream.synchronize()
    ffn_ms = f0.elapsed_time(f1) / nrep
    ffn_b = float(np.mean([ffn_bytes[i % ncyc] for i in range(nrep)]))
    peaks = load_peaks()
    achieved = ffn_b / (ffn_ms / 1e3) / 1e9
    flops = 6.0 * cfg.H * cfg.I * T * (cfg.k + (1 if cfg.shared else 0))
    tflops = flops / (ffn_ms / 1e3) / 1e12
    # AUTO takes the tensor-core kernels for MXFP4 activations at every batch size
    uses_tc = PREC == moe.MOE_ACT_MXFP4 and PATH in (moe.MOE_PATH_GEMM, moe.MOE_PATH_AUTO)
    fp4_peak = peaks["bf16_tflops"] * 4.0  # dense FP4 = 4 x dense bf16 (nominal ratio)
    t_hbm = ffn_b / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (fp4_peak * 1e12)
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": None, "kernel": "expert FFN call (plan, f16 token rows, gate/up + SwiGLU, down)",
                "peak_source": peaks["source"], "bytes_per_launch": int(ffn_b),
                "launch_ms": round(ffn_ms, 5)}
    if not uses_tc and cfg.T <= 512:
        roofline["traffic"] = measured_traffic(ffn_b)
        roofline["traffic_source"] = "ncu dram__bytes_read.sum + dram__bytes_write.sum of k_ffn_mma " \
                                     "(profiles/k_ffn_mma_decode64_t5.json), scaled by activated bytes"
    if uses_tc:
        roofline["kernel"] = "expert FFN on tcgen05 kind::mxf4 (gate/up + SwiGLU + requant, down)"
        roofline["tensor"] = {
            "achieved_tflops": round(tflops, 1), "fp4_peak_tflops": round(fp4_peak, 1),
            "frac_of_fp4_peak": round(tflops / fp4_peak, 4),
            "fp4_peak_source": "measured bf16 burst x 4 (nominal dense FP4/bf16 ratio)",
            "flops_per_launch": flops,
            "attainable_frac": round(max(t_hbm, t_tc) / (ffn_ms / 1e3), 4),
            "bound_by": "hbm" if t_hbm >= t_tc else "tensor"}
    layer_gbs = bytes_per_call / (ms_local / 1e3) / 1e9

    # ---- end to end through the C ABI with host buffers ------------------------
    xh = [torch.from_numpy(a.view(np.int16)).pin_memory() for a in xs_np]
    yh = torch.empty((T, cfg.H), dtype=torch.int16).pin_memory()
    xd = torch.empty_like(xs[0])
    n_e2e = min(args.steps, 2000)
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            xd.copy_(xh[i % NX], non_blocking=True)
            ex, sh = layers[i % NL]
            moe.moe_layer_forward(xd, Wd, bd, ex, sh, shape, y, ws, PATH, PREC, stream=stream)
            yh.copy_(y, non_blocking=True)
        stream.synchronize()
        g0 = torch.cuda.Event(enable_timing=True)
        g1 = torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for i in range(n_e2e):
            xd.copy_(xh[i % NX], non_blocking=True)
            ex, sh = layers[i % NL]
            moe.moe_layer_forward(xd, Wd, bd, ex, sh, shape, y, ws, PATH, PREC, stream=stream)
            yh.copy_(y, non_blocking=True)
        g1.record(stream)
        stream.synchronize()
    e2e_ms = g0.elapsed_time(g1) / n_e2e
    e2e = {"value": round(T / (e2e_ms / 1e3), 1), "unit": "tokens/s",
           "h2d_bytes_per_step": T * cfg.H * 2, "d2h_bytes_per_step": T * cfg.H * 2,
           "ms_per_step": round(e2e_ms, 5), "api": "moe_layer_forward (eager, ctypes)"}

    # route (fused for T <= 32) + gate/up + down + combine; the tensor-core path
    # adds the activation gather and the work-item plan
    launches_per_step = (4 if T <= 32 else 6) + (2 if uses_tc else 0)
    clocks = sampler.summary(h0, h1)
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32" if PREC == moe.MOE_ACT_EXACT else "mxfp4 x mxfp4 -> f32",
        "data": "synthetic",
        "config": {"workload": cfg.name, "T": T, "H": cfg.H, "I": cfg.I, "E": cfg.E, "k": cfg.k,
                   "shared": cfg.shared, "weights": "MXFP4 (E2M1 + E8M0 per 32)",
                   "activations": "bf16" if PREC == moe.MOE_ACT_EXACT else "MXFP4 (quantised)",
                   "accumulate": "f32", "path": args.path,
                   "layer_copies": NL,
                   "l2": f"inputs larger than L2: {NL} layer copies "
                         f"({NL * cfg.E * expert_bytes(cfg) / 1e9:.2f} GB) cycled",
                   "parallelism": f"independent streams x{world}"},
        "layer_hbm_gbs": round(layer_gbs, 1),
        "activated_bytes_per_call": int(bytes_per_call),
        "roofline": roofline, "clocks": clocks, "e2e": e2e,
        "step_ms_pctl": step_pctl,
        "gpu_launches": launches_per_step * args.steps,
    }
    extra = {}
    if not args.no_extra and args.workload == DEFAULT_WORKLOAD and rank == 0:
        extra = run_extra(cfg, layers, Wd, bd, stream, dev, args)
    if extra:
        out["extra"] = extra
    ctx = {"L": L, "cfg": cfg, "xs_np": xs_np}
    return out, ctx


def run_extra(cfg, layers, Wd, bd, stream, dev, args):
    """The same layer at the other batch size of the decode/verify workload."""
    import torch
    from routed_expert_ffn_fp32_b200 import moe, synth
    res = {}
    for T in (1,) if cfg.T != 1 else (5,):
        shape = moe.shape_of(T, cfg.H, cfg.I, cfg.E, cfg.k)
        ws = moe.make_workspace(shape, moe.MOE_PATH_AUTO, moe.MOE_ACT_EXACT, cfg.shared, dev,
                                stream)
        y = torch.empty((T, cfg.H), dtype=torch.int16, device=dev)
        idx = torch.empty((T, cfg.k), dtype=torch.int32, device=dev)
        wts = torch.empty((T, cfg.k), dtype=torch.float32, device=dev)
        xs = [torch.from_numpy(synth.activations(cfg, 7000 + i, T).view(np.int16)).to(dev)
              for i in range(8)]
        NL = len(layers)
        graphs, nbytes = [], []
        with torch.cuda.stream(stream):
            for i in range(NL):
                ex, sh = layers[i]
                moe.moe_layer_forward(xs[i % 8], Wd, bd, ex, sh, shape, y, ws,
                                      moe.MOE_PATH_AUTO, moe.MOE_ACT_EXACT, idx, wts,
                                      stream=stream)
                stream.synchronize()
                nbytes.append(activated_bytes(cfg, np.bincount(idx.cpu().numpy().reshape(-1),
                                                               minlength=cfg.E)))
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    moe.moe_layer_forward(xs[i % 8], Wd, bd, ex, sh, shape, y, ws,
                                          moe.MOE_PATH_AUTO, moe.MOE_ACT_EXACT, idx, wts,
                                          stream=stream)
                graphs.append(g)
            for i in range(args.warmup):
                graphs[i % NL].replay()
            stream.synchronize()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            n = max(args.steps, 1000)
            a.record(stream)
            for i in range(n):
                graphs[i % NL].replay()
            b.record(stream)
            stream.synchronize()
        ms = a.elapsed_time(b) / n
        gbs = float(np.mean(nbytes)) / (ms / 1e3) / 1e9
        res[f"T{T}"] = {"tokens_per_s": round(T / (ms / 1e3), 1), "ms_per_step": round(ms, 5),
                        "layer_hbm_gbs": round(gbs, 1),
                        "activated_bytes_per_call": int(np.mean(nbytes))}
    return res


# ----------------------------------------------------- batch-size sweep ----
def run_sweep(args, local_rank):
    """Eight independent copies of the fine-grained layer (Zipf 1.2 routing),
    called in turn so every call reads cold weights; for each batch size the
    CUDA-core path (exact and MXFP4 activations) and the tensor-core path
    (MXFP4 activations) are timed as whole layers.  The crossover is the
    smallest batch at which the tensor-core path beats the CUDA-core path at
    the same precision."""
    import torch
    from routed_expert_ffn_fp32_b200 import build, moe, synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    build.build()
    moe.load_library()
    base = synth.SWEEP
    NL = synth.SWEEP_LAYERS
    L = synth.layer(base, seed=0)
    ex0 = moe.Experts.from_numpy(L["experts"], dev)
    sh0 = moe.Experts.from_numpy(L["shared"], dev)
    fields = ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s")
    layers = [(ex0, sh0)] + [
        (moe.Experts(**{f: getattr(ex0, f).clone() for f in fields}),
         moe.Experts(**{f: getattr(sh0, f).clone() for f in fields})) for _ in range(NL - 1)]
    Wd = torch.from_numpy(L["W_r"]).to(dev)
    bd = torch.from_numpy(L["bias"]).to(dev)
    stream = torch.cuda.Stream(dev)
    variants = [("gemv_exact", moe.MOE_PATH_GEMV, moe.MOE_ACT_EXACT),
                ("gemv_mxfp4", moe.MOE_PATH_GEMV, moe.MOE_ACT_MXFP4),
                ("gemm_mxfp4", moe.MOE_PATH_GEMM, moe.MOE_ACT_MXFP4)]
    rows = []
    for T in synth.SWEEP_T:
        cfg = base.with_T(T)
        shape = moe.shape_of(T, cfg.H, cfg.I, cfg.E, cfg.k)
        NX = 4
        xs = [torch.from_numpy(synth.activations(cfg, 9000 + i, T).view(np.int16)).to(dev)
              for i in range(NX)]
        y = torch.empty((T, cfg.H), dtype=torch.int16, device=dev)
        idx = torch.empty((T, cfg.k), dtype=torch.int32, device=dev)
        wts = torch.empty((T, cfg.k), dtype=torch.float32, device=dev)
        row = {"T": T}
        nbytes = []
        for name, path, prec in variants:
            ws = moe.make_workspace(shape, path, prec, True, dev, stream)
            ncyc = int(np.lcm(NL, NX))
            graphs = []
            with torch.cuda.stream(stream):
                for i in range(ncyc):
                    ex, sh = layers[i % NL]
                    moe.moe_layer_forward(xs[i % NX], Wd, bd, ex, sh, shape, y, ws, path, prec,
                                          idx, wts, stream=stream)
                    if name == "gemv_exact":
                        stream.synchronize()
                        nbytes.append(activated_bytes(
                            cfg, np.bincount(idx.cpu().numpy().reshape(-1), minlength=cfg.E)))
                stream.synchronize()
                for i in range(ncyc):
                    ex, sh = layers[i % NL]
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=stream):
                        moe.moe_layer_forward(xs[i % NX], Wd, bd, ex, sh, shape, y, ws, path,
                                              prec, idx, wts, stream=stream)
                    graphs.append(g)
                for i in range(max(args.warmup, 3)):
                    graphs[i % ncyc].replay()
                stream.synchronize()
                n = max(ncyc, min(200, int(2e5 / T)))
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                for i in range(n):
                    graphs[i % ncyc].replay()
                b.record(stream)
                stream.synchronize()
            assert moe.moe_get_error(ws, stream) == 0
            ms = a.elapsed_time(b) / n
            row[name] = {"tokens_per_s": round(T / (ms / 1e3), 1), "ms_per_step": round(ms, 5)}
            del graphs, ws
        act = float(np.mean(nbytes))
        row["activated_bytes_per_call"] = int(act)
        for name, _, _ in variants:
            row[name]["hbm_gbs"] = round(act / (row[name]["ms_per_step"] / 1e3) / 1e9, 1)
        rows.append(row)
    cross = next((r["T"] for r in rows
                  if r["gemm_mxfp4"]["tokens_per_s"] > r["gemv_mxfp4"]["tokens_per_s"]), None)
    peaks = load_peaks()
    return {"metric": "MoE layer tokens/s over the batch sweep (cold weights, 8 layers)",
            "unit": "tokens/s", "n_gpus": 1, "data": "synthetic",
            "config": {"workload": base.name, "layers": NL, "T": list(synth.SWEEP_T),
                       "weights_gb": round(NL * (cfg.E + 1) * expert_bytes(cfg) / 1e9, 2)},
            "hbm_peak_gbs": peaks["hbm_gbs"], "sweep": rows,
            "crossover_T_gemm_over_gemv_mxfp4": cross}


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


def measured_traffic(bytes_per_launch: float):
    """DRAM bytes per FFN call from the committed ncu record of the decode GEMV,
    scaled by the activated bytes of this workload (traffic grows with them);
    None once the kernel source has changed since the counters were taken, or
    for another kernel."""
    import hashlib
    rec = os.path.join(ROOT, "profiles", "k_ffn_mma_decode64_t5.json")
    if not os.path.exists(rec):
        return None
    d = json.load(open(rec))
    src = os.path.join(ROOT, d["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != d["source_sha256"]:
        return None
    return int(d["dram_bytes_per_call"] / d["algorithmic_bytes_per_call"] * bytes_per_launch)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "source": "measured (MEASURED_PEAKS.json: STREAM-style copy)"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


# ------------------------------------------------------- oracle on the CPU ---
def oracle_sample(cfg, L, x_bits, budget_s: float):
    """Time the fp64 oracle on whole tokens of the workload until budget_s."""
    import oracle as O
    t0 = time.perf_counter()
    tokens = 0
    calls = 0
    while True:
        row = x_bits[tokens % x_bits.shape[0]: tokens % x_bits.shape[0] + 1]
        O.layer_forward(row, L["W_r"], L["bias"], L["experts"], L["shared"], cfg.k)
        tokens += 1
        calls += 1
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
    cfg = ctx["cfg"]
    v, n, dt = oracle_sample(cfg, ctx["L"], ctx["xs_np"][0], budget_s)
    return {"value": round(v, 3), "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} tokens of {cfg.name} (one token per oracle call, fp64 numpy; "
                      f"{dt:.1f} s)"}


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
            "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E,
                       "k": cfg.k, "sample": "one token of the batch per step"},
            "cpu_baseline": {"value": round(v, 3), "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "sample": "one token per step, fp64 numpy oracle"},
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
