#!/usr/bin/env python3
"""Benchmark of the MXFP4 MoE layer on B200: tokens/s of one layer step.

A step is one ``moe_forward`` over one batch of tokens (RMSNorm, router, top-k,
grouping, gate_up + SwiGLU, down + weighted combine + residual).  Inputs are
seeded synthetic tensors of the workload's shapes (``synth``) and are resident
in HBM before the timed region; the L2 is flushed (256 MiB write, then a 256 MiB read) before every
step, outside the step's events.

The line is headlined by the largest single-GPU workload, the skewed-routing
gpt-oss-120b batch (T = 16384, E = 128, tensor-bound: the "% of FP4 tensor peak"
half of the metric).  The gpt-oss-20b decode batch (T = 16, E = 32, HBM-bound:
the "% of HBM bandwidth" half) is measured in the same run and reported under
``"decode"`` with its own timing, roofline and end-to-end figures.

The end-to-end figure (``e2e``) times ``moe_forward_host`` per step: x from pinned host
memory in, y to pinned host memory out, the batch cut into chunks whose copies run on
their own streams under the neighbouring chunks' layers (``--e2e-chunk`` sets the chunk;
by default the library picks it).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--path auto|gemv|gemm]
    python bench.py --impl reference ...   # the CPU oracle on the host cores, same metric

Under torchrun (N > 1) every rank runs its own batch (token data parallel,
weights replicated, no collective on the data path); the step time is the max
over ranks and ``value`` counts the tokens of all ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MoE-layer tokens/s on 1 B200; % of FP4 tensor peak (prefill) / HBM BW (decode)"
HEADLINE_CONFIG = "skew_120b"
DECODE_CONFIG = "decode_20b"
WORKLOAD_TEXT = {
    "tiny": "tiny MoE layer: T=32, d=128, I=128, E=4, top-2, MXFP4 block 32",
    "decode_20b": "gpt-oss-20b MoE layer, decode: T=16, d=2880, I=2880, E=32, top-4, MXFP4 experts",
    "prefill_20b": "gpt-oss-20b MoE layer, prefill: T=4096, d=2880, I=2880, E=32, top-4, MXFP4 experts",
    "moe_120b": "gpt-oss-120b MoE layer: T=8192, d=2880, I=2880, E=128, top-4, MXFP4 experts",
    "skew_120b": "skewed routing: T=16384, d=I=2880, E=128, top-4, Zipf(1.2) router bias, MXFP4 experts",
}
KERNELS = ["route", "group", "pack", "gate_up", "down", "combine"]
KERNELS_FUSED_GROUP = ["route", "pack", "gate_up", "down", "combine"]   # small batches: grouping in the router
KERNELS_FUSED = ["route", "pack", "gate_up", "down"]     # ... and the combine in the down GEMM
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# dense tensor-core rate of each MMA kind relative to bf16 (NVIDIA's B200 figures:
# bf16 2.25, fp8 4.5, fp4 9 PFLOP/s dense)
RATE_VS_BF16 = {"fp8": 2.0, "fp4": 4.0}
CSRC = os.path.join(ROOT, "mxfp4_expert_gemm_b200", "csrc")
# source files whose code a kernel's counters depend on (the kernel's file and its headers)
KERNEL_SOURCES = {
    "gate_up": ["moe_mx.cu", "moe_internal.cuh", "sm100_ptx.cuh"],
    "down": ["moe_mx.cu", "moe_internal.cuh", "sm100_ptx.cuh"],
    "route": ["moe_route.cu", "moe_route_mma.cu", "moe_internal.cuh", "sm100_ptx.cuh"],
    "group": ["moe_route.cu", "moe_internal.cuh"],
    "pack": ["moe_route.cu", "moe_internal.cuh"],
    "combine": ["moe_route.cu", "moe_internal.cuh"],
}


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default=None, choices=list(synth.CONFIGS),
                    help="measure this workload alone (default: the skewed 120b batch, plus the 20b decode batch)")
    ap.add_argument("--path", default="auto", choices=["auto", "gemv", "gemm"])
    ap.add_argument("--act", default="bf16", choices=["bf16", "mxfp8", "mxfp4"],
                    help="activation format of the expert GEMMs: exact bf16 (the layer as stated), MXFP8 or MXFP4")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch every step from the host instead of "
                    "replaying a captured CUDA graph")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU-baseline sample budget per workload")
    ap.add_argument("--e2e-chunk", type=int, default=0,
                    help="tokens per chunk of the end-to-end call (0: the library's choice)")
    ap.add_argument("--tp", action="store_true",
                    help="tensor parallelism over the intermediate features: every rank holds a slice of I "
                         "for all experts and runs the whole batch; one all-reduce of the partial outputs")
    return ap.parse_args(argv)


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def rank_rows(rank, T):
    """Token rows of this rank's batch: rank r processes global rows [r*T, (r+1)*T) (weak scaling)."""
    return np.arange(rank * T, (rank + 1) * T)


def max_over_ranks(value, pg, device="cuda"):
    """Max of a per-rank float over all ranks (identity without a process group)."""
    if pg is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank, world, steps, total_ms):
    """Whole-job tokens/s: the tokens of all ranks over the slowest rank's time."""
    return tokens_per_rank * world * steps / (total_ms * 1e-3)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def code_sha(text: str) -> str:
    """Hash of a CUDA/C++ source with its comments and whitespace removed: a capture stays
    valid across comment edits and goes stale with any change to the code itself."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return hashlib.sha256("".join(text.split()).encode()).hexdigest()[:16]


def file_sha(path):
    with open(path, encoding="utf-8") as f:
        return code_sha(f.read())


def sources_sha(files) -> str:
    """Hash of the code (without comments) of several source files, in the given order."""
    text = "".join(open(os.path.join(CSRC, f), encoding="utf-8").read() + "\n" for f in files)
    return code_sha(text)


def traffic_key(config_name, act="bf16"):
    return config_name if act == "bf16" else f"{config_name}/{act}"


def ncu_traffic(kernel_key, config_name, act="bf16"):
    """Per-launch DRAM bytes of a kernel from a committed ncu capture, while the capture still
    matches the code of the kernel and its headers (captures of the MXFP8 activation format
    are filed under "<config>/mxfp8"); None otherwise."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        ent = d.get(traffic_key(config_name, act), {}).get(kernel_key)
        if not ent:
            return None
        if sources_sha(ent["sources"]) != ent["source_sha"]:
            return None
        return ent["dram_bytes_per_launch"]
    except Exception:
        return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index, period_s=0.002):
        self.samples, self.reasons, self.ok = [], set(), False
        self.period = period_s
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

    def _sample(self):
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for bit, name in self.REASONS.items():
                if r & bit:
                    self.reasons.add(name)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ------------------------------------------------------------------------------ inputs


def slice_inputs(cfg, i0, i1):
    """MXFP4 weights (quantized on the GPU) of the slice [i0, i1) of the intermediate features:
    W1's gate rows [i0, i1) and up rows [I + i0, I + i1), W2's columns [i0, i1)."""
    import torch
    import mxfp4_expert_gemm_b200 as moe
    E, d, I, Ir = cfg.E, cfg.d, cfg.I, i1 - i0
    W = [torch.empty(sh, dtype=torch.uint8, device="cuda")
         for sh in (*moe.mxfp4_shapes(E, 2 * Ir, d), *moe.mxfp4_shapes(E, d, Ir))]
    for e in range(E):
        w1 = synth.w1_expert(cfg, e)
        w1s = np.ascontiguousarray(np.concatenate([w1[i0:i1], w1[I + i0:I + i1]]))
        w2s = np.ascontiguousarray(synth.w2_expert(cfg, e)[:, i0:i1])
        moe.moe_mxfp4_quantize(torch.from_numpy(w1s).cuda(), W[0][e:e + 1], W[1][e:e + 1], role="gate_up")
        moe.moe_mxfp4_quantize(torch.from_numpy(w2s).cuda(), W[2][e:e + 1], W[3][e:e + 1], role="down")
    torch.cuda.synchronize()
    return W


def device_inputs(cfg, rank):
    """Hidden rows (this rank's tokens), router, and MXFP4 weights quantized on the GPU."""
    import torch
    import mxfp4_expert_gemm_b200 as moe
    rows = rank_rows(rank, cfg.T)
    x = synth.hidden_rows(cfg, rows) if rank else synth.hidden(cfg)
    gamma, rw, rb = synth.norm_weight(cfg), synth.router_weight(cfg), synth.router_bias(cfg)
    E, d, I = cfg.E, cfg.d, cfg.I
    dev = "cuda"
    s1c, s1s = moe.mxfp4_shapes(E, 2 * I, d)
    s2c, s2s = moe.mxfp4_shapes(E, d, I)
    w1c = torch.empty(s1c, dtype=torch.uint8, device=dev)
    w1s = torch.empty(s1s, dtype=torch.uint8, device=dev)
    w2c = torch.empty(s2c, dtype=torch.uint8, device=dev)
    w2s = torch.empty(s2s, dtype=torch.uint8, device=dev)
    for e in range(E):
        moe.moe_mxfp4_quantize(torch.from_numpy(synth.w1_expert(cfg, e)).to(dev), w1c[e:e + 1], w1s[e:e + 1],
                               role="gate_up")
        moe.moe_mxfp4_quantize(torch.from_numpy(synth.w2_expert(cfg, e)).to(dev), w2c[e:e + 1], w2s[e:e + 1],
                               role="down")
    torch.cuda.synchronize()
    xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
    return dict(x=x, gamma=gamma, rw=rw, rb=rb, x_dev=xt, gamma_dev=torch.from_numpy(gamma).to(dev),
                rw_dev=torch.from_numpy(rw).to(dev), rb_dev=torch.from_numpy(rb).to(dev),
                W=(w1c, w1s, w2c, w2s))


# ------------------------------------------------------------------------------ CPU oracle timing


def oracle_inputs(cfg, x, tokens):
    """The oracle's inputs for a sample of tokens: router tensors and the MXFP4 weights of the
    experts the oracle's own routing picks for them (the other experts are never read)."""
    import oracle
    gamma, rw, rb = synth.norm_weight(cfg), synth.router_weight(cfg), synth.router_bias(cfg)
    used = np.unique(oracle.route(x[tokens], gamma, rw, rb, cfg.k, cfg.rms_eps)["idx"])
    E, d, I = cfg.E, cfg.d, cfg.I
    ow = (np.zeros((E, 2 * I, d // 2), np.uint8), np.zeros((E, 2 * I, d // 32), np.uint8),
          np.zeros((E, d, I // 2), np.uint8), np.zeros((E, d, I // 32), np.uint8))
    for e in used.tolist():
        ow[0][e], ow[1][e] = oracle.quantize(synth.w1_expert(cfg, e))
        ow[2][e], ow[3][e] = oracle.quantize(synth.w2_expert(cfg, e))
    return dict(x=x, gamma=gamma, rw=rw, rb=rb, oracle_W=ow)


def time_oracle(cfg, inp, tokens_per_call, budget_s=None, steps=None, warmup=0, act="bf16", vary=True):
    """Time the CPU oracle (as it stands) on calls of ``tokens_per_call`` consecutive tokens of
    the workload (the next tokens each call, or with ``vary`` False the first ones every
    call); run until ``budget_s`` seconds (after at least one call) or for ``warmup + steps``
    calls.  Returns (tokens/s, threads, sample description)."""
    import oracle
    T = cfg.T
    n = tokens_per_call
    times, done, i = [], 0, 0
    t_start = time.perf_counter()
    while True:
        toks = ((np.arange(n) + (i if vary else 0) * n) % T).astype(np.int32)
        t0 = time.perf_counter()
        oracle.moe_forward(inp["x"], inp["gamma"], inp["rw"], inp["rb"], *inp["oracle_W"], I=cfg.I, k=cfg.k,
                           eps=cfg.rms_eps, limit=cfg.swiglu_limit, tokens=toks, act=act)
        dt = time.perf_counter() - t0
        if i >= warmup:
            times.append(dt)
            done += n
        i += 1
        if steps is not None:
            if i >= warmup + steps:
                break
        elif time.perf_counter() - t_start >= budget_s and times:
            break
    total = sum(times)
    which = "consecutive tokens" if vary else "the batch's first tokens every time"
    sample = (f"{len(times)} oracle forward(s) of {n} token(s) each ({which}) from the {cfg.name} batch "
              f"({total:.1f} s, fp64, all host threads)")
    return done / total, os.cpu_count(), sample


def cpu_tokens_per_call(cfg):
    """A bounded oracle sample: one call is a few seconds of host work at gpt-oss width."""
    return min(cfg.T, 256)


# ------------------------------------------------------------------------------ our arm


ACT_DTYPE = {"bf16": "mxfp4xbf16", "mxfp8": "mxfp4xmxfp8", "mxfp4": "mxfp4xmxfp4"}
ACT_NOTE = {
    "bf16": ("MXFP4 (E2M1 + E8M0) weights x bf16 activations, each carried into the tensor cores as two E4M3 "
             "terms with their block scales; fp32 accumulation"),
    "mxfp8": "MXFP4 weights x MXFP8 (E4M3) activations; fp32 accumulation",
    "mxfp4": "MXFP4 weights x MXFP4 (E2M1) activations (FP4 x FP4 MMA); fp32 accumulation",
}
ACT_TEXT = {
    "bf16": "bf16, exact (each value carried into the MMA as two E4M3 terms)",
    "mxfp8": "MXFP8 (E4M3 in 32-value blocks)",
    "mxfp4": "MXFP4 (E2M1 in 32-value blocks, the weights' rule)",
}


class L2Flush:
    """Before every step: write a 256 MiB buffer (twice the L2), then read another one.
    The write evicts everything the previous step left in L2; the read evicts the write's
    own dirty lines (written back here, outside the step's events) so that the step does
    not pay for the flush's write-backs.  The step starts with nothing of its own in L2."""

    def __init__(self, device="cuda"):
        import torch
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=device)
        self.r = torch.zeros(256 << 20, dtype=torch.uint8, device=device)

    def __call__(self):
        import torch
        self.w.zero_()
        torch.sum(self.r, dtype=torch.int32)


L2_TEXT = ("flushed before every step: a 256 MiB write, then a 256 MiB read that writes the "
           "dirty lines back (both outside the step events)")


def measure(cfg, args, rank, world, local_rank, pg, want_cpu):
    """One workload: timed steps (graph replay), per-kernel times, roofline, end to end,
    clocks and the CPU oracle baseline.  Returns the workload's record."""
    import torch
    import mxfp4_expert_gemm_b200 as moe
    inp = device_inputs(cfg, rank)
    dims = moe.make_dims(cfg.d, cfg.I, cfg.E, cfg.k, cfg.rms_eps, cfg.swiglu_limit, path=args.path, act=args.act)
    ws = moe.new_workspace(dims, cfg.T)
    y = torch.empty_like(inp["x_dev"])
    flush = L2Flush()
    W = inp["W"]
    fwd = (dims, inp["x_dev"], inp["gamma_dev"], inp["rw_dev"], inp["rb_dev"], *W, ws)

    def plain_step():
        moe.moe_forward(*fwd, y=y)

    for _ in range(max(3, args.warmup)):
        flush()
        plain_step()
    torch.cuda.synchronize()
    st = moe.moe_device_status(ws)
    if st != moe.MOE_OK:
        raise moe.MoeError(st, "device status after warm-up")
    path_used = moe.resolved_path(dims, cfg.T)

    K = args.steps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    for e in [*starts, *stops]:
        e.record()  # creates the underlying CUDA events
    torch.cuda.synchronize()
    use_graph = not args.no_graph
    graph = None
    if use_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            plain_step()
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    # ---- timed region: the layer as a user runs it (one graph replay per step)
    with ClockSampler(local_rank) as clk:
        for i in range(K):
            flush()
            starts[i].record()
            if use_graph:
                graph.replay()
            else:
                plain_step()
            stops[i].record()
        torch.cuda.synchronize()
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    total_ms = float(sum(a.elapsed_time(b) for a, b in zip(starts, stops)))
    plain_step()
    launches = moe.last_launch_count() * K   # kernels per forward x timed steps
    del graph

    # ---- instrumented pass (outside the timed region): the same steps with a CUDA event
    # pair around each of the library's launches, replayed from one graph
    kev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * len(KERNELS))]
    for e in kev:
        e.record()
    torch.cuda.synchronize()

    def timed_step():
        moe.moe_forward_timed(*fwd, y=y, events=kev)

    kgraph = None
    if use_graph:
        kgraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(kgraph):
            timed_step()
    else:
        timed_step()
    n_timed = moe.last_launch_count()
    names = {len(KERNELS): KERNELS, len(KERNELS_FUSED_GROUP): KERNELS_FUSED_GROUP}.get(n_timed, KERNELS_FUSED)
    per_kernel = {name: [] for name in names[:n_timed]}
    for i in range(K):
        flush()
        if use_graph:
            kgraph.replay()
        else:
            timed_step()
        torch.cuda.synchronize()
        for j, name in enumerate(names[:n_timed]):
            per_kernel[name].append(kev[2 * j].elapsed_time(kev[2 * j + 1]))
    del kgraph
    st = moe.moe_device_status(ws)
    if st != moe.MOE_OK:
        raise moe.MoeError(st, "device status after the timed steps")
    kern_ms = {name: statistics.mean(v) for name, v in per_kernel.items()}
    total_ms = max_over_ranks(total_ms, pg)

    # ---- end to end through the public API with host buffers (pinned): moe_forward_host
    # stages x and y through the device in chunks whose copies, on their own streams,
    # overlap the layer of the neighbouring chunks
    x_host = torch.empty(inp["x_dev"].shape, dtype=torch.bfloat16, pin_memory=True)
    x_host.copy_(inp["x_dev"].cpu())
    y_host = torch.empty_like(x_host, pin_memory=True)
    e_starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    e_stops = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    x_dev2 = torch.empty_like(inp["x_dev"])
    chunk = min(args.e2e_chunk or moe.moe_host_chunk_tokens(dims, cfg.T), cfg.T)
    n_chunks = (cfg.T + chunk - 1) // chunk
    last = cfg.T - (n_chunks - 1) * chunk
    need = max(moe.moe_workspace_bytes(dims, chunk), moe.moe_workspace_bytes(dims, last))
    ws_e2e = ws if ws.numel() >= need else torch.zeros(need, dtype=torch.uint8, device=ws.device)
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_step():
        moe.moe_forward_host(dims, x_host, inp["gamma_dev"], inp["rw_dev"], inp["rb_dev"], *W, ws_e2e, x_dev2, y,
                             y_host=y_host, chunk_tokens=chunk, h2d_stream=h2d, d2h_stream=d2h)

    e2e_graph = None
    if use_graph:
        e2e_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(e2e_graph):
            e2e_step()
        e2e_graph.replay()
        torch.cuda.synchronize()
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    for i in range(K):
        flush()
        e_starts[i].record()
        if use_graph:
            e2e_graph.replay()
        else:
            e2e_step()
        e_stops[i].record()
    torch.cuda.synchronize()
    e2e_ms = float(sum(a.elapsed_time(b) for a, b in zip(e_starts, e_stops)))
    e2e_ms = max_over_ranks(e2e_ms, pg)
    del e2e_graph
    assert moe.moe_device_status(ws) == moe.MOE_OK
    assert moe.moe_device_status(ws_e2e) == moe.MOE_OK

    # ---- roofline of the dominant kernel (gate_up) and of the layer
    peaks, peak_src = load_peaks()
    counts = np.bincount(moe.moe_route(dims, inp["x_dev"], inp["gamma_dev"], inp["rw_dev"], inp["rb_dev"],
                                       ws)["topk_idx"].cpu().numpy().ravel(), minlength=cfg.E)
    used = int(np.count_nonzero(counts))
    P = cfg.T * cfg.k
    d, I = cfg.d, cfg.I
    w1_bytes = 2 * I * d // 2 + (d // 32) * 2 * I
    w2_bytes = d * I // 2 + (I // 32) * d
    gu_ms = kern_ms["gate_up"]
    layer_ms = total_ms / K
    traffic = ncu_traffic("gate_up", cfg.name, args.act)
    if (P / cfg.E) <= 24:   # few tokens per expert: the weight stream bounds the layer
        # expert weights streamed once + activations in / out (bf16: two E4M3 bytes per value;
        # MXFP8: one; MXFP4: half; block scales not counted)
        act_b = {"bf16": 2.0, "mxfp8": 1.0, "mxfp4": 0.5}[args.act]
        alg = int(used * w1_bytes + act_b * (P * d + P * I))
        achieved = alg / (gu_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "kernel": "gate_up (mx_expert_kernel<GATE_UP>)", "achieved": round(achieved, 1),
                "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                "algorithmic_bytes_per_launch": alg, "launch_ms": round(gu_ms, 5),
                "peak_source": f"hbm_gbs, {peak_src}"}
        layer_bytes = used * (w1_bytes + w2_bytes)
        gbps = layer_bytes / (layer_ms * 1e-3) / 1e9
        roof["layer"] = {"unique_expert_bytes": layer_bytes, "experts_used": used, "achieved_GBps": round(gbps, 1),
                         "frac_of_peak": round(gbps / peak, 4), "frac_of_8TBps": round(gbps * 1e9 / 8e12, 4)}
    else:                   # many tokens per expert: the tensor cores bound the layer
        alg = 4 * d * I * P
        achieved = alg / (gu_ms * 1e-3) / 1e12
        fp8_peak = round(RATE_VS_BF16["fp8"] * peaks["bf16_tflops"], 1)
        fp4_peak = round(RATE_VS_BF16["fp4"] * peaks["bf16_tflops"], 1)
        cols = 2 if args.act == "bf16" else 1   # MMA columns per token
        # the MMA's own rate: E2M1 x E4M3 (kind::mxf8f6f4) at the fp8 rate, FP4 x FP4 (kind::mxf4)
        # at the FP4 rate
        fp4_mma = args.act == "mxfp4"
        mma_peak = fp4_peak if fp4_mma else fp8_peak
        roof = {"bound": "tensor", "kernel": "gate_up (mx_expert_kernel<GATE_UP>)", "achieved": round(achieved, 1),
                "peak": mma_peak, "unit": "TFLOP/s", "frac": round(achieved / mma_peak, 4), "traffic": traffic,
                "algorithmic_flops_per_launch": alg, "launch_ms": round(gu_ms, 5),
                "peak_source": (f"4 x bf16_tflops burst ({peak_src}): the FP4 x FP4 MMA (kind::mxf4) runs at "
                                "the FP4 rate" if fp4_mma else
                                f"2 x bf16_tflops burst ({peak_src}): the block-scaled E2M1 x E4M3 MMA "
                                "(kind::mxf8f6f4) runs at the fp8 rate"),
                "mma_flops_per_launch": cols * alg, "mma_frac": round(cols * achieved / mma_peak, 4),
                "mma_note": ("each bf16 activation enters the MMA as two E4M3 columns (hi and lo terms), so the "
                             "MMA executes 2x the algorithmic flops" if cols == 2 else
                             "one MMA column per token"),
                "frac_of_fp4_peak": round(achieved / fp4_peak, 4),
                "fp4_peak": fp4_peak, "fp4_peak_source": f"4 x bf16_tflops burst ({peak_src})"}
        layer_flops = 6 * d * I * P
        tfl = layer_flops / (layer_ms * 1e-3) / 1e12
        roof["layer"] = {"flops": layer_flops, "achieved_TFLOPs": round(tfl, 1),
                         "frac_of_fp8_peak": round(tfl / fp8_peak, 4), "frac_of_fp4_peak": round(tfl / fp4_peak, 4)}

    rec = {
        "value": round(job_throughput(cfg.T, world, K, total_ms), 1), "unit": "tokens/s",
        "ms_per_step": round(total_ms / K, 5),
        "config": {"workload": WORKLOAD_TEXT[cfg.name], "name": cfg.name, "tokens_per_gpu": cfg.T,
                   "global_batch": cfg.T * world, "path": path_used, "parallelism": f"dp{world}",
                   "activations": ACT_TEXT[args.act],
                   "l2": L2_TEXT,
                   "timing": "sum of per-step CUDA events on the launching stream; max over ranks",
                   "launch": "CUDA graph replay per step" if use_graph else "host launches per step",
                   "kernel_timing": "separate pass of the same steps with CUDA events around each kernel"},
        "kernel_ms": {k_: round(v, 5) for k_, v in kern_ms.items()},
        "roofline": roof,
        "e2e": {"value": round(job_throughput(cfg.T, world, K, e2e_ms), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": int(inp["x_dev"].numel() * 2), "d2h_bytes_per_step": int(y.numel() * 2),
                "api": "moe_forward_host (pinned host x in, pinned host y out)", "chunks": n_chunks,
                "chunk_tokens": chunk},
        "gpu_launches": launches,
        "clocks": clk.summary(),
    }
    del ws, ws_e2e, flush, W, inp["W"]
    if want_cpu:
        n = cpu_tokens_per_call(cfg)
        v, cores, sample = time_oracle(cfg, oracle_inputs(cfg, inp["x"], np.arange(n)), n,
                                       budget_s=args.cpu_seconds, act=args.act, vary=False)
        rec["cpu_baseline"] = {"value": round(v, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                               "sample": sample}
    torch.cuda.empty_cache()
    return rec


def measure_tp(cfg, args, rank, world, local_rank, pg):
    """Tensor parallelism over I: the whole batch on every rank, each rank its slice of the
    intermediate features; per step the slice's partial forward, one all-reduce of the fp32
    partial outputs (NCCL), and the residual pass.  Host launches (no graph around the
    collective); step time = max over ranks; total work fixed (strong scaling)."""
    import torch
    import mxfp4_expert_gemm_b200 as moe
    i0, i1 = moe.intermediate_slices(cfg.I, world)[rank]
    x = synth.hidden(cfg)
    dev = "cuda"
    x_dev = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
    gamma = torch.from_numpy(synth.norm_weight(cfg)).to(dev)
    rw, rb = torch.from_numpy(synth.router_weight(cfg)).to(dev), torch.from_numpy(synth.router_bias(cfg)).to(dev)
    W = slice_inputs(cfg, i0, i1)
    dims = moe.make_dims(cfg.d, i1 - i0, cfg.E, cfg.k, cfg.rms_eps, cfg.swiglu_limit, path=args.path, act=args.act)
    ws = moe.new_workspace(dims, cfg.T)
    part = torch.empty((cfg.T, cfg.d), dtype=torch.float32, device=dev)
    y = torch.empty_like(x_dev)
    flush = L2Flush(dev)

    def step():
        moe.moe_forward_partial(dims, x_dev, gamma, rw, rb, *W, ws, y_partial=part)
        n = moe.last_launch_count()
        if pg:
            pg.all_reduce(part)
        moe.moe_residual_norm(x_dev, part, y=y)
        return n + moe.last_launch_count()

    for _ in range(max(3, args.warmup)):
        flush()
        step()
    torch.cuda.synchronize()
    if moe.moe_device_status(ws) != moe.MOE_OK:
        raise RuntimeError("device status after warm-up")
    K = args.steps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    launches = 0
    with ClockSampler(local_rank) as clk:
        for i in range(K):
            flush()
            starts[i].record()
            launches += step()
            stops[i].record()
        torch.cuda.synchronize()
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    total_ms = max_over_ranks(float(sum(a.elapsed_time(b) for a, b in zip(starts, stops))), pg)
    if moe.moe_device_status(ws) != moe.MOE_OK:
        raise RuntimeError("device status after the timed steps")
    return {"value": round(job_throughput(cfg.T, 1, K, total_ms), 1), "unit": "tokens/s",
            "ms_per_step": round(total_ms / K, 5),
            "config": {"workload": WORKLOAD_TEXT[cfg.name], "name": cfg.name, "global_batch": cfg.T,
                       "parallelism": f"tp{world}", "slice": [i0, i1], "path": moe.resolved_path(dims, cfg.T),
                       "collective": "NCCL all-reduce (sum) of the fp32 partial outputs [T, d] per step",
                       "l2": L2_TEXT,
                       "timing": "sum of per-step CUDA events on the launching stream; max over ranks",
                       "launch": "host launches per step"},
            "gpu_launches": launches, "clocks": clk.summary()}


def run_ours(args, rank, world, local_rank):
    import torch
    torch.cuda.set_device(local_rank)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        pg = dist
    want_cpu = (rank == 0 and world == 1 and not args.no_cpu_baseline)
    if args.tp:
        rec = measure_tp(synth.CONFIGS[args.config or HEADLINE_CONFIG], args, rank, world, local_rank, pg)
        line = {"metric": METRIC, "value": rec["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": max(3, args.warmup), "ms_per_step": rec["ms_per_step"], "higher_is_better": True,
                "scaling": "strong", "vs_baseline": None,
                "dtype": ACT_DTYPE[args.act], "data": "synthetic",
                "config": rec["config"], "gpu_launches": rec["gpu_launches"], "clocks": rec["clocks"]}
        if rank == 0:
            print(json.dumps(line), flush=True)
        if pg:
            pg.barrier()
            pg.destroy_process_group()
        return
    names = [args.config] if args.config else [HEADLINE_CONFIG, DECODE_CONFIG]
    recs = [measure(synth.CONFIGS[n], args, rank, world, local_rank, pg, want_cpu) for n in names]
    head = recs[0]
    line = {"metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": head["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": ACT_DTYPE[args.act],
            "dtype_note": ACT_NOTE[args.act],
            "data": "synthetic"}
    for key in ("config", "kernel_ms", "roofline", "e2e", "gpu_launches", "clocks", "cpu_baseline"):
        if key in head:
            line[key] = head[key]
    if len(recs) > 1:
        line["decode"] = recs[1]
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


# ------------------------------------------------------------------------------ reference arm


def run_reference(args, rank, world):
    if rank != 0:
        return
    cfg = synth.CONFIGS[args.config or HEADLINE_CONFIG]
    x = synth.hidden(cfg)
    # one token per step keeps --steps K --warmup W within minutes on the host cores
    n = 1
    calls = args.warmup + args.steps
    inp = oracle_inputs(cfg, x, (np.arange(calls * n)) % cfg.T)
    t0 = time.perf_counter()
    v, cores, sample = time_oracle(cfg, inp, n, steps=args.steps, warmup=args.warmup, act=args.act)
    wall = time.perf_counter() - t0
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(n / v * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD_TEXT[cfg.name], "name": cfg.name, "tokens_per_step": n},
            "cpu_baseline": {"kind": "oracle", "cores": cores, "sample": sample, "value": round(v, 4)},
            "e2e": {"value": round(v, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "wall_s": round(wall, 1)}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank, world, local_rank = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
