"""Benchmark of the double-binary layer forward on B200.

Headline workload: the DBF full-weight MLP layer (DBF page, section 2 form
with ell = 1): M = 4096 inputs, N = 11008 outputs, R = 5888 (~1.97
bits/weight), bf16 activations ~ N(0, 1), iid +-1 factors, fp16
lognormal(0, 0.5) scales. One step runs the whole forward (gamma scaling,
sign accumulation over B2, beta scaling, sign accumulation over B1, alpha
scaling, write) twice: once in the decode regime (1 token) and once in the
prefill regime (2048 tokens). Reported: tokens/s for the whole job, the
decode call against the HBM roofline and the prefill call against the
tensor-core roofline.

The other four layer configurations are timed too, each against its own
roofline and beside the fp64 oracle on the same token rows ("configs"): the
tiny layer (256 x 256, R = 16, 4 fp32 tokens), the LoRDBA adapter branch
(4096 x 4096, R = 64) at 1, 4, 16 and 64 tokens, 32 adapters (R = 32,
ell = 2) routed over 256 tokens in one segmented call, and the large
prefill layer (M = N = R = 8192) at 8192 tokens.

L2: every headline step reads a different one of 24 device copies of the
layer (24 x 11.2 MB, more than twice the 126 MB L2), so the sign matrices
come from HBM; the per-configuration calls are timed one by one with a
256 MB buffer written between calls (L2 flushed). Multi-GPU (torchrun):
each rank runs the same per-GPU work (weak scaling); the timing is the max
over ranks.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
python bench.py --profile NAME   (three calls of one configuration and exit,
                                  for ncu captures: decode, prefill, tiny,
                                  adapter64, segmented, large_prefill)
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import dbf_synth as S  # noqa: E402

METRIC = "DBF layer tokens/s; HBM GB/s (decode) & tensor TFLOP/s (prefill) vs roofline"
WORKLOAD = "dbf_mlp"
T_DECODE = 1
T_PREFILL = 2048
COPIES = 24
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_traffic(key: str, src: str):
    """DRAM bytes per launch from profiles/traffic.txt, or None when the
    kernel source changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    with open(os.path.join(ROOT, src), "rb") as f:
        digest = hashlib.sha256(f.read()).hexdigest()[:16]
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 3 and parts[0] == key and not line.startswith("#"):
                return float(parts[2]) if parts[1] == digest else None
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.proc = None
        self.thread = None

    def __enter__(self):
        cmd = ["nvidia-smi", "-i", str(self.index), "--query-gpu=clocks.sm,clocks.max.sm,power.draw,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
               "--format=csv,noheader,nounits", "-lms", "100"]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self

        def reader():
            for line in self.proc.stdout:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 7:
                    self.samples.append(parts)

        self.thread = threading.Thread(target=reader, daemon=True)
        self.thread.start()
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = []
        smax = None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        seen = set()
        for p in self.samples:
            try:
                sm.append(float(p[0]))
                smax = float(p[1])
            except ValueError:
                continue
            for name, val in zip(names, p[3:7]):
                if val.lower() == "active":
                    seen.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(seen),
                "samples": len(sm)}


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank timing over all ranks (the job's time is the slowest
    rank's); the identity without a process group."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world: int, tokens_per_step: int, steps: int, elapsed_ms: float) -> float:
    """Whole-job tokens/s: every rank processes tokens_per_step per step."""
    return world * tokens_per_step * steps / (elapsed_ms * 1e-3)


def algorithmic(w, T, act_bytes=2, R=None, layers=1):
    """Algorithmic bytes and flops of one forward call: the packed signs and
    the scales of 'layers' layers, x in and y out (act_bytes per value)."""
    R = w.R if R is None else R
    sign_bytes = layers * R * (w.M + w.N) / 8
    scale_bytes = layers * 2 * w.ell * (w.M + w.N + R)
    io_bytes = T * w.M * act_bytes + T * w.N * act_bytes
    flops = 2 * T * w.ell * R * (w.M + w.N)
    return sign_bytes + scale_bytes + io_bytes, flops


ORACLE_ROWS = 128   # prefill rows of the oracle sample (first, last, every 256-token tile)


def oracle_rows(w):
    return S.sample_rows_per_tile(w.seed, T_PREFILL, ORACLE_ROWS, 256)


def oracle_sample_rate(w, L, x_dec, x_pre, rows, nthreads):
    """The fp64 oracle on a bounded sample: tokens / second on host cores."""
    import oracle
    t0 = time.perf_counter()
    oracle.forward(L, x_dec, nthreads=nthreads)
    oracle.forward(L, x_pre, rows=rows, nthreads=nthreads)
    dt = time.perf_counter() - t0
    return (1 + len(rows)) / dt, dt


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def bench_config(w):
    """The workload description both arms print (identical dicts)."""
    return {"workload": w.description, "decode_tokens": T_DECODE, "prefill_tokens": T_PREFILL,
            "l2": f"inputs larger than L2: {COPIES} rotating copies of the layer weights",
            "oracle_sample": f"1 decode token + {ORACLE_ROWS} fixed seeded rows of the {T_PREFILL}-token prefill "
                             "(first, last, and rows of every 256-token tile)"}


def run_reference(args, rank, world):
    """Reference arm: the fp64 CPU oracle, timed on the host cores, on the
    same sample the other arm's cpu_baseline uses."""
    import oracle
    w = S.WORKLOADS[WORKLOAD]
    if world > 1 and rank != 0:
        return
    L = S.workload_layers(w)[0]
    x_dec = S.make_x(w.seed, T_DECODE, w.M, "bf16")
    x_pre = S.make_x(w.seed + 100, T_PREFILL, w.M, "bf16")
    rows = oracle_rows(w)
    nthreads = oracle.default_threads()
    for _ in range(args.warmup):
        oracle_sample_rate(w, L, x_dec, x_pre, rows[:8], nthreads)
    tokens = 0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_rate(w, L, x_dec, x_pre, rows, nthreads)
        tokens += 1 + len(rows)
    dt = time.perf_counter() - t0
    value = tokens / dt
    sample = (f"per step: 1 decode token + {len(rows)} of the {T_PREFILL} prefill tokens (fixed seeded rows); "
              f"CPU {cpu_model()}")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(w),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": nthreads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def oracle_rate(fn, tokens, min_s=0.3):
    """tokens / second of repeated oracle calls (at least min_s of work)."""
    n, t0 = 0, time.perf_counter()
    while True:
        fn()
        n += 1
        dt = time.perf_counter() - t0
        if dt >= min_s:
            return n * tokens / dt


def measure_configs(dbf, dev, stream, run_oracle):
    """Every layer configuration timed one call at a time (L2 flushed before
    each call by writing a 256 MB buffer, outside the timed events), against
    its roofline, beside the fp64 oracle on the same token rows."""
    import torch
    pk, pk_kind = peaks()
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    f16 = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.float16)).to(dev)
    bf16 = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    dev_layer = lambda L: dbf.Layer.from_signs(torch.from_numpy(L.b1).to(dev), torch.from_numpy(L.b2).to(dev),
                                               f16(L.alpha), f16(L.beta), f16(L.gamma))
    nthreads = None
    if run_oracle:
        import oracle
        nthreads = oracle.default_threads()

    def graph_ms(fn, n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(n):
                fn()
        g.replay()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            g.replay()
            b.record(stream)
        torch.cuda.synchronize(dev)
        del g
        return a.elapsed_time(b)

    def timed(fn, n):
        """Device time per call with L2 flushed before each call: CUDA graphs
        of n x [flush, call] and of n x [flush], the difference over n (no
        host launch cost, no idle gaps between the timing events)."""
        with torch.cuda.stream(stream):
            for _ in range(3):
                fn()
        torch.cuda.synchronize(dev)
        both = graph_ms(lambda: (flush_buf.zero_(), fn()), n)
        flush_only = graph_ms(lambda: flush_buf.zero_(), n)
        return max_over_ranks(max(1e3 * (both - flush_only) / n, 1e-3), dev)

    def entry(kernel, T, us, nbytes, flops, bound):
        e = {"kernel": kernel, "tokens": T, "us_per_call": us, "tokens_per_s": T / (us * 1e-6),
             "GB_per_s": nbytes / (us * 1e-6) / 1e9, "TFLOP_per_s": flops / (us * 1e-6) / 1e12,
             "algorithmic_bytes": nbytes, "flops": flops, "bound": bound, "l2": "flushed before each call (256 MB write)", "timing": "CUDA graphs of [flush, call] minus graphs of [flush]"}
        if bound == "hbm":
            e.update(peak=pk["hbm_gbs"], unit="GB/s", frac=e["GB_per_s"] / pk["hbm_gbs"],
                     peak_source=f"{pk_kind} copy bandwidth")
        else:
            e.update(peak=pk["bf16_tflops"], unit="TFLOP/s", frac=e["TFLOP_per_s"] / pk["bf16_tflops"],
                     peak_source=f"{pk_kind} bf16 dense (fp16 runs at the same rate)")
        return e

    out = {}
    # ---- tiny layer: 4 fp32 tokens
    w = S.WORKLOADS["tiny"]
    L = S.workload_layers(w)[0]
    dl = dev_layer(L)
    xh = S.make_x(w.seed, 4, w.M, "f32")
    x = torch.from_numpy(xh).to(dev)
    y = torch.empty((4, w.N), dtype=torch.float32, device=dev)
    ws = dbf.alloc_workspace(dbf.workspace_bytes(dl, 4), dev)
    us = timed(lambda: dbf.forward(dl, x, y=y, ws=ws, stream=stream), 50)
    nb, fl = algorithmic(w, 4, act_bytes=4)
    e = entry(f"{w.description}: decode path, {dbf.forward_launches(dl, 4)} launch", 4, us, nb, fl, "hbm")
    if run_oracle:
        e["oracle_tokens_per_s"] = oracle_rate(lambda: oracle.forward(L, xh, nthreads=nthreads), 4)
        e["oracle_tokens_per_s_1thread"] = oracle_rate(lambda: oracle.forward(L, xh, nthreads=1), 4)
    out["tiny_T4"] = e
    # ---- LoRDBA adapter branch at 1, 4, 16, 64 tokens
    w = S.WORKLOADS["adapter"]
    L = S.workload_layers(w)[0]
    dl = dev_layer(L)
    for T in w.tokens:
        xh = S.make_x(w.seed, T, w.M, "bf16")
        x = bf16(xh)
        y = torch.empty((T, w.N), dtype=torch.bfloat16, device=dev)
        ws = dbf.alloc_workspace(dbf.workspace_bytes(dl, T), dev)
        us = timed(lambda: dbf.forward(dl, x, y=y, ws=ws, stream=stream), 50)
        nb, fl = algorithmic(w, T)
        e = entry(f"{w.description}: decode path, {dbf.forward_launches(dl, T)} launch(es)", T, us, nb, fl, "hbm")
        if run_oracle:
            e["oracle_tokens_per_s"] = oracle_rate(lambda: oracle.forward(L, xh, nthreads=nthreads), T)
            e["oracle_tokens_per_s_1thread"] = oracle_rate(lambda: oracle.forward(L, xh, nthreads=1), T)
        out[f"adapter_T{T}"] = e
    # ---- DBF MLP layer, decode (1 token) and prefill (2048 tokens)
    w = S.WORKLOADS["dbf_mlp"]
    L = S.workload_layers(w)[0]
    dl = dev_layer(L)
    for T, seed in ((1, w.seed), (T_PREFILL, w.seed + 100)):
        xh = S.make_x(seed, T, w.M, "bf16")
        x = bf16(xh)
        y = torch.empty((T, w.N), dtype=torch.bfloat16, device=dev)
        ws = dbf.alloc_workspace(dbf.workspace_bytes(dl, T), dev)
        us = timed(lambda: dbf.forward(dl, x, y=y, ws=ws, stream=stream), 50 if T == 1 else 10)
        nb, fl = algorithmic(w, T)
        path = "decode" if T == 1 else "prefill"
        e = entry(f"{w.description}: {path} path, {dbf.forward_launches(dl, T)} launch(es)", T, us, nb, fl,
                  "hbm" if T == 1 else "tensor")
        if run_oracle:
            rows = None if T == 1 else oracle_rows(w)
            e["oracle_tokens_per_s"] = oracle_rate(lambda: oracle.forward(L, xh, rows=rows, nthreads=nthreads),
                                                   T if rows is None else len(rows))
            e["oracle_sample"] = "all tokens" if rows is None else f"{len(rows)} fixed seeded rows"
        out[f"dbf_mlp_T{T}"] = e
    # ---- 32 adapters (R = 32, ell = 2) over 256 tokens routed by id
    w = S.WORKLOADS["segmented"]
    Ls = S.workload_layers(w)
    table = dbf.AdapterTable([dev_layer(La) for La in Ls], dev)
    seg = S.make_segments(w.seed, 256, w.num_adapters)
    xh = S.make_x(w.seed, 256, w.M, "bf16")[seg.order]
    x = bf16(np.ascontiguousarray(xh))
    y = torch.empty((256, w.N), dtype=torch.bfloat16, device=dev)
    offs = torch.from_numpy(seg.offsets.astype(np.int32)).to(dev)
    ids = torch.from_numpy(seg.adapter.astype(np.int32)).to(dev)
    ws = dbf.alloc_workspace(dbf.segmented_workspace_bytes(w.R, w.ell, 256), dev)
    us = timed(lambda: dbf.forward_segmented(table, offs, ids, x, y=y, ws=ws, stream=stream), 50)
    nb, fl = algorithmic(w, 256, layers=w.num_adapters)
    e = entry(f"{w.description}: one segmented call ({len(seg.adapter)} segments), two launches", 256, us, nb, fl,
              "hbm")
    if run_oracle:
        e["oracle_tokens_per_s"] = oracle_rate(
            lambda: oracle.forward_segmented(Ls, seg.offsets, seg.adapter, xh, nthreads=nthreads), 256)
        e["oracle_tokens_per_s_1thread"] = oracle_rate(
            lambda: oracle.forward_segmented(Ls, seg.offsets, seg.adapter, xh, nthreads=1), 256)
    out["segmented_T256"] = e
    del table
    # ---- large prefill layer, M = N = R = 8192 at 8192 tokens
    w = S.WORKLOADS["large_prefill"]
    L = S.workload_layers(w)[0]
    dl = dev_layer(L)
    T = 8192
    xh = S.make_x(w.seed, T, w.M, "bf16")
    x = bf16(xh)
    y = torch.empty((T, w.N), dtype=torch.bfloat16, device=dev)
    ws = dbf.alloc_workspace(dbf.workspace_bytes(dl, T), dev)
    us = timed(lambda: dbf.forward(dl, x, y=y, ws=ws, stream=stream), 10)
    nb, fl = algorithmic(w, T)
    e = entry(f"{w.description}: prefill path (fp16 operand pre-pass + one tcgen05 launch of both stages, tiles claimed at run time)", T, us, nb, fl,
              "tensor")
    if run_oracle:
        rows = S.sample_rows_per_tile(w.seed, T, ORACLE_ROWS, 256)
        e["oracle_tokens_per_s"] = oracle_rate(lambda: oracle.forward(L, xh, rows=rows, nthreads=nthreads), len(rows))
        e["oracle_sample"] = f"{len(rows)} fixed seeded rows"
    out[f"large_prefill_T{T}"] = e
    if run_oracle:
        out["oracle_threads"] = nthreads
        out["oracle_cpu"] = cpu_model()
    del flush_buf, x, y, ws
    torch.cuda.empty_cache()
    return out


def profile_calls(name: str, calls: int = 3):
    """Three forward calls of one configuration on cuda:0 (seeded synthetic
    inputs as in the timed runs), synchronised, for a profiler to capture."""
    import torch
    import double_binary_rank_b200 as dbf
    dev = torch.device("cuda", 0)
    f16 = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.float16)).to(dev)
    bf16 = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    dev_layer = lambda L: dbf.Layer.from_signs(torch.from_numpy(L.b1).to(dev), torch.from_numpy(L.b2).to(dev),
                                               f16(L.alpha), f16(L.beta), f16(L.gamma))
    if name == "backward":
        # the DBF MLP layer's gradients at the prefill size (the bench's backward call)
        w = S.WORKLOADS["dbf_mlp"]
        L = S.workload_layers(w)[0]
        dl = dev_layer(L)
        x = bf16(S.make_x(w.seed + 100, T_PREFILL, w.M, "bf16"))
        dy = bf16(S.make_x(w.seed + 200, T_PREFILL, w.N, "bf16"))
        signs_t = dbf.transposed_signs(dl)
        ws = dbf.alloc_workspace(dbf.backward_workspace_bytes(dl, T_PREFILL), dev)
        grads = dbf.backward(dl, x, dy, signs_t=signs_t, ws=ws)
        fn = lambda: dbf.backward(dl, x, dy, signs_t=signs_t, grads=grads, ws=ws)
    elif name == "mbok":
        # the multi-boolean-kernel layer (4096 -> 4096, K = 3) at the prefill size
        mb = S.make_mbok_layer(0xDBF00006, 4096, 4096, 3)
        ml = dbf.MbokLayer.from_signs(torch.from_numpy(mb.w).to(dev), f16(mb.s_in), f16(mb.s_out))
        x = bf16(S.make_x(0xDBF00006, T_PREFILL, 4096, "bf16"))
        y = torch.empty((T_PREFILL, 4096), dtype=torch.bfloat16, device=dev)
        ws = dbf.alloc_workspace(dbf.mbok_workspace_bytes(ml, T_PREFILL), dev)
        fn = lambda: dbf.mbok_forward(ml, x, y=y, ws=ws)
    elif name == "factorize":
        # one outer iteration of the factorisation of an 11008 x 4096 fp32
        # weight at k = 5888, 4 ADMM steps per factor (the bench's call);
        # one call only (over a thousand launches)
        n, m, k = 11008, 4096, 5888
        gen = torch.Generator(device=dev)
        gen.manual_seed(0xDBF00001)
        W = torch.randn((n, m), device=dev, generator=gen)
        U0 = 0.1 * torch.randn((n, k), device=dev, generator=gen)
        V0 = 0.1 * torch.randn((k, m), device=dev, generator=gen)
        ws = dbf.alloc_workspace(dbf.factorize_workspace_bytes(n, m, k, 1, 24), dev)
        fn = lambda: dbf.factorize(W, U0, V0, outer=1, admm_iters=4, objective=False, ws=ws)
        calls = 1
    elif name == "segmented_prefill":
        # 32 adapters (4096 -> 4096, R = 128, two envelopes), 256 tokens each,
        # through the host-planned segmented forward (grouped GEMMs)
        n_ad, per, M = 32, 256, 4096
        layers = [dev_layer(S.make_layer(0xDBF00007, M, M, 128, 2, 0.5, adapter=a)) for a in range(n_ad)]
        offs = np.arange(0, (n_ad + 1) * per, per, dtype=np.int32)
        ids = np.arange(n_ad, dtype=np.int32)
        x = torch.randn((n_ad * per, M), device=dev).to(torch.bfloat16)
        y = torch.empty((n_ad * per, M), dtype=torch.bfloat16, device=dev)
        ws = dbf.alloc_workspace(dbf.segmented_planned_workspace_bytes(layers, offs, ids, M, M, n_ad * per), dev)
        fn = lambda: dbf.forward_segmented_planned(layers, offs, ids, x, y=y, ws=ws)
    elif name == "segmented":
        w = S.WORKLOADS["segmented"]
        Ls = S.workload_layers(w)
        table = dbf.AdapterTable([dev_layer(La) for La in Ls], dev)
        seg = S.make_segments(w.seed, 256, w.num_adapters)
        x = bf16(np.ascontiguousarray(S.make_x(w.seed, 256, w.M, "bf16")[seg.order]))
        y = torch.empty((256, w.N), dtype=torch.bfloat16, device=dev)
        offs = torch.from_numpy(seg.offsets.astype(np.int32)).to(dev)
        ids = torch.from_numpy(seg.adapter.astype(np.int32)).to(dev)
        ws = dbf.alloc_workspace(dbf.segmented_workspace_bytes(w.R, w.ell, 256), dev)
        fn = lambda: dbf.forward_segmented(table, offs, ids, x, y=y, ws=ws)
    else:
        wname, T, kind = {"decode": ("dbf_mlp", 1, "bf16"), "prefill": ("dbf_mlp", T_PREFILL, "bf16"),
                          "tiny": ("tiny", 4, "f32"), "adapter64": ("adapter", 64, "bf16"),
                          "large_prefill": ("large_prefill", 8192, "bf16")}[name]
        w = S.WORKLOADS[wname]
        L = S.workload_layers(w)[0]
        dl = dev_layer(L)
        xh = S.make_x(w.seed, T, w.M, kind)
        x = torch.from_numpy(xh).to(dev) if kind == "f32" else bf16(xh)
        y = torch.empty((T, w.N), dtype=torch.float32 if kind == "f32" else torch.bfloat16, device=dev)
        ws = dbf.alloc_workspace(dbf.workspace_bytes(dl, T), dev)
        fn = lambda: dbf.forward(dl, x, y=y, ws=ws, static_weights=True)
    for _ in range(calls):
        fn()
    torch.cuda.synchronize(dev)
    print(f"profile {name}: {calls} calls done")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", choices=["decode", "prefill", "tiny", "adapter64", "segmented", "large_prefill",
                                          "backward", "segmented_prefill", "mbok", "factorize"],
                    help="run three calls of one configuration and exit (no timing; for ncu captures)")
    args = ap.parse_args()
    if args.profile:
        profile_calls(args.profile)
        return
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist
    import double_binary_rank_b200 as dbf

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    w = S.WORKLOADS[WORKLOAD]
    L = S.workload_layers(w)[0]
    base = dbf.Layer.from_signs(torch.from_numpy(L.b1).to(dev), torch.from_numpy(L.b2).to(dev),
                                torch.from_numpy(L.alpha.view(np.float16)).to(dev),
                                torch.from_numpy(L.beta.view(np.float16)).to(dev),
                                torch.from_numpy(L.gamma.view(np.float16)).to(dev))
    layers = [base] + [dbf.Layer(base.M, base.N, base.R, base.ell, base.b1.clone(), base.b2.clone(),
                                 base.alpha.clone(), base.beta.clone(), base.gamma.clone())
                       for _ in range(COPIES - 1)]
    x_dec_h = S.make_x(w.seed, T_DECODE, w.M, "bf16")
    x_pre_h = S.make_x(w.seed + 100, T_PREFILL, w.M, "bf16")
    to_dev = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    x_dec, x_pre = to_dev(x_dec_h), to_dev(x_pre_h)
    y_dec = torch.empty((T_DECODE, w.N), dtype=torch.bfloat16, device=dev)
    y_pre = torch.empty((T_PREFILL, w.N), dtype=torch.bfloat16, device=dev)
    ws_dec = dbf.alloc_workspace(dbf.workspace_bytes(base, T_DECODE), dev)
    ws_pre = dbf.alloc_workspace(dbf.workspace_bytes(base, T_PREFILL), dev)
    stream = torch.cuda.Stream(device=dev)

    def step(i, ev=None):
        Lk = layers[i % COPIES]
        if ev is not None:
            ev[0].record(stream)
        dbf.forward(Lk, x_dec, y=y_dec, ws=ws_dec, static_weights=True, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        dbf.forward(Lk, x_pre, y=y_pre, ws=ws_pre, static_weights=True, stream=stream)
        if ev is not None:
            ev[2].record(stream)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    torch.cuda.synchronize(dev)

    # events around the decode and the prefill call of every 8th timed step
    # (at least three): they give the split of a step between the two calls
    # and the kernels' durations for the rooflines; the other steps carry
    # none, because an event recorded between two launches ends the
    # programmatic overlap of a kernel's start with the previous one's tail
    ev_every = 8 if args.steps >= 24 else 1
    evs = {i: [torch.cuda.Event(enable_timing=True) for _ in range(3)] for i in range(0, args.steps, ev_every)}
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            t_start.record(stream)
            for i in range(args.steps):
                step(i, evs.get(i))
            t_end.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), dev)
    evs = list(evs.values())
    dec_us = max_over_ranks(statistics.mean(1e3 * e[0].elapsed_time(e[1]) for e in evs), dev)
    pre_us = max_over_ranks(statistics.mean(1e3 * e[1].elapsed_time(e[2]) for e in evs), dev)
    tokens_per_step = T_DECODE + T_PREFILL
    value = weak_scaling_value(world, tokens_per_step, args.steps, elapsed_ms)

    # ---- end to end through the public API: host buffers, copies timed.
    # Every step copies its inputs in from pinned host memory and its outputs
    # (both y) back out; the copies run on their own streams, double
    # buffered, so that step i's output copy and step i+1's input copy
    # overlap step i+1's compute (the link is full duplex).
    x_dec_pin = torch.from_numpy(x_dec_h.view(np.int16)).view(torch.bfloat16).pin_memory()
    x_pre_pin = torch.from_numpy(x_pre_h.view(np.int16)).view(torch.bfloat16).pin_memory()
    y_dec_pin = torch.empty((T_DECODE, w.N), dtype=torch.bfloat16).pin_memory()
    y_pre_pin = torch.empty((T_PREFILL, w.N), dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(3, args.steps // 5)
    h2d_s, d2h_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    xd2 = [x_dec, torch.empty_like(x_dec)]
    xp2 = [x_pre, torch.empty_like(x_pre)]
    yd2 = [y_dec, torch.empty_like(y_dec)]
    yp2 = [y_pre, torch.empty_like(y_pre)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        b = i & 1
        Lk = layers[i % COPIES]
        with torch.cuda.stream(h2d_s):
            if i >= 2:
                h2d_s.wait_event(ev_comp[b])       # step i-2 has read this input buffer
            xd2[b].copy_(x_dec_pin, non_blocking=True)
            xp2[b].copy_(x_pre_pin, non_blocking=True)
            ev_in[b].record(h2d_s)
        stream.wait_event(ev_in[b])
        if i >= 2:
            stream.wait_event(ev_out[b])           # step i-2's outputs have left this buffer
        dbf.forward(Lk, xd2[b], y=yd2[b], ws=ws_dec, static_weights=True, stream=stream)
        dbf.forward(Lk, xp2[b], y=yp2[b], ws=ws_pre, static_weights=True, stream=stream)
        ev_comp[b].record(stream)
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(ev_comp[b])
            y_dec_pin.copy_(yd2[b], non_blocking=True)
            y_pre_pin.copy_(yp2[b], non_blocking=True)
            ev_out[b].record(d2h_s)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d_s.wait_event(e0)
    d2h_s.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i)
    stream.wait_event(ev_out[0])
    stream.wait_event(ev_out[1])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    e2e_value = weak_scaling_value(world, tokens_per_step, e2e_steps, e2e_ms)
    h2d = x_dec_pin.numel() * 2 + x_pre_pin.numel() * 2
    d2h = y_dec_pin.numel() * 2 + y_pre_pin.numel() * 2

    # ---- decode calls back to back (one token through the rotating layer
    # copies, as through the layers of a model): per-call time when nothing
    # else runs in between
    dec_launches = dbf.forward_launches(base, T_DECODE)
    pre_launches = dbf.forward_launches(base, T_PREFILL)
    # (captured in a CUDA graph, so that host launch cost is not timed)
    n_stream = 4 * COPIES
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(n_stream):
            dbf.forward(layers[i % COPIES], x_dec, y=y_dec, ws=ws_dec, static_weights=True, stream=stream)
    graph.replay()
    torch.cuda.synchronize(dev)
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        s0.record(stream)
        graph.replay()
        s1.record(stream)
    torch.cuda.synchronize(dev)
    stream_us = max_over_ranks(1e3 * s0.elapsed_time(s1) / n_stream, dev)
    del graph

    # ---- a dependent chain, as through the layers of a served model: the
    # input of call k+1 is the first M outputs of call k (one token). The
    # chain's copies have alpha scaled by 2^-12 (exact) so that values stay
    # finite over the chain; the work per call is the same.
    chain = [dbf.Layer(Lk.M, Lk.N, Lk.R, Lk.ell, Lk.b1, Lk.b2, Lk.alpha * (2.0 ** -12), Lk.beta, Lk.gamma)
             for Lk in layers]
    ybuf = [torch.empty((T_DECODE, w.N), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    ybuf[1][:, :w.M].copy_(x_dec)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(n_stream):
            src, dst = ybuf[(i + 1) % 2], ybuf[i % 2]
            dbf.forward(chain[i % COPIES], src[:, :w.M], y=dst, ws=ws_dec, static_weights=True, stream=stream)
    graph.replay()
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        s0.record(stream)
        graph.replay()
        s1.record(stream)
    torch.cuda.synchronize(dev)
    chain_us = max_over_ranks(1e3 * s0.elapsed_time(s1) / n_stream, dev)
    chain_finite = bool(torch.isfinite(ybuf[(n_stream - 1) % 2].float()).all())
    del graph, chain

    # ---- backward of the prefill batch (gradients through the layer for
    # training), timed separately: not part of the forward step above
    dy_h = S.make_x(w.seed + 200, T_PREFILL, w.N, "bf16")
    dy = to_dev(dy_h)
    signs_t = dbf.transposed_signs(base, stream=stream)
    ws_bwd = dbf.alloc_workspace(dbf.backward_workspace_bytes(base, T_PREFILL), dev)
    with torch.cuda.stream(stream):
        grads = dbf.backward(base, x_pre, dy, signs_t=signs_t, ws=ws_bwd, stream=stream)
        for _ in range(2):
            dbf.backward(base, x_pre, dy, signs_t=signs_t, grads=grads, ws=ws_bwd, stream=stream)
    torch.cuda.synchronize(dev)
    n_bwd = 5
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        b0.record(stream)
        for _ in range(n_bwd):
            dbf.backward(base, x_pre, dy, signs_t=signs_t, grads=grads, ws=ws_bwd, stream=stream)
        b1.record(stream)
    torch.cuda.synchronize(dev)
    bwd_us = max_over_ranks(1e3 * b0.elapsed_time(b1) / n_bwd, dev)

    # ---- multi-boolean-kernel layer (4096 -> 4096, K = 3 kernels) on the
    # prefill batch, timed separately
    mb = S.make_mbok_layer(0xDBF00006, w.M, w.M, 3)
    f16t = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.float16)).to(dev)
    mlayer = dbf.MbokLayer.from_signs(torch.from_numpy(mb.w).to(dev), f16t(mb.s_in), f16t(mb.s_out))
    y_mb = torch.empty((T_PREFILL, mb.N), dtype=torch.bfloat16, device=dev)
    ws_mb = dbf.alloc_workspace(dbf.mbok_workspace_bytes(mlayer, T_PREFILL), dev)
    with torch.cuda.stream(stream):
        for _ in range(3):
            dbf.mbok_forward(mlayer, x_pre, y=y_mb, ws=ws_mb, stream=stream)
    torch.cuda.synchronize(dev)
    m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_mb = 10
    with torch.cuda.stream(stream):
        m0.record(stream)
        for _ in range(n_mb):
            dbf.mbok_forward(mlayer, x_pre, y=y_mb, ws=ws_mb, stream=stream)
        m1.record(stream)
    torch.cuda.synchronize(dev)
    mb_us = max_over_ranks(1e3 * m0.elapsed_time(m1) / n_mb, dev)
    mb_flops = 2 * T_PREFILL * mb.K * mb.M * mb.N

    # ---- segmented prefill planned on the host: 32 adapters (4096 -> 4096,
    # R = 128, two envelopes), 256 tokens each, one forward per segment
    n_ad, per = 32, 256
    seg_layers = []
    for a in range(n_ad):
        La = S.make_layer(0xDBF00007, w.M, w.M, 128, 2, 0.5, adapter=a)
        seg_layers.append(dbf.Layer.from_signs(torch.from_numpy(La.b1).to(dev), torch.from_numpy(La.b2).to(dev),
                                               f16t(La.alpha), f16t(La.beta), f16t(La.gamma)))
    seg_offs = np.arange(0, (n_ad + 1) * per, per, dtype=np.int32)
    seg_ids = np.arange(n_ad, dtype=np.int32)
    x_seg = torch.randn((n_ad * per, w.M), device=dev).to(torch.bfloat16)
    y_seg = torch.empty((n_ad * per, w.M), dtype=torch.bfloat16, device=dev)
    with torch.cuda.stream(stream):
        dbf.forward_segmented_planned(seg_layers, seg_offs, seg_ids, x_seg, y=y_seg, stream=stream)
        ws_seg = dbf.alloc_workspace(dbf.segmented_planned_workspace_bytes(seg_layers, seg_offs, seg_ids, w.M, w.M,
                                                                           n_ad * per), dev)
        dbf.forward_segmented_planned(seg_layers, seg_offs, seg_ids, x_seg, y=y_seg, ws=ws_seg, stream=stream)
    torch.cuda.synchronize(dev)
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        g0.record(stream)
        for _ in range(5):
            dbf.forward_segmented_planned(seg_layers, seg_offs, seg_ids, x_seg, y=y_seg, ws=ws_seg, stream=stream)
        g1.record(stream)
    torch.cuda.synchronize(dev)
    seg_us = max_over_ranks(1e3 * g0.elapsed_time(g1) / 5, dev)
    seg_flops = 2 * n_ad * per * 2 * 128 * (w.M + w.M)

    # ---- SVID of a dense 11008 x 4096 fp32 weight (24 power iterations), the
    # projection of the factorisation and the first MBOK kernel
    Wd = torch.randn((w.N, w.M), device=dev)
    sv_signs = torch.empty((w.N, (w.M + 31) // 32), dtype=torch.int32, device=dev)
    sv_out = torch.empty(w.N, dtype=torch.float16, device=dev)
    sv_in = torch.empty(w.M, dtype=torch.float16, device=dev)
    sv_ws = dbf.alloc_workspace(int(dbf._lib.dbf_svid_scratch_bytes(w.N, w.M, 24)), dev)
    svid_call = lambda: dbf.svid(Wd, iters=24, signs=sv_signs, s_out=sv_out, s_in=sv_in, scratch=sv_ws, stream=stream)
    with torch.cuda.stream(stream):
        svid_call()
    torch.cuda.synchronize(dev)
    v0, v1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        v0.record(stream)
        for _ in range(3):
            svid_call()
        v1.record(stream)
    torch.cuda.synchronize(dev)
    svid_us = max_over_ranks(1e3 * v0.elapsed_time(v1) / 3, dev)
    # algorithmic bytes: one read of X per power iteration that ran (u and v
    # come from the same pass; converged iterations pass v on without reading
    # X), one read for the signs, the packed signs written
    svid_iters_run = dbf.svid_iterations(sv_ws, w.N, w.M, 24)
    svid_bytes = (svid_iters_run + 1) * Wd.numel() * 4 + Wd.numel() // 8
    del Wd, sv_signs, sv_ws

    # ---- DBF factorisation of an 11008 x 4096 fp32 weight at k = 5888 (the
    # DBF MLP layer's shape): one outer iteration, 4 ADMM steps per factor,
    # 24-iteration SVID projections, seeded random start
    fn, fm, fk, f_admm = w.N, w.M, w.R, 4
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed)
    Wf = (torch.randn((fn, fm), device=dev, generator=gen) * torch.exp(0.25 * torch.randn((fn, 1), device=dev, generator=gen))
          * torch.exp(0.25 * torch.randn((1, fm), device=dev, generator=gen)))
    s0 = float(Wf.square().mean().sqrt()) ** 0.5 * fk ** -0.25
    U0f = s0 * torch.randn((fn, fk), device=dev, generator=gen)
    V0f = s0 * torch.randn((fk, fm), device=dev, generator=gen)
    f_ws = dbf.alloc_workspace(dbf.factorize_workspace_bytes(fn, fm, fk, 1, 24), dev)
    dbf.factorize(Wf, U0f, V0f, outer=1, admm_iters=f_admm, objective=False, ws=f_ws, stream=stream)
    torch.cuda.synchronize(dev)
    # three timed calls, each bracketed by its own events; the median (the
    # first call after the warm-up is at times several ms slower)
    f_ms = []
    for _ in range(3):
        q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            q0.record(stream)
            dbf.factorize(Wf, U0f, V0f, outer=1, admm_iters=f_admm, objective=False, ws=f_ws, stream=stream)
            q1.record(stream)
        torch.cuda.synchronize(dev)
        f_ms.append(q0.elapsed_time(q1))
    fact_us = max_over_ranks(1e3 * sorted(f_ms)[1], dev)
    # fp32 contraction flops of one outer iteration: W V^T, V V^T, the sweep
    # inverse, the U solves; U^T W, U^T U, the sweep inverse, the V solves
    fact_flops = (2 * fn * fm * fk + 2 * fk * fk * fm + 2 * fk ** 3 + f_admm * 2 * fn * fk * fk
                  + 2 * fn * fm * fk + 2 * fk * fk * fn + 2 * fk ** 3 + f_admm * 2 * fk * fk * fm)
    del Wf, U0f, V0f, f_ws

    configs = measure_configs(dbf, dev, stream, run_oracle=(world == 1 and not args.no_cpu_baseline))

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    pk, pk_kind = peaks()
    fp32x3_peak = pk["bf16_tflops"] * (1.1 / 2.25) / 3
    b_dec, f_dec = algorithmic(w, T_DECODE)
    b_pre, f_pre = algorithmic(w, T_PREFILL)
    gbs = b_dec / (dec_us * 1e-6) / 1e9
    tfs = f_pre / (pre_us * 1e-6) / 1e12
    roof_pre = {"bound": "tensor", "achieved": tfs, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": tfs / pk["bf16_tflops"], "traffic": kernel_traffic("gemm_prefill", "double_binary_rank_b200/csrc/dbf_gemm.cu"),
                "kernel": "prefill forward (fp16 operand pre-pass + one tcgen05 launch of both stages, tiles claimed at run time), one call",
                "peak_source": f"{pk_kind} bf16 dense burst (fp16 runs at the same rate)"}
    if pk.get("bf16_tflops_sustained"):
        # the step loop keeps the tensor cores busy for the whole timed region:
        # the fraction of the sustained (power-capped) figure, for context
        roof_pre["peak_sustained"] = pk["bf16_tflops_sustained"]
        roof_pre["frac_sustained"] = tfs / pk["bf16_tflops_sustained"]
    roof_dec = {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / pk["hbm_gbs"], "traffic": kernel_traffic("decode", "double_binary_rank_b200/csrc/dbf_decode.cu"),
                "kernel": f"decode forward ({dec_launches} launch: stage 1, grid barrier, stage 2), one call inside the step",
                "peak_source": f"{pk_kind} copy bandwidth", "us_per_call": dec_us,
                "stream_us_per_call": stream_us, "stream_frac": b_dec / (stream_us * 1e-6) / 1e9 / pk["hbm_gbs"],
                "stream": f"{n_stream} independent calls back to back in a CUDA graph over the {COPIES} copies",
                "chain_us_per_call": chain_us, "chain_frac": b_dec / (chain_us * 1e-6) / 1e9 / pk["hbm_gbs"],
                "chain": f"{n_stream} dependent calls in a CUDA graph (x of call k+1 = first M outputs of call k)",
                "chain_outputs_finite": chain_finite}

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": bench_config(w),
        "arithmetic": "prefill: fp16 x fp16 tensor cores (tcgen05), fp32 accumulate; decode: u8 x s8 integer "
                      "tensor-core products of the sign bits with three int8 digits of 22-bit fixed-point "
                      "activations, exact integer sums",
        "roofline": roof_pre,
        "roofline_decode": roof_dec,
        "prefill_us_per_call": pre_us,
        "backward": {"kernel": "gradients dx, dalpha, dbeta, dgamma of the T=2048 prefill batch (two pre-passes + four tcgen05 sign GEMMs in two launches of tiles claimed at run time), one call",
                     "us_per_call": bwd_us, "achieved": 2 * f_pre / (bwd_us * 1e-6) / 1e12, "unit": "TFLOP/s",
                     "peak": pk["bf16_tflops"], "frac": 2 * f_pre / (bwd_us * 1e-6) / 1e12 / pk["bf16_tflops"]},
        "mbok": {"kernel": "multi-boolean-kernel layer 4096 -> 4096, K=3, T=2048 (fp16 pre-pass + one tcgen05 sign GEMM), one call",
                 "us_per_call": mb_us, "achieved": mb_flops / (mb_us * 1e-6) / 1e12, "unit": "TFLOP/s",
                 "peak": pk["bf16_tflops"], "frac": mb_flops / (mb_us * 1e-6) / 1e12 / pk["bf16_tflops"]},
        "segmented_prefill": {"kernel": "32 adapters 4096 -> 4096 (R=128, 2 envelopes) x 256 tokens, host-planned: one grouped pre-pass + two grouped tcgen05 GEMM launches",
                              "us_per_call": seg_us, "tokens_per_s": n_ad * per / (seg_us * 1e-6),
                              "achieved": seg_flops / (seg_us * 1e-6) / 1e12, "unit": "TFLOP/s", "peak": pk["bf16_tflops"],
                              "frac": seg_flops / (seg_us * 1e-6) / 1e12 / pk["bf16_tflops"]},
        "svid": {"kernel": "SVID of an 11008 x 4096 fp32 matrix, at most 24 power iterations, stopping once the "
                           "unit iterate moves by less than 1e-6 (signs packed, fp16 scales)",
                 "iterations_run": svid_iters_run, "us_per_call": svid_us, "achieved": svid_bytes / (svid_us * 1e-6) / 1e9, "unit": "GB/s",
                 "peak": pk["hbm_gbs"], "frac": svid_bytes / (svid_us * 1e-6) / 1e9 / pk["hbm_gbs"]},
        "factorize": {"kernel": "DBF factorisation of an 11008 x 4096 fp32 weight at k=5888: one outer iteration "
                                "(4 ADMM steps per factor; products on tcgen05 as three TF32 MMAs each, fp32 "
                                "accumulation; blocked sweep inverse; single-read SVID projections)",
                      "ms_per_outer_iteration": fact_us / 1e3, "ms_three_calls": [round(v, 2) for v in f_ms], "achieved": fact_flops / (fact_us * 1e-6) / 1e12,
                      "unit": "TFLOP/s", "bound": "tensor", "peak": fp32x3_peak,
                      "frac": fact_flops / (fact_us * 1e-6) / 1e12 / fp32x3_peak,
                      "peak_source": f"{pk_kind} bf16 dense x nominal TF32/BF16 ratio 1.1/2.25, / 3 TF32 products "
                                     "per fp32 multiply-add"},
        "configs": configs,
        "clocks": clk.summary(),
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "method": "x copied in from pinned host memory and both y copied out every step, on their own "
                          "streams with double-buffered device tensors (overlapping the next step's compute)"},
        "gpu_launches": args.steps * (dec_launches + pre_launches),
    }
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        nthreads = oracle.default_threads()
        rows = oracle_rows(w)
        rate, dt = oracle_sample_rate(w, L, x_dec_h, x_pre_h, rows, nthreads)
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                                "cpu": cpu_model(),
                                "sample": f"1 decode token + {len(rows)} fixed seeded rows of the {T_PREFILL}-token "
                                          f"prefill ({dt:.1f} s)"}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
