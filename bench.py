#!/usr/bin/env python
"""Benchmark of the NVFP4 MoE layer on B200.

Default workload: the 8192-token prefill chunk of the 512-expert, hidden 2048,
intermediate 768, top-10 NVFP4 layer with BF16 activations and Zipf(1.1)-skewed
router logits. One step = the whole layer (routing, sort/permute, gate/up grouped
GEMM + SwiGLU, down grouped GEMM + weighted combine) over one chunk, inputs
resident in HBM. Also reported: decode expert GB/s for 1/2/4/8 tokens over 8
distinct layers, end-to-end throughput through the C ABI with host buffers, the
dominant kernel's roofline, and the FP64 CPU oracle's throughput.

Multi-GPU: each rank runs its own replica on its own chunk (tokens are
independent; no data-path collective), value = all ranks' tokens / max time.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "MoE-layer prefill tok/s & decode expert GB/s on 1 B200, as % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def prefill_launches(d):
    """Kernels one grouped-GEMM forward launches: routing (top-k + histogram,
    chunk scan, scan, scatter), activation staging, the gate/up and down tile
    kernels, the gate/up and down small-expert kernels, and the combine. The
    small-expert kernels are launched whenever their staged rows fit shared
    memory (17 rows of the padded H and I, 200 KB), which holds for every
    workload here."""
    def staged(k):
        return 17 * ((k + 255) // 256 * 256 + 8) * 2 + 128
    small = staged(d.H) <= 200 * 1024 and staged(d.I) <= 200 * 1024
    return 10 if small else 8
DECODE_BYTES_PER_EXPERT = None  # set from dims: (3*I*H)/2 codes + (3*I*H)/16 scales


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class Clocks:
    """Samples the SM clock and the clock-event (throttle) reasons through NVML
    every 10 ms while the timed region runs (read-only queries)."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, index: int):
        self.index = index
        self.sm, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self.ok = False

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[self.index]) if vis else self.index
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self.nv = pynvml
            self.ok = True
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        except Exception:
            self.ok = False
        return self

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.sm.append(float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.01)

    def __exit__(self, *a):
        self._stop.set()
        if self.ok:
            self.t.join(timeout=2)

    def summary(self):
        if not self.sm:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(self.sm)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.sm), "via": "NVML, 10 ms"}


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        import datetime
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, ws: int) -> float:
    if ws == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64,
                     device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ oracle leg

def cpu_oracle_rate(layer_cpu, x, logits, K, n_tokens, x_scale=None):
    """Tokens/s of the FP64 oracle (as it stands) on a sample of n_tokens tokens."""
    import oracle
    sample = np.arange(n_tokens, dtype=np.int32)
    xs = x[:n_tokens]
    lg = logits[:n_tokens]
    t0 = time.perf_counter()
    oracle.forward(layer_cpu, xs, K=K, logits=lg, x_scale=None if x_scale is None else x_scale[:n_tokens],
                   sample=sample)
    dt = time.perf_counter() - t0
    return n_tokens / dt, dt


def oracle_baseline(layer_cpu, x, logits, K, T, seconds, x_scale=None, layers=1):
    """The bench line's `cpu_baseline`: the oracle on the first n tokens of the
    chunk, n sized from an 8-token calibration to about `seconds` of CPU work.
    `layers` > 1: one layer is timed and the rate divided by the layer count (the
    stack's layers have one shape, so the oracle's cost per layer is the same)."""
    rate, _ = cpu_oracle_rate(layer_cpu, x, logits, K, 8, x_scale)       # calibrate
    n = int(min(T, max(8, rate * seconds)))
    rate, dt = cpu_oracle_rate(layer_cpu, x, logits, K, n, x_scale)
    sample = f"first {n} of the {T} tokens of the same chunk, FP64, {dt:.1f} s wall"
    if layers > 1:
        sample += f"; one layer timed, rate divided by {layers} layers (linear extrapolation)"
    return {"value": round(rate / layers, 3), "unit": "tok/s", "cores": oracle_threads(n),
            "cpu_model": cpu_model(), "kind": "oracle", "sample": sample}


def cpu_model():
    """The host CPU's model name, as the kernel reports it."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def oracle_threads(n_tokens):
    """Worker threads the C oracle starts for n sampled tokens: one per online CPU, at most one per token."""
    return max(1, min(n_tokens, os.cpu_count() or 1))


# ------------------------------------------------------------------- workloads

def make_prefill(wl_name, dev):
    wl = synth.CONFIGS[wl_name]
    d = wl.dims
    seed = synth.workload_seed(wl)
    T = wl.tokens[0]
    layer = synth.make_layer(d, seed, device=dev)
    logits = synth.make_logits(T, d.E, seed, zipf_s=wl.zipf_s, device=dev)
    if wl.act == "int8":
        x, xs = synth.make_x_int8(T, d.H, seed, outliers=wl.outliers, device=dev)
    else:
        x, xs = synth.make_x_bf16(T, d.H, seed, outliers=wl.outliers, device=dev), None
    return wl, layer, logits, x, xs


def run_ours(args, ws, rank, local):
    import nvfp4_mixture_experts_03_b200 as nv
    dev = torch.device("cuda", local)
    pk, pk_src = peaks()
    if args.decode_only:   # profiling aid: the decode measurement alone
        return {"metric": METRIC, "decode": run_decode(args, dev, pk, pk_src)}
    wl, layer, logits, x, xs = make_prefill(args.workload, dev)
    d = wl.dims
    T = x.shape[0]
    P = T * d.K
    m = nv.MoELayer.from_layer(layer, top_k=d.K, max_tokens=T)
    out = torch.empty(T, d.H, dtype=torch.float32, device=dev)
    ws_buf = m.workspace(T)
    stream = torch.cuda.current_stream()

    def step():
        m.forward(x, logits=logits, x_scale=xs, out=out, workspace=ws_buf)

    for _ in range(args.warmup):
        step()
    st = m.status()
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")
    counts = nv.debug_buffers(T, d.E, d.K, dev)
    m.forward(x, logits=logits, x_scale=xs, out=out, workspace=ws_buf, debug=counts)
    n_used = int((counts["counts"] > 0).sum().item())

    # phase events per step -> kernel durations over the timed region
    evsets = [[torch.cuda.Event(enable_timing=True) for _ in range(nv.PHASE_EVENTS)]
              for _ in range(args.steps)]
    for evs in evsets:
        for e in evs:
            e.record()
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with Clocks(dev.index) as clk:
        t0.record()
        for i in range(args.steps):
            m.set_phase_events(evsets[i])
            step()
        t1.record()
        torch.cuda.synchronize()
    m.set_phase_events(())
    barrier(ws)
    ms = t0.elapsed_time(t1)
    ms_max = max_over_ranks(ms, ws)
    phase_ms = np.zeros(nv.PHASE_EVENTS - 1)
    for evs in evsets:
        for j in range(nv.PHASE_EVENTS - 1):
            phase_ms[j] += evs[j].elapsed_time(evs[j + 1])
    phase_ms /= args.steps
    st = m.status()
    if st != 0:
        raise RuntimeError(f"device status {st} after timed steps")

    value = ws * T * args.steps / (ms_max / 1e3)
    flops_gu = 2.0 * P * (2 * d.I) * d.H
    flops_dn = 2.0 * P * d.H * d.I
    gu_ms = phase_ms[2]
    achieved = flops_gu / (gu_ms / 1e3) / 1e12
    # The sampled SM clock stays within about 10 % of its maximum during the
    # step (sw_power_cap is flagged; far above the ~1.3 GHz of a seconds-long
    # GEMM loop), so the burst cuBLAS figure
    # is the denominator; the sustained one is context.
    peak = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    # The gate/up phase is two launches: the tensor-core tiles of the experts with
    # more than 16 pairs and the streaming kernel of the rest; its traffic is the
    # sum of both captures (None unless both match the current sources).
    t_tiles = profile_traffic("grouped_gemm_gateup", wl.name)
    t_small = profile_traffic("small_expert_gateup", wl.name)
    traffic = t_tiles + t_small if t_tiles is not None and t_small is not None else None
    roof = {"kernel": "gate/up + SwiGLU phase: grouped_gemm_kernel<0> (tensor-core tiles) + "
                      "small_expert_kernel<0> (experts with <= 16 pairs)", "bound": "tensor",
            "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "traffic": traffic,
            "traffic_parts": {"grouped_gemm_kernel<0>": t_tiles, "small_expert_kernel<0>": t_small},
            "peak_source": f"{pk_src} bf16_tflops, burst (F16 operands run at the BF16 rate); "
                           f"sustained {pk.get('bf16_tflops_sustained')} for context",
            "frac_of_sustained": round(achieved / pk.get("bf16_tflops_sustained",
                                                         FALLBACK_PEAKS["bf16_tflops_sustained"]), 4),
            "algorithmic_flops_per_launch": flops_gu}
    phases = {"routing_ms": round(phase_ms[0], 4), "stage_activations_ms": round(phase_ms[1], 4),
              "gate_up_ms": round(phase_ms[2], 4), "down_and_combine_ms": round(phase_ms[3], 4),
              "down_tflops": round(flops_dn / (phase_ms[3] / 1e3) / 1e12, 1)}

    res = {"metric": METRIC, "value": round(value, 1), "unit": "tok/s", "n_gpus": ws,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 4),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "f16 (exact NVFP4 dequant, FP32 accumulate)", "data": "synthetic",
           "config": {"workload": f"{wl.name}: {wl.note}", "tokens_per_rank": T,
                      "experts_used": n_used,
                      "l2": "inputs larger than L2 (1.27 GiB of expert planes per layer)",
                      "parallelism": f"replicas x{ws}"},
           "roofline": roof, "phases": phases, "clocks": clk.summary(),
           "gpu_launches": prefill_launches(d) * args.steps,
           "gpu_launches_by_region": {"prefill_device_timed": prefill_launches(d) * args.steps}}

    if wl.act == "int8":
        # the same tokens through the BF16-activation path (informational)
        xf = synth.make_x_f32(T, d.H, synth.workload_seed(wl), outliers=wl.outliers, device=dev)
        ob = m.forward(xf.to(torch.bfloat16), logits=logits)
        oi = m.forward(x, logits=logits, x_scale=xs)
        res["w4a8_vs_bf16_rel_l2"] = round(float(torch.linalg.vector_norm((oi - ob).double()) /
                                                 torch.linalg.vector_norm(ob.double())), 5)
        del xf, ob, oi

    # ---- end to end: host buffers, copies inside the timed region. Every step
    # copies its inputs from pinned host memory and reads its output back; the
    # copies of neighbouring steps overlap the layer (H2D, compute and D2H on
    # three streams, two device input/output buffers, events guarding reuse),
    # as a serving loop would run it.
    if not args.no_e2e:
        xh = x.cpu().pin_memory()
        lh = logits.cpu().pin_memory()
        xsh = xs.cpu().pin_memory() if xs is not None else None
        ohs = [torch.empty(T, d.H, dtype=torch.float32).pin_memory() for _ in range(2)]
        xds = [torch.empty_like(x) for _ in range(2)]
        lds = [torch.empty_like(logits) for _ in range(2)]
        xsds = [torch.empty_like(xs) if xs is not None else None for _ in range(2)]
        outs = [out, torch.empty_like(out)]
        m.set_phase_events(())      # no per-phase records in this loop
        # one workspace: every forward runs on the compute stream, one at a time
        s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()
        in_ready = [ev(), ev()]     # inputs of buffer b copied
        in_free = [ev(), ev()]      # compute done reading inputs of buffer b
        out_ready = [ev(), ev()]    # output of buffer b computed
        out_free = [ev(), ev()]     # output of buffer b copied back
        for e_ in in_free + out_free:
            e_.record(torch.cuda.current_stream())

        def e2e_step(i):
            bb = i & 1
            with torch.cuda.stream(s_in):
                s_in.wait_event(in_free[bb])
                xds[bb].copy_(xh, non_blocking=True)
                lds[bb].copy_(lh, non_blocking=True)
                if xsh is not None:
                    xsds[bb].copy_(xsh, non_blocking=True)
                in_ready[bb].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(in_ready[bb])
                s_cmp.wait_event(out_free[bb])
                m.forward(xds[bb], logits=lds[bb], x_scale=xsds[bb], out=outs[bb], workspace=ws_buf,
                          stream=s_cmp)
                in_free[bb].record(s_cmp)
                out_ready[bb].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(out_ready[bb])
                ohs[bb].copy_(outs[bb], non_blocking=True)
                out_free[bb].record(s_out)

        for i in range(max(1, args.warmup)):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier(ws)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s_in)
        for i in range(args.steps):
            e2e_step(i)
        s_in.wait_stream(s_out)
        b.record(s_in)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(b), ws)
        st = m.status()
        if st != 0:
            raise RuntimeError(f"device status {st} after the end-to-end steps")
        h2d = xh.numel() * xh.element_size() + lh.numel() * 4 + (xsh.numel() * 4 if xsh is not None else 0)
        res["e2e"] = {"value": round(ws * T * args.steps / (e_ms / 1e3), 1), "unit": "tok/s",
                      "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(ohs[0].numel() * 4),
                      "ms_per_step": round(e_ms / args.steps, 4),
                      "schedule": "H2D, layer and D2H on three streams, double-buffered across steps"}
        res["gpu_launches"] += prefill_launches(d) * args.steps
        res["gpu_launches_by_region"]["prefill_e2e_timed"] = prefill_launches(d) * args.steps

    # ---- decode expert GB/s (8 distinct layers so the L2 never holds the weights)
    if not args.no_decode:
        res["decode"] = run_decode(args, dev, pk, pk_src)
        n_dec = sum(v["timed_launches"] for k, v in res["decode"].items() if k.startswith("T"))
        res["gpu_launches"] += n_dec
        res["gpu_launches_by_region"]["decode_timed"] = n_dec

    # ---- CPU oracle baseline (rank 0, N = 1 only)
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = oracle_baseline(layer.to("cpu"), x.cpu(), logits.cpu(), d.K, T,
                                              args.cpu_seconds,
                                              xs.cpu() if xs is not None else None)
    m.close()
    return res


def run_decode(args, dev, pk, pk_src):
    """Decode expert streaming, T in {1,2,4,8}: one step = the layer over each of
    `decode_layers` distinct layers (so the L2 never holds the weights), captured
    once as a CUDA graph and replayed."""
    import nvfp4_mixture_experts_03_b200 as nv
    wl = synth.CONFIGS["decode"]
    d = wl.dims
    nl = args.decode_layers
    per_expert = (3 * d.I * d.H) // 2 + (3 * d.I * d.H) // 16
    layers = [synth.make_layer(d, synth.workload_seed(wl, l), device=dev) for l in range(nl)]
    models = [nv.MoELayer.from_layer(L, top_k=d.K, max_tokens=8) for L in layers]
    out = {}
    reps = max(args.steps, 50)
    for T in wl.tokens:
        xs = [synth.make_x_bf16(T, d.H, synth.workload_seed(wl, l) + 17 * T, outliers=True, device=dev)
              for l in range(nl)]
        lg = [synth.make_logits(T, d.E, synth.workload_seed(wl, l) + 17 * T, zipf_s=wl.zipf_s,
                                device=dev) for l in range(nl)]
        outs = [torch.empty(T, d.H, dtype=torch.float32, device=dev) for _ in range(nl)]
        uniq = 0
        for l in range(nl):
            dbg = nv.debug_buffers(T, d.E, d.K, dev)
            models[l].forward(xs[l], logits=lg[l], out=outs[l], debug=dbg)
            uniq += int((dbg["counts"] > 0).sum().item())
        ws_bufs = [mm.workspace(T) for mm in models]
        stream = torch.cuda.Stream()
        stream.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                for l in range(nl):
                    models[l].forward(xs[l], logits=lg[l], out=outs[l], workspace=ws_bufs[l], stream=stream)
            stream.synchronize()
            # no phase events inside the timed graph: event nodes would serialise the
            # programmatic-dependent launches and add their own cost
            with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
                for l in range(nl):
                    models[l].forward(xs[l], logits=lg[l], out=outs[l], workspace=ws_bufs[l], stream=stream)
        torch.cuda.current_stream().wait_stream(stream)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            g.replay()
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / reps
        for l in range(nl):
            if models[l].status() != 0:
                raise RuntimeError(f"decode layer {l} status {models[l].status()}")
        del g
        nbytes = uniq * per_expert
        gbs = nbytes / (ms / 1e3) / 1e9
        out[f"T{T}"] = {"layers": nl, "unique_experts": uniq, "bytes": nbytes,
                        "layer_us": round(ms * 1e3 / nl, 2), "GBps": round(gbs, 1),
                        "frac": round(gbs / pk["hbm_gbs"], 4), "timed_launches": reps * nl}
    out["peak"] = {"hbm_gbs": pk["hbm_gbs"], "source": pk_src}
    out["timing"] = (f"CUDA graph of the {nl}-layer step (one kernel per layer, programmatic "
                     f"dependent launch between layers), replayed {reps} times; bytes = unique "
                     f"selected experts x {per_expert:,} B")
    for mm in models:
        mm.close()
    return out


def profile_traffic(kernel_key, workload):
    """DRAM bytes per launch of `kernel_key` on `workload` from the committed ncu
    summaries (the fenced json block of profiles/*.md), or None when a source the
    kernel is built from changed since the counters were taken."""
    import glob
    import hashlib
    import re
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        m = re.search(r"```json\n(.*?)\n```", open(path).read(), re.S)
        if not m:
            continue
        try:
            rec = json.loads(m.group(1)).get("traffic", {}).get(kernel_key)
        except ValueError:
            continue
        if not rec or rec.get("workload") != workload:
            continue
        h = hashlib.sha256()
        for src in rec["sources"]:
            h.update(open(os.path.join(ROOT, src), "rb").read())
        if h.hexdigest()[:16] == rec["sources_sha256_16"]:
            return rec["dram_bytes_per_launch"]
    return None


def run_stack(args, ws, rank, local):
    """48 stacked layers (independent seeds), x <- x + layer(bf16(x)) carried in
    FP32 in place. Prefill: one step = the 4096-token chunk through all 48 layers.
    Decode: T = 1..4 through all 48 layers, captured as one CUDA graph."""
    import nvfp4_mixture_experts_03_b200 as nv
    dev = torch.device("cuda", local)
    pk, pk_src = peaks()
    wl = synth.CONFIGS["stack48"]
    d = wl.dims
    t0 = time.perf_counter()
    layers = [synth.make_layer(d, synth.workload_seed(wl, l), device=dev) for l in range(wl.layers)]
    gen_s = time.perf_counter() - t0
    Tp = 4096
    models = [nv.MoELayer.from_layer(L, top_k=d.K, max_tokens=Tp) for L in layers]
    wsb = models[0].workspace(Tp)                  # one workspace shared by the sequential layers
    lgp = [synth.make_logits(Tp, d.E, synth.workload_seed(wl, l) + 202, zipf_s=wl.zipf_s, device=dev)
           for l in range(wl.layers)]
    x0 = synth.make_x_f32(Tp, d.H, synth.workload_seed(wl) + 2, outliers=False, device=dev).contiguous()
    x = x0.clone()

    def step():
        x.copy_(x0)
        for l in range(wl.layers):
            models[l].forward(x, logits=lgp[l], out=x, accumulate=True, workspace=wsb)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(ws)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    steps = max(1, args.steps // 20)
    with Clocks(dev.index) as clk:
        a.record()
        for _ in range(steps):
            step()
        b.record()
        torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), ws) / steps
    for mm in models:
        assert mm.status() == 0
    flops = 2.0 * Tp * d.K * 3 * d.I * d.H * wl.layers
    res = {"metric": METRIC, "value": round(ws * Tp / (ms / 1e3), 1), "unit": "tok/s",
           "n_gpus": ws, "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "f16 (exact NVFP4 dequant, FP32 accumulate)", "data": "synthetic",
           "config": {"workload": f"stack48: {wl.note}; prefill chunk {Tp} tokens",
                      "resident_expert_bytes": sum(L.nbytes() for L in layers),
                      "generation_s": round(gen_s, 1),
                      "l2": "inputs larger than L2 (61 GiB of expert planes)"},
           "stack_tflops": round(flops / (ms / 1e3) / 1e12, 1), "clocks": clk.summary(),
           "gpu_launches": prefill_launches(wl.dims) * wl.layers * steps,
           "gpu_launches_by_region": {"prefill_device_timed": prefill_launches(wl.dims) * wl.layers * steps}}
    # whole-step throughput of all the layer's kernels against the sustained GEMM
    # peak (a step of 48 layers runs for tens of milliseconds under the power cap)
    sus = pk.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    res["roofline"] = {"kernel": "all kernels of the 48-layer prefill step", "bound": "tensor",
                       "achieved": res["stack_tflops"], "peak": sus, "unit": "TFLOP/s",
                       "frac": round(res["stack_tflops"] / sus, 4), "traffic": None,
                       "peak_source": f"{pk_src} bf16_tflops_sustained",
                       "algorithmic_flops_per_step": flops}
    # end to end: the chunk's FP32 hidden states from pinned host memory, the 48
    # layers, the result back to pinned host memory, all inside the timed region
    xh = x0.cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()

    def e2e_step():
        x.copy_(xh, non_blocking=True)
        for l in range(wl.layers):
            models[l].forward(x, logits=lgp[l], out=x, accumulate=True, workspace=wsb)
        oh.copy_(x, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    a.record()
    for _ in range(steps):
        e2e_step()
    b.record()
    torch.cuda.synchronize()
    e_ms = max_over_ranks(a.elapsed_time(b), ws) / steps
    for mm in models:
        assert mm.status() == 0
    res["e2e"] = {"value": round(ws * Tp / (e_ms / 1e3), 1), "unit": "tok/s",
                  "h2d_bytes_per_step": int(xh.numel() * 4), "d2h_bytes_per_step": int(oh.numel() * 4),
                  "ms_per_step": round(e_ms, 3),
                  "schedule": "H2D, 48 layers, D2H on one stream (logits stay resident)"}
    res["gpu_launches"] += prefill_launches(wl.dims) * wl.layers * steps
    res["gpu_launches_by_region"]["prefill_e2e_timed"] = prefill_launches(wl.dims) * wl.layers * steps
    # decode through the whole stack, T = 1..4, one CUDA graph per T
    per_expert = (3 * d.I * d.H) // 2 + (3 * d.I * d.H) // 16
    dec = {}
    for T in (1, 2, 3, 4):
        xd0 = synth.make_x_f32(T, d.H, synth.workload_seed(wl) + 1 + T, outliers=False, device=dev).contiguous()
        xd = xd0.clone()
        lgd = [synth.make_logits(T, d.E, synth.workload_seed(wl, l) + 101 + T, zipf_s=wl.zipf_s,
                                 device=dev) for l in range(wl.layers)]
        uniq = 0
        for l in range(wl.layers):
            dbg = nv.debug_buffers(T, d.E, d.K, dev)
            models[l].forward(xd, logits=lgd[l], out=xd, accumulate=True, workspace=wsb, debug=dbg)
            uniq += int((dbg["counts"] > 0).sum().item())
        st = torch.cuda.Stream()
        st.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(st):
            with torch.cuda.graph(g, stream=st, capture_error_mode="thread_local"):
                xd.copy_(xd0)
                for l in range(wl.layers):
                    models[l].forward(xd, logits=lgd[l], out=xd, accumulate=True, workspace=wsb, stream=st)
        torch.cuda.current_stream().wait_stream(st)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        reps = 20
        a.record()
        for _ in range(reps):
            g.replay()
        b.record()
        torch.cuda.synchronize()
        dms = a.elapsed_time(b) / reps
        gbs = uniq * per_expert / (dms / 1e3) / 1e9
        dec[f"T{T}"] = {"tokens_per_s": round(T / (dms / 1e3), 1), "ms_per_token_step": round(dms, 3),
                        "unique_experts": uniq, "GBps": round(gbs, 1), "frac": round(gbs / pk["hbm_gbs"], 4),
                        "timed_launches": reps * wl.layers}
        del g
        xg = xd.clone()   # the per-layer graph's result
        # the same 48 layers as ONE kernel launch (nvfp4_moe_forward_decode_stack)
        lga = torch.stack(lgd).contiguous()
        for _ in range(3):
            xd.copy_(xd0)
            nv.decode_stack(models, xd, lga, workspace=wsb)
        torch.cuda.synchronize()
        a.record()
        for _ in range(reps):
            xd.copy_(xd0)
            nv.decode_stack(models, xd, lga, workspace=wsb)
        b.record()
        torch.cuda.synchronize()
        assert models[0].status() == 0
        pms = a.elapsed_time(b) / reps
        pgbs = uniq * per_expert / (pms / 1e3) / 1e9
        dec[f"T{T}"]["one_launch"] = {"tokens_per_s": round(T / (pms / 1e3), 1),
                                      "ms_per_token_step": round(pms, 3), "GBps": round(pgbs, 1),
                                      "frac": round(pgbs / pk["hbm_gbs"], 4), "timed_launches": reps,
                                      "same_bits_as_per_layer": bool(torch.equal(xg, xd))}
    dec["peak"] = {"hbm_gbs": pk["hbm_gbs"], "source": pk_src}
    res["decode_stack"] = dec
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        # layer 0 on its own input bf16(x0), the stack's first step
        res["cpu_baseline"] = oracle_baseline(layers[0].to("cpu"), x0.to(torch.bfloat16).cpu(),
                                              lgp[0].cpu(), d.K, Tp, args.cpu_seconds,
                                              layers=wl.layers)
    n_dec = sum(v["timed_launches"] + v["one_launch"]["timed_launches"]
                for k, v in dec.items() if k.startswith("T"))
    res["gpu_launches"] += n_dec
    res["gpu_launches_by_region"]["decode_timed"] = n_dec
    for mm in models:
        mm.close()
    return res


# --------------------------------------------------------- reference (oracle) arm

def run_reference(args, ws, rank):
    if rank != 0:
        return None
    # the 48-layer stack's layers have the 8K layer's shape: the oracle's cost per
    # token and layer is the same, so its stack rate is the layer rate / 48
    per_layers = 48 if args.workload == "stack48" else 1
    wl = synth.CONFIGS["prefill8k" if args.workload == "stack48" else args.workload]
    d = wl.dims
    seed = synth.workload_seed(wl)
    T = wl.tokens[0]
    n = args.ref_tokens
    gen_dev = "cuda" if torch.cuda.is_available() else "cpu"   # same draw as the GPU arm
    layer = synth.make_layer(d, seed, device=gen_dev).to("cpu")
    logits = synth.make_logits(T, d.E, seed, zipf_s=wl.zipf_s, device=gen_dev).cpu()
    if wl.act == "int8":
        x, xs = synth.make_x_int8(T, d.H, seed, outliers=wl.outliers, device=gen_dev)
        x, xs = x.cpu(), xs.cpu()
    else:
        x, xs = synth.make_x_bf16(T, d.H, seed, outliers=wl.outliers, device=gen_dev).cpu(), None
    for _ in range(args.warmup):
        cpu_oracle_rate(layer, x, logits, d.K, n, xs)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        cpu_oracle_rate(layer, x, logits, d.K, n, xs)
    dt = time.perf_counter() - t0
    v = n * args.steps / dt / per_layers
    return {"impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": "tok/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt * 1e3 / args.steps, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{wl.name}: {wl.note}", "tokens_per_step": n},
            "cpu_baseline": {"value": round(v, 3), "unit": "tok/s", "cores": oracle_threads(n),
                             "cpu_model": cpu_model(), "kind": "oracle",
                             "sample": f"first {n} tokens of the {T}-token chunk per step"
                                       + (", one layer; rate divided by 48 layers" if per_layers > 1 else "")},
            "e2e": {"value": round(v, 3), "unit": "tok/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def ncu_target(case):
    """A few forwards of one case on cuda:0, for an ncu capture (-k selects the
    kernel, -s skips the first launches). prefill8k: 3 forwards of the 8192-token
    chunk; decode8: 6 forwards of 8 tokens on the decode layer; router8k /
    router8: 3 forwards of 8192 / 8 tokens whose logits come from the layer's
    router projection (BF16 W_r [512][2048])."""
    import nvfp4_mixture_experts_03_b200 as nv
    dev = torch.device("cuda", 0)
    wl = synth.CONFIGS["prefill8k" if case in ("prefill8k", "router8k") else "decode"]
    d = wl.dims
    seed = synth.workload_seed(wl)
    layer = synth.make_layer(d, seed, device=dev)
    T = wl.tokens[0] if case in ("prefill8k", "router8k") else 8
    x = synth.make_x_bf16(T, d.H, seed, outliers=wl.outliers, device=dev)
    logits = synth.make_logits(T, d.E, seed, zipf_s=wl.zipf_s, device=dev)
    wr = synth.make_router_w(d.E, d.H, seed, device=dev) if case.startswith("router") else None
    m = nv.MoELayer.from_layer(layer, top_k=d.K, max_tokens=T)
    out = torch.empty(T, d.H, device=dev)
    ws = m.workspace(T)
    for _ in range(6 if case == "decode8" else 3):
        if wr is None:
            m.forward(x, logits=logits, out=out, workspace=ws)
        else:
            m.forward(x, router_w=wr, out=out, workspace=ws)
    torch.cuda.synchronize()
    st = m.status()
    m.close()
    if st != 0:
        raise RuntimeError(f"device status {st}")
    print("ok", case, flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="prefill8k", choices=["prefill8k", "w4a8_32k", "stack48"])
    ap.add_argument("--decode-layers", type=int, default=8)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-tokens", type=int, default=16)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--decode-only", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-subrecords", action="store_true",
                    help="skip the 32K W4A8 and 48-layer stack sub-records of the default run")
    ap.add_argument("--ncu-target", choices=["prefill8k", "decode8", "router8k", "router8"],
                    help="profiling aid: a few untimed forwards of one case (for ncu), no JSON")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.ncu_target:
        ncu_target(args.ncu_target)
        return
    ws, rank, local = dist_setup()
    if args.impl == "reference":
        res = run_reference(args, ws, rank)
    elif args.workload == "stack48":
        res = run_stack(args, ws, rank, local)
    else:
        res = run_ours(args, ws, rank, local)
        # The default single-GPU run also carries the other two timed configurations
        # as sub-records: the 32768-token W4A8 chunk and the 48-layer stack.
        if args.workload == "prefill8k" and ws == 1 and not args.no_subrecords and not args.decode_only:
            torch.cuda.empty_cache()
            sub = argparse.Namespace(**vars(args))
            sub.workload, sub.no_decode, sub.steps = "w4a8_32k", True, max(5, min(args.steps, 40))
            res["w4a8_32k"] = run_ours(sub, ws, rank, local)
            torch.cuda.empty_cache()
            sub = argparse.Namespace(**vars(args))
            sub.workload, sub.steps = "stack48", max(20, min(args.steps, 100))
            res["stack48"] = run_stack(sub, ws, rank, local)
            torch.cuda.empty_cache()
            for k in ("w4a8_32k", "stack48"):
                res["gpu_launches"] += res[k]["gpu_launches"]
                res["gpu_launches_by_region"][k] = res[k]["gpu_launches"]
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
