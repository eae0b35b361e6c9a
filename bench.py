#!/usr/bin/env python
"""Benchmark of the MoE decode layer on B200: µs per layer and weight-stream
HBM GB/s (fraction of the measured peak), batch 1 / 8 / 64.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kd|reference]

One step = one pass of the whole layer (QKV projection, o-proj + residual,
router + top-k, shared expert on its side stream, routed experts, combine)
over one batch of synthetic input already resident in HBM.  The headline
line is the M=1 layer with H=7168 (256 routed experts, top-8, I=2048, bf16
weights); the M=8 verify, M=64 Zipf and 4-layer FP8 graph-stack workloads
are reported under "workloads".  L2 is flushed (256 MiB write) before every
timed step, outside the timed window.  With N > 1 (torchrun) every rank runs
an independent replica (the layer does not shard on one GPU's worth of work);
`value` is the whole-job µs per layer = max-over-ranks time / (N x layers).

--impl reference times the CPU oracle (fp64 C, the correctness reference) on
the same workload, on the host cores, rank 0 only.
"""
from __future__ import annotations

import argparse
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

METRIC = "µs per MoE decode layer & weight-stream HBM GB/s (% of peak), batch 1/8/64"
UNIT = "us/layer"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from the committed ncu capture, or None
    when there is none for this kernel/workload or its sources changed since."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        if t["kernel"] != kernel or not t["workload"].startswith(workload):
            return None
        h = hashlib.sha256()
        for src in t["source_files"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        return t["dram_bytes_per_launch"] if h.hexdigest()[:16] == t["source_sha256_16"] else None
    except Exception:
        return None


def load_peak():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, torch copy)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s"


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms while active."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines: list[str] = []
        self.thread = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.25)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self) -> dict:
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- distributed

def dist_setup(n_gpus: int):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if ws > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        pg = dist
    return ws, rank, local, pg


def _nccl(pg) -> bool:
    return pg is not None and pg.get_backend() == "nccl"


def barrier(pg, local):
    """All ranks meet (NCCL on the GPU machine; gloo in the CPU tests), then the
    local device drains."""
    import torch
    if pg is not None:
        if _nccl(pg):
            pg.barrier(device_ids=[local])
        else:
            pg.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def max_over_ranks(pg, value: float) -> float:
    if pg is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device="cuda" if _nccl(pg) else "cpu")
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_us_per_layer(ms_max: float, world_size: int, layers: int = 1) -> float:
    """Whole-job µs per layer: the slowest rank's step time over the layers
    all ranks processed in it (weak scaling: every rank runs its own step)."""
    return ms_max * 1e3 / (world_size * layers)


# --------------------------------------------------------------------------- kd arm

def to_dev_bf16(bits: np.ndarray):
    import torch
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).cuda().contiguous()


class L2Flush:
    """Write a buffer of 2x L2, then read another one, so that the step starts
    with no useful line in L2 and no dirty line left to write back."""

    def __init__(self):
        import torch
        l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
        n = max(2 * l2, 256 << 20)
        self.buf = torch.empty(n, dtype=torch.uint8, device="cuda")
        self.buf2 = torch.ones(n // 4, dtype=torch.float32, device="cuda")
        self.sink = torch.empty((), dtype=torch.float32, device="cuda")
        self.n = 0

    def __call__(self):
        import torch
        self.n += 1
        self.buf.fill_(self.n & 0xFF)
        torch.amax(self.buf2, dim=0, out=self.sink)


def layer_bytes(layer, n_active: int) -> int:
    st, ex = layer.bytes()
    return st + n_active * ex


def kernel_bytes(spec, n_active: int) -> dict:
    """Algorithmic weight bytes each main-stream kernel must read per call."""
    eb = 2 if spec.wdtype == 0 else 1
    H, I, E = spec.hidden, spec.inter, spec.n_experts
    A = spec.q_heads * spec.head_dim
    nq = (spec.q_heads + 2 * spec.kv_heads) * spec.head_dim
    sc = 0 if spec.wdtype == 0 else 4
    blk = lambda r, k: ((r + 127) // 128) * ((k + 127) // 128) * sc
    return {
        "proj": (nq * H + H * A) * eb + blk(nq, H) + blk(H, A),
        "router": E * H * eb + blk(E, H),
        "gateup": n_active * (2 * I * H * eb + 2 * blk(I, H)),
        "down": (n_active + spec.n_shared) * (H * I * eb + blk(H, I)),
    }


KNAMES = ("proj", "router", "gateup", "down")
SWEEP_M = (1, 2, 3, 4, 5, 6, 7, 8, 16, 32, 64)


def time_layer(layer, x_bits, a_bits, steps, warmup, flush, pg, local, per_kernel=True):
    """Device-timed single-layer steps (L2 flushed before each, input reset)."""
    import torch
    import moe_decode_layer_skinny_b200 as kd
    x0 = to_dev_bf16(x_bits)
    hidden = x0.clone()
    attn = to_dev_bf16(a_bits)
    M = x_bits.shape[0]
    s = torch.cuda.current_stream()
    for _ in range(warmup):
        hidden.copy_(x0)
        flush()
        layer.decode(hidden, attn, M)
    torch.cuda.synchronize()
    layer.check()
    start = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    end = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(kd.N_TIMING_EVENTS)]
           for _ in range(steps)] if per_kernel else None
    if per_kernel:
        for evs in kev:          # torch creates the CUDA event on its first record
            for e in evs:
                e.record(s)
    barrier(pg, local)
    for i in range(steps):
        hidden.copy_(x0)
        flush()
        if per_kernel:
            layer.set_timing_events(kev[i])
        start[i].record(s)
        layer.decode(hidden, attn, M)
        end[i].record(s)
    barrier(pg, local)
    if per_kernel:
        layer.set_timing_events(None)
    layer.check()
    times = [a.elapsed_time(b) for a, b in zip(start, end)]
    kt = None
    if per_kernel:
        kt = {n: statistics.mean(kev[i][j].elapsed_time(kev[i][j + 1]) for i in range(steps))
              for j, n in enumerate(KNAMES)}
    return times, kt


def time_layer_e2e(layer, x_bits, a_bits, steps, warmup, flush, pg, local):
    """Same step through the C ABI from pinned host buffers: H2D inputs, layer,
    D2H output, all inside the timed window."""
    import torch
    M = x_bits.shape[0]
    hx = torch.from_numpy(x_bits.view(np.int16).copy()).view(torch.bfloat16).pin_memory()
    ha = torch.from_numpy(a_bits.view(np.int16).copy()).view(torch.bfloat16).pin_memory()
    hout = torch.empty_like(hx).pin_memory()
    hidden = torch.empty(hx.shape, dtype=torch.bfloat16, device="cuda")
    attn = torch.empty(ha.shape, dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.current_stream()

    def step():
        hidden.copy_(hx, non_blocking=True)
        attn.copy_(ha, non_blocking=True)
        layer.decode(hidden, attn, M)
        hout.copy_(hidden, non_blocking=True)

    for _ in range(warmup):
        flush()
        step()
    torch.cuda.synchronize()
    start = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    end = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier(pg, local)
    for i in range(steps):
        flush()
        start[i].record(s)
        step()
        end[i].record(s)
    barrier(pg, local)
    layer.check()
    times = [a.elapsed_time(b) for a, b in zip(start, end)]
    return times, hx.numel() * 2 + ha.numel() * 2, hout.numel() * 2


class _DeviceView:
    def __init__(self, ptr: int, n: int):
        self.__cuda_array_interface__ = {"shape": (n,), "typestr": "<i4", "data": (int(ptr), False),
                                         "version": 3, "strides": None}


def n_active_of(layer) -> int:
    """Experts the last call touched (layer-owned device counter)."""
    import torch

    import moe_decode_layer_skinny_b200 as kd
    torch.cuda.synchronize()
    return int(torch.as_tensor(_DeviceView(layer.debug_ptr(kd.T_NACTIVE), 1), device="cuda").item())


def make_layer(w, layer_id=0):
    import moe_decode_layer_skinny_b200 as kd
    spec = kd.LayerSpec.from_dims(w.dims, wdtype=w.wdtype, layer_id=layer_id, max_tokens=w.M,
                                  router_bias=w.bias())
    return kd.Layer(spec, seed=w.seed)


def with_experts(w, n_experts: int):
    """The workload with fewer routed experts (same shapes per expert, same
    top-k): a small device footprint for profiling captures."""
    import dataclasses
    if not n_experts:
        return w
    d = dataclasses.replace(w.dims, n_experts=n_experts)
    return dataclasses.replace(w, dims=d, name=f"{w.name}_e{n_experts}",
                               zipf_s=w.zipf_s)


def bench_single(w, steps, warmup, flush, pg, local, peak):
    layer = make_layer(w)
    try:
        x, a = w.hidden_in(), w.attn_out()
        # the layer as it runs (kernels chained by programmatic dependent launch)
        times, _ = time_layer(layer, x, a, steps, warmup, flush, pg, local, per_kernel=False)
        # per-kernel durations from a separate pass with events between kernels
        # (the hook launches each kernel only after the previous one finished)
        _, kt = time_layer(layer, x, a, max(steps // 4, 5), 2, flush, pg, local, per_kernel=True)
        na = n_active_of(layer)
        ms = statistics.mean(times)
        byts = layer_bytes(layer, na)
        kb = kernel_bytes(layer.spec, na)
        res = {"us_per_layer": ms * 1e3, "p10_us": float(np.percentile(times, 10)) * 1e3,
               "p90_us": float(np.percentile(times, 90)) * 1e3, "M": w.M,
               "active_experts": na, "weight_bytes": byts,
               "hbm_gbs": byts / (ms * 1e-3) / 1e9, "tok_s": w.M / (ms * 1e-3)}
        res["hbm_frac"] = res["hbm_gbs"] / peak
        res["expert_bytes"] = layer.bytes()[1]
        res["kernels_us"] = {n: kt[n] * 1e3 for n in KNAMES}
        res["kernels_gbs"] = {n: (kb[n] / (kt[n] * 1e-3) / 1e9 if kb[n] else None) for n in KNAMES}
        return res, layer, x, a, kb, kt
    except Exception:
        layer.close()
        raise


def bench_stack(w, steps, warmup, flush, pg, local, peak, prefetch):
    import torch

    import moe_decode_layer_skinny_b200 as kd
    layers = [make_layer(w, l) for l in range(w.n_layers)]
    try:
        st = kd.Stack(layers, w.M, prefetch=prefetch)
        x0 = to_dev_bf16(w.hidden_in())
        attn = to_dev_bf16(np.concatenate([w.attn_out(l) for l in range(w.n_layers)]))
        hidden = x0.clone()
        s = torch.cuda.current_stream()
        for _ in range(warmup):
            hidden.copy_(x0)
            flush()
            st.run(hidden, attn)
        torch.cuda.synchronize()
        for L in layers:
            L.check()
        start = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        end = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        barrier(pg, local)
        for i in range(steps):
            hidden.copy_(x0)
            flush()
            start[i].record(s)
            st.run(hidden, attn)
            end[i].record(s)
        barrier(pg, local)
        times = [a.elapsed_time(b) for a, b in zip(start, end)]
        # bytes: each layer's unique weights under the routing of its own input
        byts = 0
        hidden.copy_(x0)
        per_layer = []
        for L, l in zip(layers, range(w.n_layers)):
            L.decode(hidden, attn[l * w.M:(l + 1) * w.M])
            na = n_active_of(L)
            per_layer.append(na)
            byts += layer_bytes(L, na)
        st0, ex0 = layers[0].bytes()
        st.close()
        ms = statistics.mean(times)
        return {"us_per_layer": ms * 1e3 / w.n_layers, "us_per_step": ms * 1e3,
                "M": w.M, "layers": w.n_layers, "weight_bytes": byts,
                "hbm_gbs": byts / (ms * 1e-3) / 1e9, "hbm_frac": byts / (ms * 1e-3) / 1e9 / peak,
                "tok_s": w.M / (ms * 1e-3), "l2_prefetch": bool(prefetch),
                "active_experts_per_layer": per_layer, "active_experts_layer0": per_layer[0],
                "layer0_bytes": (st0, ex0)}
    finally:
        for L in layers:
            L.close()


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


def _oracle_call(w, rows, threads, layer_id=0):
    import oracle
    import kdgen
    x = kdgen.bf16_bits_to_f32(w.hidden_in()[rows]).astype(np.float64)
    a = kdgen.bf16_bits_to_f32(w.attn_out(layer_id)[rows]).astype(np.float64)
    t0 = time.perf_counter()
    r = oracle.layer(w.dims, x, a, wdtype=w.wdtype, layer_id=layer_id,
                     bias=None if w.bias() is None else w.bias().astype(np.float64),
                     nthreads=threads, want_qkv=True)
    return time.perf_counter() - t0, len(np.unique(r["idx"]))


def cpu_baseline(w, threads, budget_s=15.0, rows=None, full_union=None, static_bytes=None,
                 expert_bytes=None):
    """The oracle as it stands (fp64 C, weights generated as it goes) on the
    host cores, timed on the workload's layer (layer 0 of a stack).  With
    `rows`, a bounded sample: only those token rows, scaled to the full layer
    by its weight bytes (the oracle's time is its weight generation, linear in
    the experts it touches): t_full = t_sample x (static + U_full expert) /
    (static + U_sample expert)."""
    rows = list(range(w.M)) if rows is None else list(rows)
    times, n_sample = [], 0
    t_end = time.time() + budget_s
    while not times or (time.time() < t_end and len(times) < 5):
        t, n_sample = _oracle_call(w, rows, threads)
        times.append(t)
    t = statistics.mean(times)
    res = {"threads": threads, "calls": len(times), "rows": len(rows), "sample_s": t}
    if len(rows) < w.M and full_union and static_bytes is not None:
        scale = (static_bytes + full_union * expert_bytes) / (static_bytes + n_sample * expert_bytes)
        res.update(us_per_layer=t * scale * 1e6, scaled=True, experts_sample=n_sample,
                   experts_full=full_union)
    else:
        res.update(us_per_layer=t * 1e6, scaled=False, experts=n_sample)
    return res


def cpu_baselines(workloads: dict, unions: dict, layer_bytes_by_wl: dict) -> dict:
    """Every workload's layer on all host cores (full layer) and on one core
    (the full layer when it is the M=1 one, else the first token row, scaled
    to the full layer by weight bytes)."""
    cores = os.cpu_count() or 1
    out = {"nproc": cores, "cpu_model": cpu_model(), "kind": "oracle", "unit": UNIT,
           "workloads": {}}
    for name, w in workloads.items():
        st, ex = layer_bytes_by_wl.get(name, (None, None))
        allc = cpu_baseline(w, cores, budget_s=10.0)
        one = cpu_baseline(w, 1, budget_s=5.0, rows=None if w.M == 1 else [0],
                           full_union=unions.get(name), static_bytes=st, expert_bytes=ex)
        out["workloads"][name] = {"all_cores": allc, "one_core": one}
    return out


def bench_sweep(dims, Ms, steps, flush, pg, local, peak) -> dict:
    """µs per layer, HBM fraction and launches at each token count M (one
    bf16 H=7168 layer; rows with 0.9 correlation at the verify shapes 4..8,
    independent otherwise)."""
    import moe_decode_layer_skinny_b200 as kd
    import kdgen
    spec = kd.LayerSpec.from_dims(dims, max_tokens=max(Ms))
    layer = kd.Layer(spec, seed=0)
    res = {}
    try:
        for M in Ms:
            rho = 0.9 if 4 <= M <= 8 else 0.0
            x = kdgen.activations(0, 0, kdgen.HIDDEN_IN, M, dims.hidden, rho)
            a = kdgen.activations(0, 0, kdgen.ATTN_OUT, M, dims.attn, rho)
            times, _ = time_layer(layer, x, a, steps, 3, flush, pg, local, per_kernel=False)
            na = n_active_of(layer)
            ms = statistics.mean(times)
            byts = layer_bytes(layer, na)
            res[str(M)] = {"us_per_layer": ms * 1e3, "active_experts": na, "weight_bytes": byts,
                           "hbm_gbs": byts / (ms * 1e-3) / 1e9,
                           "hbm_frac": byts / (ms * 1e-3) / 1e9 / peak,
                           "tok_s": M / (ms * 1e-3), "launches": layer.launches(M),
                           "rows": "correlated 0.9" if rho else "independent"}
    finally:
        layer.close()
    return res


def run_kd(args):
    import torch

    import kdgen
    import moe_decode_layer_skinny_b200 as kd
    ws, rank, local, pg = dist_setup(args.gpus)
    if ws == 1:
        torch.cuda.set_device(0)
    kd.lib()
    peak, peak_src = load_peak()
    flush = L2Flush()
    W = kdgen.WORKLOADS
    main = with_experts(W[args.workload], args.experts)
    res, layer, x, a, kb, kt = bench_single(main, args.steps, args.warmup, flush, pg, local, peak)
    dev_index = torch.cuda.current_device()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
    smi_index = int(vis[dev_index]) if len(vis) > dev_index and vis[dev_index].strip().isdigit() \
        else dev_index
    # clocks sampled during a second timed pass of the same workload (same code path)
    with ClockSampler(smi_index) as cs:
        t_end = time.time() + 1.0
        times = []
        while time.time() < t_end:
            tt, _ = time_layer(layer, x, a, max(args.steps, 50), 1, flush, pg, local,
                               per_kernel=False)
            times += tt
    clocks = cs.summary()
    e2e_times, h2d, d2h = time_layer_e2e(layer, x, a, min(args.steps, 200), args.warmup, flush, pg,
                                         local)
    launches_per_step = layer.launches(main.M)
    layer.close()
    ms = res["us_per_layer"] / 1e3
    ms_max = max_over_ranks(pg, ms)
    e2e_ms = max_over_ranks(pg, statistics.mean(e2e_times))
    out = {
        "metric": METRIC, "value": job_us_per_layer(ms_max, ws), "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded counter-based generator, random-init weights of the stated shapes",
        "config": {"workload": main.name, "desc": main.desc, "M": main.M, "hidden": main.dims.hidden,
                   "qkv": main.dims.nqkv, "attn": main.dims.attn, "experts": main.dims.n_experts,
                   "top_k": main.dims.top_k, "shared": main.dims.n_shared, "inter": main.dims.inter,
                   "weights": "bf16" if main.wdtype == 0 else "fp8-e4m3-128x128",
                   "parallelism": f"replicas x{ws}", "l2": "flushed before every timed step (2x L2 write)"},
        "hbm_gbs": res["hbm_gbs"], "hbm_frac": res["hbm_frac"], "hbm_peak_gbs": peak,
        "hbm_peak_src": peak_src, "tok_s": res["tok_s"] * ws,
        "active_experts": res["active_experts"], "weight_bytes_per_layer": res["weight_bytes"],
        "p10_us": res["p10_us"], "p90_us": res["p90_us"],
        "kernels_us": res["kernels_us"], "kernels_gbs": res["kernels_gbs"],
        "clocks": clocks,
        "e2e": {"value": job_us_per_layer(e2e_ms, ws), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
    }
    # dominant kernel of the main stream by time
    dom = max(KNAMES, key=lambda n: kt[n])
    ach = kb[dom] / (kt[dom] * 1e-3) / 1e9
    out["roofline"] = {"bound": "hbm", "kernel": dom, "achieved": ach, "peak": peak, "unit": "GB/s",
                       "frac": ach / peak, "traffic": profiled_traffic(dom, main.name),
                       "algorithmic_bytes_per_launch": kb[dom], "peak_src": peak_src}
    # secondary workloads
    unions = {main.name: res["active_experts"]}
    lbytes = {main.name: (res["weight_bytes"] - res["active_experts"] * res["expert_bytes"],
                          res["expert_bytes"])}
    if not args.main_only:
        wl = {}
        for name in ("verify8", "batch64_zipf"):
            r2, l2, *_ = bench_single(W[name], max(10, args.steps // 10), 3, flush, pg, local, peak)
            l2.close()
            wl[name] = r2
            unions[name] = r2["active_experts"]
            lbytes[name] = (r2["weight_bytes"] - r2["active_experts"] * r2["expert_bytes"],
                            r2["expert_bytes"])
        # the stack without and with the next layer's static weights prefetched
        # into L2 on a side stream (the pages' option; measured slightly slower
        # here, so the plain chain is the workload's line)
        for pf in (False, True):
            key = "stack4_fp8" + ("_prefetch" if pf else "")
            wl[key] = bench_stack(W["stack4_fp8"], max(5, args.steps // 20), 3, flush, pg, local,
                                  peak, pf)
        unions["stack4_fp8"] = wl["stack4_fp8"]["active_experts_layer0"]
        lbytes["stack4_fp8"] = wl["stack4_fp8"]["layer0_bytes"]
        out["workloads"] = wl
        out["sweep"] = bench_sweep(W["batch1"].dims, SWEEP_M, max(10, args.steps // 10), flush, pg,
                                   local, peak)
    if rank == 0 and ws == 1 and not args.no_cpu:
        names = [main.name] if args.main_only else ["batch1", "verify8", "batch64_zipf", "stack4_fp8"]
        cb = cpu_baselines({n: W[n] if n != main.name else main for n in names}, unions, lbytes)
        head = cb["workloads"][main.name]["all_cores"]
        out["cpu_baseline"] = {
            "value": head["us_per_layer"], "unit": UNIT, "cores": cb["nproc"], "kind": "oracle",
            "sample": f"{head['calls']} full {main.name} layer call(s) (M={main.M}), fp64 oracle "
                      f"generating its weights as it goes, {cb['nproc']} threads",
            "cpu_model": cb["cpu_model"], "per_workload": cb["workloads"]}
    if pg is not None:
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(out))


# --------------------------------------------------------------------------- reference arm

def run_reference(args):
    import kdgen
    import oracle
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = kdgen.WORKLOADS[args.workload]
    x = kdgen.bf16_bits_to_f32(w.hidden_in()).astype(np.float64)
    a = kdgen.bf16_bits_to_f32(w.attn_out()).astype(np.float64)
    cores = os.cpu_count() or 1
    bias = None if w.bias() is None else w.bias().astype(np.float64)
    budget = 150.0
    # one untimed warm-up call (page-in, thread start-up), then timed calls
    # until --steps are done or the time budget is spent
    oracle.layer(w.dims, x, a, wdtype=w.wdtype, bias=bias, nthreads=cores)
    t_start = time.time()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.layer(w.dims, x, a, wdtype=w.wdtype, bias=bias, nthreads=cores)
        times.append(time.perf_counter() - t0)
        if time.time() - t_start > budget:
            break
    done_w = 1
    ms = statistics.mean(times) * 1e3
    out = {
        "impl": "reference", "metric": METRIC, "value": ms * 1e3, "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "desc": w.desc, "M": w.M},
        "cpu_baseline": {"value": ms * 1e3, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{len(times)} timed full {w.name} layer call(s) of the fp64 "
                                   f"oracle ({done_w} untimed warm-up), capped at ~{budget:.0f} s"},
        "e2e": {"value": ms * 1e3, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out))


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("kd", "reference"), default="kd")
    ap.add_argument("--workload", default="batch1")
    ap.add_argument("--main-only", action="store_true", help="skip the secondary workloads")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--experts", type=int, default=0,
                    help="profiling only: routed experts of the main workload (default: its own)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_kd(args)


if __name__ == "__main__":
    main()
