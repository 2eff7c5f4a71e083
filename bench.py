"""Benchmark of the causal sliding-window GQA attention block on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cswa|reference]

One step is the whole hot path on one batch: for each layer of the nanochat-d20
shaped pair (B=8, T=2048, Hq=Hkv=10, D=128; a short layer with window 1024 and
a long layer with window 2048 = full causal) it runs the RoPE + QK-norm
prologue, attention forward, and the block backward (attention backward with the
prologue backward fused into its kernels: gradients w.r.t. the raw q, k, v).
`value` is useful fwd+bwd TFLOP/s: 12*D per visible (query, key) pair (the
pages' 3 x forward convention), masked work and recompute not counted. The
KV-cache decode workload (32 sequences, lengths U[512, 2048], window 1024) is
timed in the same run and reported under "decode" as HBM GB/s, and the
chunked-prefill workload (8 sequences, a 512-token chunk each on cache lengths
U[0, 1536], window 1024) under "prefill" as useful TFLOP/s, and the batch-1 -> 8
KV-cache replication of a 20-layer stack under "kv_replicate" as GB/s.

Under torchrun each rank runs its own batch (weak scaling, no collective on
the data path); times are the max over ranks. `--impl reference` times the
fp64 CPU oracle on a bounded sample of the same workload instead.
"""
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
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)
import workloads  # noqa: E402

METRIC = "attention fwd+bwd TFLOP/s (useful FLOPs) & % bf16 peak; decode HBM GB/s"
WORKLOAD = ("nanochat-d20 attention layer pair, fwd+bwd incl. RoPE+QK-norm prologue: B=8 T=2048 Hq=Hkv=10 "
            "D=128 bf16, windows 1024 (short layer) and 2048 (long layer)")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SUSTAINED_REGION_MS = 3000.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ distributed
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        import datetime
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def shard_seed(base_seed, rank):
    """Each rank draws its own batch: the global batch is world x B sequences."""
    return base_seed + 1000 * rank


# ------------------------------------------------------------------ FLOPs / bytes
def layer_useful_flops(B, T, Hq, D, W):
    n = B * Hq * workloads.visible_pairs(T, W)
    return 4.0 * D * n, 8.0 * D * n


def decode_bytes(lengths, Hq, Hkv, D, W):
    """Algorithmic HBM bytes of one decode step: the visible K and V rows, q, o,
    lse, the new k/v read and appended, and pos."""
    B = len(lengths)
    n = sum(min(int(p), W) + 1 if W >= 0 else int(p) + 1 for p in lengths)
    return (n * Hkv * D * 2 * 2 + B * Hq * D * 2 * 2 + B * Hq * 4 + 2 * B * Hkv * D * 2 * 2 + B * 4)


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons while running: through
    NVML every millisecond when the binding is present (NVML is set up when the sampler is
    made, before the timed region, so that a region of a few milliseconds still gets
    samples), else through nvidia-smi every 200 ms."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index):
        self.index = index
        self.rows = []  # (sm_mhz, max_mhz, [reason names])
        self.source = None
        self._stop = threading.Event()
        self._t = None
        self._nvml = None
        try:
            import pynvml
            pynvml.nvmlInit()
            h = self._nvml_handle(pynvml)
            bits = [pynvml.nvmlClocksEventReasonHwSlowdown, pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                    pynvml.nvmlClocksEventReasonSwThermalSlowdown, pynvml.nvmlClocksEventReasonSwPowerCap]
            mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self._nvml = (pynvml, h, bits, mx)
        except Exception:
            self._nvml = None

    def _nvml_handle(self, pynvml):
        try:
            uuid = str(torch.cuda.get_device_properties(self.index).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.index)

    def _run_nvml(self):
        pynvml, h, bits, mx = self._nvml
        self.source = "nvml, 1 ms"
        while not self._stop.is_set():
            sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
            r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
            self.rows.append((float(sm), float(mx), [n for n, b in zip(self.NAMES, bits) if r & b]))
            self._stop.wait(0.001)

    def _run_smi(self):
        self.source = "nvidia-smi, 200 ms"
        while not self._stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                                      "--format=csv,noheader,nounits"], capture_output=True, text=True,
                                     timeout=5).stdout.strip()
                r = [x.strip() for x in out.split(",")]
                if len(r) >= 9 and r[1].replace(".", "").isdigit():
                    self.rows.append((float(r[1]), float(r[2]),
                                      [n for i, n in enumerate(self.NAMES) if r[5 + i] == "Active"]))
            except Exception:
                pass
            self._stop.wait(0.2)

    def _run(self):
        if self._nvml is not None:
            try:
                return self._run_nvml()
            except Exception:
                pass
        self._run_smi()

    def __enter__(self):
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        self._t.join(timeout=10)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock samples"], "samples": 0}
        return {"sm_mhz": statistics.median(r[0] for r in self.rows), "sm_max_mhz": max(r[1] for r in self.rows),
                "reasons": sorted({n for r in self.rows for n in r[2]}), "samples": len(self.rows),
                "source": self.source}


# ------------------------------------------------------------------ GPU arm
def kernel_source_sha():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "causal_sliding_window_attn_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel):
    """dram bytes per launch from the committed ncu summary, if the kernel sources are unchanged."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel)
    if not d or d.get("csrc_sha") != kernel_source_sha():
        return None
    return d.get("dram_bytes_per_launch")


def flush_l2(buf):
    """Writes a 256 MB buffer (every L2 line is replaced), then reads it back, so that the
    dirty lines the write leaves are written back here and not during the timed call."""
    buf.add_(1)
    buf.amax()


def run_gpu(args, rank, world, local):
    import causal_sliding_window_attn_b200 as cswa
    cswa.lib()
    dev = torch.device("cuda", local)
    c = workloads.CONFIGS["d20"]
    B, T, Hq, Hkv, D = c["B"], c["T"], c["Hq"], c["Hkv"], c["D"]
    windows = c["windows"]
    scale = workloads.default_scale(D)
    q, k, v, do = (t.to(dev) for t in workloads.training_inputs(B, T, Hq, Hkv, D, shard_seed(c["seed"], rank)))
    # per-layer buffers (all outputs preallocated; the library allocates nothing)
    L = []
    for W in windows:
        L.append(dict(W=W, qh=torch.empty_like(q), kh=torch.empty_like(k), o=torch.empty_like(q),
                      lse=torch.empty((B, Hq, T), device=dev, dtype=torch.float32),
                      dv=torch.empty_like(v), dq=torch.empty_like(q), dk=torch.empty_like(k),
                      ws=torch.empty(cswa.attn_block_bwd_workspace_bytes(B, T, Hq, Hkv, D, W), device=dev,
                                     dtype=torch.uint8)))
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    per_op = {"prologue": 0.0, "fwd": 0.0, "bwd": 0.0}
    bwd_ms = [0.0, 0.0]

    def step(record):
        # per layer: the prologue (q, k -> q_hat, k_hat), the forward, and the block backward
        # (gradients w.r.t. the raw q, k: the prologue backward runs inside its kernels)
        for li, l in enumerate(L):
            e = [ev() for _ in range(4)] if record else None
            if record:
                e[0].record()
            cswa.attn_rope_qknorm(q, k, l["qh"], l["kh"])
            if record:
                e[1].record()
            cswa.attn_fwd(l["qh"], l["kh"], v, l["W"], scale, o=l["o"], lse=l["lse"])
            if record:
                e[2].record()
            cswa.attn_block_bwd(q, k, l["qh"], l["kh"], v, l["o"], do, l["lse"], l["W"], scale, dq=l["dq"],
                                dk=l["dk"], dv=l["dv"], workspace=l["ws"])
            if record:
                e[3].record()
                l["events"] = l.get("events", []) + [e]

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize()
    assert cswa.attn_get_status() == 0
    graph = None
    if not args.eager:
        # the step's launches captured once and replayed: the same kernels on the same
        # buffers, without the host's per-call work between them
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step(False)
        graph.replay()
        torch.cuda.synchronize()
        assert cswa.attn_get_status() == 0
    for l in L:
        l["events"] = []
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = ev(), ev()
    # the timed steps carry no events of their own (an event recorded between two launches
    # delays the second): the per-operation breakdown comes from a second, untimed pass
    with ClockSampler(local) as clocks:
        t0.record()
        for _ in range(args.steps):
            if graph is not None:
                graph.replay()
            else:
                step(False)
        t1.record()
        torch.cuda.synchronize()
    barrier(world)
    ms_total = t0.elapsed_time(t1)
    for _ in range(args.steps):
        step(True)
    torch.cuda.synchronize()
    for li, l in enumerate(L):
        for e in l["events"]:
            per_op["prologue"] += e[0].elapsed_time(e[1])
            per_op["fwd"] += e[1].elapsed_time(e[2])
            bwd_ms[li] += e[2].elapsed_time(e[3])
    per_op["bwd"] = sum(bwd_ms)
    status = cswa.attn_get_status()
    assert status == 0, f"device status {status}"

    ms_step = max_over_ranks(ms_total / args.steps, world)
    flops_f = sum(layer_useful_flops(B, T, Hq, D, W)[0] for W in windows)
    flops_b = sum(layer_useful_flops(B, T, Hq, D, W)[1] for W in windows)
    value = world * (flops_f + flops_b) / (ms_step * 1e-3) / 1e12

    pk, pk_src = peaks()
    peak_sus = pk.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    peak_burst = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    # A timed region of a few seconds or more runs into the power cap: the sustained
    # peak applies. A shorter one is a burst: the burst peak applies.
    long_region = ms_total >= SUSTAINED_REGION_MS
    peak_use = peak_sus if long_region else peak_burst
    peak_kind = (f"bf16 {'sustained' if long_region else 'burst'} ({pk_src}): timed region "
                 f"{ms_total / 1e3:.2f} s {'>=' if long_region else '<'} {SUSTAINED_REGION_MS / 1e3:.0f} s; "
                 f"burst {peak_burst}, sustained {peak_sus}")
    bwd_avg_ms = per_op["bwd"] / (2 * args.steps)
    bwd_tflops = flops_b / 2 / (bwd_avg_ms * 1e-3) / 1e12
    fwd_avg_ms = per_op["fwd"] / (2 * args.steps)
    # DRAM bytes of one attn_block_bwd call = its three launches (ncu, window-1024 layer)
    parts = [ncu_traffic(kn) for kn in ("attn_bwd_prep_kernel", "attn_bwd_kernel", "attn_bwd_dq_kernel")]
    traffic = sum(parts) if all(x is not None for x in parts) else None
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16 activations of the d20 shapes)",
        "config": {"workload": WORKLOAD, "global_batch": B * world, "seq_len": T, "parallelism": f"dp{world}",
                   "l2": "no flush: each layer's inputs (q,k,v,dO: 168 MB) exceed the 126 MB L2",
                   "launch": "eager, one C-ABI call at a time" if graph is None else
                   "one CUDA graph of the step's 10 launches, replayed once per step"},
        "pct_bf16_peak": {"of_sustained": round(value / world / peak_sus, 4),
                          "of_burst": round(value / world / peak_burst, 4), "peaks": pk_src,
                          "applies": "sustained" if long_region else "burst"},
        "breakdown_ms_per_step": {k2: round(v2 / args.steps, 4) for k2, v2 in per_op.items()},
        "fwd_tflops": round(flops_f / 2 / (fwd_avg_ms * 1e-3) / 1e12, 1),
        "bwd_tflops": round(bwd_tflops, 1),
        "bwd_tflops_fa_convention": round(bwd_tflops * 10 / 8, 1),
        "roofline": {"kernel": "attn_block_bwd call (prep + main + dq launches, prologue backward fused), "
                               "both layers", "bound": "tensor",
                     "achieved": round(bwd_tflops, 1), "peak": peak_use, "unit": "TFLOP/s",
                     "frac": round(bwd_tflops / peak_use, 4),
                     "peak_kind": peak_kind,
                     "traffic": traffic,
                     "traffic_note": "ncu dram read+write bytes of one attn_block_bwd call (prep + main + dq), "
                                     "window-1024 layer; null when the kernel sources changed since the capture",
                     "algorithmic_flops_per_launch": flops_b / 2},
        "gpu_launches": 10 * args.steps,  # per layer: prologue, fwd, bwd prep / main / dq
        "clocks": clocks.summary(),
    }
    if not args.no_configs:
        cfg_steps = max(3, args.steps // 4)
        result["gqa"] = run_config(cswa, dev, "gqa", cfg_steps, world, rank, peak_use)
        lc = run_config(cswa, dev, "long", cfg_steps, world, rank, peak_use)
        pw, pf = (workloads.visible_pairs(8192, W) for W in (2048, -1))
        lc["window_vs_full"] = {
            "useful_flop_ratio": round(pw / pf, 4),
            "time_ratio": round(lc["layers"]["2048"]["fwd_bwd_ms"] / lc["layers"]["-1"]["fwd_bwd_ms"], 4),
            "note": "window 2048 over full causal on identical inputs: useful FLOPs and measured fwd+bwd time"}
        result["long"] = lc
        result["fp8"] = run_fp8(cswa, dev, cfg_steps, world, rank, peak_use)
    if rank == 0 and not args.no_decode:
        result["decode"] = run_decode(cswa, dev, args, pk, pk_src)
        result["prefill"] = run_prefill(cswa, dev, args, pk, pk_src)
        result["kv_replicate"] = run_replicate(cswa, dev, args, pk, pk_src)
    if not args.no_e2e:
        result["e2e"] = run_e2e(cswa, dev, args, q, k, v, do, L, scale, world, flops_f + flops_b)
    return result


def run_config(cswa, dev, name, steps, world, rank, peak):
    """fwd and bwd of each layer of a training config (the GQA layer, or the long-context
    layers at window 2048 and full causal), timed with CUDA events over `steps` repetitions
    after 3 warm-ups; useful TFLOP/s per layer. Inputs exceed L2."""
    c = workloads.CONFIGS[name]
    B, T, Hq, Hkv, D = c["B"], c["T"], c["Hq"], c["Hkv"], c["D"]
    scale = workloads.default_scale(D)
    q, k, v, do = (t.to(dev) for t in workloads.training_inputs(B, T, Hq, Hkv, D, shard_seed(c["seed"], rank)))
    qh, kh = cswa.attn_rope_qknorm(q, k)
    out = {"workload": f"{name}: B={B} T={T} Hq={Hq} Hkv={Hkv} D={D} bf16, fwd+bwd per layer (attention kernels; "
                       f"prologue excluded)", "steps": steps, "layers": {}}
    for W in c["windows"]:
        o = torch.empty_like(qh)
        lse = torch.empty((B, Hq, T), device=dev, dtype=torch.float32)
        dq, dk, dv = torch.empty_like(qh), torch.empty_like(kh), torch.empty_like(v)
        ws = torch.empty(cswa.attn_bwd_workspace_bytes(B, T, Hq, Hkv, D, W), device=dev, dtype=torch.uint8)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        for i in range(3 + steps):
            e = ev[i - 3] if i >= 3 else None
            if e:
                e[0].record()
            cswa.attn_fwd(qh, kh, v, W, scale, o=o, lse=lse)
            if e:
                e[1].record()
            cswa.attn_bwd(qh, kh, v, o, do, lse, W, scale, dq=dq, dk=dk, dv=dv, workspace=ws)
            if e:
                e[2].record()
        torch.cuda.synchronize()
        assert cswa.attn_get_status() == 0
        f_ms = max_over_ranks(statistics.median(e[0].elapsed_time(e[1]) for e in ev), world)
        b_ms = max_over_ranks(statistics.median(e[1].elapsed_time(e[2]) for e in ev), world)
        ff, fb = layer_useful_flops(B, T, Hq, D, W)
        out["layers"][str(W)] = {
            "window": W, "fwd_ms": round(f_ms, 4), "bwd_ms": round(b_ms, 4), "fwd_bwd_ms": round(f_ms + b_ms, 4),
            "fwd_tflops": round(world * ff / (f_ms * 1e-3) / 1e12, 1),
            "bwd_tflops": round(world * fb / (b_ms * 1e-3) / 1e12, 1),
            "fwd_bwd_tflops": round(world * (ff + fb) / ((f_ms + b_ms) * 1e-3) / 1e12, 1),
            "frac_of_peak": round((ff + fb) / ((f_ms + b_ms) * 1e-3) / 1e12 / peak, 4)}
        del o, lse, dq, dk, dv, ws
    return out


def run_fp8(cswa, dev, steps, world, rank, peak):
    """The e4m3 forward on the d20 layers (tensorwise-quantized q_hat, k_hat, v), useful
    TFLOP/s (4 D per visible pair) per window, and the three quantizations timed apart.
    The peak is the bf16 one: FP8 tensor cores run at twice that, so "of_bf16_peak" above
    0.5 would already mean more than the fp8 roofline allows for a bf16-shaped pipeline."""
    c = workloads.CONFIGS["d20"]
    B, T, Hq, Hkv, D = c["B"], c["T"], c["Hq"], c["Hkv"], c["D"]
    scale = workloads.default_scale(D)
    q, k, v, _ = (t.to(dev) for t in workloads.training_inputs(B, T, Hq, Hkv, D, shard_seed(c["seed"], rank)))
    qh, kh = cswa.attn_rope_qknorm(q, k)
    desc = torch.empty(3, device=dev, dtype=torch.float32)
    q8 = torch.empty(qh.shape, device=dev, dtype=torch.uint8)
    k8 = torch.empty(kh.shape, device=dev, dtype=torch.uint8)
    v8 = torch.empty(v.shape, device=dev, dtype=torch.uint8)

    def quantize():
        cswa.attn_quantize_fp8(qh, q8, desc[0:1])
        cswa.attn_quantize_fp8(kh, k8, desc[1:2])
        cswa.attn_quantize_fp8(v, v8, desc[2:3])
    out = {"workload": f"d20 layers: B={B} T={T} Hq=Hkv={Hq} D={D}, e4m3 q_hat/k_hat/v (tensorwise scales), "
                       "attention forward on the e4m3 tensor cores", "steps": steps, "layers": {}}
    o = torch.empty_like(qh)
    lse = torch.empty((B, Hq, T), device=dev, dtype=torch.float32)
    for W in c["windows"]:
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        for i in range(3 + steps):
            e = ev[i - 3] if i >= 3 else None
            if e:
                e[0].record()
            quantize()
            if e:
                e[1].record()
            cswa.attn_fwd_fp8(q8, k8, v8, desc, W, scale, o=o, lse=lse)
            if e:
                e[2].record()
        torch.cuda.synchronize()
        assert cswa.attn_get_status() == 0
        qms = max_over_ranks(statistics.median(e[0].elapsed_time(e[1]) for e in ev), world)
        fms = max_over_ranks(statistics.median(e[1].elapsed_time(e[2]) for e in ev), world)
        ff, _ = layer_useful_flops(B, T, Hq, D, W)
        tf = world * ff / (fms * 1e-3) / 1e12
        out["layers"][str(W)] = {"window": W, "fwd_ms": round(fms, 4), "fwd_tflops": round(tf, 1),
                                 "of_bf16_peak": round(tf / world / peak, 4), "quantize_ms": round(qms, 4)}
    return out


def run_decode(cswa, dev, args, pk, pk_src):
    c = workloads.DECODE
    B, Hq, Hkv, D, Tmax, W = c["B"], c["Hq"], c["Hkv"], c["D"], c["Tmax"], c["window"]
    lengths, kraw, vc, qraw, knraw, vn = workloads.decode_inputs(**c)
    kraw, vc, qraw, knraw, vn = (t.to(dev) for t in (kraw, vc, qraw, knraw, vn))
    pos = lengths.to(dev)
    _, kc = cswa.attn_rope_qknorm(None, kraw)
    qd, kn = cswa.attn_rope_qknorm(qraw, knraw, pos=pos)
    o = torch.empty_like(qd)
    lse = torch.empty((B, Hq), device=dev, dtype=torch.float32)
    ws = torch.empty(cswa.attn_decode_workspace_bytes(B, Hq, D, Tmax, W), device=dev, dtype=torch.uint8)
    flush = torch.empty(256 * 1024 * 1024 // 4, device=dev, dtype=torch.float32)
    reps = max(20, args.steps)
    times = []
    for i in range(5 + reps):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        cswa.attn_decode(qd, kc, vc, pos, W, k_new=kn, v_new=vn, o=o, lse=lse, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        if i >= 5:
            times.append(e0.elapsed_time(e1))
    assert cswa.attn_get_status() == 0
    ms = statistics.median(times)
    nbytes = decode_bytes(lengths.tolist(), Hq, Hkv, D, W)
    gbs = nbytes / (ms * 1e-3) / 1e9
    hbm = pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    return {"workload": "KV-cache decode: 32 sequences, lengths U[512,2048] (seed 4), Hq=Hkv=10, D=128, "
                        "Tmax=2176, window 1024, append of the new k/v",
            "us_per_step": round(ms * 1e3, 2), "us_p10": round(np.percentile(times, 10) * 1e3, 2),
            "us_p90": round(np.percentile(times, 90) * 1e3, 2), "value": round(gbs, 1), "unit": "GB/s",
            "l2": "flushed (256 MB written, then read back) before every call", "gpu_launches_per_step": 1,
            "roofline": {"kernel": "attn_decode (one launch: chunks, merge by the last chunk CTA)", "bound": "hbm",
                         "achieved": round(gbs, 1),
                         "peak": hbm, "unit": "GB/s", "frac": round(gbs / hbm, 4),
                         "traffic": ncu_traffic("decode_chunk_kernel"), "algorithmic_bytes": nbytes,
                         "peak_kind": pk_src}}


def run_prefill(cswa, dev, args, pk, pk_src):
    """Chunked prefill: a 512-token chunk per sequence against its KV cache (one launch:
    the tensor-core forward over the cache with the append fused), useful FLOPs = 4 D per
    visible pair."""
    c = workloads.PREFILL
    B, Hq, Hkv, D, T, Tmax, W = c["B"], c["Hq"], c["Hkv"], c["D"], c["T"], c["Tmax"], c["window"]
    lengths, kraw, vc, qraw, knraw, vn = workloads.prefill_inputs(**c)
    kraw, vc, qraw, knraw, vn = (t.to(dev) for t in (kraw, vc, qraw, knraw, vn))
    pos = lengths.to(dev)
    _, kc = cswa.attn_rope_qknorm(None, kraw)
    q, kn = cswa.attn_rope_qknorm(qraw, knraw, pos=pos)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, T), device=dev, dtype=torch.float32)
    flush = torch.empty(256 * 1024 * 1024 // 4, device=dev, dtype=torch.float32)
    reps = max(20, args.steps)
    times = []
    for i in range(5 + reps):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        # the same chunk is appended every call: the caches end up identical each time
        cswa.attn_prefill(q, kc, vc, pos, W, k_new=kn, v_new=vn, o=o, lse=lse)
        e1.record()
        torch.cuda.synchronize()
        if i >= 5:
            times.append(e0.elapsed_time(e1))
    assert cswa.attn_get_status() == 0
    ms = statistics.median(times)
    flops = 4 * D * Hq * workloads.prefill_pairs(lengths.tolist(), T, W)
    tf = flops / (ms * 1e-3) / 1e12
    peak = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    return {"workload": "chunked prefill: 8 sequences, a 512-token chunk each on cache lengths U[0,1536] "
                        "(seed 5), Hq=Hkv=10, D=128, Tmax=2048, window 1024, append of the chunk's k/v",
            "us_per_step": round(ms * 1e3, 2), "us_p10": round(np.percentile(times, 10) * 1e3, 2),
            "us_p90": round(np.percentile(times, 90) * 1e3, 2), "value": round(tf, 1), "unit": "TFLOP/s",
            "l2": "flushed (256 MB written, then read back) before every call", "gpu_launches_per_step": 1,
            "roofline": {"kernel": "attn_prefill (forward over the cache, append fused)", "bound": "tensor",
                         "achieved": round(tf, 1), "peak": peak, "unit": "TFLOP/s", "frac": round(tf / peak, 4),
                         "traffic": ncu_traffic("attn_fwd_kernel_prefill"),
                         "traffic_note": "ncu dram read+write bytes of the prefill launch",
                         "algorithmic_flops": flops, "peak_kind": f"bf16 burst ({pk_src})"}}


def run_replicate(cswa, dev, args, pk, pk_src):
    """Batch-1 -> 8 cache replication over a 20-layer d20 stack: a 1024-token prompt
    copied into 8 sample rows of (20, 8, 2048, 10, 128) k and v caches."""
    n_layers, rows, Tmax, N, Hkv, D = 20, 1024, 2048, 8, 10, 128
    ks = torch.randn((n_layers, 1, Tmax, Hkv, D), device=dev).to(torch.bfloat16)
    vs = torch.randn((n_layers, 1, Tmax, Hkv, D), device=dev).to(torch.bfloat16)
    kd = torch.empty((n_layers, N, Tmax, Hkv, D), device=dev, dtype=torch.bfloat16)
    vd = torch.empty_like(kd)
    times = []
    for i in range(3 + 10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        cswa.attn_kv_replicate(ks, vs, kd, vd, rows)
        e1.record()
        torch.cuda.synchronize()
        if i >= 3:
            times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    row = Hkv * D * 2
    nbytes = 2 * n_layers * rows * row * (1 + N)  # k and v: the prompt read once, written N times
    gbs = nbytes / (ms * 1e-3) / 1e9
    hbm = pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    return {"workload": "batch-1 -> 8 KV-cache replication: 20 layers, 1024-token prompt, Hkv=10, D=128, Tmax=2048",
            "us_per_step": round(ms * 1e3, 1), "value": round(gbs, 1), "unit": "GB/s",
            "l2": "inputs and outputs (1.9 GB) exceed L2", "gpu_launches_per_step": 1,
            "roofline": {"kernel": "attn_kv_replicate (broadcast kernel: each prompt vector read once, "
                                   "stored to the N samples)", "bound": "hbm",
                         "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s", "frac": round(gbs / hbm, 4),
                         "traffic": ncu_traffic("kv_replicate_kernel"), "algorithmic_bytes": nbytes,
                         "peak_kind": pk_src}}


def run_e2e(cswa, dev, args, q, k, v, do, L, scale, world, flops):
    """The same step through the public API with pinned HOST buffers: every step copies
    its inputs (q, k, v, dO) to the device and the layer outputs (o, dq, dk, dv) back.
    The copies run on two copy streams (host-to-device, device-to-host) and the compute on
    a third, with the device buffers doubled, so that step i's compute overlaps step i+1's
    input copy and step i-1's output copy; events order every use of a buffer. The timed
    region runs from before the first copy to after the last output copy."""
    hq, hk, hv, hdo = (t.cpu().pin_memory() for t in (q, k, v, do))
    ins = [(q, k, v, do), tuple(torch.empty_like(t) for t in (q, k, v, do))]
    outs = []  # [buffer][layer] -> dict of device outputs and lse
    for b in range(2):
        per = []
        for l in L:
            if b == 0:
                per.append({n: l[n] for n in ("o", "dq", "dk", "dv", "lse")})
            else:
                per.append({n: torch.empty_like(l[n]) for n in ("o", "dq", "dk", "dv", "lse")})
        outs.append(per)
    host_out = [[{n: torch.empty(l[n].shape, dtype=l[n].dtype, pin_memory=True) for n in ("o", "dq", "dk", "dv")}
                 for l in L] for _ in range(2)]
    B, T, Hq, D = q.shape
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdo))
    d2h = sum(h.numel() * h.element_size() for hl in host_out[0] for h in hl.values())
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    in_ready = [ev(), ev()]   # inputs of buffer b copied in
    in_free = [ev(), ev()]    # the compute has read buffer b's inputs
    out_ready = [ev(), ev()]  # outputs of buffer b computed
    out_free = [ev(), ev()]   # buffer b's outputs copied out
    started = [False, False]

    def step(i):
        b = i & 1
        qb, kb, vb, dob = ins[b]
        with torch.cuda.stream(s_in):
            if started[b]:
                s_in.wait_event(in_free[b])
            for d, h in zip(ins[b], (hq, hk, hv, hdo)):
                d.copy_(h, non_blocking=True)
            in_ready[b].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(in_ready[b])
            if started[b]:
                s_cmp.wait_event(out_free[b])
            for l, ob in zip(L, outs[b]):
                cswa.attn_rope_qknorm(qb, kb, l["qh"], l["kh"])
                cswa.attn_fwd(l["qh"], l["kh"], vb, l["W"], scale, o=ob["o"], lse=ob["lse"])
                cswa.attn_block_bwd(qb, kb, l["qh"], l["kh"], vb, ob["o"], dob, ob["lse"], l["W"], scale,
                                    dq=ob["dq"], dk=ob["dk"], dv=ob["dv"], workspace=l["ws"])
            in_free[b].record(s_cmp)
            out_ready[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(out_ready[b])
            for ob, hb in zip(outs[b], host_out[b]):
                for n, h in hb.items():
                    h.copy_(ob[n], non_blocking=True)
            out_free[b].record(s_out)
        started[b] = True

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize()
    steps = max(10, args.steps // 2)  # the pipeline's fill and drain are spread over the steps
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream(dev)
    e0.record(cur)
    for st in (s_in, s_cmp, s_out):
        st.wait_event(e0)
    for i in range(steps):
        step(i)
    for st in (s_in, s_cmp, s_out):
        cur.wait_stream(st)
    e1.record(cur)
    torch.cuda.synchronize()
    barrier(world)
    assert cswa.attn_get_status() == 0
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    return {"value": round(world * flops / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "ms_per_step": round(ms, 3),
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "how": "pinned host q,k,v,dO -> device, both layers fwd+bwd, o/dq/dk/dv -> pinned host; copies on "
                   "two copy streams overlap the neighbouring steps' compute (device buffers doubled)"}


# ------------------------------------------------------------------ CPU (oracle) arm
REF_UNIT = ("one (sequence, head) unit of the d20 layer pair: the B=1, Hq=Hkv=1 slice (T=2048, D=128) of one "
            "sequence and head, both windows (1024 and 2048), prologue + fwd + bwd + prologue bwd")


class OracleUnits:
    """The fp64 oracle on (sequence, head) units of the d20 layer pair: per unit, the
    prologue, forward, backward and prologue backward of one head of one sequence, for
    both layers. Units cycle through the heads of sequence 0."""

    def __init__(self, seed_offset=0):
        import oracle
        self.oracle = oracle
        c = workloads.CONFIGS["d20"]
        self.c = c
        self.scale = workloads.default_scale(c["D"])
        self.q, self.k, self.v, self.do = workloads.training_inputs(1, c["T"], c["Hq"], c["Hkv"], c["D"],
                                                                    c["seed"] + seed_offset)
        self.pos = oracle.row_positions(1, c["T"])
        self.n = 0

    def run_one(self):
        """Runs the next unit; returns its useful FLOPs (12 D per visible pair, both layers)."""
        o, c = self.oracle, self.c
        hs = slice(self.n % c["Hq"], self.n % c["Hq"] + 1)
        self.n += 1
        qf, kf, vf, dof = (t[:, :, hs].float().numpy().astype(np.float64) for t in (self.q, self.k, self.v, self.do))
        flops = 0.0
        for W in c["windows"]:
            qh = o.prologue(qf, self.pos, workloads.ROPE_BASE, workloads.EPS)
            kh = o.prologue(kf, self.pos, workloads.ROPE_BASE, workloads.EPS)
            o.attention_fwd(qh, kh, vf, W, self.scale)
            dqh, dkh, _ = o.attention_bwd(qh, kh, vf, dof, W, self.scale)
            o.prologue_bwd(qf, dqh, self.pos, workloads.ROPE_BASE, workloads.EPS)
            o.prologue_bwd(kf, dkh, self.pos, workloads.ROPE_BASE, workloads.EPS)
            flops += 12.0 * c["D"] * workloads.visible_pairs(c["T"], W)
        return flops


def cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count()


def oracle_sample(seconds_budget, seed_offset=0):
    """Times the oracle on units until the budget is spent. Returns (TFLOP/s, description, cores)."""
    u = OracleUnits(seed_offset)
    flops, units = 0.0, 0
    t0 = time.perf_counter()
    while True:
        flops += u.run_one()
        units += 1
        if time.perf_counter() - t0 >= seconds_budget:
            break
    dt = time.perf_counter() - t0
    desc = f"{units} units, each {REF_UNIT}; fp64 numpy oracle, {dt:.1f} s"
    return flops / dt / 1e12, desc, cpu_cores()


def run_reference(args, rank, world):
    """The oracle as the reference arm. One step = one unit (a stated subset of the
    workload, see REF_UNIT), timed on the host; ms_per_step is that measured time."""
    if rank != 0:
        return None
    u = OracleUnits()
    for _ in range(args.warmup):
        u.run_one()
    flops, times = 0.0, []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        flops += u.run_one()
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = flops / total / 1e12
    cores = cpu_cores()
    sample = f"{args.steps} steps of one unit each ({REF_UNIT}), {total:.1f} s in total"
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "sample of the " + WORKLOAD + ": " + REF_UNIT + " per step",
                       "global_batch": 1, "seq_len": 2048, "parallelism": "host cores"},
            "cpu_baseline": {"kind": "oracle", "value": value, "unit": "TFLOP/s", "cores": cores, "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=800)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cswa", choices=["cswa", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="budget of the cpu_baseline oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the GQA and long-context sub-keys")
    ap.add_argument("--eager", action="store_true",
                    help="time the training steps as separate calls instead of replaying a CUDA graph of the step")
    args = ap.parse_args()
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            res = run_reference(args, rank, world)
        else:
            if args.warmup < 3:
                raise SystemExit("timing rules need at least 3 warm-up steps")
            res = run_gpu(args, rank, world, local)
            if rank == 0 and not args.no_cpu_baseline:
                v, desc, cores = oracle_sample(args.cpu_seconds)
                res["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                       "sample": desc}
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
