#!/usr/bin/env python
"""MoE-layer throughput of the ternary MoE block forward on B200.

One run measures the four synthetic workloads in turn and prints one JSON line: the
headline (top-level keys) is the 35B-A3B-class decode layer (d=2048, 256 experts, top-8 +
shared expert, ffn 512, PQ2_0 experts, rank-512 correction), where one step = one forward
at each decode batch size b in {1, 8, 32, 64} (105 tokens), each call on the next of 40
independent layers (9.1 GB of weights, far above the 126 MB L2, so every call reads its
weights from HBM).  "workloads" holds the same figures for every workload: a3b_decode,
a3b_prefill (4096 tokens), flashnext_decode (d=3072, 512 experts, top-10 + shared, PTQ1_0,
b in {1, 16, 64}, 48 layers) and flashnext_prefill (16384 tokens, Zipf-loaded router).
Metric: tokens/s over the whole job, with the roofline fraction of the dominant kernel.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl scion|reference]

The block does not shard across GPUs (one GPU per layer replica): with N > 1 each
rank runs an independent replica (weak scaling); NCCL is used only for the barrier
and the max-over-ranks of the timed region.  `--impl reference` times the CPU
oracle (the plain fp64 reference) on the host cores instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s (decode b=1..64, prefill 4K/16K); % HBM or bf16 roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_traffic(workload, stage):
    """DRAM bytes per launch of `stage` measured by ncu for `workload` (profiles/dram_traffic.txt),
    or None when no capture of the current kernel is recorded."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        for line in f:
            parts = line.split("#", 1)[0].split()
            if len(parts) == 3 and parts[0] == workload and parts[1] == stage:
                return None if parts[2] == "null" else float(parts[2])
    return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="all",
                    help="all (the four measured workloads, a3b_decode first as the headline) or one name")
    ap.add_argument("--impl", default="scion", choices=["scion", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=0, help="override the number of cycled layers")
    ap.add_argument("--packed-corr", action="store_true",
                    help="ternary correction factors (PQ2_0 blocks) instead of the workload's bf16 ones")
    ap.add_argument("--stream-min-tokens", type=int, default=0,
                    help="decode batches of at least this many tokens use the persistent expert kernels")
    ap.add_argument("--decode-tc", type=int, default=0, choices=[0, 1],
                    help="1: tcgen05 expert GEMMs for those batches, 0: the mma.sync bulk-copy ring kernels")
    ap.add_argument("--prefill-reduce", action="store_true",
                    help="prefill: fp32 reductions into out from the down projection instead of per-entry rows "
                         "summed in slot order")
    return ap.parse_args()


# ------------------------------------------------------------------- algorithmic work
def workload_bytes(cfg, T, U, cb=2.0):
    """Algorithmic HBM bytes of one forward: U active experts' packed banks, the dense
    bf16 weights (router + delta, shared expert), the correction factors (cb bytes per
    weight: 2 for bf16, 34/128 for PQ2_0 blocks), x in and out."""
    bb = 34 if cfg.fmt == 0 else 28
    per_expert = 3 * cfg.ffn * cfg.d * bb // 128
    fixed = (2 * cfg.n_experts * cfg.d + 3 * cfg.shared_ffn * cfg.d) * 2 + 2 * cfg.rank * cfg.d * cb
    return U * per_expert + fixed + T * cfg.d * (2 + 4)


def stage_bytes(cfg, T, U, cb=2.0):
    """Algorithmic bytes per launch of each kernel stage (cb as in workload_bytes)."""
    bb = 34 if cfg.fmt == 0 else 28
    d, F, k, Fs, r, E = cfg.d, cfg.ffn, cfg.top_k, cfg.shared_ffn, cfg.rank, cfg.n_experts
    return {
        "router_f32": 2 * E * d * 4 + T * d * 2 + T * E * 4,
        "xproj": ((0 if cfg.router_f32 else 2 * E * d) + 2 * Fs * d) * 2 + r * d * cb + T * d * 2 + T * E * 4
        + T * (Fs + r) * 2,
        "route": T * E * 4 + T * k * 12 + E * 12,
        "gateup": U * 2 * F * d * bb // 128 + T * d * 2 + T * k * F * 2,
        "down_routed": U * F * d * bb // 128 + T * k * F * 2 + T * d * 4,
        "down_dense": d * Fs * 2 + d * r * cb + T * (Fs + r) * 2 + T * d * 4,
    }


def stage_flops(cfg, T):
    """Algorithmic tensor-core FLOPs per launch of each GEMM stage (no padding counted)."""
    d, F, k, Fs, r, E = cfg.d, cfg.ffn, cfg.top_k, cfg.shared_ffn, cfg.rank, cfg.n_experts
    return {
        "router_f32": 2 * T * 2 * E * d,
        "xproj": 2 * T * ((0 if cfg.router_f32 else 2 * E * d) + 2 * Fs * d + r * d),
        "gateup": 2 * T * k * 2 * d * F,
        "down_routed": 2 * T * k * d * F,
        "down_dense": 2 * T * d * (Fs + r),
    }


def workload_flops(cfg, T):
    return 2 * T * (cfg.top_k * 3 * cfg.d * cfg.ffn + 3 * cfg.d * cfg.shared_ffn + 2 * cfg.n_experts * cfg.d
                    + 2 * cfg.rank * cfg.d)


# ------------------------------------------------------------------- ranks
def max_over_ranks(v, world, device):
    """Maximum of a per-rank float over the process group (the job's time is its slowest rank)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist

    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world, tokens_per_step, steps, ms_max):
    """Whole-job throughput: every rank runs its own replica (weak scaling) on the same schedule,
    so the job processes world x tokens_per_step x steps tokens in the slowest rank's time."""
    return world * tokens_per_step * steps / (ms_max / 1000.0)


# ------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons of one GPU through NVML (read-only)."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, torch_dev):
        self.samples, self.reasons, self.ok = [], set(), False
        self._stop = threading.Event()
        try:
            import pynvml
            import torch

            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(torch_dev).uuid)
            h = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                hi = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(hi)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    h = hi
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(0)
            self.h, self.nv = h, pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover
            self.err = str(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                mask = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if mask & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        # re-entered once per timed region; the samples accumulate over all of them
        if self.ok:
            self._stop.clear()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------- oracle baseline
def oracle_sample(cfg, batches):
    """Host-generated layer 0 of the workload and its oracle; returns (oracle layer, xs)."""
    import oracle
    from workloads import synth

    L = synth.layer_host(cfg, 0)
    banks = {n: oracle.pack(cfg.fmt, L[n + "_codes"], L[n + "_scales"]) for n in ("gate", "up", "down")}
    for n in ("gate", "up", "down"):
        del L[n + "_codes"]
    ol = oracle.OracleLayer(
        d=cfg.d, n_experts=cfg.n_experts, top_k=cfg.top_k, ffn=cfg.ffn, fmt=cfg.fmt, w_router=L["w_router"],
        w_delta=L["w_delta"], gate_exps=banks["gate"], up_exps=banks["up"], down_exps=banks["down"],
        shared_ffn=cfg.shared_ffn, sh_gate=L.get("sh_gate"), sh_up=L.get("sh_up"), sh_down=L.get("sh_down"),
        rank=cfg.rank, corr_a=L.get("corr_a"), corr_b=L.get("corr_b"))
    xs = [synth.x_host(cfg, T) for T in batches]
    return ol, xs


# Token counts of the bounded oracle samples of the prefill workloads: the first tokens of a
# batch drawn like the workload's (same router, same x distribution, Zipf load included).
PREFILL_SAMPLE_TOKENS = {"a3b_prefill": 256, "flashnext_prefill": 128}


def oracle_batches(cfg):
    """The batches one oracle step runs: the workload's own decode batches, or a bounded sample
    of a prefill batch."""
    if max(cfg.tokens) <= 64:
        return list(cfg.tokens)
    return [PREFILL_SAMPLE_TOKENS.get(cfg.name, 64)]


def cpu_baseline(cfg, seconds=5.0):
    """The oracle as it stands on the host cores: its batch set repeated for about `seconds` of
    CPU work (at least once, at most 6x that)."""
    import oracle

    batches = oracle_batches(cfg)
    ol, xs = oracle_sample(cfg, batches)
    t0 = time.perf_counter()
    reps = 0
    while True:
        for x in xs:
            oracle.forward(ol, x)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= seconds or dt * (reps + 1) / reps > 6 * seconds:
            break
    ntok = sum(batches) * reps
    what = ("one forward per batch %s" % batches if max(cfg.tokens) <= 64 else
            "one forward of the first %d tokens of a %d-token batch" % (batches[0], cfg.tokens[0]))
    return {"value": ntok / dt, "unit": "tokens/s", "cores": oracle.cores_used(), "kind": "oracle",
            "sample": "%s layer 0 (host-generated), %d x %s = %d tokens, %.1f s" % (cfg.name, reps, what, ntok, dt)}


def run_reference(args, rank):
    """The oracle arm: plain fp64 C reference on the host cores, rank 0 only.  A step is the
    headline workload's own step (one forward at each of its decode batch sizes, or a bounded
    sample of its prefill batch) on layer 0; the other workloads get bounded samples too."""
    if rank != 0:
        return
    import oracle
    from workloads import synth

    names = workload_names(args)
    cfg = synth.CONFIGS[names[0]]
    batches = oracle_batches(cfg)
    ol, xs = oracle_sample(cfg, batches)
    for _ in range(args.warmup):
        for x in xs:
            oracle.forward(ol, x)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for x in xs:
            oracle.forward(ol, x)
    dt = time.perf_counter() - t0
    v = sum(batches) * args.steps / dt
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(cfg, args),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": oracle.cores_used(), "kind": "oracle",
                             "sample": "each step: one forward per batch %s on layer 0 of %s" % (batches, cfg.name)},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    if len(names) > 1:
        line["workloads"] = {n: {"cpu_baseline": cpu_baseline(synth.CONFIGS[n], 3.0)} for n in names[1:]}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- GPU arm
ALL_WORKLOADS = ("a3b_decode", "a3b_prefill", "flashnext_decode", "flashnext_prefill")


def workload_names(args):
    """The workloads of one run, the headline first."""
    return list(ALL_WORKLOADS) if args.workload == "all" else [args.workload]


def workload_config(cfg, args, n_layers=None, weight_bytes=None):
    c = {"workload": cfg.name, "d": cfg.d, "experts": cfg.n_experts, "top_k": cfg.top_k, "ffn": cfg.ffn,
         "shared_ffn": cfg.shared_ffn, "rank": cfg.rank, "format": "PQ2_0" if cfg.fmt == 0 else "PTQ1_0",
         "correction": "PQ2_0 blocks" if args.packed_corr else "bf16", "batches": list(cfg.tokens),
         "decode_expert_kernels": "tcgen05" if args.decode_tc else "mma.sync ring",
         "prefill_combine": "fp32 reductions" if args.prefill_reduce else "slot-order rows",
         "tokens_per_step": sum(cfg.tokens)}
    if cfg.zipf_s is not None:
        c["router_load"] = "Zipf(%.1f) over a seeded permutation of the experts" % cfg.zipf_s
    if n_layers is not None:
        c["layers_cycled"] = n_layers
    if weight_bytes is not None:
        c["l2"] = "inputs larger than L2: %.1f GB of layers cycled" % (weight_bytes / 1e9)
    return c


def build_layers(cfg, args, dev, n_layers, max_T):
    import torch

    import ternary_quantized_moe_b200 as tq
    from workloads import synth

    layers = []
    for l in range(n_layers):
        W = synth.layer_device(cfg, l, dev)
        banks = {n: tq.scion_pack_device(cfg.fmt, W.pop(n + "_codes"), W.pop(n + "_scales")) for n in
                 ("gate", "up", "down")}
        corr = dict(corr_a=W.get("corr_a"), corr_b=W.get("corr_b"))
        if args.packed_corr and cfg.rank:
            # ternary correction factors with the experts' code and scale distributions
            corr = {}
            for name, rows, K in (("corr_a", cfg.rank, cfg.d), ("corr_b", cfg.d, cfg.rank)):
                g = torch.Generator(device=dev)
                g.manual_seed(7000 + 31 * l + rows)
                u = torch.randint(0, 10, (rows, K), generator=g, device=dev)
                codes = torch.where(u < 4, 0, torch.where(u < 7, 1, -1)).to(torch.int8)
                scales = (torch.rand((rows, K // 128), generator=g, device=dev) * 0.015 + 0.005).half()
                corr[name] = tq.scion_pack_device(synth.PQ2_0, codes, scales.view(torch.int16))
        layers.append(tq.scion_layer_create(
            d=cfg.d, n_experts=cfg.n_experts, top_k=cfg.top_k, ffn=cfg.ffn, fmt=cfg.fmt, w_router=W["w_router"],
            w_router_delta=W["w_delta"], gate_exps=banks["gate"], up_exps=banks["up"], down_exps=banks["down"],
            shared_ffn=cfg.shared_ffn, sh_gate=W.get("sh_gate"), sh_up=W.get("sh_up"), sh_down=W.get("sh_down"),
            rank=cfg.rank, max_tokens=max_T, corr_packed=1 if args.packed_corr and cfg.rank else 0, **corr))
        del banks, W
        if args.stream_min_tokens:
            tq.scion_layer_set_option(layers[-1], tq.SCION_OPT_STREAM_MIN_TOKENS, args.stream_min_tokens)
        tq.scion_layer_set_option(layers[-1], tq.SCION_OPT_DECODE_TC, args.decode_tc)
        if args.prefill_reduce:
            tq.scion_layer_set_option(layers[-1], tq.SCION_OPT_DETERMINISTIC, 0)
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return layers


def measure(cfg, args, rank, world, dev, peaks, peak_src, clocks):
    """Every figure of one workload: device-timed throughput, per-kernel times, rooflines, per
    batch size, end to end through the host-buffer entry point, and the oracle baseline."""
    import torch
    import torch.distributed as dist

    import ternary_quantized_moe_b200 as tq
    from workloads import synth

    n_layers = args.layers or cfg.n_layers
    batches = list(cfg.tokens)
    max_T = max(batches)
    layers = build_layers(cfg, args, dev, n_layers, max_T)
    cb = 34.0 / 128.0 if args.packed_corr else 2.0
    weight_bytes = sum(tq.scion_layer_device_bytes(L) for L in layers)

    xs = {T: synth.x_device(cfg, T, dev) for T in batches}
    outs = {T: torch.empty((T, cfg.d), dtype=torch.float32, device=dev) for T in batches}
    stream = torch.cuda.current_stream(dev)
    nb = len(batches)

    def step(s):
        for i, T in enumerate(batches):
            tq.scion_moe_forward(xs[T], T, layers[(s * nb + i) % n_layers], outs[T], stream)

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()

    def timed(fn, K):
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for s in range(K):
            fn(s)
        e1.record(stream)
        e1.synchronize()
        ms = e0.elapsed_time(e1)
        barrier()
        return max_over_ranks(ms, world, dev)

    for s in range(max(3, args.warmup)):
        step(s)
    K = args.steps

    # ---- headline: device-timed region, inputs resident in HBM
    launches0 = tq.scion_kernel_launches()
    with clocks:
        ms = timed(step, K)
    launches = tq.scion_kernel_launches() - launches0
    tokens_per_step = sum(batches)
    value = job_tokens_per_s(world, tokens_per_step, K, ms)

    # ---- per-kernel device time (CUDA events around every launch, same schedule)
    barrier()
    tq.scion_profile_begin(int(launches) + 64)
    for s in range(K):
        step(s)
    stages = tq.scion_profile_end()

    # ---- realised routing: distinct active experts of every (layer, batch) pair
    U = {}
    counts = torch.empty(cfg.n_experts, dtype=torch.int32, device=dev)
    for li in range(n_layers):
        for T in batches:
            tq.scion_moe_forward_debug(xs[T], T, layers[li], outs[T], stream, counts=counts)
            U[(li, T)] = int((counts > 0).sum().item())
    sched = [((s * nb + i) % n_layers, T) for s in range(K) for i, T in enumerate(batches)]
    bytes_total = sum(workload_bytes(cfg, T, U[(li, T)], cb) for li, T in sched)
    # the active experts' packed banks alone (U distinct experts per call)
    expert_bytes = sum(U[(li, T)] * 3 * cfg.ffn * cfg.d * (34 if cfg.fmt == 0 else 28) // 128 for li, T in sched)
    sbytes, sflops = {}, {}
    min_ring = args.stream_min_tokens or 16
    for li, T in sched:
        sb, sf = stage_bytes(cfg, T, U[(li, T)], cb), stage_flops(cfg, T)
        if T < min_ring and (T + 7) // 8 <= 2 and cfg.shared_ffn + cfg.rank > 0:
            # below the ring threshold the dense down projection runs inside the gate/up launch
            sb["gateup"] += sb.pop("down_dense")
            sf["gateup"] += sf.pop("down_dense")
        for k_, v in sb.items():
            sbytes[k_] = sbytes.get(k_, 0) + v
        for k_, v in sf.items():
            sflops[k_] = sflops.get(k_, 0) + v
    flops_total = sum(workload_flops(cfg, T) for _, T in sched)

    # ---- per batch size (each batch alone, cycling layers)
    per_batch = {}
    if nb > 1:
        for T in batches:
            def one(s, T=T):
                tq.scion_moe_forward(xs[T], T, layers[s % n_layers], outs[T], stream)
            msT = timed(one, K)
            bT = sum(workload_bytes(cfg, T, U[(s % n_layers, T)], cb) for s in range(K))
            per_batch[str(T)] = {"tokens_per_s": job_tokens_per_s(world, T, K, msT),
                                 "us_per_call": 1000.0 * msT / K,
                                 "hbm_frac": (bT / (msT / 1000.0)) / (peaks["hbm_gbs"] * 1e9)}

    # ---- end to end through the host-buffer entry point (pinned host x in, out back to host)
    xh = {T: xs[T].cpu().pin_memory() for T in batches}
    oh = {T: torch.empty((T, cfg.d), dtype=torch.float32).pin_memory() for T in batches}

    def step_host(s):
        for i, T in enumerate(batches):
            tq.scion_moe_forward_host(xh[T], T, layers[(s * nb + i) % n_layers], oh[T], stream)

    ms_e2e = timed(step_host, K)
    e2e = {"value": job_tokens_per_s(world, tokens_per_step, K, ms_e2e), "unit": "tokens/s",
           "h2d_bytes_per_step": sum(T * cfg.d * 2 for T in batches),
           "d2h_bytes_per_step": sum(T * cfg.d * 4 for T in batches)}

    # ---- roofline of the dominant kernel
    decode = max_T <= 64
    work = sbytes if decode else sflops  # the roofline is taken on a stage that moves weights / does MMAs
    dom = max((k_ for k_ in stages if stages[k_][1] > 0 and work.get(k_, 0) > 0), key=lambda k_: stages[k_][0])
    dom_ms, dom_n = stages[dom]
    if decode:
        achieved = (sbytes[dom] / dom_n) / (dom_ms / dom_n / 1000.0) / 1e9
        roof = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": load_traffic(cfg.name, dom), "peak_source": peak_src,
                "bytes_per_launch": sbytes[dom] / dom_n, "us_per_launch": 1000.0 * dom_ms / dom_n}
    else:
        achieved = sflops[dom] / (dom_ms / 1000.0) / 1e12  # the dominant kernel's own FLOPs / its time
        roof = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"], "traffic": load_traffic(cfg.name, dom),
                "peak_source": peak_src, "flops_per_launch": sflops[dom] / dom_n,
                "us_per_launch": 1000.0 * dom_ms / dom_n}
    step_roof = {"bytes_per_step": bytes_total / K, "hbm_frac": (bytes_total / (ms / 1000.0)) / (peaks["hbm_gbs"] * 1e9),
                 "tflops": flops_total / (ms / 1000.0) / 1e12,
                 "tflops_frac": flops_total / (ms / 1000.0) / 1e12 / peaks["bf16_tflops"],
                 "expert_bytes_per_step": expert_bytes / K,
                 "expert_stage_hbm_frac": (expert_bytes / ((stages.get("gateup", (0, 0))[0] +
                                                            stages.get("down_routed", (0, 0))[0]) / 1000.0)
                                           / (peaks["hbm_gbs"] * 1e9)) if stages.get("gateup", (0, 0))[0] > 0 else None,
                 # the same step against nominal figures: HBM3e at 8 TB/s, and the bf16 throughput
                 # a seconds-long GEMM sustains under the power cap
                 "hbm_frac_vs_nominal_8tbs": (bytes_total / (ms / 1000.0)) / 8e12,
                 "tflops_frac_vs_sustained": flops_total / (ms / 1000.0) / 1e12 /
                 peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"])}
    res = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "ms_per_step": ms / K,
        "config": workload_config(cfg, args, n_layers, weight_bytes),
        "roofline": roof, "step_roofline": step_roof,
        "stages_us_per_launch": {k_: 1000.0 * v[0] / v[1] for k_, v in stages.items() if v[1]},
        "stages_rate": {k_: (sbytes[k_] / (v[0] / 1000.0) / 1e9 if decode else
                             sflops.get(k_, 0) / (v[0] / 1000.0) / 1e12)
                        for k_, v in stages.items() if v[1] and k_ in sbytes},
        "stages_rate_unit": "GB/s" if decode else "TFLOP/s",
        "stages_share": {k_: v[0] / sum(x[0] for x in stages.values()) for k_, v in stages.items() if v[1]},
        "e2e": e2e,
        "gpu_launches": int(launches),
    }
    if per_batch:
        res["per_batch"] = per_batch
    if not decode:
        # routing of the prefill batch: empty experts and the heaviest expert's share of the entries
        tq.scion_moe_forward_debug(xs[max_T], max_T, layers[0], outs[max_T], stream, counts=counts)
        c = counts.cpu()
        res["routing"] = {"empty_experts": int((c == 0).sum()), "max_expert_tokens": int(c.max()),
                          "mean_expert_tokens": float(c.float().mean())}
    for L in layers:
        L.close()
    del layers, xs, outs, xh, oh
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(cfg)
    return res


def run_gpu(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from workloads import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    peaks, peak_src = load_peaks()
    clocks = ClockSampler(dev)  # sampled during every timed region of every workload
    names = workload_names(args)
    results = {n: measure(synth.CONFIGS[n], args, rank, world, dev, peaks, peak_src, clocks) for n in names}
    head = results[names[0]]
    line = {
        "metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": dict(head["config"], parallelism="replicas" if world > 1 else "single"),
    }
    for k_ in ("roofline", "step_roofline", "per_batch", "stages_us_per_launch", "stages_rate", "stages_rate_unit",
               "stages_share", "e2e", "gpu_launches", "cpu_baseline"):
        if k_ in head:
            line[k_] = head[k_]
    line["clocks"] = clocks.summary()
    if len(names) > 1:
        line["workloads"] = results
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_quantize(args):
    """The float -> ternary quantizers over one 35B-A3B-class layer's expert weights (256 experts x
    (gate, up, down) x 512 x 2048 = 805M N(0,1) fp32 weights, 3.2 GB): one step = one call of the
    Lloyd quantizer (30 rounds at most) over all groups.  Device-timed with CUDA events; the
    roofline is the HBM traffic (fp32 in, int8 codes and fp16 scales out)."""
    import torch

    import ternary_quantized_moe_b200 as tq

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    n = 256 * 3 * 512 * 2048 // 128
    g = torch.Generator(device=dev)
    g.manual_seed(4242)
    w = torch.randn((n, 128), generator=g, device=dev)
    codes = torch.empty((n, 128), dtype=torch.int8, device=dev)
    scales = torch.empty(n, dtype=torch.int16, device=dev)
    bytes_per_call = n * 128 * 5 + n * 2
    res = {}
    for name, method in (("lloyd", tq.SCION_QUANT_LLOYD), ("absmean", tq.SCION_QUANT_ABSMEAN)):
        for _ in range(max(3, args.warmup)):
            tq.scion_quantize_device(method, w, codes, scales, iters=30)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            tq.scion_quantize_device(method, w, codes, scales, iters=30)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
        res[name] = {"ms_per_call": ms, "weights_per_s": n * 128 / (ms / 1000.0),
                     "hbm_gbs": bytes_per_call / (ms / 1000.0) / 1e9}
    line = {"metric": "ternary quantizer weights/s (Lloyd g128)", "value": res["lloyd"]["weights_per_s"],
            "unit": "weights/s", "n_gpus": 1, "steps": args.steps, "warmup": max(3, args.warmup),
            "ms_per_step": res["lloyd"]["ms_per_call"], "higher_is_better": True, "dtype": "f64",
            "data": "synthetic", "config": {"workload": "quantize_a3b_experts", "weights": n * 128,
                                             "l2": "inputs larger than L2: 3.2 GB"},
            "roofline": {"bound": "hbm", "achieved": res["lloyd"]["hbm_gbs"], "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": res["lloyd"]["hbm_gbs"] / peaks["hbm_gbs"], "traffic": None,
                         "peak_source": peak_src},
            "absmean": res["absmean"]}
    print(json.dumps(line))


def main():
    args = parse()
    if args.workload == "quantize_a3b_experts":
        run_quantize(args)
        return
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    run_gpu(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
