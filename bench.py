"""Benchmark of the fused MoE layer forward (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config decode|prefill|fp8|mxfp8|fp8t|skew|tiny]
                    [--impl ours|reference] [--no-cpu-baseline]

A step is one moe_forward over one batch of the workload's T tokens (router
logits, top-k, permute, [FP8 activation quantisation], gate-up GEMM, down GEMM,
combine), inputs resident in HBM.  K steps are timed on the device with CUDA
events (barrier + synchronize on both sides), max over ranks.  Every rank
runs its own replica on its own batch (tokens are independent given the
weights, so the layer shards over tokens with no collective): "scaling" is
"weak" and `value` = all ranks' tokens / the slowest rank's time.

Extra keys: `roofline` (dominant kernel, from the events the library records
at the stage boundaries inside the timed region), `cpu_baseline` (the FP64
oracle on a bounded token sample, rank 0, N=1), `e2e` (the same metric through
moe_forward_host: host->device copy of x, the layer, device->host copy of y,
every step), `clocks` (nvidia-smi samples taken during the timed region),
`gpu_launches` (kernels of this library launched in the timed region).

`--impl reference` times the oracle (the plain FP64 CPU implementation) on
the host cores instead, as the reference arm.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from expert_layer_dual_b200.configs import CONFIGS, MoEConfig  # noqa: E402
from expert_layer_dual_b200.inputs import make_layer  # noqa: E402

METRIC = "fused MoE layer tokens/s"
UNIT = "tokens/s"
# oracle token sample per step of the CPU baseline / reference arm
CPU_SAMPLE = {"tiny": 16, "decode": 64, "prefill": 16, "fp8": 8, "mxfp8": 8, "fp8t": 8, "skew": 16}


def cpu_sample(cfg: MoEConfig) -> int:
    return CPU_SAMPLE.get(cfg.name.split("-")[0], 8)


def describe(cfg: MoEConfig) -> str:
    s = f"{cfg.name}: T={cfg.T} d={cfg.d} E={cfg.E} top-{cfg.k}"
    s += f" + shared I={cfg.I}" if cfg.Is else f" I={cfg.I}"
    s += {0: ", BF16 weights", 1: ", FP8 e4m3 128x128 block-scaled weights",
          2: ", MXFP8 (e4m3, E8M0 scale per 1x32) weights and activations",
          3: ", FP8 e4m3 per-tensor weight scales, static calibrated activation scales"}[cfg.wdtype]
    if cfg.zipf_bias:
        s += ", Zipf(1.2)-biased routing"
    return s


# ------------------------------------------------------------------ ranks
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        torch.distributed.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def max_over_ranks(value: float, device) -> float:
    """Largest value over all ranks (identity without a process group)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier():
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.barrier()


# ------------------------------------------------------------------ clocks
def nvml_bus_id(dev) -> str:
    """PCI bus id of a torch CUDA device in NVML's form (the index NVML and
    nvidia-smi use need not be the CUDA index when CUDA_VISIBLE_DEVICES is set)."""
    p = torch.cuda.get_device_properties(dev)
    return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"


class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU, sampled every
    `period_s` by a thread reading NVML while the timed region runs (read
    only: no setting of the GPU is touched).  Falls back to nvidia-smi's
    100 ms loop when NVML is unavailable."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str, period_s: float = 0.005):
        self.bus_id = bus_id
        self.period = period_s
        self.lines = []
        self.proc = None
        self.path = None
        self.thread = None
        self.stop = False
        self.power_limit_w = None

    def _nvml_loop(self, nv, h):
        names = [("hw_slowdown", nv.nvmlClocksEventReasonHwSlowdown),
                 ("hw_thermal_slowdown", nv.nvmlClocksEventReasonHwThermalSlowdown),
                 ("sw_thermal_slowdown", nv.nvmlClocksEventReasonSwThermalSlowdown),
                 ("sw_power_cap", nv.nvmlClocksEventReasonSwPowerCap)]
        smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        try:
            self.power_limit_w = nv.nvmlDeviceGetEnforcedPowerLimit(h) / 1000.0
        except nv.NVMLError:
            pass
        while not self.stop:
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            except nv.NVMLError:
                break
            flags = ["Active" if r & bit else "Not Active" for _, bit in names]
            self.lines.append(", ".join(["0", str(sm), str(smax), f"{pw:.2f}", hex(r)] + flags))
            time.sleep(self.period)

    def __enter__(self):
        try:
            import threading
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByPciBusId(self.bus_id)
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, h), daemon=True)
            self.thread.start()
            time.sleep(0.05)
            return self
        except Exception:  # noqa: BLE001 -- no NVML: sample with nvidia-smi instead
            self.thread = None
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", self.bus_id, "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop = True
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.thread is not None:
            out = parse_clock_samples(self.lines)
            out["source"] = f"NVML every {self.period * 1e3:.0f} ms"
            if self.power_limit_w is not None:
                out["power_limit_w"] = self.power_limit_w
            return out
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        out = parse_clock_samples(open(self.path).read().splitlines())
        out["source"] = "nvidia-smi every 100 ms"
        return out


def parse_clock_samples(lines):
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    sm, smax, reasons, power = [], [], set(), []
    for ln in lines:
        parts = [p.strip() for p in ln.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            smax.append(float(parts[2]))
            power.append(float(parts[3]))
        except ValueError:
            continue
        for n, v in zip(names, parts[5:9]):
            if v.lower() == "active":
                reasons.add(n)
    if not sm:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
    loaded = [s for s, p in zip(sm, power) if p > 0.3 * max(power)] or sm
    return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax),
            "power_w_max": max(power), "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------------ roofline
def load_peaks(sustained: bool = False):
    """(HBM GB/s, dense BF16 TFLOP/s, source).  The BF16 figure is the burst one
    for a short timed region, the sustained (power-capped) one for a long region."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        tf = p.get("bf16_tflops_sustained", 1400.0) if sustained else p.get("bf16_tflops", 1590.0)
        return p.get("hbm_gbs", 6650.0), tf, "measured"
    return 6650.0, (1400.0 if sustained else 1590.0), "fallback"


def power_capped(clocks: dict, ms_total: float) -> bool:
    """Whether the timed region ran in the sustained regime, the one the
    sustained peak was measured in: its median SM clock under load sat below
    90% of the maximum (a power-cap flag at full clock is not that regime).
    Without clock samples: whether it was long enough to reach the cap (0.3 s)."""
    sm, smax = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    if sm and smax:
        return sm < 0.9 * smax
    return ms_total > 300.0


# DRAM traffic of the dominant kernel, from an ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum of one launch) recorded in profiles/dram_traffic.txt with a
# hash of the kernel's sources; reported only while the sources still match.
KERNEL_SOURCES = {
    "k_gateup_bf16": ["csrc/gemm_bf16.cu", "csrc/common.cuh", "csrc/grouped_common.cuh"],
    "k_gateup_bf16_wide": ["csrc/gemm_bf16_wide.cu", "csrc/common.cuh", "csrc/grouped_common.cuh"],
    "k_gateup_bf16_2sm": ["csrc/gemm_bf16_2sm.cu", "csrc/common.cuh", "csrc/grouped_common.cuh"],
    "k_gateup_fp8": ["csrc/gemm_fp8.cu", "csrc/common.cuh", "csrc/grouped_common.cuh"],
    "k_gateup_mx": ["csrc/gemm_mx.cu", "csrc/common.cuh", "csrc/grouped_common.cuh"],
    "k_gateup_f8t": ["csrc/gemm_f8t.cu", "csrc/common.cuh", "csrc/grouped_common.cuh"],
}


def kernel_source_hash(kernel: str) -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "expert_layer_dual_b200", rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """(bytes per launch, note) if profiles/dram_traffic.txt holds a capture of
    `kernel` on `workload` taken from the current sources, else (None, why)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None, "no capture recorded"
    for line in open(path):
        parts = line.split()
        if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel and parts[1] == workload:
            if parts[3] != kernel_source_hash(kernel):
                return None, "kernel changed since the capture"
            return int(parts[2]), "ncu capture, profiles/dram_traffic.txt"
    return None, "no capture for this workload"


def gateup_kernel(cfg: MoEConfig, T: int, num_sms: int) -> str:
    """Name of the gate-up kernel moe_forward launches for this shape: the
    library's dispatch rule for BF16 (use_pair_gateup in launch.h: the CTA-pair
    kernel over x copied into the permuted row order from 256 rows per expert
    on average, the one-CTA gathering kernel below)."""
    del num_sms
    if cfg.wdtype != 0:
        return "k_gateup_" + {1: "fp8", 2: "mx", 3: "f8t"}[cfg.wdtype]
    return "k_gateup_bf16_2sm" if T * cfg.k >= 256 * cfg.E else "k_gateup_bf16"


def router_ksplit(T: int, d: int, E: int) -> int:
    """The library's K split of the router GEMM (router_ksplit in router.cu)."""
    tiles = -(-T // 128) * -(-E // 64)
    nk, ks = d // 64, 1
    while ks < 8 and tiles * ks * 2 <= 148 and nk // (ks * 2) >= 4:
        ks *= 2
    return ks


def kernels_per_step(cfg: MoEConfig, T: int) -> int:
    """Kernels of this library one moe_forward launches, by its dispatch: the
    router (with the top-k fused into it when one CTA covers a tile's whole K
    and E <= 64, else followed by the top-k kernel), the permute (one kernel for at most
    1024 assignments, else count, scan and scatter), gate-up, down and
    combine, plus the activation quantiser on the FP8 paths and the copy of x
    into the permuted row order before the CTA-pair BF16 gate-up."""
    router = 1 if router_ksplit(T, cfg.d, cfg.E) == 1 and cfg.E <= 64 else 2
    permute = 1 if T * cfg.k <= 1024 else 3
    a_prep = 1 if cfg.wdtype or T * cfg.k >= 256 * cfg.E else 0
    return router + permute + 3 + a_prep


def gateup_algorithmic(cfg: MoEConfig, T: int, n_active: int):
    """Algorithmic work of one gate-up launch: FLOPs, and bytes = the weights
    of every expert that received tokens (+ shared) read once, x read once,
    h written once."""
    R = T * cfg.k + (T if cfg.Is else 0)
    wbytes = 1 if cfg.wdtype else 2
    groups = n_active + (1 if cfg.Is else 0)
    flops = 2.0 * R * cfg.d * 2 * cfg.I
    byts = groups * 2 * cfg.I * cfg.d * wbytes + T * cfg.d * wbytes + R * cfg.I * wbytes
    if cfg.wdtype == 2:  # MXFP8: one scale byte per 32 elements of weights, x and h
        byts += (groups * 2 * cfg.I * cfg.d + T * cfg.d + R * cfg.I) // 32
    return flops, byts


def down_algorithmic(cfg: MoEConfig, T: int, n_active: int):
    R = T * cfg.k + (T if cfg.Is else 0)
    wbytes = 1 if cfg.wdtype else 2
    groups = n_active + (1 if cfg.Is else 0)
    flops = 2.0 * R * cfg.I * cfg.d
    byts = groups * cfg.d * cfg.I * wbytes + R * cfg.I * wbytes + R * cfg.d * 2
    if cfg.wdtype == 2:
        byts += (groups * cfg.d * cfg.I + R * cfg.I) // 32
    return flops, byts


# ------------------------------------------------------------------ CPU oracle
def _bits(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def oracle_static_scales(cfg: MoEConfig, inp: dict, n_tokens: int = 8):
    """Static activation scales of a per-tensor FP8 layer for the oracle runs
    without a GPU, by the oracle's per-tensor rule s = fp32(amax) / 448: over
    the first n_tokens of x, and over their gate-up output h from the
    oracle's own BF16 stages, rounded to bf16 as the library's calibration
    takes it (moe_calibrate_fp8_static does the same on the GPU with 64
    tokens)."""
    import oracle
    L, xs = oracle_sample(MoEConfig(**{**cfg.__dict__, "wdtype": 0}), inp, n_tokens)
    out = oracle.forward(L, xs)
    h = oracle.gateup(L, xs, out["perm"], out["offsets"])[:, : cfg.I]
    _, sx = oracle.quant_fp8_tensor(xs[None])
    _, sh = oracle.quant_fp8_tensor(oracle.bf16_round(h)[None])
    return (float(sx[0]), float(sh[0]))


def oracle_sample(cfg: MoEConfig, inp: dict, n_tokens: int, act=(1.0, 1.0)):
    """Host inputs of the oracle for the first n_tokens of the workload: x rows,
    the router weight and the experts the oracle's own routing selects."""
    import oracle
    oracle.build()
    n = min(n_tokens, cfg.T)
    xs = _bits(inp["x"][:n])
    rw = inp["router_w"].detach().cpu().numpy()
    bias = None if inp.get("router_bias") is None else inp["router_bias"].cpu().numpy()
    hi, lo = oracle.router_split(rw)
    lg = oracle.router_logits(xs, hi, lo, bias)
    need = np.unique(oracle.route_topk(lg.astype(np.float32), cfg.k)[0])
    w_gu = np.empty((cfg.E, 2 * cfg.I, cfg.d), np.uint16)
    w_d = np.empty((cfg.E, cfg.d, cfg.I), np.uint16)
    for e in need:
        w_gu[e] = _bits(inp["w_gu"][int(e)])
        w_d[e] = _bits(inp["w_d"][int(e)])
    L = oracle.Layer(T=n, d=cfg.d, E=cfg.E, k=cfg.k, I=cfg.I, Is=cfg.Is, w_gu=w_gu, w_d=w_d,
                     ws_gu=None if inp.get("ws_gu") is None else _bits(inp["ws_gu"]),
                     ws_d=None if inp.get("ws_d") is None else _bits(inp["ws_d"]),
                     router_w=rw, router_bias=bias, wdtype=cfg.wdtype, renorm=cfg.renorm,
                     act_sx=act[0], act_sh=act[1])
    return L, xs


def oracle_times(L, xs, repeats: int):
    """Seconds of each of `repeats` whole-layer oracle runs on the sample."""
    import oracle
    times = []
    for _ in range(repeats):
        t0 = time.perf_counter()
        oracle.forward(L, xs)
        times.append(time.perf_counter() - t0)
    return times


def run_reference(args, cfg: MoEConfig):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    inp = make_layer(cfg, device="cuda" if torch.cuda.is_available() else "cpu")
    import oracle
    # size the per-step sample so the whole run stays within a few minutes
    L1, x1 = oracle_sample(cfg, inp, 1)
    t1 = oracle_times(L1, x1, 1)
    budget = 150.0 / (args.warmup + args.steps)
    n = int(max(1, min(cpu_sample(cfg), budget / max(t1[0], 1e-3))))
    act = oracle_static_scales(cfg, inp) if cfg.wdtype == 3 else (1.0, 1.0)
    L, xs = oracle_sample(cfg, inp, n, act)
    n = xs.shape[0]
    times, cores = oracle_times(L, xs, args.warmup + args.steps), oracle.num_threads()
    timed = times[args.warmup:]
    tps = n * len(timed) / sum(timed)
    sample = f"{n} tokens of the {cfg.name} workload per step (whole layer, FP64)"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": tps, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(timed) / len(timed),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": describe(cfg)},
        "cpu_baseline": {"value": tps, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": tps, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ------------------------------------------------------------------ our arm
def run_ours(args, cfg: MoEConfig):
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    init_dist(world, "nccl")
    dev = torch.device("cuda", local)
    import expert_layer_dual_b200.moe as M

    inp = make_layer(cfg, device=dev)
    # each rank's own batch: same weights, a different draw of x
    if rank > 0:
        g = torch.Generator(device=dev).manual_seed(cfg.seed * 1000 + 500 + rank)
        inp["x"] = torch.randn(inp["x"].shape, generator=g, device=dev).to(torch.bfloat16)
    layer = M.MoELayer(cfg, inp, device=dev)
    x = inp["x"]
    y = torch.empty_like(x)
    shape = layer.shape(cfg.T)
    stream = torch.cuda.current_stream()

    # routing statistics of this batch (outside the timed region)
    logits = torch.empty((cfg.T, cfg.E), dtype=torch.float32, device=dev)
    M.router_logits(x.view(torch.uint16), layer.router_hi, layer.router_lo, layer.router_bias, logits)
    ids = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=dev)
    wts = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=dev)
    M.route_topk(logits, cfg.k, int(cfg.renorm), ids, wts)
    counts = torch.bincount(ids.view(-1).long(), minlength=cfg.E)
    n_active = int((counts > 0).sum().item())

    nev = M.PROFILE_EVENTS
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(args.steps)]
    for row in events:
        for e in row:
            e.record(stream)  # creates the event handles
    warm = [torch.cuda.Event(enable_timing=True) for _ in range(nev)]
    for e in warm:
        e.record(stream)
    for _ in range(args.warmup):
        M.forward_profiled(shape, layer.weights, x.view(torch.uint16), y.view(torch.uint16), layer.ws, warm)
    torch.cuda.synchronize()
    if layer.device_status() != M.OK:
        raise RuntimeError("device status after warm-up: " + M.status_string(layer.device_status()))

    # the timed steps: one moe_forward per step, all K of them captured in one
    # CUDA graph (the library's launches are capturable) so host launch gaps do
    # not count; each step records its stage events as event nodes of the graph,
    # so the per-stage (roofline) times come from the timed replay itself
    graph = None
    stage_source = "eager moe_forward_profiled launches (the timed steps)"
    if not args.no_graph:
        y_ref = y.clone()
        one = torch.cuda.CUDAGraph()
        with torch.cuda.graph(one):
            M.forward(shape, layer.weights, x.view(torch.uint16), y.view(torch.uint16), layer.ws)
        one.replay()
        torch.cuda.synchronize()
        if not torch.equal(y, y_ref) or layer.device_status() != M.OK:
            raise RuntimeError("graph replay does not reproduce the eager forward")
        del one
        graph = torch.cuda.CUDAGraph()
        try:
            with torch.cuda.graph(graph):
                for i in range(args.steps):
                    M.forward_profiled(shape, layer.weights, x.view(torch.uint16), y.view(torch.uint16),
                                       layer.ws, events[i])
            stage_source = "event nodes inside the timed CUDA graph replay"
        except Exception:  # noqa: BLE001 -- event nodes unavailable: time stages eagerly after
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for i in range(args.steps):
                    M.forward(shape, layer.weights, x.view(torch.uint16), y.view(torch.uint16), layer.ws)
            stage_source = "eager moe_forward_profiled pass after the timed graph replay"
        graph.replay()                                      # untimed: more warm-up steps
        torch.cuda.synchronize()
        if not torch.equal(y, y_ref) or layer.device_status() != M.OK:
            raise RuntimeError("the K-step graph does not reproduce the eager forward")
        stream = torch.cuda.current_stream()

    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(nvml_bus_id(dev)) as clocks:
        barrier()
        torch.cuda.synchronize()
        t_start.record(stream)
        if graph is not None:
            graph.replay()                                  # exactly K steps
        else:
            for i in range(args.steps):
                M.forward_profiled(shape, layer.weights, x.view(torch.uint16), y.view(torch.uint16),
                                   layer.ws, events[i])
        t_end.record(stream)
        torch.cuda.synchronize()
        barrier()
    ms_total = t_start.elapsed_time(t_end)
    ms_total = max_over_ranks(ms_total, dev)
    if graph is not None and stage_source.startswith("eager"):
        for i in range(args.steps):
            M.forward_profiled(shape, layer.weights, x.view(torch.uint16), y.view(torch.uint16),
                               layer.ws, events[i])
        torch.cuda.synchronize()
    ms_step = ms_total / args.steps
    value = world * cfg.T * args.steps / (ms_total / 1e3)

    stage_ms = {name: 0.0 for name in M.STAGES}
    for row in events:
        for j, name in enumerate(M.STAGES):
            stage_ms[name] += row[j].elapsed_time(row[j + 1]) / args.steps
    if layer.device_status() != M.OK:
        raise RuntimeError("device status after timing: " + M.status_string(layer.device_status()))

    # roofline of the dominant kernel (the gate-up GEMM)
    sustained = power_capped(clocks.summary(), ms_total)
    hbm_peak, tflops_peak, peak_kind = load_peaks(sustained)
    gu_ms = stage_ms["gemm_gateup"]
    gu_flops, gu_bytes = gateup_algorithmic(cfg, cfg.T, n_active)
    dn_flops, dn_bytes = down_algorithmic(cfg, cfg.T, n_active)
    ai = gu_flops / gu_bytes
    ridge = tflops_peak * 1e12 / (hbm_peak * 1e9) * (2 if cfg.wdtype else 1)
    if ai < ridge:
        roof = {"bound": "hbm", "achieved": gu_bytes / (gu_ms / 1e3) / 1e9, "peak": hbm_peak,
                "unit": "GB/s"}
    else:
        peak = tflops_peak * (2 if cfg.wdtype else 1)
        roof = {"bound": "tensor", "achieved": gu_flops / (gu_ms / 1e3) / 1e12, "peak": peak,
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel"] = gateup_kernel(cfg, cfg.T, torch.cuda.get_device_properties(dev).multi_processor_count)
    tf_key = ("bf16_tflops_sustained (the SM clock sat below 90% of its maximum)" if sustained
              else "bf16_tflops (burst: the SM clock stayed at its maximum)")
    roof["peak_source"] = (f"{peak_kind} MEASURED_PEAKS.json "
                           + ("hbm_gbs" if roof["bound"] == "hbm"
                              else tf_key + (" x2 (e4m3 nominal ratio)" if cfg.wdtype else "")))
    roof["traffic"], roof["traffic_source"] = recorded_traffic(roof["kernel"], cfg.name)
    roof["algorithmic_bytes"] = gu_bytes
    roof["algorithmic_flops"] = gu_flops
    roof["launch_ms"] = gu_ms
    roof["launch_ms_source"] = stage_source
    if roof["bound"] == "hbm":
        roof["peak_note"] = ("the measured peak is a device-to-device copy (half reads, half writes); "
                             "this kernel's traffic is almost all reads, which the HBM serves a little "
                             "faster, so frac can exceed 1 slightly")

    # end to end through host buffers: every step copies its x in from pinned host
    # memory, runs the forward and copies y out (moe_forward_host_async), the
    # steps pipelined over two streams with one workspace each, so one step's
    # copies overlap the other's kernels
    xh = [x.cpu().pin_memory() for _ in range(2)]
    yh = [torch.empty_like(xh[0]).pin_memory() for _ in range(2)]
    wss = [layer.ws, torch.empty_like(layer.ws)]
    streams = [torch.cuda.Stream(device=dev) for _ in range(2)]
    for i in range(max(2, args.warmup)):
        layer.forward_host_async(xh[i % 2], yh[i % 2], streams[i % 2], wss[i % 2])
    torch.cuda.synchronize()
    if not torch.equal(yh[0].to(dev), y) or layer.device_status() != M.OK:
        raise RuntimeError("the host-buffer forward does not reproduce the device forward")
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    done = [torch.cuda.Event() for _ in range(2)]
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for st in streams:
        st.wait_event(e0)
    for i in range(args.steps):
        layer.forward_host_async(xh[i % 2], yh[i % 2], streams[i % 2], wss[i % 2])
    for j, st in enumerate(streams):
        done[j].record(st)
        stream.wait_event(done[j])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    e2e = {"value": world * cfg.T * args.steps / (e2e_ms / 1e3), "unit": UNIT,
           "h2d_bytes_per_step": xh[0].numel() * xh[0].element_size(),
           "d2h_bytes_per_step": yh[0].numel() * yh[0].element_size(),
           "pipeline": "moe_forward_host_async, steps alternating over 2 streams (one workspace each)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        L, xs = oracle_sample(cfg, inp, cpu_sample(cfg), layer.act_scales)
        n, cores = xs.shape[0], oracle.num_threads()
        times = oracle_times(L, xs, 1)
        # repeat up to about 10 s of CPU work (at most 30 s)
        reps = int(min(30.0, max(10.0, times[0])) // max(times[0], 1e-3))
        if reps > 1:
            times += oracle_times(L, xs, reps - 1)
        cpu = {"value": n * len(times) / sum(times), "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"first {n} tokens of the {cfg.name} batch, whole layer in FP64, "
                         f"{len(times)} runs, {sum(times):.1f} s of CPU time"}

    launches_per_step = kernels_per_step(cfg, cfg.T)
    if rank == 0:
        out = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": {0: "bf16", 1: "f8e4m3", 2: "mxf8e4m3", 3: "f8e4m3"}[cfg.wdtype],
            "data": "synthetic",
            "config": {"workload": describe(cfg), "tokens_per_gpu": cfg.T,
                       "active_experts": n_active,
                       "l2": "no flush: the expert weights read each step "
                             f"({(gu_bytes + dn_bytes) / 1e9:.1f} GB) exceed the 126 MB L2",
                       "parallelism": f"{world} independent replicas (tokens sharded, no collective)",
                       "launch": ("one CUDA graph holding the K steps' moe_forward launches, replayed once"
                                  if graph is not None
                                  else "eager moe_forward_profiled launches")},
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks.summary(),
            "stages_ms": stage_ms,
            "tflops": cfg.flops() / (ms_step / 1e3) / 1e12 * world,
            "layer_weight_gbs": (gu_bytes + dn_bytes) / (ms_step / 1e3) / 1e9,
        }
        print(json.dumps(out), flush=True)
    if torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="skew", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-graph", action="store_true",
                    help="time eager launches with stage events instead of CUDA graph replays")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override T (a smaller case of the same layer, e.g. for profiling)")
    ap.add_argument("--experts", type=int, default=None,
                    help="override E (a smaller case of the same layer, e.g. for profiling)")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)  # at least 3 untimed warm-up steps, whatever is asked
    cfg = CONFIGS[args.config]
    if args.tokens is not None or args.experts is not None:
        import dataclasses
        cfg = dataclasses.replace(cfg, T=args.tokens or cfg.T, E=args.experts or cfg.E,
                                  name=f"{cfg.name}-T{args.tokens or cfg.T}-E{args.experts or cfg.E}")
    if args.impl == "reference":
        run_reference(args, cfg)
    else:
        run_ours(args, cfg)


if __name__ == "__main__":
    main()
