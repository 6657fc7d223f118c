#!/usr/bin/env python3
"""Benchmark of the fused RMSNorm + BitLinear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--layers L] [--secondary LIST]

Prints ONE JSON line (rank 0).  Default workload: the training-batch forward
at the 1.3B width, M = 2^8 x 2048 = 524288 tokens through the full BitLinear
set of one layer (4x 2048->2048, 2x 2048->5632, 5632->2048), each projection
group with its own fused RMSNorm + int8 quantisation: the largest
configuration that fits one GPU.  The same line carries a `secondary` list
with the prefill step at the 2.7B width (the int8 tensor-core target) and the
decode steps at the 2.7B width for 1, 8 and 32 tokens (the HBM target), each
timed in the same run with its own step time, roofline, end-to-end figure and
clock record.

A step = one pass of the whole hot path (RMSNorm, int8 quantisation, ternary
contraction, rescale: every projection of every layer set) over one batch of M
tokens, replayed as one CUDA graph.  `value` = tokens/s through one layer set
(M * L * n_gpus / step time).  Weights are packed once, before timing (offline
on the pages' terms).  Decode steps repeat the layer set over L = 32 layer
sets with distinct weights so that the packed weights (634 MB) exceed L2 and
stream from HBM every step.

--impl reference times the CPU oracle (the only reference this method has on
the box), on bounded samples of the same workload.  Multi-GPU: one process per
GPU (torchrun), token-parallel replicas with no data-path collective; a
barrier and a MAX all-reduce of the device-timed step time only.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from bitlinear_rmsnorm_quant_b200 import inputs as I  # noqa: E402
from bitlinear_rmsnorm_quant_b200 import workloads as WL  # noqa: E402

METRIC = "fused RMSNorm+BitLinear tokens/s; GB/s or int8 TOPS as % of B200 roofline"

FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
INT8_PER_BF16 = 2.0   # nominal dense ratio int8 : bf16 (4.5 : 2.25 POPS)
L2_BYTES = 126 * 1024 * 1024


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0}, "fallback"


def run_scan(args, dist):
    """The MLGRU recurrence over B x T tokens of D channels, pre-activations
    resident in HBM (4 x 32 MB in, 32 MB out: inputs larger than L2)."""
    from bitlinear_rmsnorm_quant_b200 import mmf
    B, T, D = SCAN_SHAPE
    dev = torch.device("cuda", dist.local_rank)
    gen = torch.Generator(device=dev).manual_seed(5 + dist.rank)
    mk = lambda: (torch.randn((B, T, D), generator=gen, device=dev) * 2.0).to(torch.bfloat16)
    fp, cp, gp = mk(), mk(), mk()
    h0 = torch.randn((B, D), generator=gen, device=dev)
    o = torch.empty((B, T, D), dtype=torch.bfloat16, device=dev)
    hl = torch.empty((B, D), dtype=torch.float32, device=dev)
    lib = mmf.lib()
    stream = torch.cuda.current_stream()

    def step():
        rc = lib.mmf_mlgru_scan(fp.data_ptr(), cp.data_ptr(), gp.data_ptr(), h0.data_ptr(), B, T, D, o.data_ptr(),
                                hl.data_ptr(), stream.cuda_stream)
        if rc != 0:
            raise mmf.MMFError("mmf_mlgru_scan", rc)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    dist.barrier()
    clocks = ClockSampler(dist.local_rank)
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    clocks.stop()
    dist.barrier()
    mmf.check_async()
    ms = dist.max(e0.elapsed_time(e1) / args.steps)
    # e2e: pre-activations from pinned host memory, o back to it
    h_in = [t.cpu().pin_memory() for t in (fp, cp, gp)]
    h_o = torch.empty(o.shape, dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(1, min(args.steps, 50))
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for _ in range(e2e_steps):
        for d_, h_ in zip((fp, cp, gp), h_in):
            d_.copy_(h_, non_blocking=True)
        step()
        h_o.copy_(o, non_blocking=True)
    f1.record()
    torch.cuda.synchronize()
    e2e_ms = dist.max(f0.elapsed_time(f1) / e2e_steps)
    tokens = B * T * dist.world
    nbytes = B * T * D * 2 * 4 + B * D * 4 * 2   # three inputs and o (bf16), h0 and h_last (fp32)
    peaks, peak_src = load_peaks()
    achieved = nbytes / (ms / 1e3) / 1e9
    res = {
        "metric": METRIC, "value": round(tokens / (ms / 1e3), 2),
        "unit": "tokens/s (one token through the MLGRU recurrence at the 1.3B width)",
        "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (torch normal pre-activations x2, bf16)",
        "config": {"workload": "mlgru-scan-1.3b", "B": B, "T": T, "D": D,
                   "l2": "inputs larger than L2 (4 x 32 MB)", "parallelism": f"dp{dist.world} (replicas)"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": float(peaks["hbm_gbs"]),
                     "unit": "GB/s", "frac": round(achieved / float(peaks["hbm_gbs"]), 4), "traffic": None,
                     "kernel": "mlgru_scan_kernel", "peak_source": f"{peak_src} hbm_gbs",
                     "algorithmic_bytes_per_launch": nbytes},
        "e2e": {"value": round(tokens / (e2e_ms / 1e3), 2), "unit": "tokens/s",
                "h2d_bytes_per_step": int(3 * B * T * D * 2), "d2h_bytes_per_step": int(B * T * D * 2),
                "steps": e2e_steps},
        "gpu_launches": args.steps,
        "clocks": clocks.summary(),
    }
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = scan_cpu_baseline(fp[:1, :256].cpu(), cp[:1, :256].cpu(), gp[:1, :256].cpu(), D)
    return res


def run_bwd(args, dist):
    """Backward of the three prefill projections at the 1.3B width (M = 8192):
    per projection the quantiser (the forward's codes), the two tensor-core
    products (dr = dy . w~ with the weights unpacked from their 2-bit codes,
    dW = dy^T . x_q with the codes scaled on the way in), the RMSNorm backward
    and the two-stage dgamma sum: 6 launches, all this library's kernels."""
    from bitlinear_rmsnorm_quant_b200 import mmf
    wl = WL.PREFILL_1P3B
    M = wl.M
    dev = torch.device("cuda", dist.local_rank)
    lib = mmf.lib()
    stream = torch.cuda.current_stream()
    items = []
    for j, p in enumerate(wl.projections):
        x = I.activations(wl.seed, M, p.K, index=p.input_index, device=dev)
        g = I.gamma(wl.seed, p.K, index=p.input_index, device=dev)
        W = I.latent_weights(wl.seed, p.N, p.K, index=j, device=dev)
        packed, scale = mmf.pack_ternary(W, wl.eps_w)
        del W
        dy = I.activations(wl.seed, M, p.N, index=32 + j, device=dev)
        dx = torch.empty((M, p.K), dtype=torch.bfloat16, device=dev)
        dg = torch.empty(p.K, dtype=torch.float32, device=dev)
        dW = torch.empty((p.N, p.K), dtype=torch.float32, device=dev)
        ws = torch.empty(int(lib.mmf_bwd_workspace_bytes(M, p.K, p.N)), dtype=torch.uint8, device=dev)
        items.append((p, x, g, packed, scale, dy, dx, dg, dW, ws))

    def step():
        for p, x, g, packed, scale, dy, dx, dg, dW, ws in items:
            rc = lib.mmf_bitlinear_bwd(dy.data_ptr(), x.data_ptr(), g.data_ptr(), wl.eps, packed.data_ptr(),
                                       scale.data_ptr(), M, p.K, p.N, dx.data_ptr(), dg.data_ptr(), dW.data_ptr(),
                                       ws.data_ptr(), ws.numel(), stream.cuda_stream)
            if rc != 0:
                raise mmf.MMFError("mmf_bitlinear_bwd", rc)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    dist.barrier()
    clocks = ClockSampler(dist.local_rank)
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    clocks.stop()
    dist.barrier()
    mmf.check_async()
    ms = dist.max(e0.elapsed_time(e1) / args.steps)
    flops = sum(2 * 2 * M * p.N * p.K for p in wl.projections)
    peaks, peak_src = load_peaks()
    achieved = flops / (ms / 1e3) / 1e12
    peak = float(peaks["bf16_tflops"])
    return {
        "metric": METRIC, "value": round(M * dist.world / (ms / 1e3), 2),
        "unit": "tokens/s (one token back through the three prefill projections)",
        "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded SplitMix64/Box-Muller)",
        "config": {"workload": "bwd-prefill-1.3b", "M": M, "projections": [f"{p.K}->{p.N}" for p in wl.projections],
                   "parallelism": f"dp{dist.world} (replicas)"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": None,
                     "kernel": "gemm_bwd_kernel (tcgen05 kind::f16), whole backward step",
                     "peak_source": f"{peak_src} bf16_tflops", "algorithmic_flops_per_step": flops},
        "gpu_launches": 6 * len(items) * args.steps,
        "clocks": clocks.summary(),
    }


def scan_cpu_baseline(fp, cp, gp, D):
    """The oracle's recurrence on a sample of one sequence's first 256 tokens."""
    import numpy as np

    from oracle import load
    orc = load()
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    f_, c_, g_ = bits(fp), bits(cp), bits(gp)
    t0 = time.perf_counter()
    reps = 0
    while time.perf_counter() - t0 < 5.0:
        orc.mlgru_scan(f_, c_, g_)
        reps += 1
    dt = (time.perf_counter() - t0) / reps
    return {"value": round(fp.shape[1] / dt, 2), "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"1 sequence x {fp.shape[1]} tokens x {D} channels"}


def library_int8_tops(n: int = 8192, reps: int = 5):
    """Context for the tensor roofline: a library int8 GEMM (torch._int_mm,
    cuBLASLt) at n^3 on this GPU, best of `reps`, CUDA events."""
    try:
        a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device="cuda")
        b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device="cuda")
        torch._int_mm(a, b)
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._int_mm(a, b)
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        del a, b
        return round(2.0 * n ** 3 / (best / 1e3) / 1e12, 1)
    except Exception as exc:  # the measurement is context only
        return f"unavailable: {type(exc).__name__}"


# ----------------------------------------------------------------------------- dist

class Dist:
    def __init__(self, gpus: int):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if self.world > 1:
            import torch.distributed as dist
            backend = "nccl" if torch.cuda.is_available() else "gloo"
            if backend == "nccl":
                torch.cuda.set_device(self.local_rank)
            import datetime
            dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist
        if gpus != self.world:
            raise SystemExit(f"--gpus {gpus} but WORLD_SIZE={self.world}")

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, v: float) -> float:
        if self.pg is None:
            return v
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML during the timed region."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
               0x10: "sync_boost", 0x1: "gpu_idle"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.ok = False
        self.samples, self.reasons = [], 0
        self.period = period_s
        try:
            import pynvml as N
            N.nvmlInit()
            self.N = N
            try:
                p = torch.cuda.get_device_properties(device_index)
                bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
                self.h = N.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.h = N.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = N.nvmlDeviceGetMaxClockInfo(self.h, N.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()
        self._t = None

    def _read(self):
        N = self.N
        self.samples.append(N.nvmlDeviceGetClockInfo(self.h, N.NVML_CLOCK_SM))
        try:
            self.reasons |= int(N.nvmlDeviceGetCurrentClocksEventReasons(self.h))
        except Exception:
            self.reasons |= int(N.nvmlDeviceGetCurrentClocksThrottleReasons(self.h))

    def _loop(self):
        while not self._stop.is_set():
            try:
                self._read()
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._loop, daemon=True)
            self._t.start()

    def stop(self):
        if self._t is not None:
            self._stop.set()
            self._t.join()
            try:
                self._read()
            except Exception:
                pass

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [v for k, v in self.REASONS.items() if self.reasons & k and v != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ----------------------------------------------------------------------------- workloads

WORKLOADS = {
    "decode-2.7b-m1": (lambda: WL.decode_2p7b(1), 32),
    "decode-2.7b-m8": (lambda: WL.decode_2p7b(8), 32),
    "decode-2.7b-m32": (lambda: WL.decode_2p7b(32), 32),
    "decode-370m": (lambda: WL.DECODE_370M, 160),
    "prefill-1.3b": (lambda: WL.PREFILL_1P3B, 1),
    "prefill-2.7b": (lambda: WL.PREFILL_2P7B, 1),
    "train-fwd-1.3b": (lambda: WL.TRAIN_FWD_1P3B, 1),
    "smoke-256": (lambda: WL.SMOKE, 1),
    "mlgru-scan-1.3b": (None, 1),   # the token mixer's recurrence alone (run_scan)
    "bwd-prefill-1.3b": (None, 1),  # straight-through backward of the prefill projections (run_bwd)
}
SCAN_SHAPE = (4, 2048, 2048)        # sequences, tokens, channels: 4 x 2048 tokens at the 1.3B width
DEFAULT_WORKLOAD = "train-fwd-1.3b"
DEFAULT_SECONDARY = "prefill-2.7b,decode-2.7b-m1,decode-2.7b-m8,decode-2.7b-m32"
E2E_SINGLE_SHOT_BYTES = 8 << 30     # above this x + y, the end-to-end step streams token chunks
E2E_CHUNKS = 8


def proj_bytes(M, K, N):
    """Algorithmic HBM bytes of one fused BitLinear call: packed W, x, gamma, y, beta."""
    return N * K // 4 + 2 * M * K + 4 * K + 2 * M * N + 4


def proj_ops(M, K, N):
    return 2 * M * N * K


def contraction_kernel(mmf, wl) -> str:
    """The kernel that contracts this workload's tokens with the weights, as
    the library dispatches it: the fused decode kernel (normalisation in the
    same launch, no workspace), the decode tensor-core kernel (4 .. 32 tokens)
    or the large-M tensor-core kernel."""
    p = wl.projections[0]
    if mmf.workspace_bytes(wl.M, p.K, p.N) == 0:
        return "gemv_kernel"
    return "gemv_wide_kernel" if wl.M <= 32 else "gemm_tc_kernel"


def hbm_bound(wl) -> bool:
    """Decode batches (M <= 32) are bound by streaming the packed weights: 2M
    int8 operations per 0.25 byte is below the int8 ridge point of the chip."""
    return wl.M <= 32


# ----------------------------------------------------------------------------- copy kernel

def time_hbm_copy(dev, nbytes: int = 1 << 30, reps: int = 10):
    """The library's 128-bit streaming copy (mmf_hbm_copy) on 1 GiB: read +
    write bytes per second, median of `reps` CUDA-event timings.  Stated next
    to the measured copy bandwidth the HBM fractions use."""
    from bitlinear_rmsnorm_quant_b200 import mmf
    src = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    dst = torch.empty_like(src)
    src.fill_(1)
    for _ in range(3):
        mmf.hbm_copy(src, dst)
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        mmf.hbm_copy(src, dst)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    mmf.check_async()
    ms = statistics.median(times)
    del src, dst
    return {"kernel": "hbm_copy_kernel (mmf_hbm_copy)", "bytes_copied": nbytes,
            "gbs": round(2 * nbytes / (ms / 1e3) / 1e9, 1), "ms": round(ms, 4),
            "note": "read + write bytes / time, median of %d copies of 1 GiB" % reps}


# ----------------------------------------------------------------------------- our arm

class Step:
    """One workload's step: packed weights, inputs and outputs resident on the
    device, the library calls of one step, and their CUDA graph."""

    def __init__(self, wl, L, dist, args):
        from bitlinear_rmsnorm_quant_b200 import mmf
        self.mmf = mmf
        self.wl, self.L = wl, L
        dev = torch.device("cuda", dist.local_rank)
        self.dev = dev
        M = wl.M
        seed = wl.seed + 7919 * dist.rank  # each rank draws its own tokens and weights
        # -- weights: drawn on the device, packed once (offline), fp32 freed
        self.packed, self.scales = {}, {}
        for l in range(L):
            for j, p in enumerate(wl.projections):
                W = I.latent_weights(seed, p.N, p.K, index=64 * l + j, device=dev)
                self.packed[l, j], self.scales[l, j] = mmf.pack_ternary(W, wl.eps_w)
                del W

        # -- activations and outputs: views into one flat device buffer each
        def carve(shapes):
            offs, total = [], 0
            for shp in shapes:
                offs.append(total)
                total += (math.prod(shp) + 7) // 8 * 8      # 16-byte aligned views
            flat = torch.empty(max(total, 8), dtype=torch.bfloat16, device=dev)
            return flat, [flat[o:o + math.prod(shp)].view(*shp) for o, shp in zip(offs, shapes)]

        x_keys = [(l, idx) for l in range(L) for idx, _ in wl.inputs()]
        self.x_flat, x_views = carve([(M, dict(wl.inputs())[idx]) for _, idx in x_keys])
        self.xs = dict(zip(x_keys, x_views))
        for (l, idx), xv in self.xs.items():
            xv.copy_(I.activations(seed, M, xv.shape[1], index=64 * l + idx, outlier_frac=wl.outlier_frac,
                                   device=dev))
        self.gs = {(l, idx): I.gamma(seed, K, index=64 * l + idx, device=dev)
                   for l in range(L) for idx, K in wl.inputs()}
        y_keys = [(l, j) for l in range(L) for j in range(len(wl.projections))]
        self.y_flat, y_views = carve([(M, wl.projections[j].N) for _, j in y_keys])
        self.ys = dict(zip(y_keys, y_views))
        self.groups = {}
        for j, p in enumerate(wl.projections):
            self.groups.setdefault(p.input_index, []).append(j)
        ws_need = max(max(mmf.workspace_bytes(M, wl.projections[js[0]].K,
                                              sum(wl.projections[j].N for j in js)),
                          max(mmf.workspace_bytes(M, wl.projections[j].K, wl.projections[j].N) for j in js))
                      for js in self.groups.values())
        self.ws = torch.empty(max(ws_need, 256), dtype=torch.uint8, device=dev)
        self.lib = mmf.lib()
        self.flags = 0 if args.no_pdl else mmf.FWD_PDL
        self.api, self.glu = args.api, args.glu
        self.keep = []           # ctypes arrays that must outlive the graph
        self.launches_per_step = 0
        self.bytes_per_step = 0
        self.ops_per_step = 0
        self.calls = self.make_calls(0, M, count=True)
        self.graph = None

    def make_calls(self, t0, t1, count=False):
        """The library calls of one step over tokens [t0, t1) (all of them for
        the graph; a token chunk for the streamed end-to-end step)."""
        wl, mmf, lib = self.wl, self.mmf, self.lib
        Mc = t1 - t0
        calls = []
        for l in range(self.L):
            for idx, js in sorted(self.groups.items()):
                K = wl.projections[js[0]].K
                x, g = self.xs[l, idx][t0:t1], self.gs[l, idx]
                y = {j: self.ys[l, j][t0:t1] for j in range(len(wl.projections))}
                names = [wl.projections[j].name for j in js]
                if self.glu and names == ["down"]:
                    # the channel mixer's down projection reads this layer set's gate and up
                    # outputs through the fused GLU call (SiLU(g) * u formed while normalising)
                    jg = [j for j, p in enumerate(wl.projections) if p.name == "gate"][0]
                    ju = [j for j, p in enumerate(wl.projections) if p.name == "up"][0]
                    j = js[0]
                    p = wl.projections[j]
                    calls.append((lib.mmf_bitlinear_fwd_glu,
                                  (y[jg].data_ptr(), y[ju].data_ptr(), g.data_ptr(), wl.eps,
                                   self.packed[l, j].data_ptr(), self.scales[l, j].data_ptr(), Mc, p.K, p.N,
                                   y[j].data_ptr(), self.ws.data_ptr(), self.ws.numel(), self.flags)))
                    if count:
                        self.launches_per_step += mmf.fwd_launches(Mc, p.K, p.N)
                        self.bytes_per_step += p.N * p.K // 4 + 2 * Mc * p.N + 4 + 2 * (2 * Mc * K) + 4 * K
                        self.ops_per_step += proj_ops(Mc, p.K, p.N)
                    continue
                if self.api == "group":
                    arr = mmf.projection_array([(self.packed[l, j], self.scales[l, j], y[j], wl.projections[j].N)
                                                for j in js])
                    self.keep.append(arr)
                    calls.append((lib.mmf_bitlinear_fwd_group,
                                  (x.data_ptr(), g.data_ptr(), wl.eps, Mc, K, arr, len(js), self.ws.data_ptr(),
                                   self.ws.numel(), self.flags)))
                    if count:
                        self.launches_per_step += mmf.fwd_launches(Mc, K, sum(wl.projections[j].N for j in js),
                                                                   len(js))
                else:
                    for j in js:
                        p = wl.projections[j]
                        calls.append((lib.mmf_bitlinear_fwd,
                                      (x.data_ptr(), g.data_ptr(), wl.eps, self.packed[l, j].data_ptr(),
                                       self.scales[l, j].data_ptr(), Mc, p.K, p.N, y[j].data_ptr(),
                                       self.ws.data_ptr(), self.ws.numel())))
                        if count:
                            self.launches_per_step += mmf.fwd_launches(Mc, p.K, p.N)
                if count:
                    for j in js:
                        p = wl.projections[j]
                        self.bytes_per_step += p.N * p.K // 4 + 2 * Mc * p.N + 4
                        self.ops_per_step += proj_ops(Mc, p.K, p.N)
                    self.bytes_per_step += 2 * Mc * K + 4 * K      # x and gamma once per shared input
        return calls

    @staticmethod
    def run(calls, stream_ptr):
        for f, a in calls:
            rc = f(*a, stream_ptr)
            if rc != 0:
                from bitlinear_rmsnorm_quant_b200 import mmf
                raise mmf.MMFError(f.__name__, rc)

    def quant_calls(self):
        """The step's quantiser launches alone: mmf_quantize_act over every
        shared input of every layer set (the same quantiser kernels the grouped
        calls launch, without the code-sum output), into scratch codes."""
        wl, M = self.wl, self.wl.M
        kmax = max(K for _, K in wl.inputs())
        self.q_scratch = torch.empty(M * kmax, dtype=torch.int8, device=self.dev)
        self.a_scratch = torch.empty(max(M, 4), dtype=torch.float32, device=self.dev)
        return [(self.lib.mmf_quantize_act, (self.xs[l, idx].data_ptr(), self.gs[l, idx].data_ptr(), wl.eps, M, K,
                                             self.q_scratch.data_ptr(), self.a_scratch.data_ptr()))
                for l in range(self.L) for idx, K in wl.inputs()]

    def capture_calls(self, calls):
        """A CUDA graph of `calls` (run once outside capture first: one-time
        per-device set-up)."""
        self.run(calls, torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
        self.mmf.check_async()
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        with torch.cuda.stream(cap):
            graph.capture_begin()
            self.run(calls, cap.cuda_stream)
            graph.capture_end()
        torch.cuda.synchronize()
        return graph

    def capture(self):
        self.graph = self.capture_calls(self.calls)

    def time_graph(self, steps, warmup, dist, graph=None, sample_clocks=True):
        graph = graph or self.graph
        for _ in range(warmup):
            graph.replay()
        torch.cuda.synchronize()
        self.mmf.check_async()
        clocks = ClockSampler(dist.local_rank) if sample_clocks else None
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        dist.barrier()
        torch.cuda.synchronize()
        if clocks:
            clocks.start()
        e0.record()
        for _ in range(steps):
            graph.replay()
        e1.record()
        torch.cuda.synchronize()
        if clocks:
            clocks.stop()
        dist.barrier()
        self.mmf.check_async()
        return dist.max(e0.elapsed_time(e1) / steps), (clocks.summary() if clocks else None)

    def time_e2e(self, steps, dist):
        """End to end through the C ABI with host buffers: every step copies all
        inputs from pinned host memory to the device and all outputs back.
        Small steps: one copy in, the graph, one copy out.  Large steps (x + y
        above E2E_SINGLE_SHOT_BYTES): the tokens stream in E2E_CHUNKS chunks on
        three streams (copy in, compute, copy out) so the two copy directions
        and the kernels overlap; host staging is two pinned slots per direction
        (a chunk's host bytes are its inputs)."""
        xb, yb = self.x_flat.numel() * 2, self.y_flat.numel() * 2
        if xb + yb <= E2E_SINGLE_SHOT_BYTES or self.L != 1:
            h_x = self.x_flat.cpu().pin_memory()
            h_y = torch.empty(self.y_flat.shape, dtype=torch.bfloat16).pin_memory()

            def e2e_step():
                self.x_flat.copy_(h_x, non_blocking=True)
                self.graph.replay()
                h_y.copy_(self.y_flat, non_blocking=True)

            n = max(1, min(steps, 200))
            for _ in range(3):
                e2e_step()
            torch.cuda.synchronize()
            dist.barrier()
            f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            f0.record()
            for _ in range(n):
                e2e_step()
            f1.record()
            torch.cuda.synchronize()
            dist.barrier()
            ms = dist.max(f0.elapsed_time(f1) / n)
            del h_x, h_y
            return ms, n, {"mode": "one copy in, the step's graph, one copy out"}
        wl, M = self.wl, self.wl.M
        C = E2E_CHUNKS
        bounds = [(M * i // C, M * (i + 1) // C) for i in range(C)]
        xin = [(idx, self.xs[0, idx]) for idx, _ in wl.inputs()]
        outs = [(j, self.ys[0, j]) for j in range(len(wl.projections))]
        rows = bounds[0][1] - bounds[0][0]
        h_x = [{idx: t[:rows].cpu().pin_memory() for idx, t in xin} for _ in range(2)]
        h_y = [{j: torch.empty((rows, t.shape[1]), dtype=torch.bfloat16).pin_memory() for j, t in outs}
               for _ in range(2)]
        chunk_calls = [self.make_calls(t0, t1) for t0, t1 in bounds]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        s_cmp = torch.cuda.current_stream()

        def e2e_step():
            # a step's copies in start once the previous step's kernels are done with x
            s_in.wait_stream(s_cmp)
            for c, (t0, t1) in enumerate(bounds):
                n_r = t1 - t0
                with torch.cuda.stream(s_in):
                    for idx, t in xin:
                        t[t0:t1].copy_(h_x[c % 2][idx][:n_r], non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(s_in)
                s_cmp.wait_event(ev)
                self.run(chunk_calls[c], s_cmp.cuda_stream)
                ev2 = torch.cuda.Event()
                ev2.record(s_cmp)
                s_out.wait_event(ev2)
                with torch.cuda.stream(s_out):
                    for j, t in outs:
                        h_y[c % 2][j][:n_r].copy_(t[t0:t1], non_blocking=True)
            ev3 = torch.cuda.Event()
            ev3.record(s_out)
            s_cmp.wait_event(ev3)

        n = max(1, min(steps, 5))
        e2e_step()
        torch.cuda.synchronize()
        dist.barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(s_cmp)
        for _ in range(n):
            e2e_step()
        f1.record(s_cmp)
        torch.cuda.synchronize()
        dist.barrier()
        self.mmf.check_async()
        ms = dist.max(f0.elapsed_time(f1) / n)
        del h_x, h_y
        return ms, n, {"mode": f"{C} token chunks streamed on three streams (copy in / kernels / copy out), "
                               "two pinned host slots per direction"}


def run_workload(name, args, dist, steps, warmup, peaks, peak_src, copy_gbs=None, layers=0):
    """Times one workload's step; returns its JSON object (without cpu_baseline)."""
    make, default_layers = WORKLOADS[name]
    wl = make()
    L = layers or default_layers
    st = Step(wl, L, dist, args)
    st.capture()
    ms, clocks = st.time_graph(steps, warmup, dist)
    e2e_ms, e2e_steps, e2e_mode = st.time_e2e(steps, dist)
    M = wl.M
    streamed = sum(p.N * p.K // 4 for p in wl.projections) * L + 2 * st.x_flat.numel() + 2 * st.y_flat.numel()
    l2_note = (f"inputs larger than L2: {streamed / 1e6:.0f} MB of packed weights, x and y per step > 126 MB"
               if streamed > L2_BYTES else
               f"working set below L2 ({streamed / 1e6:.1f} MB per step, not flushed): a parity-size run, "
               "not a throughput figure")
    tokens_per_step = M * L * dist.world
    value = tokens_per_step / (ms / 1e3)
    e2e_value = tokens_per_step / (e2e_ms / 1e3)
    kernel = contraction_kernel(st.mmf, wl)
    # the dominant kernel's own time: the step minus its quantiser launches,
    # which are timed alone in a graph of their own (none below 4 tokens, where
    # the decode kernel normalises and quantises in the same launch)
    split = None
    if kernel != "gemv_kernel" and not args.glu:
        qgraph = st.capture_calls(st.quant_calls())
        q_ms, _ = st.time_graph(max(3, min(steps, 50)), 3, dist, graph=qgraph, sample_clocks=False)
        del qgraph
        st.q_scratch = st.a_scratch = None
        if q_ms < ms:
            split = {"quantiser_ms_per_step": round(q_ms, 6), "kernel_ms_per_step": round(ms - q_ms, 6),
                     "quantiser_launches_per_step": L * len(wl.inputs()),
                     "method": "kernel time = step time - the step's quantiser launches timed alone "
                               "(mmf_quantize_act over the same inputs, own CUDA graph, CUDA events)"}
    k_ms = split["kernel_ms_per_step"] if split else ms
    k_launches = st.launches_per_step - (L * len(wl.inputs()) if split else 0)
    if hbm_bound(wl):
        if kernel == "gemv_kernel":
            k_bytes = st.bytes_per_step
            what = "packed weights, x and gamma once per shared input, y"
        else:
            # the contraction reads the packed weights and the codes once, writes y
            k_bytes = L * sum(sum(wl.projections[j].N * K // 4 + 2 * M * wl.projections[j].N + 4 for j in js)
                              + M * K + 8 * M
                              for K, js in ((wl.projections[js[0]].K, js) for js in st.groups.values()))
            what = "packed weights, codes and per-token sums once per shared input, y"
        achieved = k_bytes / (k_ms / 1e3) / 1e9
        step_achieved = st.bytes_per_step / (ms / 1e3) / 1e9
        peak = float(peaks["hbm_gbs"])
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "kernel": kernel, "traffic": None,
                "algorithmic_bytes_per_launch": round(k_bytes / max(k_launches, 1)),
                "kernel_launches_per_step": k_launches,
                "step_achieved": round(step_achieved, 1), "step_frac": round(step_achieved / peak, 4),
                "algorithmic_bytes_per_step": st.bytes_per_step,
                "peak_source": f"{peak_src} hbm_gbs (copy of 1 Gi bf16, read+write bytes)",
                "note": f"achieved = the kernel's algorithmic bytes ({what}) / its time per step, "
                        "inter-kernel gaps included; step_achieved = the layer's bytes / step time; traffic: "
                        "the ncu DRAM counters of this kernel are in the profiles, not measured in this run"}
        if copy_gbs:
            roof["copy_kernel_gbs"] = copy_gbs
            roof["frac_of_copy_kernel"] = round(achieved / copy_gbs, 4)
    else:
        achieved = st.ops_per_step / (k_ms / 1e3) / 1e12
        step_achieved = st.ops_per_step / (ms / 1e3) / 1e12
        # burst peak for a short step, sustained (power-capped) for a step of many ms
        long_step = (ms > 10.0 or ms * steps > 1000.0) and "bf16_tflops_sustained" in peaks
        peak_key = "bf16_tflops_sustained" if long_step else "bf16_tflops"
        peak = float(peaks[peak_key]) * INT8_PER_BF16
        burst = float(peaks["bf16_tflops"]) * INT8_PER_BF16
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "frac_of_burst": round(achieved / burst, 4),
                "frac_of_datasheet_4500": round(achieved / 4500.0, 4),
                "kernel": kernel, "traffic": None, "kernel_launches_per_step": k_launches,
                "algorithmic_ops_per_launch": round(st.ops_per_step / max(k_launches, 1)),
                "step_achieved": round(step_achieved, 1), "step_frac": round(step_achieved / peak, 4),
                "peak_source": f"{peak_src} {peak_key} x {INT8_PER_BF16} (nominal int8:bf16 dense ratio)",
                "algorithmic_ops_per_step": st.ops_per_step,
                "note": "achieved = 2MNK int8 operations / the contraction kernel's time per step; step_achieved "
                        "= the same over the whole step (quantisers included); traffic: the ncu DRAM counters "
                        "of this kernel are in the profiles, not measured in this run"}
    if split:
        roof["split"] = split
    if roof["bound"] == "tensor":
        # context: the datasheet's dense int8 figure over the whole step, and a
        # library int8 GEMM (8192^3) on this GPU, timed after this workload
        roof["step_frac_of_datasheet_4500"] = round(step_achieved / 4500.0, 4)
        lib_tops = library_int8_tops()
        roof["library_int8_gemm_tops"] = lib_tops
        if isinstance(lib_tops, float):
            roof["frac_of_library_int8_gemm"] = round(achieved / lib_tops, 4)
    res = {
        "metric": METRIC, "value": round(value, 2),
        "unit": "tokens/s (one token through one BitLinear layer set)",
        "n_gpus": dist.world, "steps": steps, "warmup": warmup, "ms_per_step": round(ms, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic (seeded SplitMix64/Box-Muller; random-init latent weights)",
        "config": {
            "workload": wl.name, "description": wl.description, "M": M, "layer_sets": L,
            "projections": [f"{p.K}->{p.N}" for p in wl.projections],
            "packed_weight_bytes": sum(p.N * p.K // 4 for p in wl.projections) * L,
            "l2": l2_note, "graph": "one CUDA graph per step",
            "parallelism": f"dp{dist.world} (token-parallel replicas)",
            "api": "mmf_bitlinear_fwd_group" if args.api == "group" else "mmf_bitlinear_fwd",
            "pdl": not args.no_pdl and args.api == "group", "launches_per_step": st.launches_per_step,
            "glu_down": bool(args.glu),
        },
        "roofline": roof,
        "e2e": {"value": round(e2e_value, 2), "unit": "tokens/s (one token through one BitLinear layer set)",
                "h2d_bytes_per_step": int(st.x_flat.numel() * 2), "d2h_bytes_per_step": int(st.y_flat.numel() * 2),
                "steps": e2e_steps, **e2e_mode},
        "gpu_launches": st.launches_per_step * steps,
        "clocks": clocks,
    }
    st.graph = None
    del st
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res, wl


# ----------------------------------------------------------------------------- oracle timing

def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def time_oracle(wl, sample_tokens: int | None, budget_s: float, max_reps: int | None = None,
                one_projection_per_rep: bool = False):
    """Times the CPU oracle (ternarised weights prepared untimed) on a bounded
    sample: rmsnorm+quant, ternary accumulation and rescale for each projection."""
    import numpy as np

    from oracle import load
    orc = load()
    M = wl.M if sample_tokens is None else min(wl.M, sample_tokens)
    prep = []
    for j, p in enumerate(wl.projections):
        W = I.latent_weights(wl.seed, p.N, p.K, index=j).numpy()
        wt, beta = orc.absmean_ternary(W, wl.eps_w)
        x = I.activations(wl.seed, M, p.K, index=p.input_index, outlier_frac=wl.outlier_frac)
        xb = x.view(torch.int16).numpy().view(np.uint16)
        g = I.gamma(wl.seed, p.K, index=p.input_index).numpy()
        prep.append((xb, g, wt, beta))
    per_proj = [[] for _ in prep]
    t_start = time.perf_counter()
    reps = 0
    while True:
        todo = [reps % len(prep)] if one_projection_per_rep else range(len(prep))
        for j in todo:
            xb, g, wt, beta = prep[j]
            t0 = time.perf_counter()
            q, a = orc.rmsnorm_quant(xb, g, wl.eps)
            acc = orc.ternary_acc(q, wt)
            orc.rescale(acc, a, beta)
            per_proj[j].append(time.perf_counter() - t0)
        reps += 1
        if max_reps is not None and reps >= max_reps and all(per_proj):
            break
        if time.perf_counter() - t_start > budget_s and all(per_proj):
            break
    t_set = sum(statistics.median(v) for v in per_proj)
    return M / t_set, M, orc.num_threads(), reps


def oracle_sample_tokens(wl, cap):
    return cap if wl.M > cap else None


def cpu_baseline_obj(wl, budget_s=12.0):
    sample = oracle_sample_tokens(wl, 512)
    tps, M, threads, reps = time_oracle(wl, sample, budget_s)
    return {"value": round(tps, 3), "unit": "tokens/s (one token through one BitLinear layer set)",
            "cores": threads, "threads": threads, "host_cores": host_cores(), "kind": "oracle",
            "sample": f"{M} tokens x all {len(wl.projections)} projections, median of {reps} rep(s); the "
                      f"contraction on OpenMP threads over (token, output row) pairs, normalisation and "
                      f"rescale on one thread; weights ternarised untimed"
                      + (f"; extrapolated linearly from {M} of {wl.M} tokens" if M < wl.M else "")}


def run_reference(args, dist: Dist):
    wl, _ = WORKLOADS[args.workload]
    wl = wl()
    if dist.rank != 0:
        return None
    sample = oracle_sample_tokens(wl, 64)
    # each step: one projection of the set (round robin) on the sampled tokens;
    # the run stops after --steps steps or 150 s, whichever comes first
    t0 = time.perf_counter()
    tps, M, threads, reps = time_oracle(wl, sample, budget_s=150.0, max_reps=max(args.steps, len(wl.projections)),
                                        one_projection_per_rep=True)
    wall = time.perf_counter() - t0
    ms_per_step = 1e3 * M / tps / len(wl.projections)
    return {
        "metric": METRIC, "impl": "reference", "value": round(tps, 3),
        "unit": "tokens/s (one token through one BitLinear layer set)",
        "n_gpus": dist.world, "steps": reps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic (seeded SplitMix64/Box-Muller; random-init latent weights)",
        "config": {"workload": wl.name, "description": wl.description, "M": wl.M,
                   "projections": [f"{p.K}->{p.N}" for p in wl.projections]},
        "cpu_baseline": {"value": round(tps, 3), "unit": "tokens/s (one token through one BitLinear layer set)",
                         "cores": threads, "threads": threads, "host_cores": host_cores(), "kind": "oracle",
                         "sample": f"{M} tokens; each step one projection (round robin); wall {wall:.1f} s"
                                   + (f"; extrapolated linearly from {M} of {wl.M} tokens" if M < wl.M else "")},
        "e2e": {"value": round(tps, 3), "unit": "tokens/s (one token through one BitLinear layer set)",
                "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------- main

def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--layers", type=int, default=0, help="layer sets per step (default per workload)")
    ap.add_argument("--secondary", default=None,
                    help="comma-separated workloads timed after the main one in the same run, or 'none' "
                         f"(default with the default workload: {DEFAULT_SECONDARY}; otherwise none)")
    ap.add_argument("--secondary-min-steps", type=int, default=200,
                    help="timed steps of each secondary workload: max(--steps, this)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-copy-kernel", action="store_true", help="skip timing mmf_hbm_copy")
    ap.add_argument("--api", choices=("group", "single"), default="group",
                    help="group: one call per set of projections sharing x; single: one call per projection")
    ap.add_argument("--glu", action="store_true",
                    help="the down projection reads the gate/up outputs through mmf_bitlinear_fwd_glu")
    ap.add_argument("--no-pdl", action="store_true", help="plain stream-ordered launches")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.secondary is None:
        args.secondary = DEFAULT_SECONDARY if args.workload == DEFAULT_WORKLOAD else "none"
    secondary = [] if args.secondary in ("", "none") else args.secondary.split(",")
    for w in secondary:
        if w not in WORKLOADS or WORKLOADS[w][0] is None:
            raise SystemExit(f"--secondary: unknown forward workload {w}")
    dist = Dist(args.gpus)
    try:
        if args.impl == "reference" and args.workload == "mlgru-scan-1.3b":
            if dist.rank == 0:
                B, T, D = SCAN_SHAPE
                g = torch.Generator().manual_seed(5)
                mk = lambda: (torch.randn((1, 256, D), generator=g) * 2.0).to(torch.bfloat16)
                cb = scan_cpu_baseline(mk(), mk(), mk(), D)
                print(json.dumps({"metric": METRIC, "impl": "reference", "value": cb["value"], "unit": cb["unit"],
                                  "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
                                  "higher_is_better": True, "config": {"workload": args.workload},
                                  "cpu_baseline": cb, "e2e": {"value": cb["value"], "unit": cb["unit"],
                                                              "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
                      flush=True)
            return 0
        if args.impl == "reference" and WORKLOADS[args.workload][0] is None:
            if dist.rank == 0:
                print(json.dumps({"impl": "reference", "unavailable":
                                  f"no oracle arm for --workload {args.workload}; use the default workload"}))
            return 0
        if args.impl == "reference":
            res = run_reference(args, dist)
            if res is not None:
                print(json.dumps(res), flush=True)
            return 0
        if not torch.cuda.is_available():
            raise SystemExit("bench.py --impl ours needs a CUDA device")
        torch.cuda.set_device(dist.local_rank)
        if args.workload in ("mlgru-scan-1.3b", "bwd-prefill-1.3b"):
            res = run_scan(args, dist) if args.workload == "mlgru-scan-1.3b" else run_bwd(args, dist)
            if dist.rank == 0:
                print(json.dumps(res), flush=True)
            return 0
        peaks, peak_src = load_peaks()
        copy = None if args.no_copy_kernel else time_hbm_copy(torch.device("cuda", dist.local_rank))
        copy_gbs = copy["gbs"] if copy else None
        res, wl = run_workload(args.workload, args, dist, args.steps, args.warmup, peaks, peak_src, copy_gbs,
                               layers=args.layers)
        if copy:
            res["hbm_copy"] = copy
        sec = []
        for w in secondary:
            r, _ = run_workload(w, args, dist, max(args.steps, args.secondary_min_steps), args.warmup, peaks,
                                peak_src, copy_gbs)
            sec.append({k: r[k] for k in ("value", "unit", "ms_per_step", "steps", "warmup", "roofline", "e2e",
                                          "gpu_launches", "clocks", "config")})
        if sec:
            res["secondary"] = sec
        if dist.rank == 0:
            if dist.world == 1 and not args.no_cpu_baseline:
                res["cpu_baseline"] = cpu_baseline_obj(wl)
            print(json.dumps(res), flush=True)
        return 0
    finally:
        dist.close()


if __name__ == "__main__":
    sys.exit(main())
