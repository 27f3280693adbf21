"""Benchmark of the W4A16 decode GEMV on B200 (one JSON line on stdout).

Headline workload: batch-1 decode through a stack of L = 16 distinct
8192 x 8192 W4 g128 layers (the LLaMA-65B attention GEMV [1,8192] x
[8192,8192]).  One step = one token through the 16 layers: layer l's output
is layer l+1's input.  The 16 packed weights (570 MB) are 4.5x the 126 MB L2,
so every layer's weights come from HBM.  The steps are replayed from a CUDA
graph and timed with CUDA events on the launching stream.

value  = effective GB/s = (packed codes + scales + zeros of all layers) / step time
e2e    = the same, through the public Python API, eager, with the step's input
         copied from pinned host memory and its output read back every step.
Extra keys: per-layer microseconds of the other workloads (LLaMA-7B set,
LLaMA-65B set, 4096^2, skinny M, the 11008 x 4096 quantize+pack), the
roofline of the GEMV kernel, the CPU oracle baseline and the SM clocks seen
during the timed region.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {ours,reference}]
"""
from __future__ import annotations

import argparse
import faulthandler
import hashlib
import json
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

faulthandler.enable()


def log(msg):
    print(f"[bench {time.strftime('%H:%M:%S')}] {msg}", file=sys.stderr, flush=True)


METRIC = "W4A16 GEMV effective GB/s & % of B200 HBM peak (M=1, K=N=8192); us/layer"
LAYERS = 16
M1, N1, K1 = 1, 8192, 8192
WEIGHT_BYTES = N1 * K1 // 2 + 2 * N1 * (K1 // 128) * 2       # codes + scales + zeros = 35,651,584
FALLBACK_HBM_GBS = 6650.0
FALLBACK_TFLOPS = 1590.0


def layer_bytes(N, K):
    return N * K // 2 + 2 * N * (K // 128) * 2


def workload_config(layers=LAYERS):
    return {"workload": f"decode token through {layers} distinct W4 g128 8192x8192 layers, M=1 "
                        "(LLaMA-65B attention GEMV [1,8192]x[8192,8192])",
            "M": M1, "N": N1, "K": K1, "group": 128, "bits": 4, "mode": "asym", "layers": layers,
            "weights_per_step_bytes": layers * WEIGHT_BYTES,
            "l2": "inputs larger than L2: 16 distinct packed weights, 570 MB vs 126 MB L2",
            "inputs": "seeded synthetic: W ~ N(0, 0.015) fp16, x ~ N(0,1) with 1% channels x20"}


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def whole_job_gbps(world, bytes_per_step, ms_per_step):
    """Weak scaling: every rank streams bytes_per_step per step; the step time is the max over ranks."""
    return world * bytes_per_step / (ms_per_step * 1e-3) / 1e9


class Dist:
    def __init__(self, gpus):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False
        if gpus != self.world and self.world > 1:
            raise SystemExit(f"--gpus {gpus} but WORLD_SIZE={self.world}")

    def init(self, backend):
        if self.world > 1:
            import datetime

            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = True

    def barrier(self):
        if self.pg:
            import torch.distributed as dist
            dist.barrier()

    def max(self, v, device):
        if not self.pg:
            return v
        import torch
        import torch.distributed as dist
        t = torch.tensor([v], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as dist
            dist.destroy_process_group()


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, read only)
# ---------------------------------------------------------------------------
_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
            0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, torch_device):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            # match the CUDA device to its NVML handle by UUID (robust to CUDA_VISIBLE_DEVICES)
            want = str(torch.cuda.get_device_properties(torch_device).uuid).lower().replace("gpu-", "")
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = (u.decode() if isinstance(u, bytes) else str(u)).lower().replace("gpu-", "")
                if u == want:
                    self._h = h
                    break
            if self._h is None:
                raise RuntimeError(f"no NVML device with UUID {want}")
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._nv = pynvml
        except Exception as e:  # no NVML: report that instead of clocks
            self.error = f"{type(e).__name__}: {e}"

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if self._h is None:
            return {"error": getattr(self, "error", "nvml unavailable")}
        names = sorted(n for b, n in _REASONS.items() if self.reasons & b)
        med = float(np.median(self.samples)) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples),
                "source": "NVML clocks + clocks-event reasons, sampled every 2 ms during the timed region"}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, STREAM-style copy)"
    return FALLBACK_HBM_GBS, "fallback 6650 GB/s (earlier measurement on this pool)"


def measured_tensor_peak():
    """Dense fp16/bf16 tensor TFLOP/s for a kernel timed alone (burst), and where it came from."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops, cuBLAS burst; fp16 runs at the bf16 rate)"
    return FALLBACK_TFLOPS, "fallback 1590 TFLOP/s (earlier measurement on this pool)"


def profiled_traffic(kernel_key):
    """DRAM bytes per launch from the committed ncu summary, if the kernel source is unchanged."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(kernel_key)
    if not d:
        return None
    src = os.path.join(ROOT, d["source"])
    with open(src, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != d["source_sha256"]:
            return None
    return d["dram_bytes_per_launch"]


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def search_workload(Wd, Xd, dev, n_alpha=20, reps=3):
    """The alpha grid search of the 11008 x 4096 layer on its 512 calibration tokens.

    A search of 1 and of n_alpha grid points is timed with CUDA events (the
    call is synchronous); their difference gives the time per grid point, the
    rest is the target product W X and the set-up, done once per search.
    """
    import torch

    import w4a16_decode_gemv_b200 as w4
    N, K = Wd.shape
    T = Xd.shape[0]
    grid = [i / (n_alpha - 1) for i in range(n_alpha)]
    ws = torch.empty(w4.search_workspace_size(N, K, T, n_alpha), dtype=torch.uint8, device=dev)

    def timed(alphas):
        best_ms, out = None, None
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record()
            out = w4.awq_search_alpha(Wd, Xd, alphas, workspace=ws)
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
            best_ms = ms if best_ms is None else min(best_ms, ms)
        return best_ms, out

    timed(grid[:1])  # warm-up (library load, first launches)
    ms1, _ = timed(grid[:1])
    msn, (losses, best) = timed(grid)
    per = (msn - ms1) / (n_alpha - 1)
    return {"N": N, "K": K, "T": T, "n_alpha": n_alpha, "ms_per_search": round(msn, 3),
            "ms_per_alpha": round(per, 4), "ms_once_per_search": round(ms1 - per, 3),
            "best_alpha": round(grid[best], 4), "losses_min_max": [min(losses), max(losses)],
            "timing": f"CUDA events around the synchronous call, best of {reps}"}


def gptq_workload(Wd, Xd, dev, reps=3):
    """GPTQ on the 11008 x 4096 layer and its 512 calibration tokens, through the product
    entry point gptq_quantize (Hessian, factor and sweep on one stream), with each of its
    three steps also timed alone (gptq_hessian, gptq_factor, gptq_sweep)."""
    import torch

    import w4a16_decode_gemv_b200 as w4
    N, K = Wd.shape
    T = Xd.shape[0]
    lib = w4.load_library()
    H = w4.gptq_hessian(Xd)
    fws = torch.empty(int(lib.gptq_factor_workspace_size(K)), dtype=torch.uint8, device=dev)
    G = w4.gptq_factor(H, workspace=fws)
    sws = torch.empty(int(lib.gptq_sweep_workspace_size(N, K, 128)), dtype=torch.uint8, device=dev)
    qws = torch.empty(int(lib.gptq_quantize_workspace_size(N, K, 128)), dtype=torch.uint8, device=dev)
    out = (torch.empty((N, K // 8), dtype=torch.int32, device=dev),
           torch.empty((N, K // 128), dtype=torch.float16, device=dev),
           torch.empty((N, K // 128), dtype=torch.float16, device=dev))

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        best = None
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
            best = ms if best is None else min(best, ms)
        return best

    q_ms = timed(lambda: w4.gptq_quantize(Wd, Xd, workspace=qws, out=out))
    h_ms = timed(lambda: w4.gptq_hessian(Xd, out=H))
    f_ms = timed(lambda: w4.gptq_factor(H, workspace=fws, out=G))
    s_ms = timed(lambda: w4.gptq_sweep(Wd, G, workspace=sws, out=out))
    sweep_flop = N * K * K  # the updates right of each block: N K^2 / 2 multiply-add pairs
    return {"N": N, "K": K, "T": T, "gptq_quantize_ms": round(q_ms, 3), "hessian_ms": round(h_ms, 4),
            "factor_ms": round(f_ms, 3), "sweep_ms": round(s_ms, 3),
            "sweep_fp64_tflops": round(sweep_flop / (s_ms * 1e-3) / 1e12, 2),
            "hessian_fp64_tflops": round(2 * T * K * K / (h_ms * 1e-3) / 1e12, 2),
            "timing": f"CUDA events, best of {reps}; gptq_quantize is the product call, the steps are timed alone"}


def w4a8_workload(dev, Ms=(1, 4, 16, 64, 128)):
    """W4A8 (progressive group quantization) at K = N = 8192: w4a8_gemm per layer in a CUDA
    graph over distinct weight copies larger than L2, random codes / s2 / zs (the time does
    not depend on the values); HBM fraction of the algorithmic bytes (codes + s2 + zs + s1)
    and int8 tensor fraction against the nominal int8 rate (2 x the measured bf16 peak)."""
    import torch

    import w4a16_decode_gemv_b200 as w4
    N = K = 8192
    gen = torch.Generator(device=dev)
    gen.manual_seed(11)
    wbytes = N * K // 2 + 2 * N * (K // 128) + 2 * N
    copies = max(2, -(-4 * 126 * 2 ** 20 // wbytes))
    layers = []
    for _ in range(copies):
        q = torch.randint(-2 ** 31, 2 ** 31 - 1, (N, K // 8), dtype=torch.int32, device=dev, generator=gen)
        s2 = torch.randint(1, 17, (N, K // 128), dtype=torch.uint8, device=dev, generator=gen)
        zs = (torch.randint(0, 16, (N, K // 128), dtype=torch.uint8, device=dev, generator=gen) * s2).to(torch.uint8)
        s1 = (torch.rand((N,), device=dev, generator=gen) * 1e-3).half()
        layers.append((q, s1, s2, zs))
    hbm_peak, _ = measured_peaks()
    tc_peak, _ = measured_tensor_peak()
    out = []
    for M in Ms:
        x8 = torch.randint(-127, 128, (M, K), dtype=torch.int8, device=dev, generator=gen)
        sx = (torch.rand((M,), device=dev, generator=gen) * 1e-2).half()
        y = torch.empty((M, N), dtype=torch.float16, device=dev)
        ws = torch.zeros(w4.w4a8_gemm_workspace_size(M, N, K), dtype=torch.uint8, device=dev)

        def fn():
            for q, s1, s2, zs in layers:
                w4.w4a8_gemm(x8, sx, q, s1, s2, zs, out=y, workspace=ws)
        try:
            us = time_graph(fn, reps=max(3, 200 // copies)) * 1e3 / copies
            w4.gemm_check(ws)
            e = {"M": M, "N": N, "K": K, "us": round(us, 3), "GBps": round(wbytes / us / 1e3, 1),
                 "hbm_frac": round(wbytes / us / 1e3 / hbm_peak, 4),
                 "path": "CUDA cores (dp4a)" if M <= 4 else "tcgen05 kind::i8 tensor cores"}
            if M > 4:
                e["int8_tops"] = round(2 * M * N * K / us / 1e6, 2)
                e["int8_tensor_frac_of_2x_bf16_peak"] = round(2 * M * N * K / us / 1e6 / (2 * tc_peak), 4)
            out.append(e)
        except Exception as ex:  # report, never hide
            out.append({"M": M, "error": str(ex)[:200]})
    return {"algorithmic_bytes": wbytes, "entries": out}


def run_ours(args, dist):
    import torch

    import w4a16_decode_gemv_b200 as w4
    from w4a16_decode_gemv_b200 import build, inputs

    dev = torch.device("cuda", dist.local)
    torch.cuda.set_device(dev)
    dist.init("nccl")
    if dist.rank == 0:
        build.build()
    dist.barrier()
    w4.load_library()
    torch.manual_seed(0)

    # ---- inputs: the 8192^2 layer of the LLaMA-65B set, quantized on the GPU
    log("drawing inputs")
    (layer,) = inputs.layer_set(inputs.LLAMA65B, only="attn_8192x8192")
    W = torch.from_numpy(layer.W).to(dev)
    log("quantize")
    q0, s0, z0 = w4.awq_quantize_pack(W)
    del W
    log("copies")
    layers = []
    for l in range(args.layers):
        if l == 0:
            layers.append((q0, s0, z0))
        else:
            layers.append((q0.clone(), s0.clone(), z0.clone()))
    L = len(layers)
    ws = torch.zeros(w4.gemm_workspace_size(M1, N1, K1), dtype=torch.uint8, device=dev)
    xbufs = [torch.empty((M1, K1), dtype=torch.float16, device=dev) for _ in range(L + 1)]
    x0 = torch.from_numpy(layer.x).to(dev)
    stream = torch.cuda.Stream(dev)

    def token():
        for l, (q, s, z) in enumerate(layers):
            w4.w4a16_gemm(xbufs[l], q, s, z, out=xbufs[l + 1], workspace=ws)

    log("eager token")
    with torch.cuda.stream(stream):
        xbufs[0].copy_(x0)
        token()
        torch.cuda.synchronize()
        log("capture")
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            token()
        log("warmup")
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize()
    w4.gemm_check(ws)

    # ---- timed region: K graph replays, events on the launching stream
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    log("timed region")
    with ClockSampler(dev) as clk:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(args.steps):
                graph.replay()
            e1.record(stream)
        torch.cuda.synchronize()
    dist.barrier()
    ms_rank = e0.elapsed_time(e1)
    ms = dist.max(ms_rank, dev)
    ms_per_step = ms / args.steps
    w4.gemm_check(ws)
    bytes_step = L * WEIGHT_BYTES
    value = whole_job_gbps(dist.world, bytes_step, ms_per_step)
    us_layer = ms_per_step * 1e3 / L

    # ---- e2e through the public API (eager), pinned host input/output every step
    log("e2e")
    e2e = measure_e2e(args, layers, ws, x0, dev, stream, dist)

    out = None
    if dist.rank == 0:
        peak, peak_src = measured_peaks()
        achieved = WEIGHT_BYTES / (us_layer * 1e-6) / 1e9
        traffic = profiled_traffic("gemv_m1_kernel M=1 8192x8192")
        roof = {"bound": "hbm", "kernel": "gemv_m1_kernel (M=1 CUDA-core GEMV, CTA-owned rows)",
                "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": traffic,
                "algorithmic_bytes_per_launch": WEIGHT_BYTES,
                "note": f"peak: {peak_src}; achieved = (codes + scales + zeros) / average launch time, "
                        "launch time = graph step time / 16 layers (inter-kernel gaps included)"}
        out = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": dist.world,
               "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
               "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
               "dtype": "u4 x f16 -> f32 accumulate", "data": "synthetic",
               "config": workload_config(L), "us_per_layer": round(us_layer, 3),
               "hbm_frac_of_measured_peak": round(achieved / peak, 4),
               "roofline": roof, "e2e": e2e, "gpu_launches": args.steps * L,
               "clocks": clk.summary()}
        if not args.skip_extras:
            log("other workloads")
            out["workloads"] = other_workloads(args, dev)
        if dist.world == 1 and not args.skip_cpu:
            # the oracle's leg: sampled rows of this run's output checked against it,
            # then the oracle itself timed on the host cores
            log("cpu baseline")
            out["parity"] = check_parity(layer, q0, s0, z0, dev)
            out["cpu_baseline"] = cpu_baseline(layer, q0, s0, z0, args.cpu_seconds)
    del graph
    dist.close()
    return out


def check_parity(layer, q, s, z, dev):
    import torch

    import oracle
    import w4a16_decode_gemv_b200 as w4
    rng = np.random.default_rng(123)
    rows = np.sort(rng.choice(layer.N, 64, replace=False))
    y = w4.w4a16_gemm(torch.from_numpy(layer.x).to(dev), q, s, z).cpu().numpy()
    qn = q.cpu().numpy().view(np.uint32)[rows]
    sn, zn = s.cpu().numpy()[rows], z.cpu().numpy()[rows]
    qo, so, zo = oracle.quantize_pack(layer.W[rows], None, 128, 4, oracle.ASYM)
    exact = bool(np.array_equal(qn, qo) and np.array_equal(sn.view(np.uint16), so.view(np.uint16))
                 and np.array_equal(zn.view(np.uint16), zo.view(np.uint16)))
    y_ref, B = oracle.gemm_ref(layer.x, oracle.dequant(qn, sn, zn))
    err = np.abs(y[:, rows].astype(np.float64) - y_ref)
    ok = bool(np.all(err <= 2e-3 * B + 1e-3))
    if not (exact and ok):
        raise SystemExit(f"parity check failed: packed bit-exact={exact}, y within tolerance={ok}")
    return {"rows_checked": len(rows), "packed_bit_exact": exact, "y_within_tol": ok,
            "max_abs_err": float(err.max()), "tolerance": "2e-3*sum|x*w_hat| + 1e-3"}


def measure_e2e(args, layers, ws, x0, dev, stream, dist):
    import torch

    import w4a16_decode_gemv_b200 as w4
    L = len(layers)
    x_host = torch.empty((M1, K1), dtype=torch.float16, pin_memory=True)
    x_host.copy_(x0.cpu())
    y_host = torch.empty((M1, N1), dtype=torch.float16, pin_memory=True)
    xb = [torch.empty((M1, K1), dtype=torch.float16, device=dev) for _ in range(L + 1)]
    steps = max(1, min(args.steps, args.e2e_steps))

    def step():
        xb[0].copy_(x_host, non_blocking=True)
        for l, (q, s, z) in enumerate(layers):
            w4.w4a16_gemm(xb[l], q, s, z, out=xb[l + 1], workspace=ws)
        y_host.copy_(xb[L], non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(max(3, min(args.warmup, 20))):
            step()
        torch.cuda.synchronize()
        dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = dist.max(e0.elapsed_time(e1), dev) / steps
    return {"value": round(dist.world * L * WEIGHT_BYTES / (ms * 1e-3) / 1e9, 1), "unit": "GB/s",
            "h2d_bytes_per_step": M1 * K1 * 2, "d2h_bytes_per_step": M1 * N1 * 2, "ms_per_step": round(ms, 4),
            "steps": steps, "how": "eager w4a16_gemm calls from Python per layer; pinned x in, y out, per step"}


def time_graph(fn, reps, warm=3):
    import torch
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            fn()
        for _ in range(warm):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(reps):
            g.replay()
        e1.record(s)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    del g
    return ms


def other_workloads(args, dev):
    """Per-layer microseconds of the other workloads, weights rotated to defeat L2."""
    import torch

    import w4a16_decode_gemv_b200 as w4
    from w4a16_decode_gemv_b200 import inputs
    res = {}
    hbm_peak, _ = measured_peaks()
    tc_peak, tc_src = measured_tensor_peak()
    res["peaks"] = {"hbm_gbs": hbm_peak, "tensor_tflops": tc_peak, "tensor_source": tc_src}
    gen = torch.Generator(device=dev)
    gen.manual_seed(7)

    def packed(N, K, copies):
        # random codes / scales / zeros: GEMV time does not depend on the values
        out = []
        for _ in range(copies):
            q = torch.randint(-2 ** 31, 2 ** 31 - 1, (N, K // 8), dtype=torch.int32, device=dev, generator=gen)
            s = (torch.rand((N, K // 128), device=dev, generator=gen) * 0.01).half()
            z = torch.randint(0, 16, (N, K // 128), device=dev, generator=gen).half()
            out.append((q, s, z))
        return out

    def copies_for(N, K):
        return max(2, -(-4 * 126 * 2 ** 20 // layer_bytes(N, K)))

    def gemm_us(M, N, K):
        ws_ = torch.zeros(w4.gemm_workspace_size(M, N, K), dtype=torch.uint8, device=dev)
        c = copies_for(N, K)
        ws_l = packed(N, K, c)
        x = torch.randn((M, K), device=dev, generator=gen).half()
        y = torch.empty((M, N), dtype=torch.float16, device=dev)

        def fn():
            for q, s, z in ws_l:
                w4.w4a16_gemm(x, q, s, z, out=y, workspace=ws_)
        ms = time_graph(fn, reps=max(3, 200 // c))
        w4.gemm_check(ws_)
        return ms * 1e3 / c

    def cublas_us(M, N, K):
        # the dense fp16 product the W4A16 path replaces (torch.matmul -> cuBLAS), for the crossover
        Ws = [torch.randn((N, K), device=dev, generator=gen).half() for _ in range(2)]
        x = torch.randn((M, K), device=dev, generator=gen).half()
        y = torch.empty((M, N), dtype=torch.float16, device=dev)

        def fn():
            for Wf in Ws:
                torch.matmul(x, Wf.t(), out=y)
        ms = time_graph(fn, reps=20)
        del Ws
        return ms * 1e3 / 2

    shapes = {"gemv_4096x4096": [(1, 4096, 4096)],
              "llama7b_decode": [(1, N, K) for _, N, K in inputs.LLAMA7B["layers"]],
              "llama65b_decode": [(1, N, K) for _, N, K in inputs.LLAMA65B["layers"]],
              "skinny_8192": [(M, 8192, 8192) for M in inputs.SKINNY_M],
              "prefill_8192": [(M, 8192, 8192) for M in (128, 200, 512)]}
    only = args.only
    if only is not None:
        # some workloads alone (for profiling): comma-separated names, or skinny_8192:M for one M
        picked = {}
        for item in only.split(","):
            name, _, m = item.partition(":")
            if name in shapes:
                picked.setdefault(name, []).extend(e for e in shapes[name] if not m or e[0] == int(m))
        shapes = picked
        only = {item.partition(":")[0] for item in only.split(",")}
    for name, lst in shapes.items():
        entries = []
        for M, N, K in lst:
            try:
                us = gemm_us(M, N, K)
                b = layer_bytes(N, K)
                e = {"M": M, "N": N, "K": K, "us": round(us, 3), "GBps": round(b / us / 1e3, 1),
                     "hbm_frac": round(b / us / 1e3 / hbm_peak, 4), "tflops": round(2 * M * N * K / us / 1e6, 2)}
                if M > 4:
                    e["path"] = "tcgen05 tensor cores" + (f", {-(-M // 256)} chunks of <= 256 tokens" if M > 256 else "")
                    e["tensor_frac"] = round(2 * M * N * K / us / 1e6 / tc_peak, 4)
                if M >= 16:
                    e["cublas_fp16_us"] = round(cublas_us(M, N, K), 3)
                entries.append(e)
            except Exception as e:  # report, never hide
                entries.append({"M": M, "N": N, "K": K, "error": str(e)[:200]})
        res[name] = entries
    if only is None or "w4a8_8192" in only:
        res["w4a8_8192"] = w4a8_workload(dev)
    if only is not None and not only & {"quantize_pack_11008x4096", "awq_search_11008x4096", "gptq_11008x4096"}:
        return res
    W, X, _ = inputs.quant_workload()
    Wd = torch.from_numpy(W).to(dev)
    Xd = torch.from_numpy(X).to(dev)
    if only is None or "awq_search_11008x4096" in only:
        res["awq_search_11008x4096"] = search_workload(Wd, Xd, dev)
    if only is None or "gptq_11008x4096" in only:
        try:
            res["gptq_11008x4096"] = gptq_workload(Wd, Xd, dev)
        except Exception as e:  # report, never hide
            res["gptq_11008x4096"] = {"error": str(e)[:300]}
    if only is not None and "quantize_pack_11008x4096" not in only:
        return res
    # quantize + pack of the 11008 x 4096 AWQ workload (4-bit asym and 3-bit sym)
    s = w4.awq_act_scale(Xd, 0.5)
    Wc = [Wd] + [Wd.clone() for _ in range(3)]   # 4 x 90 MB > L2
    outs = [(torch.empty((11008, 512), dtype=torch.int32, device=dev),
             torch.empty((11008, 32), dtype=torch.float16, device=dev),
             torch.empty((11008, 32), dtype=torch.float16, device=dev)) for _ in Wc]
    qres = []
    for bits, mode in [(4, w4.ASYM), (3, w4.SYM)]:
        def fn():
            for Wi, o in zip(Wc, outs):
                w4.awq_quantize_pack(Wi, s, 128, bits, mode, out=o)
        us = time_graph(fn, reps=20) * 1e3 / len(Wc)
        rb = 11008 * 4096 * 2 + 4096 * 2
        wb = 11008 * 4096 // 2 + 2 * 11008 * 32 * 2
        qres.append({"bits": bits, "mode": "asym" if mode == w4.ASYM else "sym", "us": round(us, 2),
                     "GBps": round((rb + wb) / us / 1e3, 1)})
    res["quantize_pack_11008x4096"] = qres
    return res


def cpu_baseline(layer, q, s, z, seconds):
    """The oracle as it stands, on this host's cores, on a bounded sample."""
    import oracle
    try:
        from threadpoolctl import threadpool_info
        blas = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
    except Exception:
        blas = []
    qn = q.cpu().numpy().view(np.uint32)
    sn, zn = s.cpu().numpy(), z.cpu().numpy()
    rows_per_call = 1024
    done_rows, t_total, calls = 0, 0.0, 0
    while t_total < seconds:
        r0 = (calls * rows_per_call) % layer.N
        t0 = time.perf_counter()
        oracle.gemm(layer.x, qn[r0:r0 + rows_per_call], sn[r0:r0 + rows_per_call], zn[r0:r0 + rows_per_call])
        t_total += time.perf_counter() - t0
        done_rows += rows_per_call
        calls += 1
    bytes_done = done_rows * layer_bytes(1, K1)
    return {"value": round(bytes_done / t_total / 1e9, 4), "unit": "GB/s",
            "cores": max(blas) if blas else len(os.sched_getaffinity(0)),
            "host_cpus": len(os.sched_getaffinity(0)), "kind": "oracle",
            "sample": f"{calls} oracle calls of {rows_per_call} rows x 8192 (dequantize in fp64 + fp64 GEMV) "
                      f"of the 8192x8192 layer, {t_total:.1f} s",
            "us_per_layer_equiv": round(t_total / (done_rows / N1) * 1e6, 1)}


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle, timed as it stands
# ---------------------------------------------------------------------------
def run_reference(args, dist):
    if dist.rank != 0:
        return None
    import oracle
    from w4a16_decode_gemv_b200 import inputs
    (layer,) = inputs.layer_set(inputs.LLAMA65B, only="attn_8192x8192")
    qo, so, zo = oracle.quantize_pack(layer.W, None, 128, 4, oracle.ASYM)
    # size each step so that warm-up + steps take about args.ref_seconds
    t0 = time.perf_counter()
    oracle.gemm(layer.x, qo[:256], so[:256], zo[:256])
    t256 = max(time.perf_counter() - t0, 1e-4)
    per_step = args.ref_seconds / max(1, args.steps + args.warmup)
    rows = int(min(N1, max(1, 256 * per_step / t256)))

    def step(i):
        r0 = (i * rows) % (N1 - rows + 1)
        oracle.gemm(layer.x, qo[r0:r0 + rows], so[r0:r0 + rows], zo[r0:r0 + rows])

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    dt = time.perf_counter() - t0
    ms = dt * 1e3 / args.steps
    val = rows * layer_bytes(1, K1) / (ms * 1e-3) / 1e9
    try:
        from threadpoolctl import threadpool_info
        blas = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
    except Exception:
        blas = []
    cores = max(blas) if blas else len(os.sched_getaffinity(0))
    sample = f"each step: oracle dequantize (fp64) + fp64 GEMV of {rows} rows x 8192 of the 8192x8192 layer"
    return {"impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s", "n_gpus": dist.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(),
            "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "note": "the reference arm is the CPU oracle (fp64 numpy), the only implementation on the pages"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=LAYERS)
    ap.add_argument("--e2e-steps", type=int, default=500)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-seconds", type=float, default=90.0)
    ap.add_argument("--skip-extras", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--only", default=None,
                    help="run some of the other workloads only, comma-separated (gemv_4096x4096, llama7b_decode, llama65b_decode, "
                         "skinny_8192 or skinny_8192:M, prefill_8192 or prefill_8192:M, w4a8_8192, quantize_pack_11008x4096, "
                         "awq_search_11008x4096, gptq_11008x4096); for profiling")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    dist = Dist(args.gpus)
    out = run_reference(args, dist) if args.impl == "reference" else run_ours(args, dist)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
