"""Benchmark of the SDM recurrent core on B200: one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl sdm|reference]

A step is one sdm_layer_forward call over one batch of synthetic input: the
product-key selection of k' and q', the record build, the state
initialisation and the recurrence (epilogue off unless --epilogue). Inputs
are resident in HBM when the timed region starts; `e2e` repeats the
measurement through the C ABI with the inputs copied from pinned host memory
and y and M_T copied back inside the timed region. With N > 1 (torchrun) each rank runs its own batch
(weak scaling, no collective on the data path); the time is the max over
ranks. `--impl reference` times the CPU oracle on a bounded sample instead
(rank 0 only).
"""

from __future__ import annotations

import argparse
import ctypes
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time
from pathlib import Path

import torch

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import sparse_memory_linear_pkm_b200 as sdm  # noqa: E402
from sparse_memory_linear_pkm_b200 import synth  # noqa: E402

METRIC = "SDM layer tokens/s (B·T) and achieved HBM/L2 GB/s vs roofline on 1 B200"
DEFAULT_WORKLOAD = "long_t1m_n262144_dv2048"
# Measured after the headline at N = 1 (device time only), so one run also
# shows the driver the smaller workloads.
EXTRA_WORKLOADS = ("d2048_h16_n1024_dv128", "d2048_h4_n16384_dv512", "d4096_h8_n16384_dv512")
FALLBACK_HBM_GBS = 6650.0
SMEM_BYTES_PER_CLK_PER_SM = 128
NVML_REASONS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
    0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
    0x100: "display_clock_setting",
}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=synth.WORKLOAD_ORDER)
    ap.add_argument("--impl", default="sdm", choices=["sdm", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--epilogue", action="store_true", help="run the RMS-norm x gate epilogue")
    ap.add_argument("--variant", default="auto", choices=["auto", "resident", "streaming", "pipelined"])
    ap.add_argument("--tile", type=int, default=0, help="force entry k of the kernel's tile table (0: automatic)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the device-time lines of the smaller workloads")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU work of the oracle sample")
    ap.add_argument("--decode", action="store_true",
                    help="time decode steps instead: one token per call (sdm_layer_step), state carried")
    ap.add_argument("--fp8-state", action="store_true",
                    help="keep the state in the block-scaled fp8 format (E4M3, scale per 16 values): the layer "
                         "(pipelined recurrence) or, with --decode, the decode step")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward instead: sdm_scan_backward and the two selection-weight backwards")
    ap.add_argument("--slot-counts", action="store_true",
                    help="time the slot utilisation histogram of the workload's write selection instead")
    return ap.parse_args()


# ------------------------------------------------------------------ ranks --

class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False

    def init(self, backend: str):
        if self.world > 1:
            import torch.distributed as dist

            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = True

    def barrier(self, device=None):
        if self.pg:
            import torch.distributed as dist

            if device is not None and device.type == "cuda":
                dist.barrier(device_ids=[device.index])
            else:
                dist.barrier()

    def max(self, x: float, device) -> float:
        if not self.pg:
            return x
        import torch.distributed as dist

        t = torch.tensor([x], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as dist

            dist.destroy_process_group()


def aggregate_value(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / max_seconds


# ----------------------------------------------------------------- clocks --

class ClockSampler:
    """Reads SM clocks and clock-event reasons through NVML during the timed
    region (read-only; no setting of the GPU is touched)."""

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples = []
        self.max_mhz = None
        self.reasons = 0
        self._stop = threading.Event()
        self._thread = None
        self._handle = None
        try:
            import pynvml

            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self._handle = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._handle, pynvml.NVML_CLOCK_SM)
            self._nvml = pynvml
        except Exception as e:  # pragma: no cover - depends on the box
            self.error = repr(e)
        self.period = period_s

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._handle, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._handle)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._handle is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self) -> dict:
        names = sorted(n for bit, n in NVML_REASONS.items() if self.reasons & bit and n != "gpu_idle")
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# -------------------------------------------------------------- roofline --

def measured_peaks() -> dict:
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        try:
            return json.loads(p.read_text())
        except Exception:
            pass
    return {}


def algorithmic_bytes_per_token_head(shape: synth.Shape, epilogue: bool, fp8_state: bool = False) -> int:
    """(2W + R) d_v sizeof(state) of state traffic, plus the per-token-head
    inputs (indices + weights, v, alpha, beta, g) and the fp32 y. The fp8
    state moves one code byte per value and one exponent byte per 16."""
    s_state = 2 if shape.state_dtype == synth.BF16 else 4
    s_in = 2 if shape.in_dtype == synth.BF16 else 4
    b = (2 * shape.W + shape.R) * shape.d_v * s_state
    if fp8_state:
        b = (2 * shape.W + shape.R) * (shape.d_v + shape.d_v // 16)
    b += (shape.W + shape.R) * 8 + shape.d_v * s_in + 2 * s_in + shape.d_v * 4
    if epilogue:
        b += shape.d_v * s_in
    return b


# The source files each timed kernel is compiled from; a recorded DRAM
# traffic figure stays valid while these files are unchanged.
KERNEL_SOURCES = {
    "k_scan_resident": ("sdm_device.cuh", "sdm_records.cuh", "sdm_scan.cuh"),
    "k_scan_streaming": ("sdm_device.cuh", "sdm_records.cuh", "sdm_scan.cuh"),
    "k_pkm_topk_fast": ("sdm_device.cuh", "pkm_topk_fast.cuh"),
    "k_scan_pipelined": ("sdm_device.cuh", "sdm_scan.cuh", "sdm_pipelined.cuh"),
}


def source_digest(kernel: str) -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        h.update(name.encode())
        h.update((ROOT / "sparse_memory_linear_pkm_b200" / "csrc" / name).read_bytes())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, kernel: str, config: str):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, when
    it was taken on the current kernel sources and the same launch
    configuration; else None."""
    p = ROOT / "profiles" / "traffic.json"
    if not p.exists():
        return None
    try:
        entry = json.loads(p.read_text()).get(workload, {}).get(kernel)
    except Exception:
        return None
    if not entry or entry.get("source_digest") != source_digest(kernel) or entry.get("config") != config:
        return None
    return entry.get("dram_bytes_per_launch")


# ------------------------------------------------------------ CPU oracle --

def oracle_sample_inputs(inp: dict, Bs: int, Ts: int) -> dict:
    f = synth.to_numpy_f32
    out = {k: f(inp[k][:Bs, :Ts]) for k in ("kp", "qp", "v", "alpha", "beta")}
    out["M0"] = f(inp["M0"])
    if "g" in inp:
        out["g"] = f(inp["g"][:Bs, :Ts])
    return out


def time_oracle(o, shape: synth.Shape, sample: dict, threads: int) -> float:
    t0 = time.perf_counter()
    o.layer_forward(sample["kp"], sample["qp"], sample["v"], sample["alpha"], sample["beta"], sample["M0"],
                    shape.W, shape.R, g=sample.get("g"), state_bf16=shape.state_dtype == synth.BF16,
                    n_threads=threads)
    return time.perf_counter() - t0


def calibrate_sample(o, shape: synth.Shape, inp: dict, threads: int, target_s: float):
    """Grows (batch rows, tokens) of the oracle sample until one run takes
    about target_s seconds (or the whole workload is covered)."""
    Bs, Ts = 1, 1
    dt = time_oracle(o, shape, oracle_sample_inputs(inp, Bs, Ts), threads)
    while dt < target_s / 2 and (Bs < shape.B or Ts < shape.T):
        scale = max(2.0, min(16.0, target_s / max(dt, 1e-3)))
        if Ts < shape.T:
            Ts = min(shape.T, int(Ts * scale))
        else:
            Bs = min(shape.B, int(Bs * scale))
        dt = time_oracle(o, shape, oracle_sample_inputs(inp, Bs, Ts), threads)
    return Bs, Ts, dt


def cpu_baseline(shape: synth.Shape, inp: dict, target_s: float, epilogue: bool) -> dict:
    import oracle

    o = oracle.get()
    threads = oracle.default_threads()
    Bs, Ts, dt = calibrate_sample(o, shape, inp, threads, target_s)
    return {"value": Bs * Ts / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"batch rows 0..{Bs - 1}, first {Ts} tokens, all {shape.H} heads "
                      f"({Bs * Ts} tokens, {dt:.1f} s){', with epilogue' if epilogue else ''}"}


# ------------------------------------------------------------------- arms --

def run_reference(args, dist: Dist):
    """The oracle, timed on the host cores on a bounded sample per step."""
    if dist.rank != 0:
        return
    import oracle

    shape = synth.WORKLOADS[args.workload]
    dev = torch.device("cuda", dist.local_rank) if torch.cuda.is_available() else torch.device("cpu")
    inp = synth.make_inputs(shape.replace(B=1, T=min(shape.T, 4096)), seed=args.seed, device=dev,
                            with_gate=args.epilogue)
    o = oracle.get()
    threads = oracle.default_threads()
    budget_s = min(args.cpu_seconds, 150.0 / max(1, args.steps + args.warmup))
    Bs, Ts, _ = calibrate_sample(o, shape.replace(B=1, T=min(shape.T, 4096)), inp, threads, budget_s)
    sample = oracle_sample_inputs(inp, Bs, Ts)
    for _ in range(args.warmup):
        time_oracle(o, shape, sample, threads)
    t = 0.0
    for _ in range(args.steps):
        t += time_oracle(o, shape, sample, threads)
    value = args.steps * Bs * Ts / t
    desc = f"batch row 0, first {Ts} tokens, all {shape.H} heads ({Bs * Ts} tokens per step)"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(shape, args, dist),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(shape: synth.Shape, args, dist: Dist) -> dict:
    return {"workload": shape.name, "B": shape.B, "T": shape.T, "H": shape.H, "sqrt_n": shape.sqrt_n, "N": shape.N,
            "d_v": shape.d_v, "W": shape.W, "R": shape.R, "in_dtype": shape.in_dtype,
            "state_dtype": shape.state_dtype, "epilogue": bool(args.epilogue), "seed": args.seed,
            "parallelism": f"rows partition: {dist.world} x {shape.B} batch rows over {dist.world} ranks, no collective"}


def _cudart():
    """The CUDA runtime torch already loaded (same context, streams and pinned
    allocations), for the caller-side cudaMemcpyAsync calls of the e2e leg."""
    import glob

    names = glob.glob(os.path.join(os.path.dirname(torch.__file__), "..", "nvidia", "cuda_runtime", "lib",
                                   "libcudart.so*"))
    names += ["libcudart.so.12", "/usr/local/cuda/lib64/libcudart.so.12"]
    for name in names:
        try:
            lib = ctypes.CDLL(name)
        except OSError:
            continue
        lib.cudaMemcpyAsync.restype = ctypes.c_int
        lib.cudaMemcpyAsync.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int,
                                        ctypes.c_void_p]
        return lib
    raise RuntimeError("no CUDA runtime library found for the e2e copies")


H2D, D2H = 1, 2  # cudaMemcpyKind


def e2e_through_c_abi(args, dist: Dist, dev, shape: synth.Shape, sh, inp: dict, g, ws, stream) -> dict:
    """End to end through the C ABI with host buffers: every step copies its
    inputs from pinned host memory (one cudaMemcpyAsync per tensor), calls
    sdm_layer_forward, and copies y and M_T back to pinned host memory, all
    inside the timed region. Copies run on two copy streams and the device
    buffers are doubled, so step k's transfers overlap steps k-1 and k+1."""
    rt = _cudart()
    lib = sdm.native.load()
    names = ("kp", "qp", "v", "alpha", "beta")
    host = {}
    for k in names:
        host[k] = torch.empty(inp[k].shape, dtype=inp[k].dtype, pin_memory=True)
        host[k].copy_(inp[k])
    M0 = inp["M0"]
    dinp = [{k: torch.empty_like(inp[k]) for k in names} for _ in range(2)]
    ys = [torch.empty((shape.B, shape.T, shape.H, shape.d_v), dtype=torch.float32, device=dev) for _ in range(2)]
    Ms = [torch.empty((shape.B,) + tuple(M0.shape), dtype=M0.dtype, device=dev) for _ in range(2)]
    # one host copy each: the D2H copies of consecutive steps are ordered on one stream
    y_host = torch.empty(ys[0].shape, dtype=torch.float32, pin_memory=True)
    M_host = torch.empty(Ms[0].shape, dtype=M0.dtype, pin_memory=True)
    nbytes = lambda t: t.numel() * t.element_size()
    h2d = sum(nbytes(t) for t in host.values())
    d2h = nbytes(y_host) + nbytes(M_host)
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_ready = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    vp = lambda t: ctypes.c_void_p(t.data_ptr())
    gptr = vp(g) if g is not None else None

    def copy(dst, src, n, kind, st):
        rc = rt.cudaMemcpyAsync(vp(dst), vp(src), n, kind, ctypes.c_void_p(st.cuda_stream))
        if rc != 0:
            raise RuntimeError(f"cudaMemcpyAsync failed with {rc}")

    def steps(n):
        h2d_s.wait_stream(stream)
        d2h_s.wait_stream(stream)
        for k in range(n):
            b = k % 2
            if k >= 2:
                h2d_s.wait_event(done[b])  # step k-2 has finished reading this input buffer
            for name in names:
                copy(dinp[b][name], host[name], nbytes(host[name]), H2D, h2d_s)
            in_ready[b].record(h2d_s)
            stream.wait_event(in_ready[b])
            if k >= 2:
                stream.wait_event(out_done[b])  # step k-2's y and M_T have left these buffers
            d = dinp[b]
            sdm.native.check(lib.sdm_layer_forward(ctypes.byref(sh), vp(d["kp"]), vp(d["qp"]), vp(d["v"]),
                                                   vp(d["alpha"]), vp(d["beta"]), gptr, vp(M0), vp(Ms[b]),
                                                   vp(ys[b]), vp(ws), nbytes(ws),
                                                   ctypes.c_void_p(stream.cuda_stream)))
            done[b].record(stream)
            d2h_s.wait_event(done[b])
            copy(y_host, ys[b], nbytes(y_host), D2H, d2h_s)
            copy(M_host, Ms[b], nbytes(M_host), D2H, d2h_s)
            out_done[b].record(d2h_s)
        stream.wait_stream(h2d_s)
        stream.wait_stream(d2h_s)

    k_e2e = max(3, min(args.steps, 20 if shape.B * shape.T * shape.H <= 2 ** 22 else 5))
    steps(2)  # warm-up
    torch.cuda.synchronize(dev)
    sdm.stream_check(dev)
    dist.barrier(dev)
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(stream)
    steps(k_e2e)
    e2.record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier(dev)
    sdm.stream_check(dev)
    e_ms = dist.max(s2.elapsed_time(e2), dev)
    del dinp, ys, Ms, host, y_host, M_host
    torch.cuda.empty_cache()
    return {"value": aggregate_value(shape.B * shape.T * k_e2e, dist.world, e_ms / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": k_e2e,
            "path": "per step through the C ABI: one cudaMemcpyAsync per input tensor from pinned host memory, "
                    "sdm_layer_forward, cudaMemcpyAsync of y and M_T to pinned host memory; copies on two copy "
                    "streams, device buffers doubled so transfers overlap the neighbouring steps' compute"}


def run_sdm(args, dist: Dist):
    if not torch.cuda.is_available():
        raise SystemExit("bench.py --impl sdm needs a CUDA device")
    dev = torch.device("cuda", dist.local_rank)
    torch.cuda.set_device(dev)
    dist.init("nccl")
    shape = synth.WORKLOADS[args.workload]
    sdm.native.load()
    inp = synth.make_inputs(shape, seed=args.seed + dist.rank, device=dev, with_gate=args.epilogue)
    if args.fp8_state:  # M0 in the block-scaled fp8 format (the quantiser is one of the library's calls)
        inp["M0"] = sdm.quantize_fp8blk(inp["M0"].float().contiguous())
    g = inp.get("g")
    y = torch.empty((shape.B, shape.T, shape.H, shape.d_v), dtype=torch.float32, device=dev)
    M_out = torch.empty((shape.B,) + tuple(inp["M0"].shape), dtype=inp["M0"].dtype, device=dev)
    sh = sdm.make_shape(shape.B, shape.T, shape.H, shape.sqrt_n, shape.W, shape.R, shape.d_v, shape.torch_in(),
                        torch.uint8 if args.fp8_state else shape.torch_state(), variant=args.variant, tile=args.tile)
    ws = torch.empty(sdm.layer_forward_workspace_bytes(sh), dtype=torch.uint8, device=dev)

    def step(events=None, src=inp):
        sdm.layer_forward(src["kp"], src["qp"], src["v"], src["alpha"], src["beta"], inp["M0"], shape.W, shape.R,
                          g=g, variant=args.variant, y=y, M_out=M_out, workspace=ws, events=events, tile=args.tile)

    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        step()
    sdm.stream_check(dev)
    # an overlapped call (token chunks) also brackets each chunk's recurrence launch
    chunks = sdm.layer_forward_chunks(sh)
    n_ev = 6 + (2 * chunks if chunks > 1 else 0)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    for row in ev:  # create the events before the timed region
        for e in row:
            e.record(stream)
    torch.cuda.synchronize(dev)

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier(dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clocks:
        start.record(stream)
        for k in range(args.steps):
            step(events=ev[k])
        end.record(stream)
        torch.cuda.synchronize(dev)
    dist.barrier(dev)
    sdm.stream_check(dev)
    ms = start.elapsed_time(end)
    ms_max = dist.max(ms, dev)
    stage_ms = [sum(ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(args.steps)) / args.steps for i in range(5)]
    # the recurrence kernel's own time a step: its launch (one pass) or the sum of its chunk launches
    kernel_ms = stage_ms[3] if chunks == 1 else sum(
        ev[k][6 + 2 * c].elapsed_time(ev[k][7 + 2 * c]) for k in range(args.steps) for c in range(chunks)) / args.steps
    tokens = shape.B * shape.T
    value = aggregate_value(tokens * args.steps, dist.world, ms_max / 1e3)

    resident = sdm.scan_variant(sh) == "resident"
    launches_per_step = int(sdm.native.load().sdm_layer_forward_launches(ctypes.byref(sh), int(args.epilogue)))
    clk = clocks.summary()
    roof = roofline_of(shape, sh, kernel_ms, args.epilogue, dev, clk, fp8_state=args.fp8_state, launches=chunks)

    e2e = None
    if not args.no_e2e:
        e2e = e2e_through_c_abi(args, dist, dev, shape, sh, inp, g, ws, stream)

    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline and not args.fp8_state:
        cpu = cpu_baseline(shape, inp, args.cpu_seconds, args.epilogue)

    if dist.rank == 0:
        l2_mb = torch.cuda.get_device_properties(dev).L2_cache_size / 2 ** 20
        in_mb = sum(t.numel() * t.element_size() for t in inp.values()) / 2 ** 20
        cfg = workload_config(shape, args, dist)
        cfg["l2"] = (f"no flush between steps: per-step inputs {in_mb:.0f} MiB and y {d2h_mib(y):.0f} MiB "
                     f"exceed the {l2_mb:.0f} MiB L2")
        cfg["variant"] = sdm.scan_variant(sh)
        if args.fp8_state:
            cfg["state_dtype"] = "fp8 E4M3, power-of-two scale per 16 values"
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": dist.world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": cfg,
                "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
                "clocks": clk,
                "stage_ms": {"select_k_and_q": stage_ms[0], "records": stage_ms[1], "state_init": stage_ms[2],
                             "scan": stage_ms[3], "epilogue": stage_ms[4], "recurrence_kernel": kernel_ms}}
        if chunks > 1:
            line["config"]["overlap"] = (f"{chunks} token chunks: each next chunk's selection on the SMs the "
                                         "recurrence leaves free; stage_ms select/records cover the first chunk, "
                                         "scan the first chunk's recurrence to the last one's end with the "
                                         "records in between; recurrence_kernel the sum of its launches")
    del ev, inp, y, M_out, ws
    torch.cuda.empty_cache()
    if dist.rank == 0:
        if dist.world == 1 and not args.no_extra and args.workload == DEFAULT_WORKLOAD and not args.fp8_state:
            line["extra_workloads"] = {name: measure_workload(name, args, dev) for name in EXTRA_WORKLOADS}
        print(json.dumps(line), flush=True)
    dist.close()


def roofline_of(shape: synth.Shape, sh, scan_ms: float, epilogue: bool, dev, clk: dict, fp8_state: bool = False,
                launches: int = 1) -> dict:
    """Roofline of the recurrence kernel: algorithmic bytes over its CUDA-event
    time (scan_ms a layer call, over `launches` launches: the token chunks of
    an overlapped call) against the measured HBM copy bandwidth (streaming,
    pipelined), or the derived shared-memory bandwidth (resident)."""
    resident = sdm.scan_variant(sh) == "resident"
    algo_bytes = algorithmic_bytes_per_token_head(shape, epilogue, fp8_state) * shape.B * shape.T * shape.H
    achieved = algo_bytes / (scan_ms / 1e3) / 1e9
    peaks = measured_peaks()
    if resident:
        mhz = clk.get("sm_max_mhz") or 1965.0
        peak = torch.cuda.get_device_properties(dev).multi_processor_count * SMEM_BYTES_PER_CLK_PER_SM * mhz / 1e3
        roof = {"bound": "smem", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "peak_source": f"derived: SMs x {SMEM_BYTES_PER_CLK_PER_SM} B/clk x {mhz:.0f} MHz "
                               "(state tile resident in shared memory)"}
    else:
        peak = peaks.get("hbm_gbs", FALLBACK_HBM_GBS)
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "peak_source": "of measured (MEASURED_PEAKS.json hbm_gbs)" if "hbm_gbs" in peaks else "of fallback"}
    kernel = {"resident": "k_scan_resident", "streaming": "k_scan_streaming",
              "pipelined": "k_scan_pipelined"}[sdm.scan_variant(sh)]
    launch_cfg = sdm.scan_describe(sh)
    traffic = recorded_traffic(shape.name, kernel, launch_cfg)
    roof.update({"traffic": None if traffic is None else traffic / launches, "kernel": kernel, "launch": launch_cfg,
                 "ms_per_launch": scan_ms / launches, "algorithmic_bytes_per_launch": algo_bytes / launches,
                 "launches_per_step": launches})
    return roof


def measure_workload(name: str, args, dev, steps: int = 5, warmup: int = 3) -> dict:
    """Device-time throughput of one more workload (same step as the headline)."""
    shape = synth.WORKLOADS[name]
    inp = synth.make_inputs(shape, seed=args.seed, device=dev)
    y = torch.empty((shape.B, shape.T, shape.H, shape.d_v), dtype=torch.float32, device=dev)
    M_out = torch.empty((shape.B,) + tuple(inp["M0"].shape), dtype=inp["M0"].dtype, device=dev)
    sh = sdm.make_shape(shape.B, shape.T, shape.H, shape.sqrt_n, shape.W, shape.R, shape.d_v, shape.torch_in(),
                        shape.torch_state())
    ws = torch.empty(sdm.layer_forward_workspace_bytes(sh), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
    for row in ev:  # create the events before the timed region
        for e in row:
            e.record(stream)

    def step(events=None):
        sdm.layer_forward(inp["kp"], inp["qp"], inp["v"], inp["alpha"], inp["beta"], inp["M0"], shape.W, shape.R,
                          y=y, M_out=M_out, workspace=ws, events=events)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for k in range(steps):
        step(ev[k])
    end.record(stream)
    torch.cuda.synchronize(dev)
    sdm.stream_check(dev)
    ms = start.elapsed_time(end) / steps
    scan_ms = sum(ev[k][3].elapsed_time(ev[k][4]) for k in range(steps)) / steps
    roof = roofline_of(shape, sh, scan_ms, False, dev, {})
    out = {"value": shape.B * shape.T / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
           "roofline": {k: roof[k] for k in ("bound", "achieved", "peak", "frac", "kernel", "launch", "ms_per_launch",
                                              "traffic")}}
    del inp, y, M_out, ws, ev
    torch.cuda.empty_cache()
    return out


def d2h_mib(y: torch.Tensor) -> float:
    return y.numel() * y.element_size() / 2 ** 20


def run_decode(args, dist: Dist):
    """Decode: every step is one sdm_layer_step call on one token per batch row
    (B rows, H heads of the workload), the state carried in place; reports the
    device time per step and the tokens per second it implies."""
    if not torch.cuda.is_available():
        raise SystemExit("bench.py --decode needs a CUDA device")
    dev = torch.device("cuda", dist.local_rank)
    torch.cuda.set_device(dev)
    dist.init("nccl")
    base = synth.WORKLOADS[args.workload]
    n_tok = args.warmup + args.steps
    shape = base.replace(T=n_tok)
    sdm.native.load()
    inp = synth.make_inputs(shape, seed=args.seed + dist.rank, device=dev)
    per_step = [{k: inp[k][:, t:t + 1].contiguous() for k in ("kp", "qp", "v", "alpha", "beta")} for t in range(n_tok)]
    M = inp["M0"].unsqueeze(0).repeat(shape.B, 1, 1, 1).contiguous()
    if args.fp8_state:
        M = sdm.quantize_fp8blk(M.float().contiguous())
    y = torch.empty((shape.B, 1, shape.H, shape.d_v), dtype=torch.float32, device=dev)
    sh = sdm.make_shape(shape.B, 1, shape.H, shape.sqrt_n, shape.W, shape.R, shape.d_v, shape.torch_in(),
                        torch.uint8 if args.fp8_state else shape.torch_state())
    ws = torch.empty(max(16, int(sdm.native.load().sdm_layer_step_workspace_bytes(ctypes.byref(sh)))),
                     dtype=torch.uint8, device=dev)

    def step(t):
        d = per_step[t]
        sdm.layer_step(d["kp"], d["qp"], d["v"], d["alpha"], d["beta"], M, shape.W, shape.R, y=y, workspace=ws)

    stream = torch.cuda.current_stream(dev)
    for t in range(args.warmup):
        step(t)
    sdm.stream_check(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier(dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clocks:
        start.record(stream)
        for t in range(args.warmup, n_tok):
            step(t)
        end.record(stream)
        torch.cuda.synchronize(dev)
    dist.barrier(dev)
    sdm.stream_check(dev)
    ms_eager = dist.max(start.elapsed_time(end), dev)
    # The same step captured once in a CUDA graph and replayed (the serving
    # path: fixed buffers, no host work per token); the state keeps evolving.
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        step(0)
    stream.wait_stream(side)
    torch.cuda.synchronize(dev)
    with torch.cuda.graph(graph):
        step(0)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize(dev)
    dist.barrier(dev)
    with ClockSampler(dev.index) as clocks:
        start.record(stream)
        for _ in range(args.steps):
            graph.replay()
        end.record(stream)
        torch.cuda.synchronize(dev)
    dist.barrier(dev)
    sdm.stream_check(dev)
    ms = dist.max(start.elapsed_time(end), dev)
    us_per_step = ms * 1e3 / args.steps
    del graph
    if dist.rank == 0:
        cfg = workload_config(shape, args, dist)
        cfg.update({"T": 1, "mode": "decode: one token per batch row per sdm_layer_step call, state carried",
                    "state_bytes": M.numel() * M.element_size()})
        if args.fp8_state:
            cfg.update({"state_dtype": "fp8 E4M3, power-of-two scale per 16 values", "variant": "single launch"})
        else:
            cfg["variant"] = sdm.scan_variant(sh)
        line = {"metric": "SDM decode step latency (one token per batch row, state carried) on 1 B200",
                "value": us_per_step, "unit": "us", "eager_us_per_step": ms_eager * 1e3 / args.steps,
                "timing": "value: one step captured in a CUDA graph and replayed; eager: one library call per step",
                "n_gpus": dist.world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": us_per_step / 1e3, "higher_is_better": False,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": cfg,
                "tokens_per_s": aggregate_value(shape.B * args.steps, dist.world, ms / 1e3),
                "gpu_launches": int(sdm.native.load().sdm_layer_step_launches(ctypes.byref(sh))) * args.steps,
                "clocks": clocks.summary()}
        print(json.dumps(line), flush=True)
    dist.close()


def run_backward(args, dist: Dist):
    """Backward: each step takes dy = dL/dy and computes the derivatives of
    the recurrence (sdm_scan_backward: dv, dalpha, dbeta, dk, dq, dM_0 with the
    forward recomputed from M_0) and of both selections' softmax weights
    (sdm_pkm_topk_backward on k' and q'), from the forward's saved selection.
    dL/dM_T is zero (reset every step). Reports tokens/s and, for the
    recurrence kernel, the shared-memory state traffic of its reverse sweep
    against the shared-memory roofline."""
    if not torch.cuda.is_available():
        raise SystemExit("bench.py --backward needs a CUDA device")
    dev = torch.device("cuda", dist.local_rank)
    torch.cuda.set_device(dev)
    dist.init("nccl")
    shape = synth.WORKLOADS[args.workload]
    sdm.native.load()
    inp = synth.make_inputs(shape, seed=args.seed + dist.rank, device=dev)
    idx_w, w_w = sdm.pkm_topk(inp["kp"], shape.W)
    idx_r, w_r = sdm.pkm_topk(inp["qp"], shape.R)
    M0 = inp["M0"].float().contiguous()
    gen = torch.Generator(device=dev).manual_seed(args.seed + 17)
    dy = torch.randn((shape.B, shape.T, shape.H, shape.d_v), generator=gen, device=dev)
    dM = torch.zeros((shape.B, shape.H, shape.N, shape.d_v), dtype=torch.float32, device=dev)
    sh = sdm.make_shape(shape.B, shape.T, shape.H, shape.sqrt_n, shape.W, shape.R, shape.d_v, shape.torch_in(),
                        torch.float32)
    ws = torch.empty(max(16, sdm.scan_backward_workspace_bytes(sh)), dtype=torch.uint8, device=dev)
    dk = torch.empty((shape.B, shape.T, shape.H, 2 * shape.sqrt_n), dtype=torch.float32, device=dev)
    dq = torch.empty_like(dk)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        dM.zero_()
        g = sdm.scan_backward(idx_w, w_w, idx_r, w_r, inp["v"], inp["alpha"], inp["beta"], M0, dy, dM, workspace=ws)
        if ev is not None:
            ev[1].record(stream)
        sdm.pkm_topk_backward(idx_w, w_w, g["dw_w"], shape.sqrt_n, dk)
        sdm.pkm_topk_backward(idx_r, w_r, g["dw_r"], shape.sqrt_n, dq)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    sdm.stream_check(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier(dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clocks:
        start.record(stream)
        for k in range(args.steps):
            step(ev[k])
        end.record(stream)
        torch.cuda.synchronize(dev)
    dist.barrier(dev)
    sdm.stream_check(dev)
    ms = dist.max(start.elapsed_time(end), dev)
    scan_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    topk_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
    if dist.rank == 0:
        th = shape.B * shape.T * shape.H
        algo = 3 * (shape.W + shape.R) * shape.d_v * 4 * th
        achieved = algo / (scan_ms / 1e3) / 1e9
        clk = clocks.summary()
        mhz = clk["sm_max_mhz"] or 1965.0
        peak = torch.cuda.get_device_properties(dev).multi_processor_count * SMEM_BYTES_PER_CLK_PER_SM * mhz / 1e3
        cfg = workload_config(shape, args, dist)
        cfg.update({"mode": "backward: recurrence (forward recomputed from M_0) and both selection-weight backwards",
                    "l2": "inputs and outputs exceed L2"})
        line = {"metric": "SDM backward tokens/s (B*T) on 1 B200", "impl": "sdm",
                "value": aggregate_value(shape.B * shape.T * args.steps, dist.world, ms / 1e3), "unit": "tokens/s",
                "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
                "stage_ms": {"scan_backward": scan_ms, "pkm_topk_backward_x2": topk_ms},
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic", "config": cfg,
                "roofline": {"bound": "smem", "achieved": achieved, "peak": peak, "unit": "GB/s",
                             "frac": achieved / peak, "kernel": "k_scan_backward",
                             "algorithmic_bytes_per_launch": algo, "ms_per_launch": scan_ms,
                             "peak_source": f"derived: SMs x {SMEM_BYTES_PER_CLK_PER_SM} B/clk x {mhz:.0f} MHz"},
                "gpu_launches": 4 * args.steps, "clocks": clk}
        if dist.world == 1:
            ck = checkpoint_comparison(shape, inp, dy, dev, stream, max(2, args.steps // 2))
            if ck is not None:
                line["with_forward_checkpoints"] = ck
        print(json.dumps(line), flush=True)
    dist.close()


def _device_ms(fn, stream, reps: int) -> float:
    """Mean CUDA-event time of fn() over reps calls (after one untimed call)."""
    fn()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(reps):
        fn()
    end.record(stream)
    torch.cuda.synchronize()
    return start.elapsed_time(end) / reps


def checkpoint_comparison(shape, inp, dy, dev, stream, reps: int):
    """The whole layer's forward and backward (sdm_layer_forward,
    sdm_layer_backward), with the forward storing the backward's checkpoints
    and without: the forward's extra cost and the backward's saving. None
    where the forward does not store checkpoints for this shape."""
    sh = sdm.make_shape(shape.B, shape.T, shape.H, shape.sqrt_n, shape.W, shape.R, shape.d_v, shape.torch_in(),
                        torch.float32)
    try:
        chunk, nbytes = sdm.layer_checkpoint_size(sh)
    except sdm.SdmError:
        return None
    M0 = inp["M0"].float().contiguous()
    args = (inp["kp"], inp["qp"], inp["v"], inp["alpha"], inp["beta"], M0, shape.W, shape.R)
    box = {}
    fwd_ms = _device_ms(lambda: sdm.layer_forward(*args), stream, reps)
    fwd_ck_ms = _device_ms(lambda: box.__setitem__("ck", sdm.layer_forward_ckpt(*args)[2]), stream, reps)
    bwd_ms = _device_ms(lambda: sdm.layer_backward(*args[:6], dy, shape.W, shape.R), stream, reps)
    bwd_ck_ms = _device_ms(lambda: sdm.layer_backward(*args[:6], dy, shape.W, shape.R, checkpoints=box["ck"]),
                           stream, reps)
    sdm.stream_check(dev)
    return {"checkpoint_tokens": chunk, "checkpoint_bytes": nbytes, "layer_forward_ms": fwd_ms,
            "layer_forward_ckpt_ms": fwd_ck_ms, "layer_backward_ms": bwd_ms, "layer_backward_ckpt_ms": bwd_ck_ms,
            "note": "device time per call, CUDA events; the backward given the forward's checkpoints skips its "
                    "first pass over the tokens"}


def run_slot_counts(args, dist: Dist):
    """Slot utilisation: each step counts, per (b, h), how often every slot is
    among the W write slots of the workload's T tokens (sdm_slot_counts on the
    indices sdm_pkm_topk chose). Reports selections counted per second and the
    achieved HBM bandwidth: the index array read once plus one read and one
    write of the [B, H, N] int32 counts."""
    if not torch.cuda.is_available():
        raise SystemExit("bench.py --slot-counts needs a CUDA device")
    dev = torch.device("cuda", dist.local_rank)
    torch.cuda.set_device(dev)
    dist.init("nccl")
    shape = synth.WORKLOADS[args.workload]
    sdm.native.load()
    inp = synth.make_inputs(shape, seed=args.seed + dist.rank, device=dev)
    idx, _ = sdm.pkm_topk(inp["kp"], shape.W)
    del inp
    counts = torch.zeros((shape.B, shape.H, shape.N), dtype=torch.int32, device=dev)
    flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        flush.fill_(1)
        sdm.slot_counts(idx, shape.N, counts)
    sdm.stream_check(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    dist.barrier(dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clocks:
        for a, b in ev:
            flush.fill_(1)  # L2 flushed between steps
            a.record(stream)
            sdm.slot_counts(idx, shape.N, counts)
            b.record(stream)
        torch.cuda.synchronize(dev)
    dist.barrier(dev)
    sdm.stream_check(dev)
    total = sum(counts.sum(dtype=torch.int64, dim=-1).flatten().tolist())
    assert total == (args.warmup + args.steps) * shape.B * shape.T * shape.H * shape.W, "counts do not add up"
    ms = dist.max(sum(a.elapsed_time(b) for a, b in ev), dev)
    sel = shape.B * shape.T * shape.H * shape.W
    algo = sel * 4 + 2 * shape.B * shape.H * shape.N * 4
    if dist.rank == 0:
        gbs = algo * args.steps / (ms / 1e3) / 1e9
        peak = measured_peaks().get("hbm_gbs", FALLBACK_HBM_GBS)
        cfg = workload_config(shape, args, dist)
        cfg.update({"mode": "slot utilisation counts of the write selection", "l2": "flushed between steps"})
        line = {"metric": "SDM slot utilisation counting throughput on 1 B200", "impl": "sdm",
                "value": aggregate_value(sel * args.steps, dist.world, ms / 1e3), "unit": "selections/s",
                "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "int32", "data": "synthetic", "config": cfg,
                "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                             "frac": gbs / peak if peak else None, "algorithmic_bytes_per_launch": algo},
                "gpu_launches": args.steps, "clocks": clocks.summary()}
        print(json.dumps(line), flush=True)
    dist.close()


def main():
    args = parse_args()
    dist = Dist()
    if args.impl == "reference":
        run_reference(args, dist)
        return
    if args.decode:
        run_decode(args, dist)
        return
    if args.slot_counts:
        run_slot_counts(args, dist)
        return
    if args.backward:
        run_backward(args, dist)
        return
    run_sdm(args, dist)


if __name__ == "__main__":
    main()
