#!/usr/bin/env python
"""Benchmark of the fused MoDA operator on B200: fwd+bwd TFLOP/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the whole hot path over one batch of synthetic input
already resident in HBM: from the layer-major depth caches K_depth and
V_depth, the forward and the backward.  Where the shape allows it (every
depth block whole tokens), the kernels read the layer-major caches in place
(MODA_DEPTH_LAYER: the layer-major -> token-major transpose of the depth
repack happens inside the depth-tile loads, and dK_depth / dV_depth come back
layer-major); otherwise the step runs the repack kernel first and the
kernels read its token-major copy.  The line also reports the step with the
separate repack.  The workload is the 1.5B-scale attention layer at T = 4096
(B=2, Hq=16, Hk=4, d=128, L=16).  FLOPs are algorithmic: forward
4*B*Hq*d*(T(T+1)/2 + T*L), backward 2.5x that.

Printed (rank 0, one JSON line): the whole-job value, the same workload at
L = 0 (the FlashAttention-style reference point), the forward at T = 65536
(L = 32 and L = 0), an end-to-end figure through host buffers, the roofline of
the dominant launch, the oracle timed on the host as a CPU baseline, and the
SM clocks sampled during the timed region.

Under torchrun (N > 1) every rank runs its own batch (data parallel, weak
scaling, no collective in the operator); times are the max over ranks.
`--impl reference` times the CPU oracle on the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))

import numpy as np  # noqa: E402
import torch  # noqa: E402

from sequence_depth_attention_moda_b200 import inputs as I  # noqa: E402

WORKLOAD = I.LAYER_1P5B
LONG = I.LONG_64K
BWD_FACTOR = 2.5


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extra", action="store_true", help="skip the L=0 twin and T=64K lines")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--configs", action="store_true",
                    help="per-config kernel times against their rooflines (every workload, the "
                         "G x L x C sweep, L = 0 twins); one JSON line, one GPU")
    ap.add_argument("--decode-only", action="store_true",
                    help="time only the decoding path (one JSON line; small device footprint)")
    ap.add_argument("--launch-check", action="store_true",
                    help="start the ranks as for a run and report them (gloo, no GPU work)")
    return ap.parse_args()


def launch_ranks(args) -> None:
    """`--gpus N` (N > 1) outside torchrun: run this script again under
    torch.distributed.run with N ranks on this node, one per GPU, and exit
    with its status.  Under torchrun (WORLD_SIZE set) this does nothing."""
    if args.gpus <= 1 or "WORLD_SIZE" in os.environ:
        return
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__),
           *sys.argv[1:]]
    sys.exit(subprocess.call(cmd))


def run_launch_check(args):
    """Every rank joins a gloo group and reports its rank; rank 0 prints one
    JSON line with the ranks seen (the launch path without any GPU work)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    seen = [rank]
    if world > 1:
        import datetime
        torch.distributed.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
        out = [None] * world
        torch.distributed.all_gather_object(out, rank)
        seen = sorted(out)
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps({"launch_check": True, "n_gpus": world, "ranks": seen,
                          "parallelism": f"dp{world}" if world > 1 else "single"}), flush=True)


# ------------------------------------------------------------------ helpers --
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": pk["hbm_gbs"], "bf16_tflops": pk["bf16_tflops"],
                "bf16_tflops_sustained": pk.get("bf16_tflops_sustained", pk["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """SM clock and throttle reasons sampled (NVML, every 10 ms, from a thread)
    while the timed region runs; nvidia-smi is the fallback."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, index: int):
        self.index = index
        self.samples = []       # (sm_mhz, reasons bitmask)
        self.max_mhz = None
        self._stop = None
        self._thread = None

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
        except Exception:
            return self
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((float(mhz), int(rs)))
                except Exception:
                    pass
                self._stop.wait(0.01)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)
        return False

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "source": "nvml"}
        reasons = sorted({nm for _, rs in self.samples for nm, bit in self.REASONS.items() if rs & bit})
        return {"sm_mhz": float(np.median([m for m, _ in self.samples])), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": "nvml"}


def traffic_from_profile(kernel: str, kernel_src: str, table: str = "dram_traffic_layer_T4k.md"):
    """Per-launch DRAM bytes (read + write) of `kernel` from the committed ncu
    summary, or None when its source has changed since the capture."""
    path = os.path.join(ROOT, "profiles", table)
    if not os.path.exists(path):
        return None
    m = re.search(r"^\| %s \| (\d+) \| [^|]+ \| ([0-9a-f]{16}) \|" % re.escape(kernel),
                  open(path).read(), re.M)
    if not m:
        return None
    cur = hashlib.sha256(open(kernel_src, "rb").read()).hexdigest()[:16]
    return int(m.group(1)) if cur == m.group(2) else None


def kernel_work(w: I.Workload, stored_ds: bool):
    """(algorithmic FLOPs, bytes each kernel must move) per launch of the
    forward and of the backward's dK/dV and dQ kernels.  FLOPs: the forward's
    4*B*Hq*d*(T(T+1)/2 + T*L); the backward's five matmuls over [seq | depth]
    split as dK/dV = S^T, dP^T, dV, dK over the sequence keys and dQ = dQ over
    all keys plus S, dP, dK_d, dV_d over the depth rows (recomputation is not
    counted).  Bytes: every input read once and every output written once;
    with stored dS, the dK/dV kernel writes and the dQ kernel reads the 16 KB
    dS tiles (128 query rows x 64 keys) the causal mask needs."""
    e = 2
    mm_seq = 2.0 * w.B * w.Hq * w.d * (w.T * (w.T + 1) / 2)
    mm_dep = 2.0 * w.B * w.Hq * w.d * (w.T * w.L)
    q = w.B * w.Hq * w.T * w.d * e
    kv = w.B * w.Hk * w.T * w.d * e
    dep = w.B * w.Hk * w.T * w.L * w.d * e
    rows = w.B * w.Hq * w.T * 4
    ds = 0
    if stored_ds:
        Tq = 128 // w.G
        n_qt, n_kb = -(-w.T // Tq), -(-w.T // 64)
        per_head = sum(min(n_kb, (min(Tq * (qt + 1), w.T) - 1) // 64 + 1) if w.causal else n_kb
                       for qt in range(n_qt))
        ds = w.B * w.Hk * per_head * 16384
    return {"fwd": (w.fwd_flops(), q + 2 * kv + 2 * dep + q + rows),
            "dkdv": (4 * mm_seq, 2 * kv + 2 * q + 2 * rows + 2 * kv + ds),
            "dq": ((mm_seq + mm_dep) + 4 * mm_dep,
                   2 * q + 2 * rows + (ds + kv if stored_ds else 2 * kv) + 2 * dep + q + 2 * dep)}


# --------------------------------------------------------------- our arm ----
def layer_supported(w: I.Workload) -> bool:
    """Whether the kernels can read this workload's layer-major depth caches
    in place (the library's own shape check)."""
    import ctypes
    import sequence_depth_attention_moda_b200 as moda
    if not w.L or w.dtype != "bf16":
        return False
    sh = moda.make_shape(w.B, w.Hq, w.Hk, w.T, w.d, w.L, 0, moda.MODA_BF16, moda.MODA_DEPTH_LAYER)
    return moda.load().moda_workspace_size(ctypes.byref(sh), 0) != ctypes.c_size_t(-1).value


class Runner:
    """Device buffers and the C-ABI calls of one step.  layer=True: forward
    and backward read the layer-major depth caches in place; False: the
    repack writes token-major copies that they read."""

    def __init__(self, w: I.Workload, x, backward=True, layer=None):
        import sequence_depth_attention_moda_b200 as moda
        self.moda = moda
        self.w = w
        self.x = x
        self.backward = backward
        self.layer = layer_supported(w) if layer is None else (layer and layer_supported(w))
        dev = x["Q"].device
        self.sh = moda.make_shape(w.B, w.Hq, w.Hk, w.T, w.d, w.L, w.C,
                                  moda.MODA_FP32 if w.dtype == "fp32" else moda.MODA_BF16,
                                  moda.MODA_DEPTH_LAYER if self.layer else moda.MODA_DEPTH_FLAT)
        if self.layer:
            self.Kd, self.Vd = x["Kd_layer"], x["Vd_layer"]
        else:
            self.Kd = torch.empty(w.B, w.Hk, w.T * w.L, w.d, device=dev, dtype=w.torch_dtype()) if w.L else None
            self.Vd = torch.empty_like(self.Kd) if w.L else None
        self.O = torch.empty_like(x["Q"])
        self.LSE = torch.empty(w.B, w.Hq, w.T, device=dev, dtype=torch.float32)
        self.stored_ds = False
        if backward:
            self.nws = moda.moda_workspace_size(self.sh, 1)
            self.stored_ds = self.nws > moda.moda_workspace_size(self.sh, 2)
            self.ws = torch.empty(max(self.nws, 16), device=dev, dtype=torch.uint8)
            self.dQ = torch.empty_like(x["Q"])
            self.dK = torch.empty_like(x["K"])
            self.dV = torch.empty_like(x["V"])
            self.dKd = torch.empty_like(self.Kd) if w.L else None
            self.dVd = torch.empty_like(self.Vd) if w.L else None

    def launches_per_step(self):
        return (2 if self.w.L and not self.layer else 0) + 1 + (3 if self.backward else 0)

    def step(self, ev=None):
        """One step.  With `ev` (8 CUDA events) the repack is bracketed by
        ev[0:2] and the library records ev[2:4] around the forward kernel and
        ev[4:8] around the backward's three kernels (moda_set_phase_events)."""
        m, x = self.moda, self.x
        if ev is not None:
            ev[0].record()
        if self.w.L and not self.layer:
            m.moda_repack_depth(self.sh, x["Kd_layer"], self.Kd)
            m.moda_repack_depth(self.sh, x["Vd_layer"], self.Vd)
        if ev is not None:
            ev[1].record()
            m.moda_set_phase_events(ev[2:4])
        m.moda_fwd(self.sh, x["Q"], x["K"], x["V"], self.Kd, self.Vd, self.O, self.LSE)
        if self.backward:
            if ev is not None:
                m.moda_set_phase_events(ev[4:8])
            m.moda_bwd(self.sh, x["Q"], x["K"], x["V"], self.Kd, self.Vd, self.O, self.LSE, x["dO"],
                       self.dQ, self.dK, self.dV, self.dKd, self.dVd, self.ws, self.nws)
        if ev is not None:
            m.moda_set_phase_events([])

    def outputs(self):
        outs = [self.O, self.LSE]
        if self.backward:
            outs += [self.dQ, self.dK, self.dV] + ([self.dKd, self.dVd] if self.w.L else [])
        return outs


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """Max of a per-rank time over all ranks (NCCL on GPUs, gloo on CPUs)."""
    if world == 1:
        return v
    dev = (torch.device("cuda", torch.cuda.current_device())
           if torch.distributed.get_backend() == "nccl" else torch.device("cpu"))
    t = torch.tensor([v], device=dev, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_seed(w: I.Workload, rank: int) -> int:
    """Each rank draws its own batch (data parallel)."""
    return w.seed + 1000 * rank


def job_value(flops_per_rank: float, ms_max: float, world: int) -> float:
    """Whole-job TFLOP/s: the work of all ranks over the slowest rank's time."""
    return world * flops_per_rank / (ms_max * 1e-3) / 1e12


def time_steps(r: Runner, steps: int, warmup: int, world: int, per_call=False, clocks=None):
    """Warm up, then time exactly `steps` steps between barriers + syncs.
    Returns (ms per step, per-call mean ms or None)."""
    for _ in range(warmup):
        r.step()
    torch.cuda.synchronize()
    evs = None
    if per_call:
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(8)] for _ in range(steps)]
        for e in (e for row in evs for e in row):
            e.record()           # creates the event so its handle can be passed on
        torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    ctx = clocks if clocks is not None else _Null()
    with ctx:
        start.record()
        for i in range(steps):
            r.step(evs[i] if per_call else None)
        end.record()
        torch.cuda.synchronize()
    barrier(world)
    ms = start.elapsed_time(end) / steps
    calls = None
    if per_call:
        calls = {"repack": np.mean([e[0].elapsed_time(e[1]) for e in evs]),
                 "fwd": np.mean([e[2].elapsed_time(e[3]) for e in evs])}
        if r.backward:
            calls.update(rowdot=np.mean([e[4].elapsed_time(e[5]) for e in evs]),
                         dkdv=np.mean([e[5].elapsed_time(e[6]) for e in evs]),
                         dq=np.mean([e[6].elapsed_time(e[7]) for e in evs]),
                         bwd=np.mean([e[4].elapsed_time(e[7]) for e in evs]))
    return max_over_ranks(ms, world), calls


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def e2e_measure(w: I.Workload, x, steps: int, world: int):
    """Same step through the C ABI with host buffers: every step copies all of
    its inputs from pinned host memory to the device and all of its outputs
    back, inside the timed region.  Two buffer sets and three streams let step
    k's read-back overlap step k+1's upload and compute (PCIe is full
    duplex); events order each set's upload after its previous read-back."""
    host_in = {k: v.cpu().pin_memory() for k, v in x.items()}
    xs = [x, {k: torch.empty_like(v) for k, v in x.items()}]
    rs = [Runner(w, xs[0]), Runner(w, xs[1])]
    host_out = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in r.outputs()] for r in rs]
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out[0])
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_run = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def one(k):
        i = k % 2
        with torch.cuda.stream(s_in):
            if used[i]:
                s_in.wait_event(ev_out[i])       # set i's outputs read back, its inputs free
            for key, v in host_in.items():
                xs[i][key].copy_(v, non_blocking=True)
            ev_in[i].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(ev_in[i])
            rs[i].step()
            ev_run[i].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_run[i])
            for dst, src in zip(host_out[i], rs[i].outputs()):
                dst.copy_(src, non_blocking=True)
            ev_out[i].record(s_out)
        used[i] = True

    for k in range(2):
        one(k)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    start.record(s_in)
    for k in range(steps):
        one(k)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_run)
    end.record(s_out)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(start.elapsed_time(end) / steps, world)
    return ms, h2d, d2h


def decode_measure(w: I.Workload, rank: int, world: int, peaks, iters: int):
    """Decoding one new token per sequence over the cached keys: CUDA-event
    time per moda_decode call (inputs 1.1 GB, larger than L2), the HBM
    roofline of its algorithmic bytes (cache K, V and the depth rows read
    once; q read, o and LSE written) and tokens per second."""
    import sequence_depth_attention_moda_b200 as moda
    x = I.make_decode_inputs(w, device="cuda", seed=w.seed + 1000 * rank)
    sh = moda.make_shape(w.B, w.Hq, w.Hk, w.T, w.d, w.L, 0)
    nws = moda.moda_decode_workspace_size(sh)
    ws = torch.empty(max(nws, 16), device="cuda", dtype=torch.uint8)
    o = torch.empty_like(x["q"])
    lse = torch.empty(w.B, w.Hq, device="cuda", dtype=torch.float32)

    def call():
        moda.moda_decode(sh, x["q"], x["K"], x["V"], x["Kd"], x["Vd"], o, lse, ws, nws)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        call()
    e1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / iters, world)
    nbytes = sum(x[k].numel() * x[k].element_size() for k in ("q", "K", "V", "Kd", "Vd"))
    nbytes += o.numel() * o.element_size() + lse.numel() * 4
    gbs = nbytes / (ms * 1e-3) / 1e9
    src = os.path.join(ROOT, "sequence_depth_attention_moda_b200", "csrc", "moda_decode.cu")
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hk": w.Hk, "d": w.d, "T": w.T, "L": w.L,
            "ms": round(ms, 4), "tokens_per_s": round(world * w.B / (ms * 1e-3), 1),
            "roofline": {"kernel": "decode_mma_kernel (+ decode_combine_kernel, both timed)",
                         "bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                         "bytes_per_call": nbytes,
                         "traffic": traffic_from_profile("decode_mma_kernel", src,
                                                         "dram_traffic_decode_T32k.md")}}


def cpu_baseline_sample(w: I.Workload, x):
    """The oracle, as it stands, on one (b, hk) slice of the workload
    (forward + backward of G heads over all T tokens and L depth rows)."""
    import oracle
    from moda_cases import slice_workload, token_major, f64
    ws, xs = slice_workload(w, x, 0, 0)
    Kd, Vd = token_major(xs, ws)
    args = [f64(xs["Q"]), f64(xs["K"]), f64(xs["V"]), f64(Kd), f64(Vd)]
    dO = f64(xs["dO"])
    lib = oracle.load_library()
    t0 = time.perf_counter()
    oracle.fwd(*args, lib=lib)
    oracle.bwd(*args, dO, lib=lib)
    dt = time.perf_counter() - t0
    flops = ws.fwd_flops() * (1 + BWD_FACTOR)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.threads(lib),
            "kind": "oracle",
            "sample": f"one (b,hk) slice of the workload: B=1, Hq=G={ws.Hq}, Hk=1, T={ws.T}, "
                      f"L={ws.L}, d={ws.d}, fwd+bwd in fp64 ({1.0 / (w.B * w.Hk):.4f} of a step), "
                      f"{dt:.1f} s"}


def _rows_rate(lib, w: I.Workload, x, rows, cores: int):
    """Oracle time of the sampled query rows (b, h, t) of workload w, run
    on `cores` host threads (the row entry point releases the GIL).  Returns
    (seconds, FLOPs of those rows)."""
    import concurrent.futures as cf
    import oracle
    G, L = w.G, w.L
    f64 = {}

    def kv(b, hk):
        if (b, hk) not in f64:
            f64[(b, hk)] = (x["K"][b, hk].double().numpy(), x["V"][b, hk].double().numpy())
        return f64[(b, hk)]

    jobs = []
    for (b, h, t) in rows:
        K, V = kv(b, h // G)
        Kd = x["Kd_layer"][:, b, h // G, t].double().numpy() if L else np.zeros((0, w.d))
        Vd = x["Vd_layer"][:, b, h // G, t].double().numpy() if L else np.zeros((0, w.d))
        jobs.append((x["Q"][b, h, t].double().numpy(), K[:t + 1], V[:t + 1], Kd, Vd))
    flops = sum(4.0 * w.d * (t + 1 + L) for (_, _, t) in rows)
    t0 = time.perf_counter()
    with cf.ThreadPoolExecutor(max_workers=cores) as ex:
        list(ex.map(lambda a: oracle.row(*a, lib=lib), jobs))
    return time.perf_counter() - t0, flops


def cpu_baselines_per_config(x_c2):
    """The oracle, as it stands, on every workload of the benchmark, each on
    a bounded sample (a few seconds of host time in all): the tiny fp32
    workload in full; the 1.5B layer and the training shape on one (b, hk)
    slice, forward + backward; the T = 64K forward and the G x L sweep on
    sampled query rows.  Rates are FLOPs of the sample / its time; for the
    sampled workloads `est_s` is the whole workload's time at that rate
    (extrapolated)."""
    import oracle
    from moda_cases import slice_workload, token_major, f64
    lib = oracle.load_library()
    cores = oracle.threads(lib)
    out = {}

    def slice_rate(w, x, backward):
        ws, xs = slice_workload(w, x, 0, 0)
        Kd, Vd = token_major(xs, ws)
        a = [f64(xs["Q"]), f64(xs["K"]), f64(xs["V"]), f64(Kd), f64(Vd)]
        t0 = time.perf_counter()
        oracle.fwd(*a, lib=lib)
        if backward:
            oracle.bwd(*a, f64(xs["dO"]), lib=lib)
        dt = time.perf_counter() - t0
        fl = ws.fwd_flops() * ((1 + BWD_FACTOR) if backward else 1)
        return dt, fl, ws

    def entry(w, dt, fl, total, sample, extrapolated, threads):
        rate = fl / dt
        return {"value": round(rate / 1e12, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                "sample": sample, "sample_s": round(dt, 6), "extrapolated": extrapolated,
                "est_s": round(total / rate, 4)}

    w = I.TINY_FP32.with_(backward=True)
    x = I.make_inputs(w, device="cpu")
    Kd, Vd = token_major(x, w)
    a = [f64(x["Q"]), f64(x["K"]), f64(x["V"]), f64(Kd), f64(Vd)]
    reps = 50
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.fwd(*a, lib=lib)
    dt = (time.perf_counter() - t0) / reps
    out[w.name] = entry(w, dt, w.fwd_flops(), w.fwd_flops(),
                        f"the whole forward, fp64 (mean of {reps} runs)", False, cores)

    w = WORKLOAD
    dt, fl, ws = slice_rate(w, x_c2, True)
    out[w.name] = entry(w, dt, fl, w.fwd_flops() * (1 + BWD_FACTOR),
                        f"one (b,hk) slice (B=1, Hq={ws.Hq}, Hk=1), forward + backward", True, cores)

    w = I.TRAIN_FWD_BWD
    x = I.make_inputs(w.with_(B=1, Hq=w.G, Hk=1), device="cpu")
    dt, fl, ws = slice_rate(w.with_(B=1, Hq=w.G, Hk=1), x, True)
    out[w.name] = entry(w, dt, fl, w.fwd_flops() * (1 + BWD_FACTOR),
                        f"one (b,hk) slice (B=1, Hq={w.G}, Hk=1), forward + backward", True, cores)
    del x

    w = LONG
    x = I.make_inputs(w.with_(Hq=w.G, Hk=1), device="cpu", grad_out=False)
    rng = np.random.default_rng(11)
    rows = [(0, int(rng.integers(w.G)), int(t)) for t in np.linspace(0, w.T - 1, 128).astype(int)]
    dt, fl = _rows_rate(lib, w.with_(Hq=w.G, Hk=1), x, rows, cores)
    out[w.name] = entry(w, dt, fl, w.fwd_flops(), "128 query rows, t evenly spread over 0..T-1, forward (row entry point)",
                        True, cores)
    del x

    tot_fl = tot_dt = tot_all = 0.0
    for G in (1, 2, 4, 8):
        for L in (1, 8, 32, 64):
            w = I.Workload(f"sweep_G{G}_L{L}", B=1, Hq=G, Hk=1, d=128, T=8192, L=L, C=64, seed=7)
            x = I.make_inputs(w, device="cpu", grad_out=False)
            rows = [(0, int(rng.integers(G)), int(t)) for t in np.linspace(0, w.T - 1, 32).astype(int)]
            dt, fl = _rows_rate(lib, w, x, rows, cores)
            tot_fl += fl
            tot_dt += dt
            tot_all += 3 * w.with_(Hq=4 * G, Hk=4).fwd_flops()     # three C values, same work
            del x
    out["depth_group_sweep"] = entry(None, tot_dt, tot_fl, tot_all,
                                     "32 query rows of each (G, L) point (C does not change the work), "
                                     "forward (row entry point)", True, cores)
    return out


def run_ours(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    import sequence_depth_attention_moda_b200 as moda
    moda.load()
    peaks = load_peaks()
    w = WORKLOAD
    x = I.make_inputs(w, device="cuda", seed=rank_seed(w, rank))
    r = Runner(w, x)
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    clocks = ClockSampler(int(vis.split(",")[local]) if vis else torch.cuda.current_device())
    ms, calls = time_steps(r, args.steps, args.warmup, world, per_call=True, clocks=clocks)
    moda.moda_check_status()
    flops_step = w.fwd_flops() * (1 + BWD_FACTOR)
    value = job_value(flops_step, ms, world)
    per_gpu = value / world
    # the same step with the separate repack kernel and the token-major copies
    r_flat = Runner(w, x, layer=False)
    ms_flat, calls_flat = time_steps(r_flat, args.steps, args.warmup, world, per_call=True)
    moda.moda_check_status()
    del r_flat
    step_flat = {"value": round(job_value(flops_step, ms_flat, world), 2), "ms_per_step": round(ms_flat, 4),
                 "per_kernel_ms": {k: round(v, 4) for k, v in calls_flat.items()},
                 "launches_per_step": 6}

    # Roofline of the dominant kernel (largest mean duration) and of the
    # others: each against max(algorithmic FLOPs / tensor peak, bytes it must
    # move / HBM bandwidth) (kernel_work).
    work = kernel_work(w, stored_ds=r.stored_ds)
    names = {"fwd": "moda_fwd_sm100_kernel", "dkdv": "dkdv_kernel", "dq": "dq_kernel"}
    srcs = {"fwd": "moda_fwd_sm100.cu", "dkdv": "moda_bwd_sm100.cu", "dq": "moda_bwd_sm100.cu"}
    dom = max(names, key=lambda k: calls[k])

    def roof(k):
        flops, nbytes = work[k]
        t_tensor = flops / (peaks["bf16_tflops"] * 1e12)
        t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
        src = os.path.join(ROOT, "sequence_depth_attention_moda_b200", "csrc", srcs[k])
        out = {"kernel": names[k], "mean_ms": round(calls[k], 4), "algorithmic_flops": flops,
               "algorithmic_bytes": nbytes, "traffic": traffic_from_profile(names[k], src)}
        if t_tensor >= t_hbm:
            ach = flops / (calls[k] * 1e-3) / 1e12
            out.update(bound="tensor", achieved=round(ach, 1), peak=peaks["bf16_tflops"], unit="TFLOP/s",
                       frac=round(ach / peaks["bf16_tflops"], 4),
                       peak_source=f"{peaks['source']} bf16 dense (burst)")
        else:
            ach = nbytes / (calls[k] * 1e-3) / 1e9
            out.update(bound="hbm", achieved=round(ach, 1), peak=peaks["hbm_gbs"], unit="GB/s",
                       frac=round(ach / peaks["hbm_gbs"], 4), peak_source=f"{peaks['source']} copy bandwidth")
        return out

    roofline = roof(dom)
    roofline["per_kernel_ms"] = {k: round(v, 4) for k, v in calls.items() if not (k == "repack" and r.layer)}
    roofline_others = {k: roof(k) for k in names if k != dom}
    rep_bytes = 2 * 2 * w.B * w.Hk * w.T * w.L * w.d * 2
    rep_ach = rep_bytes / (calls_flat["repack"] * 1e-3) / 1e9
    roofline_repack = {"kernel": "repack_vec16_kernel (x2), in the step with the separate repack",
                       "bound": "hbm", "achieved": round(rep_ach, 1),
                       "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(rep_ach / peaks["hbm_gbs"], 4)}

    extra = {}
    if not args.no_extra:
        w0 = w.with_(L=0)
        x0 = dict(x)
        r0 = Runner(w0, x0)
        ms0, _ = time_steps(r0, args.steps, args.warmup, world)
        v0 = world * w0.fwd_flops() * (1 + BWD_FACTOR) / (ms0 * 1e-3) / 1e12
        extra["l0_twin"] = {"value": round(v0, 2), "ms_per_step": round(ms0, 4),
                            "ratio": round(value / v0, 4)}
        del r0
        xl = I.make_inputs(LONG, device="cuda", seed=LONG.seed + 1000 * rank, grad_out=False)
        long_res = {}
        for L in (LONG.L, 0):
            wl = LONG.with_(L=L)
            rl = Runner(wl, xl, backward=False, layer=False)   # the forward on token-major depth rows
            msl, callsl = time_steps(rl, max(3, args.steps // 4), 2, world, per_call=True)
            tf = wl.fwd_flops() / (callsl["fwd"] * 1e-3) / 1e12
            long_res[f"L{L}"] = {"fwd_tflops": round(tf, 1),
                                 "fwd_frac_of_peak": round(tf / peaks["bf16_tflops"], 4),
                                 "fwd_ms": round(callsl["fwd"], 3)}
            del rl
        long_res["fwd_vs_L0"] = round(long_res[f"L{LONG.L}"]["fwd_tflops"] / long_res["L0"]["fwd_tflops"], 4)
        extra["long_context_T64k_fwd"] = long_res
        del xl
        torch.cuda.empty_cache()
        extra["decode_T32k"] = decode_measure(I.DECODE_T32K, rank, world, peaks, max(10, args.steps // 2))
        torch.cuda.empty_cache()
        # the training-shaped step and the G x L x C sweep, one kernel call at a
        # time against max(FLOPs / peak, bytes / bandwidth) (fewer runs each)
        flush = torch.empty(256 << 20, device="cuda", dtype=torch.uint8)
        extra["train_T4k_L48"] = config_measure(I.TRAIN_FWD_BWD, peaks, flush, runs=5)
        torch.cuda.empty_cache()
        extra["depth_group_sweep"] = sweep_summary(peaks, flush, runs=5)
        del flush
        torch.cuda.empty_cache()

    e2e = None
    if not args.no_e2e:
        ms_e, h2d, d2h = e2e_measure(w, x, max(4, min(args.steps, 20)), world)
        e2e = {"value": round(world * flops_step / (ms_e * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms_e, 3),
               "pipeline": "upload / compute / read-back on three streams, two buffer sets"}

    cpu = cpu_all = None
    if world == 1 and rank == 0 and not args.no_cpu:
        cpu = cpu_baseline_sample(w, x)
        cpu_all = cpu_baselines_per_config({k: v.cpu() for k, v in x.items()})

    if rank == 0:
        line = {
            "metric": "MoDA fwd+bwd TFLOP/s (forward + backward per step from the layer-major depth cache)",
            "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "pct_of_peak_per_gpu": round(100 * per_gpu / peaks["bf16_tflops"], 2),
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hk": w.Hk, "d": w.d, "T": w.T,
                       "L": w.L, "C": w.C, "global_batch": w.B * world, "seq_len": w.T,
                       "parallelism": f"dp{world}" if world > 1 else "single",
                       "depth_layout": ("layer-major, read in place (repack fused into the depth-tile loads)"
                                        if r.layer else "token-major copy made by the repack kernel"),
                       "l2": "inputs larger than L2 (%.0f MB read per step)" %
                             (sum(t.numel() * t.element_size() for t in x.values()) / 1e6)},
            "roofline": roofline, "roofline_other_kernels": roofline_others,
            "roofline_repack": roofline_repack, "step_with_separate_repack": step_flat,
            "gpu_launches": r.launches_per_step() * args.steps,
            "clocks": clocks.summary(), "e2e": e2e, "cpu_baseline": cpu,
            "cpu_baseline_per_config": cpu_all, **extra,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


# --------------------------------------------------------- reference arm ----
def run_reference(args):
    """The CPU oracle as the reference arm: bounded sample of the workload
    per step (one (b, hk) slice), on the host cores, rank 0 only."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from moda_cases import slice_workload, token_major, f64
    w = WORKLOAD
    x = I.make_inputs(w, device="cpu")
    ws, xs = slice_workload(w, x, 0, 0)
    Kd, Vd = token_major(xs, ws)
    a = [f64(xs["Q"]), f64(xs["K"]), f64(xs["V"]), f64(Kd), f64(Vd)]
    dO = f64(xs["dO"])
    lib = oracle.load_library()

    def step():
        oracle.fwd(*a, lib=lib)
        oracle.bwd(*a, dO, lib=lib)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    flops = ws.fwd_flops() * (1 + BWD_FACTOR)
    value = flops / dt / 1e12
    sample = (f"one (b,hk) slice per step: B=1, Hq=G={ws.Hq}, Hk=1, T={ws.T}, L={ws.L}, "
              f"d={ws.d}, fwd+bwd in fp64")
    line = {"impl": "reference", "metric": "MoDA fwd+bwd TFLOP/s (forward + backward per step from the layer-major depth cache)",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hk": w.Hk, "d": w.d, "T": w.T,
                       "L": w.L, "C": w.C, "sample": sample},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.threads(lib),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _median_ms(call, runs: int, flush: torch.Tensor) -> float:
    """Median CUDA-event time of `call` over `runs` runs after 3 warm-up
    calls, with L2 flushed (a 256 MB write) before every timed run."""
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    times = []
    for _ in range(runs):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        call()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    return float(np.median(times))


def config_measure(w: I.Workload, peaks, flush: torch.Tensor, runs: int = 20, twin: bool = True):
    """One workload: repack, forward and (for training workloads) backward
    timed one call at a time; each against its attainable time
    max(FLOPs / tensor peak, algorithmic bytes / HBM bandwidth)."""
    import sequence_depth_attention_moda_b200 as moda
    e = 2 if w.dtype == "bf16" else 4
    x = I.make_inputs(w, device="cuda", grad_out=w.backward)

    def one(wl):
        r = Runner(wl, x, backward=wl.backward, layer=False)   # repack and kernels timed one by one
        r.step()                                   # fills the token-major depth tensors
        xx = r.x
        fwd = lambda: moda.moda_fwd(r.sh, xx["Q"], xx["K"], xx["V"], r.Kd, r.Vd, r.O, r.LSE)
        res = {"fwd_ms": _median_ms(fwd, runs, flush)}
        if wl.backward:
            bwd = lambda: moda.moda_bwd(r.sh, xx["Q"], xx["K"], xx["V"], r.Kd, r.Vd, r.O, r.LSE, xx["dO"],
                                        r.dQ, r.dK, r.dV, r.dKd, r.dVd, r.ws, r.nws)
            res["bwd_ms"] = _median_ms(bwd, runs, flush)
        if wl.L:
            def rep():
                moda.moda_repack_depth(r.sh, xx["Kd_layer"], r.Kd)
                moda.moda_repack_depth(r.sh, xx["Vd_layer"], r.Vd)
            res["repack_ms"] = _median_ms(rep, runs, flush)
        del r
        if wl.L and layer_supported(wl):
            # the same calls reading the layer-major caches in place (no repack)
            rl = Runner(wl, x, backward=wl.backward, layer=True)
            fwd_l = lambda: moda.moda_fwd(rl.sh, xx["Q"], xx["K"], xx["V"], rl.Kd, rl.Vd, rl.O, rl.LSE)
            res["fwd_layer_ms"] = _median_ms(fwd_l, runs, flush)
            if wl.backward:
                bwd_l = lambda: moda.moda_bwd(rl.sh, xx["Q"], xx["K"], xx["V"], rl.Kd, rl.Vd, rl.O, rl.LSE,
                                              xx["dO"], rl.dQ, rl.dK, rl.dV, rl.dKd, rl.dVd, rl.ws, rl.nws)
                res["bwd_layer_ms"] = _median_ms(bwd_l, runs, flush)
            del rl
        moda.moda_check_status()
        return res

    def roof(flops, nbytes, ms):
        t_tensor = flops / (peaks["bf16_tflops"] * 1e12) * 1e3
        t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9) * 1e3
        att = max(t_tensor, t_hbm)
        return {"ms": round(ms, 4), "tflops": round(flops / (ms * 1e-3) / 1e12, 1),
                "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1), "bound": "tensor" if t_tensor >= t_hbm else "hbm",
                "attainable_ms": round(att, 4), "frac_of_attainable": round(att / ms, 4)}

    q_el = w.B * w.Hq * w.T * w.d
    kv_el = w.B * w.Hk * w.T * w.d
    dep_el = w.B * w.Hk * w.T * w.L * w.d
    ff = w.fwd_flops()
    out = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hk": w.Hk, "d": w.d, "T": w.T, "L": w.L, "C": w.C,
           "dtype": w.dtype}
    m = one(w)
    out["fwd"] = roof(ff, e * (2 * q_el + 2 * kv_el + 2 * dep_el) + 4 * w.B * w.Hq * w.T, m["fwd_ms"])
    if w.backward:
        out["bwd"] = roof(BWD_FACTOR * ff, e * (4 * q_el + 4 * kv_el + 4 * dep_el) + 3 * 4 * w.B * w.Hq * w.T,
                          m["bwd_ms"])
    if w.L:
        rb = 2 * 2 * dep_el * e
        out["repack"] = {"ms": round(m["repack_ms"], 4), "gbs": round(rb / (m["repack_ms"] * 1e-3) / 1e9, 1),
                         "frac_of_hbm": round(rb / (m["repack_ms"] * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
    if "fwd_layer_ms" in m:
        # layer-major caches read in place: the repack's transpose inside the
        # depth-tile loads; its time against repack + the token-major calls
        lm = {"fwd_ms": round(m["fwd_layer_ms"], 4)}
        flat = m["repack_ms"] + m["fwd_ms"]
        lay = m["fwd_layer_ms"]
        if w.backward:
            lm["bwd_ms"] = round(m["bwd_layer_ms"], 4)
            flat += m["bwd_ms"]
            lay += m["bwd_layer_ms"]
        lm["calls_ms"] = round(lay, 4)
        lm["repack_plus_token_major_calls_ms"] = round(flat, 4)
        out["layer_major"] = lm
    if twin and w.L:
        m0 = one(w.with_(L=0))
        out["L0_fwd_ms"] = round(m0["fwd_ms"], 4)
        out["fwd_time_vs_L0"] = round(m0["fwd_ms"] / m["fwd_ms"], 4)   # L=0 time / time: <= 1
        if w.backward:
            out["L0_bwd_ms"] = round(m0["bwd_ms"], 4)
    del x
    torch.cuda.empty_cache()
    return out


def sweep_summary(peaks, flush, runs: int = 5):
    """The G x L x C sweep's forward against its attainable time: worst and
    median fraction over the 48 points, and the G = 1 and G = 8 points at
    L = 64, C = 64."""
    rows = []
    seen_g = set()
    for w in I.depth_group_sweep():
        rows.append(config_measure(w, peaks, flush, runs=runs, twin=w.G not in seen_g))
        seen_g.add(w.G)
    fr = sorted(r["fwd"]["frac_of_attainable"] for r in rows)
    pick = {r["workload"]: r for r in rows}
    worst = min(rows, key=lambda r: r["fwd"]["frac_of_attainable"])
    return {"points": len(rows), "runs": runs,
            "fwd_frac_of_attainable_worst": fr[0], "worst_point": worst["workload"],
            "fwd_frac_of_attainable_median": round(float(np.median(fr)), 4),
            "G1_L64_C64": pick["sweep_G1_L64_C64"]["fwd"], "G8_L64_C64": pick["sweep_G8_L64_C64"]["fwd"],
            "L0_fwd_ms": {f"G{r['Hq'] // r['Hk']}": r["L0_fwd_ms"] for r in rows if "L0_fwd_ms" in r}}


def run_configs(args):
    """Every workload's kernels against their rooflines (one GPU)."""
    torch.cuda.set_device(0)
    import sequence_depth_attention_moda_b200 as moda
    moda.load()
    peaks = load_peaks()
    flush = torch.empty(256 << 20, device="cuda", dtype=torch.uint8)
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    clocks = ClockSampler(int(vis.split(",")[0]) if vis else 0)
    with clocks:
        rows = [config_measure(w, peaks, flush) for w in (I.TINY_FP32, I.LAYER_1P5B, I.LONG_64K, I.TRAIN_FWD_BWD)]
        seen_g = set()
        for w in I.depth_group_sweep():
            rows.append(config_measure(w, peaks, flush, twin=w.G not in seen_g))
            seen_g.add(w.G)
    print(json.dumps({"metric": "per-config kernel time against max(FLOPs/peak, bytes/bandwidth)",
                      "n_gpus": 1, "runs": 20, "warmup": 3, "l2": "flushed (256 MB write) before every run",
                      "clocks": clocks.summary(),
                      "peaks": {"bf16_tflops": peaks["bf16_tflops"], "hbm_gbs": peaks["hbm_gbs"],
                                "source": peaks["source"]},
                      "configs": rows}), flush=True)


def run_decode_only(args):
    """The decoding workload alone (one GPU)."""
    torch.cuda.set_device(0)
    res = decode_measure(I.DECODE_T32K, 0, 1, load_peaks(), max(1, args.steps))
    print(json.dumps({"metric": "MoDA decoding tokens/s (one new token per sequence)",
                      "value": res["tokens_per_s"], "unit": "tokens/s", "n_gpus": 1,
                      "steps": args.steps, "warmup": 3, "higher_is_better": True,
                      "data": "synthetic", "decode": res}), flush=True)


def main():
    args = parse_args()
    launch_ranks(args)
    if args.launch_check:
        run_launch_check(args)
    elif args.impl == "reference":
        run_reference(args)
    elif args.decode_only:
        run_decode_only(args)
    elif args.configs:
        run_configs(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
