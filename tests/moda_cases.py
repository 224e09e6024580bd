"""Helpers shared by the GPU parity tests, the smoke check and the benchmark.

``run_gpu`` drives the CUDA path through the C ABI (repack, forward, optional
backward); ``oracle_*`` compute the fp64 CPU references on the same seeded
inputs, either in full or for sampled rows / sampled (b, hk) slices (rows are
independent in the forward, whole (b, hk) slices in the backward, so a sample
is checked exactly).
"""
from __future__ import annotations

import math
from typing import Dict, Iterable, List, Sequence, Tuple

import numpy as np
import torch

import oracle
import sequence_depth_attention_moda_b200 as moda
from sequence_depth_attention_moda_b200.inputs import Workload, make_inputs

# bf16 in / fp32 accumulate tolerances on the output (stated with the operator)
BF16_MAX_ABS, BF16_MEAN_ABS = 2e-2, 2e-3
FP32_MAX_ABS = 1e-4
# LSE is fp32 statistics of exactly representable scores: tight.
LSE_MAX_ABS = 1e-3
# gradients (the pages state none), each bound relative to the reference
# tensor's own scale, with no absolute floor:
#   ||g - ref||_2 <= 1e-2 * ||ref||_2
#   max |g - ref| <= 2e-2 * max |ref|
#   mean|g - ref| <= 5e-3 * mean|ref|
# Rounding a gradient to bf16 on store costs up to 2^-9 relative (about 1e-3 on
# average), and the bf16 P / dS operands of the tensor-core products add the
# same order again; a reference of exact zeros must come back exactly zero.
GRAD_NORM_REL, GRAD_MAX_REL, GRAD_MEAN_REL = 1e-2, 2e-2, 5e-3

# Every output the tests allocate sits between two guard bands of this many
# bytes filled with GUARD_BYTE, and is filled with NaN before the call: after
# the call the bands must be intact (nothing written outside the tensor) and
# no NaN may remain (every element written).
GUARD_BYTES = 4096
GUARD_BYTE = 0xA5


class Guarded:
    """Outputs allocated inside larger buffers with guard bands (a stand-in
    for a memory checker: the kernels' stores must stay inside their tensors
    and cover every element)."""

    def __init__(self):
        self.items = []

    def empty(self, name: str, shape, dtype, device, output: bool = True) -> torch.Tensor:
        """A guarded tensor; an output (not a workspace) also starts as NaN
        and must be fully written."""
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        raw = torch.full((2 * GUARD_BYTES + n,), GUARD_BYTE, dtype=torch.uint8, device=device)
        view = raw[GUARD_BYTES:GUARD_BYTES + n].view(dtype).view(*shape)
        if output:
            view.fill_(float("nan"))
        self.items.append((name, raw, n, view if output else None))
        return view

    def like(self, name: str, t: torch.Tensor) -> torch.Tensor:
        return self.empty(name, tuple(t.shape), t.dtype, t.device)

    def check(self):
        if any(raw.is_cuda for _, raw, _, _ in self.items):
            torch.cuda.synchronize()
        for name, raw, n, view in self.items:
            head, tail = raw[:GUARD_BYTES], raw[GUARD_BYTES + n:]
            assert bool((head == GUARD_BYTE).all()), f"{name}: bytes written before the tensor"
            assert bool((tail == GUARD_BYTE).all()), f"{name}: bytes written past the end of the tensor"
            if view is not None:
                assert not bool(torch.isnan(view).any()), f"{name}: elements left unwritten"


def shape_of(w: Workload, layout=moda.MODA_DEPTH_FLAT, C=None):
    return moda.make_shape(w.B, w.Hq, w.Hk, w.T, w.d, w.L, w.C if C is None else C,
                           moda.MODA_BF16 if w.dtype == "bf16" else moda.MODA_FP32, layout,
                           flags=0 if w.causal else moda.MODA_FLAG_NONCAUSAL,
                           depth_window=w.window)


def run_gpu(w: Workload, x: Dict[str, torch.Tensor], backward=None, layout=moda.MODA_DEPTH_FLAT,
            C=None, null_depth_if_empty=True, ws_mode: int = 1):
    """Repack the depth cache, run the forward (and backward) on the current
    stream; returns a dict of device tensors.  Every output (and the
    backward's workspace) is guarded (``Guarded``) and checked before
    returning.  ws_mode: the backward's workspace, moda_workspace_size(shape,
    ws_mode) bytes (1: the fastest path, 2: the least it accepts)."""
    sh = shape_of(w, layout, C)
    dev = x["Q"].device
    dt = x["Q"].dtype
    gd = Guarded()
    out = {}
    layer = layout == moda.MODA_DEPTH_LAYER
    if w.L > 0 and layer:      # the layer-major cache, read in place
        Kd, Vd = x["Kd_layer"], x["Vd_layer"]
    elif w.L > 0:
        Kd = gd.empty("Kd", (w.B, w.Hk, w.T * w.L, w.d), dt, dev)
        Vd = gd.empty("Vd", (w.B, w.Hk, w.T * w.L, w.d), dt, dev)
        moda.moda_repack_depth(sh, x["Kd_layer"], Kd)
        moda.moda_repack_depth(sh, x["Vd_layer"], Vd)
    else:
        Kd = Vd = None if null_depth_if_empty else torch.empty(0, device=dev, dtype=dt)
    out["Kd"], out["Vd"] = Kd, Vd
    O = gd.like("O", x["Q"])
    LSE = gd.empty("LSE", (w.B, w.Hq, w.T), torch.float32, dev)
    moda.moda_fwd(sh, x["Q"], x["K"], x["V"], Kd, Vd, O, LSE)
    out["O"], out["LSE"] = O, LSE
    if backward if backward is not None else w.backward:
        nws = moda.moda_workspace_size(sh, ws_mode)
        ws = gd.empty("workspace", (max(nws, 16),), torch.uint8, dev, output=False)
        dQ = gd.like("dQ", x["Q"])
        dK = gd.like("dK", x["K"])
        dV = gd.like("dV", x["V"])
        dKd = gd.like("dKd", Kd) if Kd is not None and Kd.numel() else None
        dVd = gd.like("dVd", Vd) if Vd is not None and Vd.numel() else None
        moda.moda_bwd(sh, x["Q"], x["K"], x["V"], Kd, Vd, O, LSE, x["dO"], dQ, dK, dV, dKd, dVd,
                      ws, nws)
        out.update(dQ=dQ, dK=dK, dV=dV, dKd=dKd, dVd=dVd)
    gd.check()
    if layer and w.L > 0 and out.get("dKd") is not None:
        # depth gradients came back layer-major [L, B, Hk, T, d]: token-major
        # copies for the comparisons, the raw tensors beside them
        def tm(t):
            return t.permute(1, 2, 3, 0, 4).reshape(w.B, w.Hk, w.T * w.L, w.d).contiguous()
        out["dKd_layer"], out["dVd_layer"] = out["dKd"], out["dVd"]
        out["dKd"], out["dVd"] = tm(out["dKd"]), tm(out["dVd"])
    return out


def token_major(x: Dict[str, torch.Tensor], w: Workload) -> Tuple[torch.Tensor, torch.Tensor]:
    """CPU token-major depth tensors via the oracle's repack (bytewise)."""
    if w.L == 0:
        e = torch.zeros(w.B, w.Hk, 0, w.d)
        return e, e
    res = []
    for k in ("Kd_layer", "Vd_layer"):
        src = x[k].cpu()
        if src.dtype == torch.bfloat16:
            u = src.view(torch.int16).numpy()
            res.append(torch.from_numpy(oracle.repack(u, w.B, w.Hk, w.T, w.d, w.L)).view(torch.bfloat16))
        else:
            res.append(torch.from_numpy(oracle.repack(src.numpy(), w.B, w.Hk, w.T, w.d, w.L)))
    return res[0], res[1]


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().double().numpy()


def oracle_fwd_full(w, x):
    Kd, Vd = token_major(x, w)
    return oracle.fwd(f64(x["Q"]), f64(x["K"]), f64(x["V"]), f64(Kd) if w.L else None,
                      f64(Vd) if w.L else None, causal=w.causal, window=w.window)


def oracle_bwd_full(w, x):
    Kd, Vd = token_major(x, w)
    return oracle.bwd(f64(x["Q"]), f64(x["K"]), f64(x["V"]), f64(Kd), f64(Vd), f64(x["dO"]),
                      causal=w.causal, window=w.window)


def sample_rows(w: Workload, n_random: int, seed: int = 7) -> List[Tuple[int, int, int]]:
    """(b, h, t) rows: first/last token, tile and chunk boundaries, randoms."""
    rng = np.random.default_rng(seed)
    Tq = 128 // w.G
    ts = {0, 1, w.T - 1, w.T - 2, min(w.T - 1, Tq), max(0, Tq - 1), min(w.T - 1, 127),
          min(w.T - 1, 128), min(w.T - 1, w.C), max(0, w.C - 1)}
    ts = sorted(t for t in ts if 0 <= t < w.T)
    rows = [(int(rng.integers(w.B)), int(rng.integers(w.Hq)), t) for t in ts]
    for _ in range(n_random):
        rows.append((int(rng.integers(w.B)), int(rng.integers(w.Hq)), int(rng.integers(w.T))))
    rows.append((w.B - 1, w.Hq - 1, w.T - 1))
    return rows


def oracle_rows(w: Workload, x, Kd_dev, Vd_dev, rows: Sequence[Tuple[int, int, int]]):
    """Oracle O and LSE for sampled rows, each computed from its visible rows
    alone (sequence keys and depth rows taken straight from the inputs)."""
    O = np.zeros((len(rows), w.d))
    LSE = np.zeros(len(rows))
    for i, (b, h, t) in enumerate(rows):
        hk = h // w.G
        q = f64(x["Q"][b, h, t])
        n_seq = t + 1 if w.causal else w.T
        Ks = f64(x["K"][b, hk, :n_seq])
        Vs = f64(x["V"][b, hk, :n_seq])
        if w.L:
            # layer-major source: depth row l of token t is Kd_layer[l, b, hk, t];
            # a window keeps the last w.window layers
            l0 = w.L - w.window if w.window else 0
            Kdep = f64(x["Kd_layer"][l0:, b, hk, t])
            Vdep = f64(x["Vd_layer"][l0:, b, hk, t])
        else:
            Kdep = Vdep = np.zeros((0, w.d))
        O[i], LSE[i] = oracle.row(q, Ks, Vs, Kdep, Vdep)
    return O, LSE


def slice_workload(w: Workload, x, b: int, hk: int):
    """The independent (b, hk) slice as a B=1, Hk=1 problem (CPU tensors)."""
    G = w.G
    ws = w.with_(B=1, Hq=G, Hk=1)
    xs = {"Q": x["Q"][b:b + 1, hk * G:(hk + 1) * G].cpu(),
          "K": x["K"][b:b + 1, hk:hk + 1].cpu(), "V": x["V"][b:b + 1, hk:hk + 1].cpu(),
          "Kd_layer": x["Kd_layer"][:, b:b + 1, hk:hk + 1].cpu(),
          "Vd_layer": x["Vd_layer"][:, b:b + 1, hk:hk + 1].cpu()}
    if "dO" in x:
        xs["dO"] = x["dO"][b:b + 1, hk * G:(hk + 1) * G].cpu()
    return ws, xs


def err_stats(got, ref) -> Tuple[float, float]:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if got.size == 0:
        return 0.0, 0.0
    d = np.abs(got - ref)
    return float(d.max()), float(d.mean())


def assert_out_close(got, ref, dtype: str, what: str):
    mx, mean = err_stats(got, ref)
    assert np.all(np.isfinite(np.asarray(got, dtype=np.float64))), f"{what}: non-finite values"
    if dtype == "fp32":
        assert mx <= FP32_MAX_ABS, f"{what}: max-abs {mx:.3e} > {FP32_MAX_ABS}"
    else:
        assert mx <= BF16_MAX_ABS and mean <= BF16_MEAN_ABS, \
            f"{what}: max-abs {mx:.3e} (<= {BF16_MAX_ABS}), mean-abs {mean:.3e} (<= {BF16_MEAN_ABS})"


def grad_errors(got, ref) -> Dict[str, float]:
    """Normwise, max and mean errors of a gradient and the reference scales."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = np.abs(got - ref)
    return {"norm_err": float(np.sqrt((d * d).sum())), "norm_ref": float(np.sqrt((ref * ref).sum())),
            "max_err": float(d.max()), "max_ref": float(np.abs(ref).max()),
            "mean_err": float(d.mean()), "mean_ref": float(np.abs(ref).mean())}


def assert_grad_close(got, ref, what: str):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, f"{what}: shape {got.shape} != {ref.shape}"
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    if ref.size == 0:
        return
    e = grad_errors(got, ref)
    if e["norm_ref"] == 0.0:
        assert e["max_err"] == 0.0, f"{what}: reference is exactly zero, max-abs {e['max_err']:.3e}"
        return
    ok = (e["norm_err"] <= GRAD_NORM_REL * e["norm_ref"] and e["max_err"] <= GRAD_MAX_REL * e["max_ref"]
          and e["mean_err"] <= GRAD_MEAN_REL * e["mean_ref"])
    assert ok, (f"{what}: normwise {e['norm_err'] / e['norm_ref']:.3e} (<= {GRAD_NORM_REL}), "
                f"max-abs {e['max_err']:.3e} (<= {GRAD_MAX_REL * e['max_ref']:.3e}), "
                f"mean-abs {e['mean_err']:.3e} (<= {GRAD_MEAN_REL * e['mean_ref']:.3e})")
