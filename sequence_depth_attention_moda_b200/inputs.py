"""Seeded synthetic inputs shaped like the MoDA kernel workloads.

This module holds the workload table and the random draws only; it contains
none of the operator's arithmetic, so both the CUDA path and the CPU oracle can
be fed from it.  Every tensor is drawn in a fixed order from one
``torch.Generator`` seeded per workload, as fp32 normals (optionally scaled by
1/sqrt(d)), then rounded once to the workload's storage dtype.

Shapes follow the tensor layouts of the "moda-attention 0.1.0" PyPI page
("Using the Kernel Directly"): Q [B,Hq,T,d], K,V [B,Hk,T,d].  The depth cache
is drawn in its natural layer-major form [L,B,Hk,T,d] (paper summary,
"Hardware-Efficient Implementation"); the token-major [B,Hk,T*L,d] tensors the
kernels read are produced from it by the depth repack.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hk: int
    d: int
    T: int
    L: int
    C: int
    dtype: str = "bf16"          # storage / input dtype: "bf16" or "fp32"
    qk_scaled: bool = False      # Q and K drawn as N(0,1)/sqrt(d)
    backward: bool = False       # the workload includes the backward pass
    seed: int = 1000
    causal: bool = True          # False: every row sees all T sequence keys
    window: int = 0              # > 0: each token's last `window` depth rows only

    @property
    def G(self) -> int:
        return self.Hq // self.Hk

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def fwd_flops(self) -> float:
        """Algorithmic forward FLOPs: 4*B*Hq*d*(T(T+1)/2 + T*L)."""
        return 4.0 * self.B * self.Hq * self.d * (self.T * (self.T + 1) / 2 + self.T * self.L)


# The five kernel workloads (seed = 1000 + index; sweep points add 100*k).
TINY_FP32 = Workload("tiny_fp32", B=1, Hq=4, Hk=2, d=64, T=32, L=8, C=16,
                     dtype="fp32", seed=1001)
LAYER_1P5B = Workload("layer_1p5b_T4k", B=2, Hq=16, Hk=4, d=128, T=4096, L=16, C=64,
                      qk_scaled=True, backward=True, seed=1002)
LONG_64K = Workload("long_context_T64k", B=1, Hq=16, Hk=4, d=128, T=65536, L=32, C=64,
                    seed=1003)
TRAIN_FWD_BWD = Workload("train_T4k_L48", B=8, Hq=32, Hk=8, d=128, T=4096, L=48, C=64,
                         backward=True, seed=1005)

# Decoding: one new token per sequence over T cached keys (its L depth rows).
DECODE_T32K = Workload("decode_T32k_L48", B=8, Hq=32, Hk=8, d=128, T=32768, L=48, C=64, seed=1006)

WORKLOADS: Dict[str, Workload] = {w.name: w for w in (TINY_FP32, LAYER_1P5B, LONG_64K, TRAIN_FWD_BWD,
                                                      DECODE_T32K)}


def depth_group_sweep() -> List[Workload]:
    """Depth/group sweep at T=8192, Hk=4, d=128: G x L x C grid."""
    out = []
    k = 0
    for G in (1, 2, 4, 8):
        for L in (1, 8, 32, 64):
            for C in (32, 64, 128):
                out.append(Workload(f"sweep_G{G}_L{L}_C{C}", B=1, Hq=4 * G, Hk=4, d=128,
                                    T=8192, L=L, C=C, seed=1004 + 100 * k))
                k += 1
    return out


def make_inputs(w: Workload, device="cpu", seed: Optional[int] = None,
                grad_out: Optional[bool] = None) -> Dict[str, torch.Tensor]:
    """Draw one batch of inputs for workload ``w``.

    Returns a dict with Q, K, V, Kd_layer, Vd_layer (layer-major depth cache,
    [L,B,Hk,T,d]) and, when the workload has a backward pass (or grad_out is
    True), dO.  Tensors are contiguous, on ``device``, in ``w``'s dtype.
    """
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed if seed is None else seed)
    dt = w.torch_dtype()
    inv = 1.0 / (w.d ** 0.5)

    def draw(shape, scaled=False):
        x = torch.randn(shape, generator=g, device=dev, dtype=torch.float32)
        if scaled:
            x.mul_(inv)
        return x.to(dt).contiguous()

    out = {
        "Q": draw((w.B, w.Hq, w.T, w.d), w.qk_scaled),
        "K": draw((w.B, w.Hk, w.T, w.d), w.qk_scaled),
        "V": draw((w.B, w.Hk, w.T, w.d)),
        "Kd_layer": draw((w.L, w.B, w.Hk, w.T, w.d), w.qk_scaled),
        "Vd_layer": draw((w.L, w.B, w.Hk, w.T, w.d)),
    }
    if w.backward if grad_out is None else grad_out:
        out["dO"] = draw((w.B, w.Hq, w.T, w.d))
    return out


def make_decode_inputs(w: Workload, device="cpu", seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Decoding inputs for workload ``w``: q [B,Hq,d] (the new token's
    queries), K, V [B,Hk,T,d] (the cache, the new token's own key last) and
    Kd, Vd [B,Hk,L,d] (the new token's depth rows), drawn in that order like
    make_inputs."""
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed if seed is None else seed)
    dt = w.torch_dtype()
    inv = 1.0 / (w.d ** 0.5)

    def draw(shape, scaled=False):
        x = torch.randn(shape, generator=g, device=dev, dtype=torch.float32)
        if scaled:
            x.mul_(inv)
        return x.to(dt).contiguous()

    return {
        "q": draw((w.B, w.Hq, w.d), w.qk_scaled),
        "K": draw((w.B, w.Hk, w.T, w.d), w.qk_scaled),
        "V": draw((w.B, w.Hk, w.T, w.d)),
        "Kd": draw((w.B, w.Hk, w.L, w.d), w.qk_scaled),
        "Vd": draw((w.B, w.Hk, w.L, w.d)),
    }
