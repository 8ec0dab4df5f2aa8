"""Seeded synthetic inputs for the MoE layer workloads.

This module only draws random numbers and lays them out. It holds none of the
layer's arithmetic: no routing, no capacity, no expert math. Both the CUDA
path's tests/bench and the CPU oracle's tests take their inputs from here.

Workloads (the shapes the pages' discussion turns on, made concrete):

* ``tiny``            N=64,    d=128,  f=256,   E=8,   K=2, W=4, dropless
* ``mixtral_prefill`` N=4096,  d=4096, f=14336, E=8,   K=2, W=8, dropless,
                      uniform router init
* ``e128_skew``       N=8192,  d=2048, f=768,   E=128, K=8, W=8, cf=1.25,
                      Zipf(s=1.1) per-expert router bias
* ``decode``          N=16,    d=7168, f=2048,  E=256, K=8, W=8, dropless
* ``stack4``          N=32768, d=4096, f=1536,  E=64,  K=6, W=8, L=4 layers,
                      cf in {1.0, 1.25, 2.0} x Zipf s in {0, 1.2}
* ``residual_top1``   N=4096,  d=4096, f=14336, E=8,   K=1, W=8, dropless, plus a
                      shared dense SwiGLU MLP of width 14336 (Residual-MoE)

Recipe (one ``torch.Generator`` per call, ``manual_seed(seed)``; draw order
x, router, W1, W3, W2; layer ``l`` of a stack re-seeds with ``seed + 1000*l``
and skips x):

* hidden states x ~ N(0, 1), rounded to bf16 (round-to-nearest-even);
* router weight Wr [E][d] fp32 ~ N(0, 1/d) (std 1/sqrt(d)), or, for the
  ``uniform`` init, U(-1/sqrt(d), 1/sqrt(d));
* expert weights W1, W3 [E][f][d] and W2 [E][d][f] ~ N(0, 0.02^2) (std 0.02),
  rounded to bf16;
* Zipf(s) bias: bias[e] = -s * ln(e + 1), computed in float64, stored fp32
  (expert 0 hottest); s = 0 means no bias (None);
* ``stack4_affinity`` replaces each layer's router by one that leans on the
  previous layer's with its experts permuted (``affine_router``), so that the
  inter-layer expert affinity a trained model shows is present.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    N: int
    d: int
    f: int
    E: int
    K: int
    W: int
    cf: float = 0.0          # <= 0 means dropless
    s: float = 0.0           # Zipf exponent of the per-expert bias; 0 = none
    router: str = "normal"   # "normal" (N(0,1/d)) or "uniform" (U(+-1/sqrt d))
    layers: int = 1
    shared_f: int = 0        # width of the shared dense MLP (Residual-MoE); 0 = none
    slot_major: bool = False  # drop priority: first choices before second choices
    reroute: bool = False     # move overflowed assignments to the next-best non-full expert
    fp8: bool = False         # e4m3 dispatch payload and gate/up GEMM
    affinity: float = 0.0     # stacks: correlation of a layer's router with the previous one's
    fp8_return: bool = False  # FP8 path: expert outputs travel back as e4m3 + block exponents
    y_f16: bool = False       # expert outputs travel back as fp16 codes + block exponents

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", N=64, d=128, f=256, E=8, K=2, W=4),
    "mixtral_prefill": Workload("mixtral_prefill", N=4096, d=4096, f=14336, E=8, K=2, W=8,
                                router="uniform"),
    "e128_skew": Workload("e128_skew", N=8192, d=2048, f=768, E=128, K=8, W=8, cf=1.25, s=1.1),
    "decode": Workload("decode", N=16, d=7168, f=2048, E=256, K=8, W=8),
    "stack4": Workload("stack4", N=32768, d=4096, f=1536, E=64, K=6, W=8, cf=1.25, s=0.0,
                       layers=4),
    # Residual-MoE: top-1 routed experts plus a shared dense MLP of the same width
    "residual_top1": Workload("residual_top1", N=4096, d=4096, f=14336, E=8, K=1, W=8,
                              router="uniform", shared_f=14336),
    # the 128-expert skewed layer with slot-major drop priority (first choices first)
    "e128_skew_slot_major": Workload("e128_skew_slot_major", N=8192, d=2048, f=768, E=128, K=8,
                                     W=8, cf=1.25, s=1.1, slot_major=True),
    # the same with overflowed assignments re-routed to the next-best non-full expert
    "e128_skew_reroute": Workload("e128_skew_reroute", N=8192, d=2048, f=768, E=128, K=8, W=8,
                                  cf=1.25, s=1.1, reroute=True),
    # the FP8 payload (e4m3 rows, e4m3 gate/up GEMM) on the Mixtral-shaped and 128-expert layers
    "mixtral_prefill_fp8": Workload("mixtral_prefill_fp8", N=4096, d=4096, f=14336, E=8, K=2,
                                    W=8, router="uniform", fp8=True),
    "e128_skew_fp8": Workload("e128_skew_fp8", N=8192, d=2048, f=768, E=128, K=8, W=8, cf=1.25,
                              s=1.1, fp8=True),
    # the FP8 path with the FP8 return payload as well (expert outputs as e4m3 codes with one
    # power-of-two exponent per 32 columns)
    "mixtral_prefill_fp8_return": Workload("mixtral_prefill_fp8_return", N=4096, d=4096, f=14336,
                                           E=8, K=2, W=8, router="uniform", fp8=True,
                                           fp8_return=True),
    "e128_skew_fp8_return": Workload("e128_skew_fp8_return", N=8192, d=2048, f=768, E=128, K=8,
                                     W=8, cf=1.25, s=1.1, fp8=True, fp8_return=True),
    # the weight-bound decode layer and the 4-layer stack on the FP8 path
    "decode_fp8": Workload("decode_fp8", N=16, d=7168, f=2048, E=256, K=8, W=8, fp8=True),
    # the stack with inter-layer expert affinity planted in the routers (rho = 0.9): the routing
    # structure a trained model shows, for the placement report
    "stack4_affinity": Workload("stack4_affinity", N=32768, d=4096, f=1536, E=64, K=6, W=8,
                                cf=1.25, layers=4, affinity=0.9),
    "stack4_fp8": Workload("stack4_fp8", N=32768, d=4096, f=1536, E=64, K=6, W=8, cf=1.25,
                           layers=4, fp8=True),
    # the Mixtral-shaped layer with half the experts and tokens (same rows per expert,
    # same GEMM tiles): a smaller case of the same kernels, for hardware-counter captures
    "mixtral_prefill_half": Workload("mixtral_prefill_half", N=2048, d=4096, f=14336, E=4, K=2,
                                     W=4, router="uniform"),
    "mixtral_prefill_half_fp8": Workload("mixtral_prefill_half_fp8", N=2048, d=4096, f=14336,
                                         E=4, K=2, W=4, router="uniform", fp8=True),
}

STACK_GRID_CF = (1.0, 1.25, 2.0)
STACK_GRID_S = (0.0, 1.2)


def zipf_bias(E: int, s: float) -> Optional[torch.Tensor]:
    """bias[e] = -s*ln(e+1) (float64, stored fp32); None when s == 0."""
    if s == 0.0:
        return None
    return torch.tensor([-s * math.log(e + 1.0) for e in range(E)], dtype=torch.float64).to(
        torch.float32)


def affine_router(w: Workload, seed: int, layer: int, device: str = "cpu") -> torch.Tensor:
    """Router [E][d] fp32 of layer ``layer`` of a stack with planted inter-layer affinity
    (``w.affinity`` = rho > 0): R_0 = Z_0 and R_l = rho * R_{l-1}[pi_l] + sqrt(1 - rho^2) * Z_l,
    where Z_l ~ N(0, 1/d) and pi_l is a permutation of the experts, both drawn from a generator
    seeded ``seed + 1000*l + 7``. Row e of layer l leans on row pi_l[e] of layer l-1, so tokens
    that chose expert pi_l[e] tend to choose expert e next (the residual stream changes little
    from one layer to the next). Every entry keeps variance 1/d."""
    rho = w.affinity
    r = None
    for j in range(layer + 1):
        g = torch.Generator(device=device)
        g.manual_seed(seed + 1000 * j + 7)
        z = torch.randn(w.E, w.d, generator=g, device=device,
                        dtype=torch.float32) * (1.0 / math.sqrt(w.d))
        if j == 0:
            r = z
        else:
            perm = torch.randperm(w.E, generator=g, device=device)
            r = rho * r[perm] + math.sqrt(1.0 - rho * rho) * z
    return r


def make_layer_inputs(w: Workload, seed: int = 0, device: str = "cpu", layer: int = 0,
                      with_x: bool = True) -> dict:
    """Draw one layer's inputs. Returns a dict of tensors on ``device``.

    Keys: x (bf16 [N][d], only when ``with_x``), w_router (fp32 [E][d]),
    bias (fp32 [E] or None), w1, w3 (bf16 [E][f][d]), w2 (bf16 [E][d][f]).
    """
    g = torch.Generator(device=device)
    g.manual_seed(seed + 1000 * layer)
    out = {}
    if with_x:
        out["x"] = torch.randn(w.N, w.d, generator=g, device=device,
                               dtype=torch.float32).to(torch.bfloat16)
    if w.router == "uniform":
        bound = 1.0 / math.sqrt(w.d)
        wr = torch.rand(w.E, w.d, generator=g, device=device, dtype=torch.float32)
        out["w_router"] = (wr * 2.0 - 1.0) * bound
    else:
        out["w_router"] = torch.randn(w.E, w.d, generator=g, device=device,
                                      dtype=torch.float32) * (1.0 / math.sqrt(w.d))
    if w.affinity > 0.0:  # drawn above to keep the draw order; replaced by the planted router
        out["w_router"] = affine_router(w, seed, layer, device)
    b = zipf_bias(w.E, w.s)
    out["bias"] = None if b is None else b.to(device)
    for name, shape in (("w1", (w.E, w.f, w.d)), ("w3", (w.E, w.f, w.d)), ("w2", (w.E, w.d, w.f))):
        t = torch.empty(shape, device=device, dtype=torch.bfloat16)
        # draw expert by expert to bound the fp32 temporary
        for e in range(w.E):
            t[e] = (torch.randn(shape[1:], generator=g, device=device, dtype=torch.float32)
                    * 0.02).to(torch.bfloat16)
        out[name] = t
    return out


def make_shared_inputs(w: Workload, seed: int = 0, device: str = "cpu", layer: int = 0) -> dict:
    """Weights of the shared dense MLP (drawn after the layer's own inputs, from seed + 500):
    ws1, ws3 [f_s][d], ws2 [d][f_s], bf16 ~ N(0, 0.02^2)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed + 500 + 1000 * layer)
    out = {}
    for name, shape in (("ws1", (w.shared_f, w.d)), ("ws3", (w.shared_f, w.d)),
                        ("ws2", (w.d, w.shared_f))):
        out[name] = (torch.randn(shape, generator=g, device=device, dtype=torch.float32)
                     * 0.02).to(torch.bfloat16)
    return out


def random_small_workload(rng: "torch.Generator", max_n: int = 16, max_e: int = 8) -> Workload:
    """A random tiny shape for brute-force checks (N<=max_n, E<=max_e)."""
    def ri(lo, hi):
        return int(torch.randint(lo, hi + 1, (1,), generator=rng).item())
    E = ri(1, max_e)
    K = ri(1, E)
    W = [w for w in range(1, E + 1) if E % w == 0][ri(0, len([w for w in range(1, E + 1) if E % w == 0]) - 1)]
    n_per = ri(1, max(1, max_n // W))
    N = n_per * W
    cf = [0.0, 0.5, 1.0, 1.25, 2.0][ri(0, 4)]
    s = [0.0, 1.1][ri(0, 1)]
    return Workload("rand", N=N, d=8 * ri(1, 4), f=8 * ri(1, 4), E=E, K=K, W=W, cf=cf, s=s)
