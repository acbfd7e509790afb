"""Seeded synthetic inputs for RACE attention workloads.

This module only draws random numbers; it holds none of the method's arithmetic.
Both the CUDA path and the CPU oracle receive exactly the tensors produced here.

Every tensor of every head comes from its own torch.Generator, seeded from
(seed, tensor id, head), so any head can be regenerated alone.  Values are drawn
in float64 and rounded once (round-to-nearest-even) to the workload dtype.
Streams on the CPU and on a CUDA device differ; a test that compares devices
generates on one device and copies.

Workloads (sizes of the published configurations of the method's evaluation,
drawn synthetically; the pages name no dataset for these scale tests):
  * iid:       q, k, v ~ N(0, 1)
  * clustered: m unit centroid directions per head shared by q and k; each token
               independently picks a centroid uniformly (separate draws for q and
               k) and adds N(0, sigma^2 I) noise; v ~ N(0, 1)
  * W ~ N(0, 1) of shape [L, d, P], float32; dO ~ N(0, 1) for backward workloads.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional, Sequence

import torch

T_Q, T_K, T_V, T_DO, T_W, T_CENTROID, T_ASSIGN_Q, T_ASSIGN_K = range(8)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    H: int                 # batch * heads (W is shared by all of them)
    N: int
    d: int
    L: int
    P: int
    tau: float
    causal: bool
    dtype: str             # "bf16" or "fp32"
    chunk: int = 0         # 0 = library default
    clusters: int = 0      # 0 = iid q/k
    sigma: float = 0.3
    backward: bool = False
    seed: int = 1
    batch: int = 1

    @property
    def R(self) -> int:
        return 1 << self.P

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {w.name: w for w in [
    Workload("noncausal_fp32_h1_n1024_d64_L4_P4", H=1, N=1024, d=64, L=4, P=4,
             tau=0.5, causal=False, dtype="fp32", seed=1),
    Workload("causal_bf16_h8_n16384_d64_L8_P6_clustered32", H=8, N=16384, d=64, L=8,
             P=6, tau=0.5, causal=True, dtype="bf16", chunk=128, clusters=32, seed=2),
    Workload("noncausal_bf16_b2h16_n262144_d64_L16_P6", H=32, N=262144, d=64, L=16,
             P=6, tau=0.5, causal=False, dtype="bf16", seed=3, batch=2),
    Workload("causal_bf16_h8_n4194304_d64_L16_P8_clustered256", H=8, N=4194304, d=64,
             L=16, P=8, tau=0.25, causal=True, dtype="bf16", chunk=256, clusters=256,
             seed=4),
    Workload("causal_fwdbwd_bf16_h4_n12582912_d64_L8_P6", H=4, N=12582912, d=64, L=8,
             P=6, tau=0.5, causal=True, dtype="bf16", chunk=256, backward=True, seed=5),
]}

SMALL = "noncausal_fp32_h1_n1024_d64_L4_P4"
HEADLINE = "causal_bf16_h8_n4194304_d64_L16_P8_clustered256"


def _gen(seed: int, tensor: int, head: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + tensor * 10_007 + head * 101 + 17) % (2 ** 63))
    return g


def _normal(shape, g, device, dtype):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float64).to(dtype)


def make_W(wl: Workload, device="cpu") -> torch.Tensor:
    g = _gen(wl.seed, T_W, 0, device)
    return _normal((wl.L, wl.d, wl.P), g, device, torch.float32)


def make_head(wl: Workload, head: int, device="cpu", N: Optional[int] = None,
              with_dout: Optional[bool] = None) -> Dict[str, torch.Tensor]:
    """q, k, v (and dO) of one head, each [N, d] in the workload dtype."""
    N = wl.N if N is None else N
    dt = wl.torch_dtype
    out = {}
    if wl.clusters:
        gc = _gen(wl.seed, T_CENTROID, head, device)
        cen = torch.randn((wl.clusters, wl.d), generator=gc, device=device,
                          dtype=torch.float64)
        cen = cen / cen.norm(dim=1, keepdim=True)
        for name, t_x, t_a in (("q", T_Q, T_ASSIGN_Q), ("k", T_K, T_ASSIGN_K)):
            ga = _gen(wl.seed, t_a, head, device)
            a = torch.randint(0, wl.clusters, (N,), generator=ga, device=device)
            gx = _gen(wl.seed, t_x, head, device)
            eps = torch.randn((N, wl.d), generator=gx, device=device, dtype=torch.float64)
            out[name] = (cen[a] + wl.sigma * eps).to(dt)
            del eps, a
    else:
        out["q"] = _normal((N, wl.d), _gen(wl.seed, T_Q, head, device), device, dt)
        out["k"] = _normal((N, wl.d), _gen(wl.seed, T_K, head, device), device, dt)
    out["v"] = _normal((N, wl.d), _gen(wl.seed, T_V, head, device), device, dt)
    if wl.backward if with_dout is None else with_dout:
        out["dout"] = _normal((N, wl.d), _gen(wl.seed, T_DO, head, device), device, dt)
    return out


def make_inputs(wl: Workload, device="cpu", N: Optional[int] = None,
                heads: Optional[Sequence[int]] = None,
                with_dout: Optional[bool] = None) -> Dict[str, torch.Tensor]:
    """All heads stacked: q, k, v (and dout) are [H, N, d]; W is [L, d, P] float32."""
    heads = range(wl.H) if heads is None else heads
    N = wl.N if N is None else N
    want_do = wl.backward if with_dout is None else with_dout
    names = ["q", "k", "v"] + (["dout"] if want_do else [])
    res = {n: torch.empty((len(heads), N, wl.d), dtype=wl.torch_dtype, device=device)
           for n in names}
    for i, h in enumerate(heads):
        one = make_head(wl, h, device, N, want_do)
        for n in names:
            res[n][i].copy_(one[n])
        del one
    res["W"] = make_W(wl, device)
    return res
