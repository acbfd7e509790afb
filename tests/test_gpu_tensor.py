"""GPU parity of the tensor-core (tcgen05) path against the float64 oracle.

bf16 q, k, v (the oracle reads the same bf16 values, upcast), float32 W; outputs
compared in float32 (out_dtype = fp32) with max|diff| <= 2e-3 * max|V|, the bf16
criterion of the method's evaluation.  Shapes cover one and several row groups,
one and several segments (multi-segment causal sweeps start from scanned segment
sums), ragged tails and the 128-token chunk edges.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_lsh_sketch_race_b200 import inputs as I
from linear_lsh_sketch_race_b200 import race_attn as ra

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 2e-3


def _np(t):
    return t.detach().to(torch.float64).cpu().numpy()


def _run(N, H, L, P, tau, causal, clusters=0, seed=1, sigma=0.3):
    wl = I.Workload("t", H=H, N=N, d=64, L=L, P=P, tau=tau, causal=causal, dtype="bf16",
                    clusters=clusters, seed=seed, sigma=sigma)
    x = I.make_inputs(wl, "cpu")
    g = {k: v.to(DEV) for k, v in x.items()}
    out, den = ra.forward(g["q"], g["k"], g["v"], g["W"], tau, causal,
                          out_dtype=torch.float32, impl="tensor", return_den=True)
    torch.cuda.synchronize()
    assert ra.race_device_status() == 0
    ref, rden = oracle.forward_heads(_np(x["q"]), _np(x["k"]), _np(x["v"]), _np(x["W"]),
                                     tau, causal)
    vmax = np.abs(_np(x["v"])).max()
    err = np.abs(_np(out) - ref).max() / vmax
    derr = np.abs(_np(den) - rden).max() / np.abs(rden).max()
    return err, derr


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("N", [1, 100, 128, 129, 1000])
def test_tensor_small(causal, N):
    err, derr = _run(N, H=2, L=2, P=6, tau=0.5, causal=causal, seed=N)
    assert err <= TOL, err
    assert derr <= 1e-2, derr


@pytest.mark.parametrize("L,P,tau", [(1, 7, 0.5), (4, 6, 0.5), (2, 8, 0.25), (3, 8, 0.25),
                                     (5, 7, 0.4)])
@pytest.mark.parametrize("causal", [True, False])
def test_tensor_table_shapes(L, P, tau, causal):
    err, _ = _run(700, H=3, L=L, P=P, tau=tau, causal=causal, clusters=16, seed=L * 10 + P)
    assert err <= TOL, err


def test_tensor_multi_segment_causal():
    # few heads and row groups: the plan splits the sequence into segments
    err, _ = _run(5000, H=1, L=2, P=6, tau=0.5, causal=True, seed=3)
    assert err <= TOL, err


def test_tensor_sharp_clusters():
    err, _ = _run(1500, H=2, L=2, P=8, tau=0.25, causal=True, clusters=4, sigma=0.3 / 8,
                  seed=5)
    assert err <= TOL, err


def test_tensor_matches_simt_path():
    wl = I.Workload("t", H=2, N=3000, d=64, L=4, P=6, tau=0.5, causal=True, dtype="bf16",
                    seed=8)
    x = {k: v.to(DEV) for k, v in I.make_inputs(wl, "cpu").items()}
    a = ra.forward(x["q"], x["k"], x["v"], x["W"], wl.tau, True, out_dtype=torch.float32,
                   impl="tensor")
    b = ra.forward(x["q"], x["k"], x["v"], x["W"], wl.tau, True, out_dtype=torch.float32,
                   impl="simt")
    vmax = x["v"].float().abs().max().item()
    assert (a - b).abs().max().item() / vmax <= TOL


@pytest.mark.parametrize("name", ["causal_bf16_h8_n16384_d64_L8_P6_clustered32"])
def test_tensor_full_config_causal_16k(name):
    wl = I.WORKLOADS[name]
    x = I.make_inputs(wl, "cpu")
    g = {k: v.to(DEV) for k, v in x.items()}
    out = ra.forward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out_dtype=torch.float32)
    ref, _ = oracle.forward_heads(_np(x["q"]), _np(x["k"]), _np(x["v"]), _np(x["W"]),
                                  wl.tau, True)
    vmax = np.abs(_np(x["v"])).max()
    assert np.abs(_np(out) - ref).max() / vmax <= TOL
