"""Full-size backward: the published forward+backward workload and the long-context
workload, in the launch configuration the benchmark times.

The float64 oracle cannot run a 12M-token backward, so these cases check what can be
computed exactly at any size:

  * causal rows: dq_i depends only on keys and values j <= i and on row i's own
    upstream gradient and output, so the oracle backward over the first R0 tokens
    gives the exact dq of those rows;
  * sum over keys of dv_j equals the sum over queries of dO_i (each row's attention
    weights, divided by its denominator, sum to one);
  * dq_i . q_i = 0 and dk_j . k_j = 0 (the output depends on q and k only through
    q / |q| and k / |k|);
  * every gradient is finite.

Tolerances: the backward receives the GPU forward's bf16 output (the oracle uses its own),
so prefix rows are held to 2 * TOL_BWD relative to max|dq_ref| (see
test_gpu_tensor_backward.py for the derivation of TOL_BWD = 1e-2).  The sum and
orthogonality identities are exact in real arithmetic; with bf16 gradients each entry
carries a relative rounding of at most 2^-9, so they are checked to 1e-2 of the norms
involved.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_lsh_sketch_race_b200 import inputs as I
from linear_lsh_sketch_race_b200 import race_attn as ra

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_BWD = 1e-2
R0 = 1024


def _run(name, heads_checked):
    wl = I.WORKLOADS[name]
    x = I.make_inputs(wl, DEV, with_dout=True)
    q, k, v, W, g = x["q"], x["k"], x["v"], x["W"], x["dout"]
    out, den = ra.forward(q, k, v, W, wl.tau, True, return_den=True)     # bf16, as benchmarked
    dq, dk, dv, dW = ra.backward(q, k, v, W, wl.tau, True, out, g, den=den)
    torch.cuda.synchronize()
    assert ra.race_device_status() == 0
    assert torch.isfinite(dW).all()
    for h in range(wl.H):   # one head at a time: float copies of a 12M-token head are 3 GB
        for t in (dq[h], dk[h], dv[h]):
            assert torch.isfinite(t).all(), h
        # sum_j dv_j = sum_i dO_i, per column
        dvh, gh = dv[h].float(), g[h].float()
        sdv, sdo = dvh.sum(dim=0), gh.sum(dim=0)
        scale = dvh.norm(dim=0) + gh.norm(dim=0)
        assert ((sdv - sdo).abs() <= 1e-2 * scale).all(), (h, ((sdv - sdo).abs() / scale).max().item())
        del dvh, gh
        # gradients orthogonal to their inputs, row by row
        for gx, xx in ((dq[h], q[h]), (dk[h], k[h])):
            gf, xf = gx.float(), xx.float()
            dot = (gf * xf).sum(dim=-1).abs()
            lim = 1e-2 * gf.norm(dim=-1) * xf.norm(dim=-1) + 1e-30
            assert (dot <= lim).all(), (h, (dot / lim).max().item())
            del gf, xf, dot, lim

    # exact dq on the first R0 rows from the oracle over the prefix
    Wn = W.double().cpu().numpy()
    for h in heads_checked:
        f = lambda t: t[h, :R0].double().cpu().numpy()  # noqa: E731
        dq_ref, _, _, _ = oracle.backward(f(q), f(k), f(v), Wn, wl.tau, True, f(g))
        err = np.abs(f(dq) - dq_ref).max() / np.abs(dq_ref).max()
        assert err <= 2 * TOL_BWD, (h, err)


@pytest.fixture(autouse=True)
def _free_memory():
    yield
    torch.cuda.empty_cache()


def test_fwdbwd_12m_tokens_4_heads():
    _run("causal_fwdbwd_bf16_h4_n12582912_d64_L8_P6", heads_checked=(0, 3))


def test_fwdbwd_4m_tokens_8_heads_long_context_shape():
    _run("causal_bf16_h8_n4194304_d64_L16_P8_clustered256", heads_checked=(0, 7))
