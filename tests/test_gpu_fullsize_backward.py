"""Backward of the published workloads against the float64 oracle.

* The causal 16K-token workload (8 heads, L = 8, P = 6): every gradient in full.
* The forward+backward workload's kernels (4 heads, L = 8, P = 6, tau = 0.5, iid inputs)
  at N = 262,144, where the plan cuts each (head, row group) into the same 18 segments as
  at N = 12,582,912: every gradient in full.
* The 12M-token forward+backward workload and the 4M-token long-context workload at full
  size, in the benchmark's launch configuration (float32 outputs and gradients, so that
  the comparison sees the kernels' own error): the exact dq of the first rows from the
  oracle over the prefix (causal: dq_i depends only on tokens j <= i), and identities
  that hold exactly at any size:
    - sum over keys of dv_j equals the sum over queries of dO_i (each row's weights,
      divided by its denominator, sum to one);
    - dq_i . q_i = 0 and dk_j . k_j = 0 (the output depends on q and k only through
      q / |q| and k / |k|; the normalisation Jacobian is applied last, in float32);
    - every gradient is finite.

Tolerance: 3 * 2^-8 of max|dG_ref| per gradient tensor, the bound derived in
test_gpu_tensor_backward.py from the bf16 operands of the tensor cores; the backward
receives the oracle's output o where the oracle has it, the GPU forward's float32 output
otherwise.  The sum identity is held to the same relative bound against the sums of
absolute values (each dv_j carries at most that relative error, and the errors of
neighbouring keys, which read the same rounded state, need not cancel).  GPU tensors are
released before any assertion, so that a failing case cannot hold device memory.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_lsh_sketch_race_b200 import inputs as I
from linear_lsh_sketch_race_b200 import race_attn as ra

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_BWD = 3 * 2.0 ** -8
R0 = 1024


@pytest.fixture(autouse=True)
def _free_memory():
    yield
    torch.cuda.empty_cache()


def _f32(t):
    return t.float().cpu().numpy()


def _errors(got, refs):
    return {name: float(np.abs(g.double().cpu().numpy() - r).max() / np.abs(r).max())
            for name, g, r in zip(("dq", "dk", "dv", "dW"), got, refs)}


def _oracle_backward_per_head(pool, wl, x):
    """oracle.backward of every head on the host cores in parallel; dW summed."""
    W = x["W"].double().cpu().numpy()
    tasks = [(_f32(x["q"][h]), _f32(x["k"][h]), _f32(x["v"][h]), W, wl.tau, wl.causal,
              _f32(x["dout"][h])) for h in range(wl.H)]
    res = pool.starmap(oracle.backward, tasks, chunksize=1)
    return (np.stack([r[0] for r in res]), np.stack([r[1] for r in res]),
            np.stack([r[2] for r in res]), np.sum([r[3] for r in res], axis=0))


def _oracle_out_per_head(pool, wl, x):
    W = x["W"].double().cpu().numpy()
    tasks = [(_f32(x["q"][h]), _f32(x["k"][h]), _f32(x["v"][h]), W, wl.tau, wl.causal)
             for h in range(wl.H)]
    return np.stack([r[0] for r in pool.starmap(oracle.forward, tasks, chunksize=1)])


def _full_compare(pool, wl):
    x = I.make_inputs(wl, "cpu", with_dout=True)
    g = {k: v.to(DEV) for k, v in x.items()}
    out = torch.from_numpy(_oracle_out_per_head(pool, wl, x)).float().to(DEV)
    grads = ra.backward(g["q"], g["k"], g["v"], g["W"], wl.tau, wl.causal, out, g["dout"],
                        grad_dtype=torch.float32)
    torch.cuda.synchronize()
    status = ra.race_device_status()
    grads = [t.cpu() for t in grads]
    del g, out
    assert status == 0
    errs = _errors(grads, _oracle_backward_per_head(pool, wl, x))
    assert max(errs.values()) <= TOL_BWD, errs


def test_causal_16k_backward_in_full(oracle_pool):
    _full_compare(oracle_pool, I.WORKLOADS["causal_bf16_h8_n16384_d64_L8_P6_clustered32"])


def test_fwdbwd_workload_kernels_at_262k_in_full(oracle_pool):
    wl = I.WORKLOADS["causal_fwdbwd_bf16_h4_n12582912_d64_L8_P6"].replace(N=262144)
    _full_compare(oracle_pool, wl)


def _full_size_checks(name, heads_checked):
    """Runs the workload and returns the worst ratio of each check to its bound (<= 1
    passes); every GPU tensor is freed on return."""
    wl = I.WORKLOADS[name]
    x = I.make_inputs(wl, DEV, with_dout=True)
    q, k, v, W, g = x["q"], x["k"], x["v"], x["W"], x["dout"]
    out, den = ra.forward(q, k, v, W, wl.tau, True, return_den=True, out_dtype=torch.float32)
    dq, dk, dv, dW = ra.backward(q, k, v, W, wl.tau, True, out, g, den=den,
                                 grad_dtype=torch.float32)
    torch.cuda.synchronize()
    res = {"status": ra.race_device_status(), "finite": bool(torch.isfinite(dW).all())}
    worst_sum = worst_orth = 0.0
    for h in range(wl.H):
        for t in (dq[h], dk[h], dv[h]):
            res["finite"] &= bool(torch.isfinite(t).all())
        # sum_j dv_j = sum_i dO_i, per column, against the sums of absolute values
        sdv, sdo = dv[h].double().sum(dim=0), g[h].double().sum(dim=0)
        scale = dv[h].double().abs().sum(dim=0) + g[h].double().abs().sum(dim=0)
        worst_sum = max(worst_sum, ((sdv - sdo).abs() / (TOL_BWD * scale)).max().item())
        # gradients orthogonal to their inputs, row by row
        for gx, xx in ((dq[h], q[h]), (dk[h], k[h])):
            xf = xx.float()
            dot = (gx * xf).sum(dim=-1).abs()
            lim = 1e-5 * gx.norm(dim=-1) * xf.norm(dim=-1) + 1e-30
            worst_orth = max(worst_orth, (dot / lim).max().item())
            del xf, dot, lim
    res["sum"], res["orth"] = worst_sum, worst_orth
    # exact dq on the first R0 rows from the oracle over the prefix
    Wn = W.double().cpu().numpy()
    res["prefix"] = 0.0
    for h in heads_checked:
        f = lambda t: t[h, :R0].double().cpu().numpy()  # noqa: E731
        dq_ref, _, _, _ = oracle.backward(f(q), f(k), f(v), Wn, wl.tau, True, f(g))
        err = np.abs(f(dq) - dq_ref).max() / np.abs(dq_ref).max()
        res["prefix"] = max(res["prefix"], err / TOL_BWD)
    return res


def _run_full_size(name, heads_checked):
    res = _full_size_checks(name, heads_checked)
    torch.cuda.empty_cache()
    assert res["status"] == 0 and res["finite"], res
    assert res["sum"] <= 1 and res["orth"] <= 1 and res["prefix"] <= 1, res


def test_fwdbwd_12m_tokens_4_heads():
    _run_full_size("causal_fwdbwd_bf16_h4_n12582912_d64_L8_P6", heads_checked=(0, 3))


def test_fwdbwd_4m_tokens_8_heads_long_context_shape():
    _run_full_size("causal_bf16_h8_n4194304_d64_L16_P8_clustered256", heads_checked=(0, 7))
