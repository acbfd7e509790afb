"""GPU parity of the tensor-core (tcgen05) backward against the float64 oracle.

bf16 q, k, v, dO and bf16 gradients dq, dk, dv; dW in float32.  Errors are measured
per gradient as max|dG - dG_ref| / max|dG_ref|.  A gradient that is exactly zero
(dq, dk at N = 1) is measured against 0.1 * max|dv_ref|.

The parity cases pass the oracle's own output o (float32) to the backward, so that
they measure the backward alone: the backward uses o only through
-(g_i . o_i)/den'_i, and with a sharp kernel o_i is close to the v_j it averages,
so the forward's own error (2e-3 * max|V|) would come back amplified by that
cancellation.  One case runs the GPU forward's output through, with a looser bound.

Bound TOL_BWD = 1e-2, derived: the operands that enter in bf16 are g/den' (one
rounding, 2^-9 relative: the computed gradient is the exact gradient for an upstream
gradient perturbed by that much), p(k) or p(q) in the in-chunk product and the masked
in-chunk weights (2^-9 each), and the stored gradients themselves (2^-9 relative to
each entry).  Four such terms give at most 4 * 2^-9 ~ 7.8e-3 relative to the largest
entry; the state enters as a bf16 hi + lo pair and -(g . o)/den' as a hi + lo pair,
so neither adds a term of that size.  Observed errors are 2e-3 .. 6e-3.
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


def _np(t):
    return t.detach().to(torch.float64).cpu().numpy()


def _case(N, H, L, P, tau, causal, seed=3, clusters=0):
    wl = I.Workload("t", H=H, N=N, d=64, L=L, P=P, tau=tau, causal=causal, dtype="bf16",
                    seed=seed, clusters=clusters, backward=True)
    x = I.make_inputs(wl, "cpu")
    return wl, x, {k: v.to(DEV) for k, v in x.items()}


def _errors(got, refs):
    gscale = np.abs(refs[2]).max()
    out = {}
    for name, g, ref in zip(("dq", "dk", "dv", "dW"), got, refs):
        denom = max(np.abs(ref).max(), 0.1 * gscale)
        out[name] = np.abs(_np(g) - ref).max() / denom
    return out


def _run(wl, x, g, gpu_out=False, den=None):
    if gpu_out:
        out = ra.forward(g["q"], g["k"], g["v"], g["W"], wl.tau, wl.causal,
                         out_dtype=torch.float32)
    else:
        o, _ = oracle.forward_heads(_np(x["q"]), _np(x["k"]), _np(x["v"]), _np(x["W"]),
                                    wl.tau, wl.causal)
        out = torch.from_numpy(o).float().to(DEV)
    grads = ra.backward(g["q"], g["k"], g["v"], g["W"], wl.tau, wl.causal, out, g["dout"],
                        den=den, impl="tensor")
    torch.cuda.synchronize()
    assert ra.race_device_status() == 0
    assert all(t.dtype == torch.bfloat16 for t in grads[:3]) and grads[3].dtype == torch.float32
    return grads, out


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("L,P", [(1, 8), (2, 7), (4, 6)])
@pytest.mark.parametrize("N", [1, 100, 1000])
def test_tensor_backward_parity(causal, L, P, N):
    wl, x, g = _case(N, 2, L, P, 0.5, causal, seed=N + L)
    grads, _ = _run(wl, x, g)
    refs = oracle.backward_heads(_np(x["q"]), _np(x["k"]), _np(x["v"]), _np(x["W"]),
                                 wl.tau, causal, _np(x["dout"]))
    errs = _errors(grads, refs)
    assert max(errs.values()) <= TOL_BWD, errs


def test_tensor_backward_sharp_kernel_two_tables():
    wl, x, g = _case(3000, 2, 2, 8, 0.25, True, seed=11)
    grads, _ = _run(wl, x, g)
    refs = oracle.backward_heads(_np(x["q"]), _np(x["k"]), _np(x["v"]), _np(x["W"]),
                                 wl.tau, True, _np(x["dout"]))
    errs = _errors(grads, refs)
    assert max(errs.values()) <= TOL_BWD, errs


def test_tensor_backward_ragged_chunk_edges():
    # lengths at and around the 128-token chunk, several segments of unequal length
    for N in (127, 128, 129, 640, 1537):
        wl, x, g = _case(N, 1, 2, 7, 0.5, True, seed=N)
        grads, _ = _run(wl, x, g)
        refs = oracle.backward_heads(_np(x["q"]), _np(x["k"]), _np(x["v"]), _np(x["W"]),
                                     wl.tau, True, _np(x["dout"]))
        errs = _errors(grads, refs)
        assert max(errs.values()) <= TOL_BWD, (N, errs)


def test_tensor_backward_with_gpu_forward_output():
    # end to end: o from the GPU forward; its error (<= 2e-3 * max|V|) reaches the
    # gradients through -(g . o)/den', amplified where o_i is close to v_j
    wl, x, g = _case(1000, 2, 4, 6, 0.5, True, seed=5)
    grads, _ = _run(wl, x, g, gpu_out=True)
    refs = oracle.backward_heads(_np(x["q"]), _np(x["k"]), _np(x["v"]), _np(x["W"]),
                                 wl.tau, True, _np(x["dout"]))
    errs = _errors(grads, refs)
    assert max(errs.values()) <= 2 * TOL_BWD, errs


def test_tensor_backward_saved_den_matches_recompute():
    wl, x, g = _case(700, 2, 2, 7, 0.5, True, seed=9)
    out, den = ra.forward(g["q"], g["k"], g["v"], g["W"], wl.tau, True,
                          out_dtype=torch.float32, return_den=True)
    a = ra.backward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out, g["dout"],
                    impl="tensor")
    b = ra.backward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out, g["dout"], den=den,
                    impl="tensor")
    torch.cuda.synchronize()
    for x1, x2 in zip(a, b):
        assert (x1.float() - x2.float()).abs().max().item() <= 1e-2 * x1.float().abs().max().item()


def test_tensor_backward_agrees_with_simt_path():
    wl, x, g = _case(900, 2, 4, 6, 0.5, True, seed=21)
    out = ra.forward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out_dtype=torch.float32)
    tc = ra.backward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out, g["dout"],
                     impl="tensor")
    si = ra.backward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out, g["dout"],
                     impl="simt")
    torch.cuda.synchronize()
    for name, a, b in zip(("dq", "dk", "dv", "dW"), tc, si):
        err = (a.float() - b.float()).abs().max().item() / b.float().abs().max().item()
        assert err <= 2 * TOL_BWD, (name, err)


def test_tensor_backward_unsupported_shape_rejected():
    # rows of 256 sketch rows are required: L * 2^P = 192 is not a multiple of 256
    wl, x, g = _case(64, 1, 3, 6, 0.5, True)
    out = ra.forward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out_dtype=torch.float32)
    with pytest.raises(ra.RaceError) as e:
        ra.backward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out, g["dout"],
                    impl="tensor")
    assert e.value.status == ra.RACE_ERR_UNSUPPORTED
