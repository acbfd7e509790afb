"""GPU parity of the tensor-core (tcgen05) backward against the float64 oracle.

bf16 q, k, v, dO; dq, dk, dv written in float32 (grad_dtype) so that the kernels' own
error is measured without a final bf16 rounding of the gradients; dW in float32.  Each
gradient tensor G is held to max|dG - dG_ref| <= TOL_BWD * max|dG_ref|.  With one token
dq, dk and dW are zero in exact arithmetic and are measured against max|dv_ref|.

TOL_BWD = 3 * 2^-8 (about 1.17e-2), derived from the arithmetic of the kernels: the
tensor cores read bf16 operands, whose unit roundoff is u = 2^-8.  A gradient entry that
comes from few products (the in-chunk terms of the first rows of a sequence, or a nearly
one-hot soft assignment) carries the rounding of the corner probability p (u), of the
in-chunk weight or weight-gradient it multiplies (u), and of the 1/den' factor folded
into p(q) on the key side (u), with nothing to cancel them.  The forward output is a
weighted mean whose numerator and denominator use the same rounded weights, which is why
it meets 2e-3; its gradients are not normalised.  A float64 emulation of the kernels'
rounding points attributes the error to these roundings (each alone 1e-3 to 2.2e-3 of
max|G| on these cases; the roundings on the state side alone stay below 1e-3).  Measured
maxima on this file's cases lie between 1.2e-3 and 7.8e-3.  The CUDA-core path, float32
throughout, is held to 1e-5 (test_gpu_parity.py).

The parity cases pass the oracle's own output o (float32) to the backward, so that
they measure the backward alone: the backward uses o only through -(g_i . o_i), and
with a sharp kernel o_i is close to the v_j it averages, so an error of the forward
would come back through that difference.  One case runs the GPU forward's output
through.  A second set checks that bf16 gradients are the float32 ones rounded once.
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


def _np(t):
    return t.detach().to(torch.float64).cpu().numpy()


def _case(N, H, L, P, tau, causal, seed=3, clusters=0, sigma=0.3):
    wl = I.Workload("t", H=H, N=N, d=64, L=L, P=P, tau=tau, causal=causal, dtype="bf16",
                    seed=seed, clusters=clusters, sigma=sigma, backward=True)
    x = I.make_inputs(wl, "cpu")
    return wl, x, {k: v.to(DEV) for k, v in x.items()}


def _errors(got, refs, N):
    out = {}
    for name, g, ref in zip(("dq", "dk", "dv", "dW"), got, refs):
        denom = np.abs(ref).max()
        if N == 1 and name != "dv":
            denom = np.abs(refs[2]).max()
        out[name] = float(np.abs(_np(g) - ref).max() / denom)
    return out


def _refs(wl, x):
    return oracle.backward_heads(_np(x["q"]), _np(x["k"]), _np(x["v"]), _np(x["W"]),
                                 wl.tau, wl.causal, _np(x["dout"]))


def _run(wl, x, g, gpu_out=False, den=None, grad_dtype=torch.float32):
    if gpu_out:
        out = ra.forward(g["q"], g["k"], g["v"], g["W"], wl.tau, wl.causal,
                         out_dtype=torch.float32)
    else:
        o, _ = oracle.forward_heads(_np(x["q"]), _np(x["k"]), _np(x["v"]), _np(x["W"]),
                                    wl.tau, wl.causal)
        out = torch.from_numpy(o).float().to(DEV)
    grads = ra.backward(g["q"], g["k"], g["v"], g["W"], wl.tau, wl.causal, out, g["dout"],
                        den=den, impl="tensor", grad_dtype=grad_dtype)
    torch.cuda.synchronize()
    assert ra.race_device_status() == 0
    assert all(t.dtype == grad_dtype for t in grads[:3]) and grads[3].dtype == torch.float32
    return grads, out


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("L,P", [(1, 8), (2, 7), (4, 6)])
@pytest.mark.parametrize("N", [1, 100, 1000])
def test_tensor_backward_parity(causal, L, P, N):
    wl, x, g = _case(N, 2, L, P, 0.5, causal, seed=N + L)
    grads, _ = _run(wl, x, g)
    errs = _errors(grads, _refs(wl, x), N)
    assert max(errs.values()) <= TOL_BWD, errs


def test_tensor_backward_sharp_kernel_two_tables():
    wl, x, g = _case(3000, 2, 2, 8, 0.25, True, seed=11)
    grads, _ = _run(wl, x, g)
    errs = _errors(grads, _refs(wl, x), 3000)
    assert max(errs.values()) <= TOL_BWD, errs


def test_tensor_backward_long_context_shape():
    """16 tables of 256 buckets, tau = 0.25, 256 clusters: the 4M-token workload's shape."""
    wl, x, g = _case(3000, 2, 16, 8, 0.25, True, seed=4, clusters=256)
    grads, _ = _run(wl, x, g)
    errs = _errors(grads, _refs(wl, x), 3000)
    assert max(errs.values()) <= TOL_BWD, errs


def test_tensor_backward_near_one_hot_assignments():
    """Tight clusters (noise 0.3/8 per coordinate) at tau = 0.25: nearly one-hot phi."""
    wl, x, g = _case(1500, 2, 2, 8, 0.25, True, seed=5, clusters=4, sigma=0.3 / 8)
    grads, _ = _run(wl, x, g)
    errs = _errors(grads, _refs(wl, x), 1500)
    assert max(errs.values()) <= TOL_BWD, errs


@pytest.mark.parametrize("P", [7, 8])
def test_tensor_backward_ragged_chunk_edges(P):
    # lengths at and around the 128-token chunk, several segments of unequal length (at
    # P = 8 the causal sweeps run as the two-CTA pipelined kernel)
    for N in (127, 128, 129, 640, 1537):
        wl, x, g = _case(N, 1, 2, P, 0.5, True, seed=N)
        grads, _ = _run(wl, x, g)
        errs = _errors(grads, _refs(wl, x), N)
        assert max(errs.values()) <= TOL_BWD, (N, errs)


def test_tensor_backward_with_gpu_forward_output():
    # end to end: o from the GPU forward (float32 output)
    wl, x, g = _case(1000, 2, 4, 6, 0.5, True, seed=5)
    grads, _ = _run(wl, x, g, gpu_out=True)
    errs = _errors(grads, _refs(wl, x), 1000)
    assert max(errs.values()) <= TOL_BWD, errs


def test_tensor_backward_bf16_gradients_are_rounded_float32_gradients():
    wl, x, g = _case(700, 2, 2, 7, 0.5, True, seed=9)
    f32, out = _run(wl, x, g)
    b16, _ = _run(wl, x, g, grad_dtype=torch.bfloat16)
    # the float32 results of two runs differ only in the order of float32 additions into
    # shared accumulators; the bf16 gradients are those results rounded once, which is
    # within one bf16 unit in the last place (2^-7 relative) of the other run's value
    for a, b in zip(f32[:3], b16[:3]):
        lim = 2.0 ** -7 * a.abs() + 1e-6 * a.abs().max()
        assert ((b.float() - a).abs() <= lim).all()
    assert (f32[3] - b16[3]).abs().max().item() <= 1e-5 * f32[3].abs().max().item()


def test_tensor_backward_saved_den_matches_recompute():
    wl, x, g = _case(700, 2, 2, 7, 0.5, True, seed=9)
    out, den = ra.forward(g["q"], g["k"], g["v"], g["W"], wl.tau, True,
                          out_dtype=torch.float32, return_den=True)
    kw = dict(impl="tensor", grad_dtype=torch.float32)
    a = ra.backward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out, g["dout"], **kw)
    b = ra.backward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out, g["dout"], den=den,
                    **kw)
    torch.cuda.synchronize()
    # the same kernels with den' from the saved den (times L) or recomputed: they differ
    # in the last bits of den' and in the order of float32 additions
    for x1, x2 in zip(a, b):
        assert (x1 - x2).abs().max().item() <= 1e-5 * x1.abs().max().item()


def test_tensor_backward_agrees_with_simt_path():
    wl, x, g = _case(900, 2, 4, 6, 0.5, True, seed=21)
    out = ra.forward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out_dtype=torch.float32)
    tc = ra.backward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out, g["dout"],
                     impl="tensor", grad_dtype=torch.float32)
    si = ra.backward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out, g["dout"],
                     impl="simt", grad_dtype=torch.float32)
    torch.cuda.synchronize()
    for name, a, b in zip(("dq", "dk", "dv", "dW"), tc, si):
        err = (a - b).abs().max().item() / b.abs().max().item()
        assert err <= TOL_BWD, (name, err)


def test_tensor_backward_unsupported_shape_rejected():
    # rows of 256 sketch rows are required: L * 2^P = 192 is not a multiple of 256
    wl, x, g = _case(64, 1, 3, 6, 0.5, True)
    out = ra.forward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out_dtype=torch.float32)
    with pytest.raises(ra.RaceError) as e:
        ra.backward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out, g["dout"],
                    impl="tensor")
    assert e.value.status == ra.RACE_ERR_UNSUPPORTED
