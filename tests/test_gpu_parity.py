"""GPU parity: the CUDA library against the float64 oracle on identical seeded inputs.

Tolerances (max over all elements, normalised by max|V| for outputs since outputs
are convex combinations of V rows, and by max|G_ref| of the same gradient tensor G):
  * CUDA-core path (float32 arithmetic, float32 outputs and gradients): 1e-5 for the
    backward; 1e-5 (float32 inputs) and 2e-5 (bf16 inputs) for the forward
  * bf16 inputs on the tensor-core path: 2e-3 (bf16 operands, float32 accumulation)
The oracle receives the exact values the GPU receives (bf16 inputs upcast).  Where a
gradient is zero in exact arithmetic (dq, dk and hence dW with a single token: o_0 = v_0
does not depend on q or k), it is measured against max|dv_ref|, the natural scale.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_lsh_sketch_race_b200 import inputs as I
from linear_lsh_sketch_race_b200 import race_attn as ra

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _np(t):
    return t.detach().to(torch.float64).cpu().numpy()


def _case(N, H=2, L=3, P=4, tau=0.5, causal=True, dtype="bf16", clusters=0, seed=7,
          backward=False):
    wl = I.Workload("t", H=H, N=N, d=64, L=L, P=P, tau=tau, causal=causal, dtype=dtype,
                    clusters=clusters, seed=seed, backward=backward)
    x = I.make_inputs(wl, "cpu")
    return wl, x, {k: v.to(DEV) for k, v in x.items()}


def _oracle_fwd(wl, x):
    return oracle.forward_heads(_np(x["q"]), _np(x["k"]), _np(x["v"]), _np(x["W"]),
                                wl.tau, wl.causal)


def _rel_err(got, ref, scale):
    return float(np.abs(_np(got) - ref).max() / scale)


# ------------------------------------------------------------------------- hash
@pytest.mark.parametrize("P", [1, 5, 8])
def test_hash_matches_oracle(P):
    wl, x, g = _case(N=77, H=2, L=3, P=P, tau=0.4, dtype="fp32")
    phi = ra.hash(g["q"], g["W"], wl.tau, out_dtype=torch.float32)
    ref = np.stack([oracle.phi(_np(x["q"])[h], _np(x["W"]), wl.tau) for h in range(2)])
    assert np.abs(_np(phi) - ref).max() <= 2e-6 * ref.max()
    # each softmax block sums to 1, so each phi block sums to 1/sqrt(L)
    blocks = _np(phi).reshape(2, 77, 3, 1 << P).sum(-1)
    assert np.allclose(blocks, 1 / np.sqrt(3), rtol=1e-5)
    phib = ra.hash(g["q"].bfloat16(), g["W"], wl.tau, out_dtype=torch.bfloat16)
    refb = np.stack([oracle.phi(_np(x["q"].bfloat16())[h], _np(x["W"]), wl.tau)
                     for h in range(2)])
    assert np.all(np.abs(_np(phib) - refb) <= 2.0 ** -8 * np.abs(refb) + 1e-30)


# ------------------------------------------------------------------------- forward
def test_forward_fp32_small_config_parity():
    """Non-causal fp32 workload (N = 1024, L = 4, P = 4): the 1e-5 criterion."""
    wl = I.WORKLOADS[I.SMALL]
    x = I.make_inputs(wl, "cpu")
    g = {k: v.to(DEV) for k, v in x.items()}
    out, den = ra.forward(g["q"], g["k"], g["v"], g["W"], wl.tau, wl.causal,
                          return_den=True)
    ref, rden = _oracle_fwd(wl, x)
    scale = np.abs(_np(x["v"])).max()
    assert _rel_err(out, ref, scale) <= 1e-5
    assert np.abs(_np(den) - rden).max() <= 1e-5 * rden.max()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 31, 33, 200, 1031])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_forward_simt_parity(causal, N, dtype):
    wl, x, g = _case(N=N, H=3, L=3, P=5, causal=causal, dtype=dtype, seed=N)
    out = ra.forward(g["q"], g["k"], g["v"], g["W"], wl.tau, causal,
                     out_dtype=torch.float32, impl="simt")
    ref, _ = _oracle_fwd(wl, x)
    tol = 1e-5 if dtype == "fp32" else 2e-5
    assert _rel_err(out, ref, np.abs(_np(x["v"])).max()) <= tol


@pytest.mark.parametrize("P,L,tau", [(8, 2, 0.25), (6, 4, 0.5), (2, 7, 1.0)])
def test_forward_simt_clustered_and_table_shapes(P, L, tau):
    wl, x, g = _case(N=300, H=2, L=L, P=P, tau=tau, causal=True, clusters=8, seed=P)
    out = ra.forward(g["q"], g["k"], g["v"], g["W"], tau, True, out_dtype=torch.float32,
                     impl="simt")
    ref, _ = _oracle_fwd(wl, x)
    assert _rel_err(out, ref, np.abs(_np(x["v"])).max()) <= 2e-5


def test_forward_simt_bf16_output_rounding():
    wl, x, g = _case(N=150, causal=True)
    out = ra.forward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, impl="simt")
    assert out.dtype == torch.bfloat16
    ref, _ = _oracle_fwd(wl, x)
    assert np.all(np.abs(_np(out) - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6)


def test_forward_outputs_convex_and_causal_prefix():
    wl, x, g = _case(N=500, causal=True, seed=3)
    out = ra.forward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out_dtype=torch.float32,
                     impl="simt")
    o = _np(out)
    v = _np(x["v"])
    cmax = np.maximum.accumulate(v, axis=1)
    cmin = np.minimum.accumulate(v, axis=1)
    assert np.all(o <= cmax + 1e-5) and np.all(o >= cmin - 1e-5)
    short = ra.forward(g["q"][:, :123].contiguous(), g["k"][:, :123].contiguous(),
                       g["v"][:, :123].contiguous(), g["W"], wl.tau, True,
                       out_dtype=torch.float32, impl="simt")
    assert np.abs(_np(short) - o[:, :123]).max() <= 1e-5


def test_caller_workspace_and_spec_form():
    wl, x, g = _case(N=257, causal=True, seed=11)
    a = ra.make_args(g["q"], g["W"], wl.tau, True)
    need = ra.race_workspace_size(a)
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    o1 = ra.forward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, workspace=ws)
    o2 = torch.empty_like(g["q"])
    H, N, d = g["q"].shape
    ra.race_forward(g["q"], g["k"], g["v"], g["W"], o2, N, H, d, wl.L, wl.P, wl.tau, 1)
    torch.cuda.synchronize()
    ref, _ = _oracle_fwd(wl, x)
    scale = np.abs(_np(x["v"])).max()
    assert _rel_err(o1, ref, scale) <= 2e-3
    assert _rel_err(o2, ref, scale) <= 2e-3
    assert ra.race_device_status() == 0


# ------------------------------------------------------------------------- backward
def _oracle_bwd(wl, x):
    return oracle.backward_heads(_np(x["q"]), _np(x["k"]), _np(x["v"]), _np(x["W"]),
                                 wl.tau, wl.causal, _np(x["dout"]))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 45, 300])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_backward_simt_parity(causal, N, dtype):
    wl, x, g = _case(N=N, H=2, L=3, P=4, tau=0.6, causal=causal, dtype=dtype, seed=N + 5,
                     backward=True)
    o, _ = _oracle_fwd(wl, x)
    out = torch.from_numpy(o).float().to(DEV)
    grads = ra.backward(g["q"], g["k"], g["v"], g["W"], wl.tau, causal, out, g["dout"],
                        impl="simt", grad_dtype=torch.float32)
    refs = _oracle_bwd(wl, x)
    check_grads(grads, refs, 1e-5, N)


def test_backward_simt_bf16_gradients_are_rounded_float32_gradients():
    wl, x, g = _case(N=300, causal=True, backward=True, seed=2)
    out = ra.forward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out_dtype=torch.float32,
                     impl="simt")
    f32 = ra.backward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out, g["dout"],
                      impl="simt", grad_dtype=torch.float32)
    b16 = ra.backward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out, g["dout"],
                      impl="simt", grad_dtype=torch.bfloat16)
    # two runs differ in the order of float32 atomic additions; a bf16 result is the
    # float32 result of its own run rounded once: within one bf16 ulp (2^-7 relative)
    for a, b in zip(f32[:3], b16[:3]):
        assert b.dtype == torch.bfloat16
        assert ((b.float() - a).abs() <= 2.0 ** -7 * a.abs() + 1e-6 * a.abs().max()).all()


def check_grads(got, refs, tol, N):
    """max|dG - dG_ref| <= tol * max|dG_ref| per gradient tensor.  With one token, dq, dk
    and dW are zero in exact arithmetic and are measured against max|dv_ref|."""
    errs = {}
    for name, g, ref in zip(("dq", "dk", "dv", "dW"), got, refs):
        denom = np.abs(ref).max()
        if N == 1 and name != "dv":
            denom = np.abs(refs[2]).max()
        errs[name] = np.abs(_np(g) - ref).max() / denom
    assert max(errs.values()) <= tol, errs
    return errs


def test_backward_with_saved_den_matches_recompute():
    wl, x, g = _case(N=200, causal=True, dtype="fp32", backward=True, seed=4)
    out, den = ra.forward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, return_den=True,
                          impl="simt")
    a = ra.backward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out, g["dout"],
                    impl="simt")
    b = ra.backward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out, g["dout"],
                    den=den, impl="simt")
    for x1, x2 in zip(a, b):
        assert (x1 - x2).abs().max().item() <= 1e-5 * x1.abs().max().item()
