"""Degenerate inputs on both kernel families: all-zero rows and rows of norm ~1e4 in q
and k, forward and backward, against the float64 oracle.

A zero vector is normalised by max(|x|, 1e-12), so its projections are 0 and its soft
assignment is uniform over the corners; the derivative of x / max(|x|, 1e-12) at x = 0
is the identity divided by 1e-12, so the gradients of zero rows are of order 1e12 times
those of other rows.  Each gradient is therefore compared separately on the zero rows and
on the other rows, each part against its own largest reference entry.  Large-norm rows
must give the same outputs as the unscaled rows (the method only sees x / |x|); they are
made by scaling rows by 2^10, which is exact in bf16 and in the float32 arithmetic of the
norms, so the outputs agree to float32 rounding.

Tolerances as in the parity files: 2e-3 * max|V| for tensor-core outputs, 3 * 2^-8 of the
largest reference entry for tensor-core gradients (see test_gpu_tensor_backward.py), and
the float32 bounds (2e-5 outputs with bf16 inputs, 1e-5 gradients) on the CUDA-core path.
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


def _inputs(N, H, L, P, tau, causal, seed):
    wl = I.Workload("edge", H=H, N=N, d=64, L=L, P=P, tau=tau, causal=causal, dtype="bf16",
                    seed=seed, backward=True)
    x = I.make_inputs(wl, "cpu")
    gen = torch.Generator().manual_seed(seed)
    zero_q = torch.randperm(N, generator=gen)[: max(1, N // 16)]
    zero_k = torch.randperm(N, generator=gen)[: max(1, N // 16)]
    big_q = torch.randperm(N, generator=gen)[: max(1, N // 16)]
    big_k = torch.randperm(N, generator=gen)[: max(1, N // 16)]
    for name, zero, big in (("q", zero_q, big_q), ("k", zero_k, big_k)):
        t = x[name].float()
        t[:, big] = t[:, big] * 1024.0          # norm ~8e3: exact power-of-two scaling
        t[:, zero] = 0.0
        x[name] = t.to(torch.bfloat16)
    return wl, x, {"q": zero_q, "k": zero_k}


CASES = [
    dict(impl="tensor", L=2, P=8, tau=0.25, causal=True),
    dict(impl="tensor", L=4, P=6, tau=0.5, causal=False),
    dict(impl="simt", L=3, P=4, tau=0.5, causal=True),
]


@pytest.mark.parametrize("c", CASES, ids=lambda c: f"{c['impl']}_P{c['P']}_"
                         f"{'causal' if c['causal'] else 'noncausal'}")
def test_zero_and_large_norm_rows(c):
    N, H = 700, 2
    wl, x, zeros = _inputs(N, H, c["L"], c["P"], c["tau"], c["causal"], seed=c["P"])
    g = {k: v.to(DEV) for k, v in x.items()}
    f = {k: _np(v) for k, v in x.items()}
    out = ra.forward(g["q"], g["k"], g["v"], g["W"], wl.tau, wl.causal,
                     out_dtype=torch.float32, impl=c["impl"])
    ref_o, _ = oracle.forward_heads(f["q"], f["k"], f["v"], f["W"], wl.tau, wl.causal)
    vmax = np.abs(f["v"]).max()
    tol = 2e-3 if c["impl"] == "tensor" else 2e-5
    assert np.isfinite(_np(out)).all()
    assert np.abs(_np(out) - ref_o).max() / vmax <= tol

    o32 = torch.from_numpy(ref_o).float().to(DEV)
    grads = ra.backward(g["q"], g["k"], g["v"], g["W"], wl.tau, wl.causal, o32, g["dout"],
                        impl=c["impl"], grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ra.race_device_status() == 0
    refs = oracle.backward_heads(f["q"], f["k"], f["v"], f["W"], wl.tau, wl.causal,
                                 f["dout"])
    gtol = 3 * 2.0 ** -8 if c["impl"] == "tensor" else 1e-5
    for name, got, ref in zip(("dq", "dk", "dv", "dW"), grads, refs):
        got = _np(got)
        assert np.isfinite(got).all(), name
        if name in ("dq", "dk"):
            zmask = np.zeros(N, dtype=bool)
            zmask[zeros[name[1]].numpy()] = True
            for part in (zmask, ~zmask):
                r, gg = ref[:, part], got[:, part]
                err = np.abs(gg - r).max() / np.abs(r).max()
                assert err <= gtol, (name, part.sum(), err)
        else:
            err = np.abs(got - ref).max() / np.abs(ref).max()
            assert err <= gtol, (name, err)


def test_large_norm_rows_match_their_directions():
    wl, x, _ = _inputs(500, 2, 2, 8, 0.25, True, seed=3)
    g = {k: v.to(DEV) for k, v in x.items()}
    out = ra.forward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out_dtype=torch.float32)
    # every row of q and k scaled by 2^10 (exact in bf16): the same directions
    out2 = ra.forward(g["q"] * 1024, g["k"] * 1024, g["v"], g["W"], wl.tau, True,
                      out_dtype=torch.float32)
    torch.cuda.synchronize()
    vmax = g["v"].float().abs().max().item()
    assert (out - out2).abs().max().item() / vmax <= 1e-5
