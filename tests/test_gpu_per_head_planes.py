"""One set of hash planes per head (race_args_t.w_per_head): W and dW of shape
[H, L, 64, P].  The pages train the sketch end to end ([JA] §2.2 differentiability), which
with several heads means each head may learn its own planes.

* Forward and backward against the oracle run head by head with that head's planes
  (tensor-core path within 2e-3 * max|V| and 3 * 2^-8 of each gradient's largest entry;
  CUDA-core path 2e-5 / 1e-5, as in the parity files).
* With every head given the same planes, the outputs equal the shared-plane call and the
  per-head dW sum to the shared dW.
* The layer with per-head planes takes a gradient step on them.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_lsh_sketch_race_b200 import inputs as I
from linear_lsh_sketch_race_b200 import layer as LY
from linear_lsh_sketch_race_b200 import race_attn as ra

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _f64(t):
    return t.detach().double().cpu().numpy()


def _case(N, H, L, P, tau, causal, seed):
    wl = I.Workload("ph", H=H, N=N, d=64, L=L, P=P, tau=tau, causal=causal, dtype="bf16",
                    seed=seed, backward=True)
    x = I.make_inputs(wl, "cpu")
    gen = torch.Generator().manual_seed(seed + 100)
    Wh = torch.randn((H, L, 64, P), generator=gen, dtype=torch.float32)
    return wl, x, Wh


CASES = [dict(impl="tensor", L=2, P=8, tau=0.25, causal=True),
         dict(impl="tensor", L=4, P=6, tau=0.5, causal=False),
         dict(impl="simt", L=3, P=4, tau=0.5, causal=True)]


@pytest.mark.parametrize("c", CASES, ids=lambda c: f"{c['impl']}_P{c['P']}")
def test_per_head_planes_against_oracle(c):
    N, H = 600, 3
    wl, x, Wh = _case(N, H, c["L"], c["P"], c["tau"], c["causal"], seed=c["P"])
    g = {k: v.to(DEV) for k, v in x.items()}
    Wd = Wh.to(DEV)
    out, den = ra.forward(g["q"], g["k"], g["v"], Wd, wl.tau, wl.causal,
                          out_dtype=torch.float32, impl=c["impl"], return_den=True)
    f = {k: _f64(v) for k, v in x.items()}
    Wn = _f64(Wh)
    ref_o = np.stack([oracle.forward(f["q"][h], f["k"][h], f["v"][h], Wn[h], wl.tau,
                                     wl.causal)[0] for h in range(H)])
    vmax = np.abs(f["v"]).max()
    tol = 2e-3 if c["impl"] == "tensor" else 2e-5
    assert np.abs(_f64(out) - ref_o).max() / vmax <= tol
    o32 = torch.from_numpy(ref_o).float().to(DEV)
    dq, dk, dv, dW = ra.backward(g["q"], g["k"], g["v"], Wd, wl.tau, wl.causal, o32,
                                 g["dout"], impl=c["impl"], grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ra.race_device_status() == 0
    assert dW.shape == (H, wl.L, 64, wl.P)
    refs = [oracle.backward(f["q"][h], f["k"][h], f["v"][h], Wn[h], wl.tau, wl.causal,
                            f["dout"][h]) for h in range(H)]
    gtol = 3 * 2.0 ** -8 if c["impl"] == "tensor" else 1e-5
    for i, (name, got) in enumerate(zip(("dq", "dk", "dv", "dW"), (dq, dk, dv, dW))):
        ref = np.stack([r[i] for r in refs])
        err = np.abs(_f64(got) - ref).max() / np.abs(ref).max()
        assert err <= gtol, (name, err)


@pytest.mark.parametrize("impl", ["tensor", "simt"])
def test_identical_per_head_planes_equal_shared_planes(impl):
    N, H, L, P = 500, 4, 4, 6
    wl, x, _ = _case(N, H, L, P, 0.5, True, seed=11)
    g = {k: v.to(DEV) for k, v in x.items()}
    W = g["W"]
    Wrep = W.unsqueeze(0).expand(H, L, 64, P).contiguous()
    kw = dict(out_dtype=torch.float32, impl=impl)
    a = ra.forward(g["q"], g["k"], g["v"], W, wl.tau, True, **kw)
    b = ra.forward(g["q"], g["k"], g["v"], Wrep, wl.tau, True, **kw)
    vmax = g["v"].float().abs().max().item()
    assert (a - b).abs().max().item() <= 1e-5 * vmax
    ga = ra.backward(g["q"], g["k"], g["v"], W, wl.tau, True, a, g["dout"], impl=impl,
                     grad_dtype=torch.float32)
    gb = ra.backward(g["q"], g["k"], g["v"], Wrep, wl.tau, True, a, g["dout"], impl=impl,
                     grad_dtype=torch.float32)
    torch.cuda.synchronize()
    for t1, t2 in zip(ga[:3], gb[:3]):
        assert (t1 - t2).abs().max().item() <= 1e-5 * t1.abs().max().item()
    assert (gb[3].sum(0) - ga[3]).abs().max().item() <= 1e-5 * ga[3].abs().max().item()


def test_hash_with_per_head_planes():
    N, H, L, P = 77, 2, 3, 5
    wl, x, Wh = _case(N, H, L, P, 0.4, False, seed=3)
    phi = ra.hash(x["q"].float().to(DEV), Wh.to(DEV), wl.tau)
    for h in range(H):
        ref = oracle.phi(_f64(x["q"][h]), _f64(Wh[h]), wl.tau)
        assert np.abs(_f64(phi[h]) - ref).max() <= 2e-6 * ref.max()


def test_layer_with_per_head_planes_trains_them():
    torch.manual_seed(4)
    layer = LY.init_like_attention(LY.RaceMultiHeadAttention(
        128, 2, L=4, P=6, tau=0.5, causal=True, per_head_planes=True, impl="simt",
        device=DEV, dtype=torch.float32, seed=5))
    assert layer.planes.shape == (2, 4, 64, 6)
    x = torch.randn(2, 300, 128, device=DEV)
    target = torch.randn(2, 300, 128, device=DEV)
    loss0 = ((layer(x) - target) ** 2).mean()
    loss0.backward()
    gW = layer.planes.grad
    assert gW.shape == layer.planes.shape and torch.isfinite(gW).all()
    assert (gW[0] - gW[1]).abs().max() > 0          # the heads' planes get their own gradients
    with torch.no_grad():
        layer.planes -= (0.05 / gW.norm()) * gW
        loss1 = ((layer(x) - target) ** 2).mean()
    assert loss1.item() < loss0.item()
