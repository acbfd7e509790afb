"""The multi-head attention layer around RACE (linear_lsh_sketch_race_b200.layer).

* The float32 layer on the CUDA-core kernels against a float64 reference of the whole
  layer: projections in float64 with the same weights, RACE attention and its gradients
  from the oracle.  Parameter gradients of every projection and of the hash planes.
* The bf16 layer (tensor-core kernels): the autograd gradients of q, k, v and W equal
  the library's backward on the same tensors, and the RACE gradients match the oracle
  given the layer's own bf16 q, k, v.
* Training use of dW: one SGD step on the hash planes along -dW lowers the loss.

Tolerances: the float32 path 1e-4 of each gradient's largest entry (the RACE kernels
meet 1e-5; the projections and the float32 matmuls around them add float32 rounding over
sums of d_model = 128 and 2 x 64 x heads terms); the bf16 path 3 * 2^-8 as derived in
test_gpu_tensor_backward.py.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_lsh_sketch_race_b200 import layer as LY
from linear_lsh_sketch_race_b200 import race_attn as ra

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _f64(t):
    return t.detach().double().cpu().numpy()


def _reference(layer, x, g_y):
    """Float64 forward and backward of the whole layer with the layer's weights."""
    B, N, _ = x.shape
    H, d = layer.heads, layer.head_dim
    X = _f64(x)
    Wq, Wk, Wv, Wo = (_f64(m.weight) for m in (layer.wq, layer.wk, layer.wv, layer.wo))
    Pl = _f64(layer.planes)
    G = _f64(g_y)
    split = lambda t: t.reshape(B, N, H, d).transpose(0, 2, 1, 3).reshape(B * H, N, d)  # noqa
    merge = lambda t: t.reshape(B, H, N, d).transpose(0, 2, 1, 3).reshape(B, N, H * d)  # noqa
    q, k, v = split(X @ Wq.T), split(X @ Wk.T), split(X @ Wv.T)
    o, _ = oracle.forward_heads(q, k, v, Pl, layer.tau, layer.causal)
    y = merge(o) @ Wo.T
    dWo = np.einsum("bno,bni->oi", G, merge(o))
    do = split(G @ Wo)
    dq, dk, dv, dP = oracle.backward_heads(q, k, v, Pl, layer.tau, layer.causal, do)
    dWq = np.einsum("bno,bni->oi", merge(dq), X)
    dWk = np.einsum("bno,bni->oi", merge(dk), X)
    dWv = np.einsum("bno,bni->oi", merge(dv), X)
    dx = merge(dq) @ Wq + merge(dk) @ Wk + merge(dv) @ Wv
    return y, {"wq": dWq, "wk": dWk, "wv": dWv, "wo": dWo, "planes": dP, "x": dx}


def _grads(layer, x):
    return {"wq": layer.wq.weight.grad, "wk": layer.wk.weight.grad,
            "wv": layer.wv.weight.grad, "wo": layer.wo.weight.grad,
            "planes": layer.planes.grad, "x": x.grad}


@pytest.mark.parametrize("causal", [True, False])
def test_float32_layer_against_float64_reference(causal):
    torch.manual_seed(0)
    layer = LY.init_like_attention(LY.RaceMultiHeadAttention(
        128, 2, L=3, P=5, tau=0.5, causal=causal, impl="simt", device=DEV,
        dtype=torch.float32, seed=1))
    x = torch.randn(2, 300, 128, device=DEV, requires_grad=True)
    y = layer(x)
    g_y = torch.randn_like(y)
    y.backward(g_y)
    torch.cuda.synchronize()
    assert ra.race_device_status() == 0
    y_ref, refs = _reference(layer, x, g_y)
    assert np.abs(_f64(y) - y_ref).max() / np.abs(y_ref).max() <= 1e-4
    for name, got in _grads(layer, x).items():
        ref = refs[name]
        err = np.abs(_f64(got) - ref).max() / np.abs(ref).max()
        assert err <= 1e-4, (name, err)


def test_bf16_layer_gradients_are_the_library_backward():
    torch.manual_seed(1)
    layer = LY.init_like_attention(LY.RaceMultiHeadAttention(
        256, 4, L=4, P=6, tau=0.5, causal=True, device=DEV, dtype=torch.bfloat16, seed=2))
    x = torch.randn(2, 1000, 256, device=DEV, dtype=torch.bfloat16)
    B, N, _ = x.shape
    q = layer._split(layer.wq(x), B, N).detach().requires_grad_(True)
    k = layer._split(layer.wk(x), B, N).detach().requires_grad_(True)
    v = layer._split(layer.wv(x), B, N).detach().requires_grad_(True)
    W = layer.planes.detach().clone().requires_grad_(True)
    o = LY.race_attention(q, k, v, W, layer.tau, True)
    g = torch.randn_like(o)
    o.backward(g)
    out, den = ra.forward(q.detach(), k.detach(), v.detach(), W.detach(), layer.tau, True,
                          return_den=True)
    lib = ra.backward(q.detach(), k.detach(), v.detach(), W.detach(), layer.tau, True, out,
                      g, den=den)
    torch.cuda.synchronize()
    # the same kernels on the same tensors: results differ at most by the order of float32
    # additions into shared accumulators, i.e. one bf16 unit in the last place (2^-7)
    close = lambda a, b: bool(((a.float() - b.float()).abs() <=  # noqa: E731
                               2.0 ** -7 * b.float().abs() + 1e-5 * b.float().abs().max()).all())
    assert close(o.detach(), out)
    for a, b in zip((q.grad, k.grad, v.grad, W.grad), lib):
        assert close(a, b)
    # the RACE gradients against the oracle on the layer's own bf16 tensors (float32 out)
    f = {n: _f64(t) for n, t in (("q", q), ("k", k), ("v", v), ("W", W), ("g", g))}
    o_ref, _ = oracle.forward_heads(f["q"], f["k"], f["v"], f["W"], layer.tau, True)
    g32 = ra.backward(q.detach(), k.detach(), v.detach(), W.detach(), layer.tau, True,
                      torch.from_numpy(o_ref).float().to(DEV), g, grad_dtype=torch.float32)
    refs = oracle.backward_heads(f["q"], f["k"], f["v"], f["W"], layer.tau, True, f["g"])
    for name, a, r in zip(("dq", "dk", "dv", "dW"), g32, refs):
        err = np.abs(_f64(a) - r).max() / np.abs(r).max()
        assert err <= 3 * 2.0 ** -8, (name, err)


@pytest.mark.parametrize("dtype,impl", [(torch.float32, "simt"), (torch.bfloat16, "auto")])
def test_sgd_step_on_the_hash_planes_lowers_the_loss(dtype, impl):
    torch.manual_seed(2)
    layer = LY.init_like_attention(LY.RaceMultiHeadAttention(
        128, 2, L=4, P=6, tau=0.5, causal=True, impl=impl, device=DEV, dtype=dtype, seed=3))
    for p in (layer.wq.weight, layer.wk.weight, layer.wv.weight, layer.wo.weight):
        p.requires_grad_(False)
    x = torch.randn(1, 700, 128, device=DEV, dtype=dtype)
    target = torch.randn(1, 700, 128, device=DEV, dtype=dtype)

    def loss_of():
        return ((layer(x).float() - target.float()) ** 2).mean()

    loss0 = loss_of()
    loss0.backward()
    gW = layer.planes.grad
    assert torch.isfinite(gW).all() and gW.abs().max() > 0
    eta = 0.05 if dtype == torch.float32 else 0.5
    with torch.no_grad():
        step = eta / gW.norm()
        layer.planes -= step * gW
        loss1 = loss_of()
    assert loss1.item() < loss0.item()
    if dtype == torch.float32:
        # first-order decrease: loss1 ~ loss0 - step |gW|^2
        predicted = loss0.item() - step.item() * gW.norm().item() ** 2
        assert abs(loss1.item() - predicted) <= 0.5 * (loss0.item() - predicted)
