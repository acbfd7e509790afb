"""Streaming (race_forward_stream): RACE attention over consecutive blocks of a sequence
with the sketch state carried between calls, as in chunked prefill and in decoding.

* Blocks of unequal length, processed one after another with the carried state, give the
  outputs of one causal call over the whole sequence (tensor-core and CUDA-core paths).
* Token-by-token decoding (N = 1 per call) gives the same outputs.
* The state after the last block is the bucket aggregation of the whole sequence,
  sum_j p(k_j)^T [v_j | 1] with p the unscaled corner probabilities, checked against the
  oracle; it can be updated in place.
* Non-causal blocks attend to every key of the block and of earlier blocks.

Tolerances: outputs against the oracle 2e-3 * max|V| (tensor cores) / 2e-5 (CUDA cores,
bf16 inputs); with L <= 3 tables and every output read through the bf16 copy of the state
(decoding), the few-table bound of test_gpu_tensor.py (4e-3) applies; the state is a float32 sum of the same terms in another order on the CUDA
cores (1e-5 of its largest entry) and of bf16-rounded corner probabilities on the tensor
cores (each term within 2^-8, so 2^-8 of the sum of absolute values, the masses being
positive).
"""
import numpy as np
import pytest
import torch

import oracle
from linear_lsh_sketch_race_b200 import inputs as I
from linear_lsh_sketch_race_b200 import race_attn as ra

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _f64(t):
    return t.detach().double().cpu().numpy()


def _case(N, H, L, P, tau, seed, dtype="bf16"):
    wl = I.Workload("stream", H=H, N=N, d=64, L=L, P=P, tau=tau, causal=True, dtype=dtype,
                    seed=seed, clusters=8)
    x = I.make_inputs(wl, "cpu")
    return wl, x, {k: v.to(DEV) for k, v in x.items()}


def _oracle_state(x, W, tau):
    """sum_j p(k_j)^T [v_j | 1] per head, p = phi * sqrt(L) (unscaled corner probs), and
    the same sum of absolute values of the terms."""
    L = W.shape[0]
    states, absums = [], []
    for h in range(x["k"].shape[0]):
        p = oracle.phi(_f64(x["k"][h]), _f64(W), tau) * np.sqrt(L)
        vv = np.concatenate([_f64(x["v"][h]), np.ones((p.shape[0], 1))], axis=1)
        states.append(p.T @ vv)
        absums.append(p.T @ np.abs(vv))
    return np.stack(states), np.stack(absums)


@pytest.mark.parametrize("impl,L,P,tau", [("tensor", 2, 8, 0.25), ("tensor", 4, 6, 0.5),
                                          ("simt", 3, 4, 0.5)])
def test_blocks_with_carried_state_equal_one_call(impl, L, P, tau):
    N, H = 1000, 2
    wl, x, g = _case(N, H, L, P, tau, seed=P)
    whole = ra.forward(g["q"], g["k"], g["v"], g["W"], tau, True, out_dtype=torch.float32,
                       impl=impl)
    cuts = [0, 129, 130, 700, N]
    state = None
    outs = []
    for s0, s1 in zip(cuts[:-1], cuts[1:]):
        sl = lambda t: t[:, s0:s1].contiguous()  # noqa: E731
        o, state = ra.forward_stream(sl(g["q"]), sl(g["k"]), sl(g["v"]), g["W"], tau, True,
                                     state=state, out_dtype=torch.float32, impl=impl)
        outs.append(o)
    torch.cuda.synchronize()
    assert ra.race_device_status() == 0
    got = torch.cat(outs, dim=1)
    vmax = g["v"].float().abs().max().item()
    ref, _ = oracle.forward_heads(_f64(x["q"]), _f64(x["k"]), _f64(x["v"]), _f64(x["W"]),
                                  tau, True)
    tol = 2e-3 if impl == "tensor" else 2e-5
    assert np.abs(_f64(got) - ref).max() / vmax <= tol
    assert (got - whole).abs().max().item() / vmax <= tol
    # the final state: the bucket aggregation of the whole sequence
    S, Sabs = _oracle_state(x, x["W"], tau)
    assert state.shape == (H, L << P, 65)
    if impl == "tensor":
        assert (np.abs(_f64(state) - S) <= 2.0 ** -8 * Sabs + 1e-6 * np.abs(S).max()).all()
    else:
        assert np.abs(_f64(state) - S).max() <= 1e-5 * np.abs(S).max()


@pytest.mark.parametrize("impl,L,P", [("tensor", 2, 7), ("tensor", 8, 6), ("simt", 2, 7)])
def test_token_by_token_decoding(impl, L, P):
    N, H, tau = 64, 2, 0.5
    wl, x, g = _case(N, H, L, P, tau, seed=9)
    state = torch.zeros(ra.state_shape(H, L, P), dtype=torch.float32, device=DEV)
    outs = []
    for i in range(N):
        sl = lambda t: t[:, i:i + 1].contiguous()  # noqa: E731
        o, state = ra.forward_stream(sl(g["q"]), sl(g["k"]), sl(g["v"]), g["W"], tau, True,
                                     state=state, out_dtype=torch.float32, impl=impl,
                                     inplace=True)
        outs.append(o)
    torch.cuda.synchronize()
    assert ra.race_device_status() == 0
    got = torch.cat(outs, dim=1)
    ref, _ = oracle.forward_heads(_f64(x["q"]), _f64(x["k"]), _f64(x["v"]), _f64(x["W"]),
                                  tau, True)
    vmax = np.abs(_f64(x["v"])).max()
    tol = (2e-3 if L > 3 else 4e-3) if impl == "tensor" else 2e-5
    assert np.abs(_f64(got) - ref).max() / vmax <= tol


def test_noncausal_block_attends_to_block_and_history():
    N, H, L, P, tau = 600, 2, 4, 6, 0.5
    wl, x, g = _case(N, H, L, P, tau, seed=4)
    s = 250
    sl = lambda t, a, b: t[:, a:b].contiguous()  # noqa: E731
    _, state = ra.forward_stream(sl(g["q"], 0, s), sl(g["k"], 0, s), sl(g["v"], 0, s), g["W"],
                                 tau, True, out_dtype=torch.float32)
    o, _ = ra.forward_stream(sl(g["q"], s, N), sl(g["k"], s, N), sl(g["v"], s, N), g["W"],
                             tau, False, state=state, out_dtype=torch.float32)
    torch.cuda.synchronize()
    # reference: every query of the second block attends to all N keys
    f = {k: _f64(v) for k, v in x.items()}
    ref = np.stack([oracle.forward_rows(f["q"][h], f["k"][h], f["v"][h], f["W"], tau, False,
                                        np.arange(s, N))[0] for h in range(H)])
    vmax = np.abs(f["v"]).max()
    assert np.abs(_f64(o) - ref).max() / vmax <= 2e-3
