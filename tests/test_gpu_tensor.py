"""GPU parity of the tensor-core (tcgen05) path against the float64 oracle.

bf16 q, k, v (the oracle reads the same bf16 values, upcast), float32 W; outputs
compared in float32 (out_dtype = fp32) with max|diff| <= 2e-3 * max|V|, the bf16
criterion of the method's evaluation.  Shapes cover one and several row groups,
one and several segments (multi-segment causal sweeps start from scanned segment
sums), ragged tails and the 128-token chunk edges.

One case uses a looser bound (TOL_FEW): with only L <= 3 tables and a sharp kernel
(tau = 0.25, P = 8) the estimate averages over few tables, and the bf16 roundings (unit
roundoff 2^-8) of phi(q), phi(k) and of one of (state, in-chunk weight) each perturb a
weight a_ij by up to 2^-8 relative; the output error is then at most about
3 * 2^-8 * max|v_j - o_i| <= 6 * 2^-8 * max|V| ~ 2.3e-2 * max|V|.  Observed errors sit
near 2e-3; the test allows 4e-3.
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
TOL_FEW = 4e-3


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


@pytest.mark.parametrize("L,P,tau", [(1, 7, 0.5), (4, 6, 0.5), (4, 8, 0.25), (5, 7, 0.4)])
@pytest.mark.parametrize("causal", [True, False])
def test_tensor_table_shapes(L, P, tau, causal):
    err, _ = _run(700, H=3, L=L, P=P, tau=tau, causal=causal, clusters=16, seed=L * 10 + P)
    assert err <= TOL, err


@pytest.mark.parametrize("L", [2, 3])
def test_tensor_few_tables_sharp_kernel(L):
    err, _ = _run(700, H=3, L=L, P=8, tau=0.25, causal=True, clusters=16, seed=L * 10 + 8)
    assert err <= TOL_FEW, err


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


# ------------------------------------------------------------------ full-size workloads
def _full(name, device_inputs=True):
    wl = I.WORKLOADS[name]
    x = I.make_inputs(wl, DEV)
    return wl, x


def _oracle_rows(wl, x, head, rows):
    hi = int(max(rows)) + 1 if wl.causal else wl.N
    f = lambda t: t[head, :hi].double().cpu().numpy()  # noqa: E731
    W = x["W"].double().cpu().numpy()
    return oracle.forward_rows(f(x["q"]), f(x["k"]), f(x["v"]), W, wl.tau, wl.causal,
                               np.asarray(rows))


def _oracle_tail_rows(pool, wl, x, head, n_rows):
    """Causal outputs of the last n_rows rows of one head from the definition: the keys
    are cut into ranges whose unnormalised sums (oracle.partial_sums) the host cores
    compute in parallel; the range that overlaps the rows carries the causal mask."""
    N = wl.N
    r0 = N - n_rows
    rows = np.arange(r0, N)
    qr = x["q"][head, r0:].double().cpu().numpy()
    kh = x["k"][head].float().cpu().numpy()        # exact: the inputs are bf16
    vh = x["v"][head].float().cpu().numpy()
    W = x["W"].double().cpu().numpy()
    span = 65536
    tasks = [(qr, kh[s:min(s + span, r0)], vh[s:min(s + span, r0)], W, wl.tau, None)
             for s in range(0, r0, span)]
    mask = (np.arange(r0, N)[None, :] <= rows[:, None]).astype(np.float64)
    tasks.append((qr, kh[r0:], vh[r0:], W, wl.tau, mask))
    num = np.zeros((n_rows, wl.d))
    den = np.zeros(n_rows)
    for a, b in pool.starmap(oracle.partial_sums, tasks, chunksize=1):
        num += a
        den += b
    return num / den[:, None]


def test_tensor_headline_4m_causal_rows_and_properties(oracle_pool):
    """The causal 4M-token workload (8 heads, L = 16, P = 8, tau = 0.25) in the launch
    configuration the benchmark times.  Compared element by element with the oracle:
    rows at the start (chunk and segment edges) and the last 256 rows of two heads,
    whose state has absorbed every earlier key; every row is checked for convexity and a
    prefix run for causality."""
    name = "causal_bf16_h8_n4194304_d64_L16_P8_clustered256"
    wl, x = _full(name)
    q, k, v, W = x["q"], x["k"], x["v"], x["W"]
    out = ra.forward(q, k, v, W, wl.tau, True, out_dtype=torch.float32)
    outb = ra.forward(q, k, v, W, wl.tau, True)            # the benchmark's bf16 output
    torch.cuda.synchronize()
    assert ra.race_device_status() == 0
    vmax = v.float().abs().max().item()
    # bf16 output is the float32 output rounded once
    assert ((outb.float() - out).abs() <= out.abs() * 2.0 ** -7 + 1e-6 * vmax).all()
    rows = [0, 1, 2, 127, 128, 129, 255, 256, 1000, 4095, 8191, 12345, 16383]
    for head in (0, 5):
        ref, _ = _oracle_rows(wl, x, head, rows)
        got = out[head, rows].double().cpu().numpy()
        assert np.abs(got - ref).max() / vmax <= TOL, head
    for head in (3, 7):
        ref = _oracle_tail_rows(oracle_pool, wl, x, head, 256)
        got = out[head, wl.N - 256:].double().cpu().numpy()
        assert np.abs(got - ref).max() / vmax <= TOL, head
    # convexity: every o_i lies within the running column range of v_0..v_i
    for head in range(wl.H):
        vf = v[head].float()
        hi = torch.cummax(vf, dim=0).values
        lo = torch.cummin(vf, dim=0).values
        assert (out[head] <= hi + 1e-4 * vmax).all() and (out[head] >= lo - 1e-4 * vmax).all()
    # causality: a run on the first 2^20 tokens gives the same rows
    Np = 1 << 20
    short = ra.forward(q[:, :Np].contiguous(), k[:, :Np].contiguous(), v[:, :Np].contiguous(),
                       W, wl.tau, True, out_dtype=torch.float32)
    assert (short - out[:, :Np]).abs().max().item() <= 1e-5 * vmax


def test_tensor_noncausal_262k_all_rows_of_two_heads(oracle_pool):
    """The non-causal throughput workload (2 x 16 heads, N = 262,144, L = 16, P = 6):
    every output row of two heads against the oracle's sketch form."""
    name = "noncausal_bf16_b2h16_n262144_d64_L16_P6"
    wl, x = _full(name)
    out = ra.forward(x["q"], x["k"], x["v"], x["W"], wl.tau, False, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ra.race_device_status() == 0
    vmax = x["v"].float().abs().max().item()
    W = x["W"].double().cpu().numpy()
    heads = (0, 31)
    tasks = [(x["q"][h].float().cpu().numpy(), x["k"][h].float().cpu().numpy(),
              x["v"][h].float().cpu().numpy(), W, wl.tau, False) for h in heads]
    refs = oracle_pool.starmap(oracle.forward, tasks, chunksize=1)
    for h, (ref, _) in zip(heads, refs):
        got = out[h].double().cpu().numpy()
        assert np.abs(got - ref).max() / vmax <= TOL, h
