"""Pins of the float64 oracle against facts fixed outside the oracle itself.

Every test here runs on the CPU.  Each pin is chosen so that a plausible slip in
the oracle (a dropped 1/sqrt(L), a wrong sign in the corner set, a transposed
projection, an exclusive instead of inclusive causal mask, a missing softmax
Jacobian term) breaks at least one of them:

* closed forms of the angular kernel and of the SRP collision probability
  (hand-derived golden values);
* the soft hash for one hyperplane (hand-derived golden values) and the exact
  identity softmax-over-corners == product of logistic factors;
* Monte-Carlo collision rate of the hard hash vs (1 - theta/pi)^P;
* E_W[phi(q).phi(k)] vs a Gauss-Hermite quadrature of the per-plane collision
  function, and Sheppard's law in the tau -> 0 limit;
* brute force: blocked sketch form == O(N^2) definition, causal prefix property,
  convexity of the outputs;
* convergence to exact angular attention as L grows (slope -1/2);
* gradients: central finite differences and torch float64 autograd of an
  independently written forward.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _pair_at_angle(theta, d, rng):
    a = rng.standard_normal(d)
    a /= np.linalg.norm(a)
    b = rng.standard_normal(d)
    b -= a * (a @ b)
    b /= np.linalg.norm(b)
    return a, math.cos(theta) * a + math.sin(theta) * b


# --------------------------------------------------------------------------- #
# closed forms
# --------------------------------------------------------------------------- #
def test_angular_kernel_golden():
    g = json.load(open(os.path.join(GOLDEN, "angular_kernel.json")))
    rng = np.random.default_rng(0)
    for c in g["cases"]:
        th = float(Fraction(c["theta_over_pi"])) * math.pi
        q, k = _pair_at_angle(th, 8, rng)
        got = oracle.angular_kernel(3.0 * q[None], 0.5 * k[None], c["P"])[0, 0]
        assert got == pytest.approx(float(Fraction(c["value"])), abs=1e-12)


def test_soft_hash_single_plane_golden():
    g = json.load(open(os.path.join(GOLDEN, "soft_hash_p1.json")))
    for c in g["cases"]:
        W = np.array(c["w"], dtype=np.float64).reshape(1, 2, 1)
        p = oracle.soft_hash(np.array([c["x"]]), W, c["tau"])[0, 0]
        t = c["two_u_over_tau"]
        assert p[1] == pytest.approx(1.0 / (1.0 + math.exp(-t)), abs=1e-14)
        assert p[0] == pytest.approx(1.0 / (1.0 + math.exp(t)), abs=1e-14)
        assert p[1] == pytest.approx(float(c["p_plus_decimal"]), abs=1e-11)


@pytest.mark.parametrize("P", [1, 3, 6, 8])
@pytest.mark.parametrize("tau", [0.25, 0.5, 2.0])
def test_corner_softmax_is_product_of_logistic_factors(P, tau):
    """softmax_b(<c_b,u>/tau) == prod_p sigmoid(2 c_bp u_p / tau), an exact identity:
    the numerator factorises over planes and the normaliser is prod_p 2cosh(u_p/tau)."""
    rng = np.random.default_rng(P)
    L, d, n = 3, 16, 20
    W = rng.standard_normal((L, d, P))
    x = rng.standard_normal((n, d)) * 3.0
    p = oracle.soft_hash(x, W, tau)
    xh = x / np.linalg.norm(x, axis=1, keepdims=True)
    u = np.einsum("nd,ldp->nlp", xh, W)
    bits = (np.arange(1 << P)[:, None] >> np.arange(P)[None, :]) & 1   # [R, P]
    sp = 1.0 / (1.0 + np.exp(-2.0 * u / tau))                           # sigma(+2u/tau)
    sm = 1.0 / (1.0 + np.exp(2.0 * u / tau))                            # sigma(-2u/tau)
    fac = np.where(bits[None, None], sp[:, :, None, :], sm[:, :, None, :])
    assert np.allclose(p, fac.prod(axis=-1), rtol=1e-12, atol=1e-300)


def test_phi_blocks_sum_and_range():
    rng = np.random.default_rng(3)
    L, d, P, n = 5, 64, 6, 50
    W = rng.standard_normal((L, d, P))
    f = oracle.phi(rng.standard_normal((n, d)), W, 0.5)
    blocks = f.reshape(n, L, 1 << P)
    assert np.allclose(blocks.sum(-1), 1.0 / math.sqrt(L), rtol=1e-13)
    assert (f > 0).all() and (f < 1).all()
    # phi(x).phi(x) summed over tables of a softmax block is at most 1
    assert (np.einsum("nk,nk->n", f, f) <= 1.0 + 1e-12).all()


def test_zero_vector_gives_uniform_assignment():
    W = np.random.default_rng(4).standard_normal((2, 8, 3))
    p = oracle.soft_hash(np.zeros((1, 8)), W, 0.3)
    assert np.allclose(p, 1.0 / 8, rtol=1e-14)


# --------------------------------------------------------------------------- #
# LSH facts
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("P", [1, 4, 6, 8])
def test_hard_hash_collision_rate(P):
    """Signed random projections collide with probability (1 - theta/pi)^P."""
    rng = np.random.default_rng(10 + P)
    n_draw = 100_000
    for theta in (0.1, 0.7, 1.3, 2.1, 3.0):
        q, k = _pair_at_angle(theta, 64, rng)
        W = rng.standard_normal((n_draw, 64, P))
        hq = oracle.hard_hash(q[None], W)[0]
        hk = oracle.hard_hash(k[None], W)[0]
        rate = np.mean(hq == hk)
        p = (1.0 - theta / math.pi) ** P
        sig = math.sqrt(max(p * (1 - p), 1e-12) / n_draw)
        assert abs(rate - p) <= 5 * sig + 1e-9, (theta, rate, p)


def test_soft_hash_tends_to_hard_hash():
    """At tau -> 0 each softmax block becomes the one-hot of the SRP bucket id."""
    rng = np.random.default_rng(5)
    L, d, P = 6, 32, 5
    W = rng.standard_normal((L, d, P))
    x = rng.standard_normal((40, d))
    p = oracle.soft_hash(x, W, 1e-6)
    h = oracle.hard_hash(x, W)
    onehot = np.zeros_like(p)
    np.put_along_axis(onehot, h[..., None], 1.0, axis=-1)
    # a plane with |u| < ~1e-4 would not have saturated; the seeded draw has none
    assert np.abs(p - onehot).max() < 1e-6


def _kappa_quadrature(theta, tau, n=96):
    """E[(1 + tanh(a/tau) tanh(b/tau))/2] for (a, b) standard normal with
    correlation cos(theta), by tensor Gauss-Hermite quadrature."""
    x, w = np.polynomial.hermite.hermgauss(n)
    rho = math.cos(theta)
    a = math.sqrt(2.0) * x[:, None]
    b = rho * a + math.sqrt(max(1.0 - rho * rho, 0.0)) * math.sqrt(2.0) * x[None, :]
    f = 0.5 * (1.0 + np.tanh(a / tau) * np.tanh(b / tau))
    return float((w[:, None] * w[None, :] * f).sum() / math.pi)


def test_kappa_quadrature_matches_sheppard_at_small_tau():
    """Sheppard: P(sign a == sign b) = 1 - theta/pi.  The soft collision function
    approaches it as tau shrinks (the quadrature of a near-step is only good to
    ~1e-2 at tau = 0.1, so the check is on the trend and a loose bound)."""
    for theta in (0.3, 1.0, 2.0):
        gaps = [abs(_kappa_quadrature(theta, t, n=250) - (1 - theta / math.pi))
                for t in (0.4, 0.1)]
        assert gaps[1] < 1e-2 and gaps[1] < gaps[0] / 3, (theta, gaps)


@pytest.mark.parametrize("tau", [0.5, 1.0])
def test_expected_soft_kernel_is_kappa_power(tau):
    """E_W[phi(q).phi(k)] = kappa_tau(theta)^P: planes are independent and the pair
    of projections of one plane is a correlated Gaussian pair.  The mean over L
    tables is a Monte-Carlo estimate of it."""
    rng = np.random.default_rng(21)
    P, d, L = 4, 32, 20_000
    for theta in (0.4, 1.2, 2.4):
        q, k = _pair_at_angle(theta, d, rng)
        W = rng.standard_normal((L, d, P))
        pq = oracle.soft_hash(q[None], W, tau)[0]
        pk = oracle.soft_hash(k[None], W, tau)[0]
        per_table = np.sum(pq * pk, axis=1)                 # L iid samples
        est = float(oracle.phi(q[None], W, tau)[0] @ oracle.phi(k[None], W, tau)[0])
        assert est == pytest.approx(per_table.mean(), rel=1e-12)
        target = _kappa_quadrature(theta, tau) ** P
        se = per_table.std() / math.sqrt(L)
        assert abs(est - target) <= 5 * se, (theta, est, target, se)


# --------------------------------------------------------------------------- #
# brute force and invariants
# --------------------------------------------------------------------------- #
def _rand_case(rng, N, d=16, L=3, P=3):
    q = rng.standard_normal((N, d))
    k = rng.standard_normal((N, d))
    v = rng.standard_normal((N, d))
    W = rng.standard_normal((L, d, P))
    return q, k, v, W


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,block", [(1, 4), (7, 3), (64, 16), (131, 32)])
def test_blocked_equals_direct(causal, N, block):
    rng = np.random.default_rng(N)
    q, k, v, W = _rand_case(rng, N)
    o1, d1 = oracle.forward(q, k, v, W, 0.4, causal, block=block)
    o2, d2 = oracle.direct_forward(q, k, v, W, 0.4, causal)
    assert np.allclose(o1, o2, rtol=1e-12, atol=1e-12)
    assert np.allclose(d1, d2, rtol=1e-12)
    rows = np.array(sorted({0, N // 2, N - 1}))
    o3, d3 = oracle.forward_rows(q, k, v, W, 0.4, causal, rows, block=5)
    assert np.allclose(o3, o2[rows], rtol=1e-12, atol=1e-12)


def test_partial_sums_over_a_key_split_give_the_definition():
    """Unnormalised sums over disjoint key ranges add up to the O(N^2) definition: their
    sum divided by the summed mass is o_i, the summed mass is den_i, and a causal mask
    over the last range reproduces the causal rows."""
    rng = np.random.default_rng(31)
    N = 50
    q, k, v, W = _rand_case(rng, N)
    for causal in (False, True):
        o, den = oracle.direct_forward(q, k, v, W, 0.4, causal)
        rows = np.array([3, 29, 49])
        num = np.zeros((len(rows), v.shape[1]))
        mass = np.zeros(len(rows))
        for s, e in ((0, 17), (17, 18), (18, 50)):
            mask = (np.arange(s, e)[None, :] <= rows[:, None]) if causal else None
            a, b = oracle.partial_sums(q[rows], k[s:e], v[s:e], W, 0.4, mask, block=4)
            num += a
            mass += b
        assert np.allclose(mass, den[rows], rtol=1e-12)
        assert np.allclose(num / mass[:, None], o[rows], rtol=1e-12, atol=1e-13)
        o2, d2 = oracle.forward_rows(q, k, v, W, 0.4, causal, rows)
        assert np.allclose(num / mass[:, None], o2, rtol=1e-12, atol=1e-13)


def test_direct_matches_pure_python_loops():
    """A third route written with scalar loops on a 5-token case."""
    rng = np.random.default_rng(8)
    N, d, L, P, tau = 5, 3, 2, 2, 0.6
    q, k, v, W = _rand_case(rng, N, d, L, P)

    def p_of(x, l):
        nx = math.sqrt(sum(t * t for t in x))
        u = [sum(W[l, e, p] * x[e] / nx for e in range(d)) for p in range(P)]
        logits = [sum((1 if (b >> p) & 1 else -1) * u[p] for p in range(P)) / tau
                  for b in range(1 << P)]
        m = max(logits)
        e = [math.exp(t - m) for t in logits]
        return [t / sum(e) for t in e]

    for causal in (False, True):
        o, _ = oracle.direct_forward(q, k, v, W, tau, causal)
        for i in range(N):
            num = [0.0] * d
            den = 0.0
            for j in range(N):
                if causal and j > i:
                    continue
                a = sum(sum(x * y for x, y in zip(p_of(q[i], l), p_of(k[j], l)))
                        for l in range(L)) / L
                den += a
                for c in range(d):
                    num[c] += a * v[j, c]
            assert np.allclose(o[i], [t / den for t in num], rtol=1e-12)


def test_causal_row_equals_noncausal_on_prefix():
    rng = np.random.default_rng(9)
    q, k, v, W = _rand_case(rng, 40)
    oc, _ = oracle.forward(q, k, v, W, 0.5, True, block=7)
    for i in (0, 1, 13, 39):
        on, _ = oracle.forward(q[:i + 1], k[:i + 1], v[:i + 1], W, 0.5, False, block=7)
        assert np.allclose(oc[i], on[i], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_outputs_are_convex_combinations(causal):
    rng = np.random.default_rng(11)
    q, k, v, W = _rand_case(rng, 90)
    o, den = oracle.forward(q, k, v, W, 0.3, causal, block=16)
    assert (den > 0).all()
    for i in range(len(o)):
        vv = v[: i + 1] if causal else v
        assert (o[i] >= vv.min(0) - 1e-12).all() and (o[i] <= vv.max(0) + 1e-12).all()
    if causal:
        assert np.allclose(o[0], v[0], rtol=1e-13)


def test_degenerate_identical_keys_return_mean_value():
    """All keys equal: every weight a_ij is the same, so o_i is the plain mean."""
    rng = np.random.default_rng(12)
    N, d = 20, 16
    q = rng.standard_normal((N, d))
    k = np.tile(rng.standard_normal((1, d)), (N, 1))
    v = rng.standard_normal((N, d))
    W = rng.standard_normal((4, d, 3))
    o, _ = oracle.forward(q, k, v, W, 0.5, False)
    assert np.allclose(o, v.mean(0), rtol=1e-12, atol=1e-13)
    oc, _ = oracle.forward(q, k, v, W, 0.5, True, block=6)
    assert np.allclose(oc, np.cumsum(v, 0) / np.arange(1, N + 1)[:, None], rtol=1e-12)


# --------------------------------------------------------------------------- #
# convergence (the error bound's variance term falls as 1/sqrt(L))
# --------------------------------------------------------------------------- #
def test_converges_to_exact_angular_attention():
    rng = np.random.default_rng(13)
    N, d, P = 24, 16, 4
    q = rng.standard_normal((N, d))
    k = np.concatenate([q[:12] + 0.3 * rng.standard_normal((12, d)),
                        rng.standard_normal((12, d))])
    v = rng.standard_normal((N, d))
    exact = oracle.exact_angular_attention(q, k, v, P, causal=False)
    Ls = [16, 64, 256, 1024, 4096]
    errs = []
    for L in Ls:
        e = []
        for seed in range(6):
            W = np.random.default_rng(1000 + 7 * seed + L).standard_normal((L, d, P))
            o, _ = oracle.forward(q, k, v, W, 1e-4, False)
            e.append(np.sqrt(np.mean((o - exact) ** 2)))
        errs.append(np.mean(e))
    slope = np.polyfit(np.log(Ls), np.log(errs), 1)[0]
    assert -0.65 < slope < -0.35, (slope, errs)
    assert errs[-1] < 0.02 * np.sqrt(np.mean(v ** 2))


def test_soft_estimator_limit_is_kappa_attention():
    """For tau > 0 the L -> inf limit is attention with weights kappa_tau(theta)^P."""
    rng = np.random.default_rng(14)
    N, d, P, tau, L = 6, 16, 3, 0.5, 60_000
    q = rng.standard_normal((N, d))
    k = rng.standard_normal((N, d))
    v = rng.standard_normal((N, d))
    W = rng.standard_normal((L, d, P))
    o, _ = oracle.forward(q, k, v, W, tau, False)
    c = np.clip(oracle.normalize(q) @ oracle.normalize(k).T, -1, 1)
    K = np.vectorize(lambda t: _kappa_quadrature(math.acos(t), tau))(c) ** P
    target = K @ v / K.sum(1, keepdims=True)
    assert np.abs(o - target).max() < 0.01


# --------------------------------------------------------------------------- #
# gradients
# --------------------------------------------------------------------------- #
def _loss(q, k, v, W, tau, causal, g):
    o, _ = oracle.direct_forward(q, k, v, W, tau, causal)
    return float(np.sum(o * g))


@pytest.mark.parametrize("causal", [False, True])
def test_backward_finite_differences(causal):
    rng = np.random.default_rng(15 + causal)
    N, d, L, P, tau = 5, 4, 2, 2, 0.7
    q, k, v, W = _rand_case(rng, N, d, L, P)
    g = rng.standard_normal((N, d))
    dq, dk, dv, dW = oracle.backward(q, k, v, W, tau, causal, g, block=2)
    dq2, dk2, dv2, dW2 = oracle.direct_backward(q, k, v, W, tau, causal, g)
    for a, b in ((dq, dq2), (dk, dk2), (dv, dv2), (dW, dW2)):
        assert np.allclose(a, b, rtol=1e-10, atol=1e-12)
    h = 1e-6
    for name, X, G in (("q", q, dq), ("k", k, dk), ("v", v, dv), ("W", W, dW)):
        num = np.zeros_like(X)
        it = np.nditer(X, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            Xp = X.copy(); Xp[idx] += h
            Xm = X.copy(); Xm[idx] -= h
            args = {"q": q, "k": k, "v": v, "W": W}
            args[name] = Xp
            fp = _loss(args["q"], args["k"], args["v"], args["W"], tau, causal, g)
            args[name] = Xm
            fm = _loss(args["q"], args["k"], args["v"], args["W"], tau, causal, g)
            num[idx] = (fp - fm) / (2 * h)
        scale = max(np.abs(num).max(), 1e-3)
        assert np.abs(num - G).max() <= 1e-6 * scale, (name, np.abs(num - G).max(), scale)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_against_torch_autograd(causal):
    """torch float64 autograd of a forward written independently (logistic-factor
    form of the soft hash, dense masked attention) must give the oracle's gradient."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(17 + causal)
    N, d, L, P, tau = 37, 8, 3, 4, 0.45
    q, k, v, W = _rand_case(rng, N, d, L, P)
    g = rng.standard_normal((N, d))
    tq, tk, tv, tW = (torch.tensor(a, dtype=torch.float64, requires_grad=True)
                      for a in (q, k, v, W))
    bits = torch.tensor((np.arange(1 << P)[:, None] >> np.arange(P)[None, :]) & 1,
                        dtype=torch.bool)

    def feat(x):
        xh = x / x.norm(dim=1, keepdim=True).clamp_min(1e-12)
        u = torch.einsum("nd,ldp->nlp", xh, tW)
        s = torch.sigmoid(2 * u / tau)                         # [n, L, P]
        f = torch.where(bits[None, None], s[:, :, None, :], 1 - s[:, :, None, :]).prod(-1)
        return f.reshape(x.shape[0], -1) / math.sqrt(L)

    A = feat(tq) @ feat(tk).T
    if causal:
        A = torch.tril(A)
    o = A @ tv / A.sum(1, keepdim=True)
    (o * torch.tensor(g)).sum().backward()
    dq, dk, dv, dW = oracle.backward(q, k, v, W, tau, causal, g, block=8)
    for a, t in ((dq, tq), (dk, tk), (dv, tv), (dW, tW)):
        ref = t.grad.numpy()
        assert np.allclose(a, ref, rtol=1e-9, atol=1e-11 * np.abs(ref).max())


def test_backward_uses_given_output():
    """Passing the oracle's own output changes nothing."""
    rng = np.random.default_rng(19)
    q, k, v, W = _rand_case(rng, 30)
    g = rng.standard_normal(v.shape)
    o, _ = oracle.forward(q, k, v, W, 0.5, True)
    a = oracle.backward(q, k, v, W, 0.5, True, g)
    b = oracle.backward(q, k, v, W, 0.5, True, g, out=o)
    for x, y in zip(a, b):
        assert np.allclose(x, y, rtol=1e-13, atol=1e-15)


def test_multihead_wrappers():
    rng = np.random.default_rng(20)
    H, N, d = 3, 17, 8
    q, k, v = (rng.standard_normal((H, N, d)) for _ in range(3))
    W = rng.standard_normal((2, d, 3))
    g = rng.standard_normal((H, N, d))
    o, den = oracle.forward_heads(q, k, v, W, 0.5, True, block=5)
    dq, dk, dv, dW = oracle.backward_heads(q, k, v, W, 0.5, True, g, block=5)
    tot = np.zeros_like(W)
    for h in range(H):
        oh, dh = oracle.forward(q[h], k[h], v[h], W, 0.5, True)
        assert np.allclose(o[h], oh) and np.allclose(den[h], dh)
        tot += oracle.backward(q[h], k[h], v[h], W, 0.5, True, g[h])[3]
    assert np.allclose(dW, tot)


# --------------------------------------------------------------------------- #
# hard-hash RACE (classic count arrays)
# --------------------------------------------------------------------------- #
def test_hard_forward_matches_scalar_loops():
    """A second route with explicit loops over tables and keys on a small case."""
    rng = np.random.default_rng(40)
    N, d, L, P = 23, 5, 3, 2
    q, k, v, W = _rand_case(rng, N, d, L, P)
    for causal in (False, True):
        o, den = oracle.hard_forward(q, k, v, W, causal)
        hq, hk = oracle.hard_hash(q, W), oracle.hard_hash(k, W)
        for i in range(N):
            cnt, acc = 0, np.zeros(d)
            for j in range(N):
                if causal and j > i:
                    continue
                m = sum(int(hq[i, l] == hk[j, l]) for l in range(L))
                cnt += m
                acc += m * v[j]
            assert den[i] == cnt
            assert np.allclose(o[i], acc / cnt if cnt else 0.0, rtol=1e-13, atol=1e-14)


def test_hard_forward_is_the_soft_estimator_as_tau_goes_to_zero():
    """With tau -> 0 every soft assignment is one-hot at the hard bucket, so the soft
    weights phi(q).phi(k) become (number of colliding tables) / L."""
    rng = np.random.default_rng(41)
    q, k, v, W = _rand_case(rng, 40, 8, 4, 3)
    o_h, den_h = oracle.hard_forward(q, k, v, W, True)
    with np.errstate(invalid="ignore"):   # rows with no collision: 0/0 in the soft form
        o_s, den_s = oracle.direct_forward(q, k, v, W, 1e-6, True)
    ok = den_h > 0
    assert ok.sum() > 30
    assert np.allclose(den_s[ok] * 4, den_h[ok], rtol=1e-6, atol=1e-6)
    assert np.allclose(o_s[ok], o_h[ok], rtol=1e-6, atol=1e-6)


def test_hard_counts_are_histograms_and_give_the_noncausal_estimator():
    rng = np.random.default_rng(42)
    q, k, v, W = _rand_case(rng, 200, 8, 5, 4)
    C, S = oracle.hard_counts(k, v, W)
    assert (C.sum(axis=1) == 200).all()
    assert np.allclose(S.sum(axis=1), np.tile(v.sum(axis=0), (5, 1)))
    hq = oracle.hard_hash(q, W)
    num = sum(S[l, hq[:, l]] for l in range(5))
    den = sum(C[l, hq[:, l]] for l in range(5))
    o, den2 = oracle.hard_forward(q, k, v, W, False)
    assert (den == den2).all()
    nz = den > 0
    assert np.allclose(num[nz] / den[nz, None], o[nz], rtol=1e-12)
