"""Classic RACE with hard hashes (race_hard_forward, race_hard_hash) against the oracle.

Bucket ids and collision counts are integers and are compared exactly.  The sign of each
projection x . W_l[:,p] is decided in float32 by the kernels and in float64, after
normalising x, by the oracle; both decide the same wherever the projection is clear of
zero.  The exactness cases therefore use inputs on which no projection can be near zero:
odd integer planes and integer rows whose coordinates sum to an odd number, so every
projection is an odd integer (exact in float32; at least 1 / |x| after normalising).  On
real-valued inputs the ids are checked to agree wherever the projection exceeds the float32
rounding bound of its 64-term dot product.  Outputs are float32 sums of exact values in
another order: 1e-5 * max|V|.
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


def _case(N, H, L, P, causal, seed, dtype="bf16", clusters=0):
    wl = I.Workload("hard", H=H, N=N, d=64, L=L, P=P, tau=1.0, causal=causal, dtype=dtype,
                    seed=seed, clusters=clusters)
    return wl, I.make_inputs(wl, "cpu")


def _odd_rows(shape, gen, dtype):
    """Integer rows in [-8, 8] whose coordinates sum to an odd number."""
    x = torch.randint(-8, 9, shape, generator=gen)
    even = (x.sum(dim=-1) % 2) == 0
    x[..., 0] = torch.where(even, torch.where(x[..., 0] < 8, x[..., 0] + 1, x[..., 0] - 1),
                            x[..., 0])
    return x.to(dtype)


def _integer_case(N, H, L, P, causal, seed, dtype="bf16"):
    wl, x = _case(N, H, L, P, causal, seed, dtype)
    gen = torch.Generator().manual_seed(seed + 1000)
    for name in ("q", "k"):
        x[name] = _odd_rows(x[name].shape, gen, x[name].dtype)
    W = torch.randint(0, 4, x["W"].shape, generator=gen) * 2 - 3     # -3, -1, 1, 3
    x["W"] = W.to(torch.float32)
    return wl, x


@pytest.mark.parametrize("P", [1, 4, 8])
def test_bucket_ids_exact(P):
    wl, x = _integer_case(500, 2, 5, P, False, seed=P)
    ids = ra.hard_hash(x["q"].to(DEV), x["W"].to(DEV))
    ref = np.stack([oracle.hard_hash(_f64(x["q"][h]), _f64(x["W"])) for h in range(2)])
    assert (ids.cpu().numpy().astype(np.int64) == ref).all()


def test_bucket_ids_real_valued_agree_outside_the_rounding_margin():
    wl, x = _case(2000, 2, 8, 8, False, seed=5)
    ids = ra.hard_hash(x["q"].to(DEV), x["W"].to(DEV)).cpu().numpy().astype(np.int64)
    X, Wn = _f64(x["q"]), _f64(x["W"])
    u = np.einsum("hnd,ldp->hnlp", X, Wn)
    bound = 2 * 64 * 2.0 ** -24 * np.einsum("hnd,ldp->hnlp", np.abs(X), np.abs(Wn))
    bits_gpu = (ids[..., None] >> np.arange(8)) & 1
    bits_ref = (u >= 0).astype(np.int64)
    differ = bits_gpu != bits_ref
    assert not (differ & (np.abs(u) > bound)).any()
    assert differ.sum() <= 0.001 * differ.size


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,L,P,dtype", [(1, 3, 4, "fp32"), (300, 4, 6, "bf16"),
                                         (1000, 16, 8, "bf16"), (777, 8, 3, "fp32")])
def test_hard_forward_against_oracle(causal, N, L, P, dtype):
    wl, x = _integer_case(N, 2, L, P, causal, seed=N + P, dtype=dtype)
    g = {k: v.to(DEV) for k, v in x.items()}
    out, cnt = ra.hard_forward(g["q"], g["k"], g["v"], g["W"], causal, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ra.race_device_status() == 0
    for h in range(2):
        o_ref, den_ref = oracle.hard_forward(_f64(x["q"][h]), _f64(x["k"][h]), _f64(x["v"][h]),
                                             _f64(x["W"]), causal)
        assert (cnt[h].cpu().numpy() == den_ref).all(), h
        vmax = np.abs(_f64(x["v"])).max()
        assert np.abs(_f64(out[h]) - o_ref).max() <= 1e-5 * vmax, h


def test_hard_forward_no_collision_gives_zero():
    # one query far from every key in every table: out = 0, count = 0
    wl, x = _case(64, 1, 2, 8, True, seed=3)
    q = x["q"].clone()
    W = x["W"]
    # a query whose projections all have the opposite sign of key 0's
    k0 = x["k"][0, 0].float()
    q[0, 0] = (-k0).to(q.dtype)
    g = {k: v.to(DEV) for k, v in x.items()}
    out, cnt = ra.hard_forward(q.to(DEV), g["k"], g["v"], g["W"], True, out_dtype=torch.float32)
    torch.cuda.synchronize()
    o_ref, den_ref = oracle.hard_forward(_f64(q[0]), _f64(x["k"][0]), _f64(x["v"][0]),
                                         _f64(W), True)
    assert den_ref[0] == 0 and cnt[0, 0].item() == 0
    assert (out[0, 0] == 0).all()


def test_hard_forward_262k_sampled_rows():
    """262,144 tokens, 4 heads, 16 tables of 256 buckets, integer inputs as above (several
    segments per head: the scanned prefix of the count arrays is exercised)."""
    N, H, L, P = 262144, 4, 16, 8
    wl, x = _integer_case(N, H, L, P, True, seed=7)
    g = {k: v.to(DEV) for k, v in x.items()}
    out, cnt = ra.hard_forward(g["q"], g["k"], g["v"], g["W"], True, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ra.race_device_status() == 0
    W = _f64(x["W"])
    vmax = np.abs(_f64(x["v"])).max()
    for h in (0, 3):
        hk = oracle.hard_hash(_f64(x["k"][h]), W)              # [N, L]
        V = _f64(x["v"][h])
        rows = [0, 127, 128, 5000, 131071, N - 1]
        hq = oracle.hard_hash(_f64(x["q"][h][rows]), W)
        for r, i in enumerate(rows):
            m = (hk[: i + 1] == hq[r][None, :]).sum(axis=1)    # colliding tables per key
            den = int(m.sum())
            assert cnt[h, i].item() == den, (h, i)
            ref = (m[:, None] * V[: i + 1]).sum(axis=0) / den if den else np.zeros(64)
            assert np.abs(_f64(out[h, i]) - ref).max() <= 1e-5 * vmax, (h, i)
