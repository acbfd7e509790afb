"""Synthetic inputs (no GPU): the workload table matches the five published configurations of
the method's evaluation, generation is deterministic per (seed, tensor, head), and the
clustered recipe has the structure it states."""
import torch

from linear_lsh_sketch_race_b200 import inputs as I

# (H = batch * heads, N, d, L, P, tau, causal, dtype, chunk, clusters, backward, batch)
TABLE = {
    "noncausal_fp32_h1_n1024_d64_L4_P4": (1, 1024, 64, 4, 4, 0.5, False, "fp32", 0, 0, False, 1),
    "causal_bf16_h8_n16384_d64_L8_P6_clustered32":
        (8, 16384, 64, 8, 6, 0.5, True, "bf16", 128, 32, False, 1),
    "noncausal_bf16_b2h16_n262144_d64_L16_P6":
        (32, 262144, 64, 16, 6, 0.5, False, "bf16", 0, 0, False, 2),
    "causal_bf16_h8_n4194304_d64_L16_P8_clustered256":
        (8, 4194304, 64, 16, 8, 0.25, True, "bf16", 256, 256, False, 1),
    "causal_fwdbwd_bf16_h4_n12582912_d64_L8_P6":
        (4, 12582912, 64, 8, 6, 0.5, True, "bf16", 256, 0, True, 1),
}


def test_workload_table_matches_the_configurations():
    assert set(I.WORKLOADS) == set(TABLE)
    for name, row in TABLE.items():
        w = I.WORKLOADS[name]
        got = (w.H, w.N, w.d, w.L, w.P, w.tau, w.causal, w.dtype, w.chunk, w.clusters,
               w.backward, w.batch)
        assert got == row, name
    assert I.HEADLINE == "causal_bf16_h8_n4194304_d64_L16_P8_clustered256"


def _small(name, **kw):
    return I.WORKLOADS[name].replace(N=512, **kw)


def test_generation_is_deterministic_and_per_head():
    wl = _small("causal_bf16_h8_n4194304_d64_L16_P8_clustered256")
    a = I.make_inputs(wl, "cpu", with_dout=True)
    b = I.make_inputs(wl, "cpu", with_dout=True)
    for key in a:
        assert torch.equal(a[key], b[key]), key
    # one head regenerated alone equals that head of the full draw
    one = I.make_inputs(wl, "cpu", heads=[3])
    assert torch.equal(one["q"][0], a["q"][3]) and torch.equal(one["v"][0], a["v"][3])
    # another seed gives other tensors
    c = I.make_inputs(wl.replace(seed=wl.seed + 1), "cpu")
    assert not torch.equal(c["q"], a["q"])


def test_dtypes_and_shapes():
    for name in TABLE:
        w = _small(name, H=2)
        x = I.make_inputs(w, "cpu", with_dout=True)
        for key in ("q", "k", "v", "dout"):
            assert x[key].shape == (2, 512, 64) and x[key].dtype == w.torch_dtype, (name, key)
        assert x["W"].shape == (w.L, 64, w.P) and x["W"].dtype == torch.float32


def _mean_pair_dot(x):
    """Mean of x_i . x_j over ordered pairs i != j."""
    x = x.double()
    n = x.shape[0]
    tot = x.sum(dim=0)
    return ((tot @ tot) - x.pow(2).sum()).item() / (n * (n - 1))


def test_clustered_rows_share_their_centroids():
    # q_i = c_a(i) + sigma * noise with unit centroids: two rows share a centroid with
    # probability 1/m and then have expected dot product 1, otherwise 0 on average (the dot
    # products of different random centroids add a spread of a few tenths of 1/m); iid rows
    # have mean pair dot product 0 (standard error about 8 sqrt(2) / N here)
    n = 4096
    for name, m in (("causal_bf16_h8_n16384_d64_L8_P6_clustered32", 32),
                    ("causal_bf16_h8_n4194304_d64_L16_P8_clustered256", 256)):
        wl = I.WORKLOADS[name].replace(H=1)
        x = I.make_inputs(wl, "cpu", N=n)
        for key in ("q", "k"):
            got = _mean_pair_dot(x[key][0])
            assert 0.5 / m < got < 2.0 / m, (name, key, got)
        # squared norms: 1 + d sigma^2 on average
        assert abs(x["q"][0].double().pow(2).sum(dim=1).mean().item() - (1 + 64 * wl.sigma ** 2)) < 0.2
    iid = I.make_inputs(I.WORKLOADS["noncausal_bf16_b2h16_n262144_d64_L16_P6"].replace(H=1),
                        "cpu", N=n)
    assert abs(_mean_pair_dot(iid["q"][0])) < 0.01
    assert abs(iid["q"][0].double().pow(2).sum(dim=1).mean().item() - 64) < 1.0
