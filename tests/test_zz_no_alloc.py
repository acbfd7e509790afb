"""race_forward_noalloc: the forward with its scratch in a fixed device array.

The GPU cases call the allocation-free entry point twice in a row through the C ABI
and compare both results with race_forward_ex (which takes stream-ordered scratch of
its own) on the same inputs.  Both run the same kernels; only the order of the
floating-point additions into the shared accumulators can differ, so the bound is
1e-4 * max|V| on float32 outputs.  A second call that saw the first call's leftovers
(an accumulator not cleared) would be off by a whole output.

The size check runs on the host before any device work, so it is tested without a GPU.
"""
import numpy as np
import pytest
import torch

from linear_lsh_sketch_race_b200 import inputs as I
from linear_lsh_sketch_race_b200 import race_attn as ra

DEV = "cuda"
TOL = 1e-4

CASES = [
    # causal bf16, P = 8, 16 tables: norm pre-pass, segment sums + scan, sweep
    dict(N=8192, H=2, L=16, P=8, tau=0.25, causal=True, dtype="bf16"),
    # non-causal bf16: sketch build, total scan, readout
    dict(N=3000, H=2, L=4, P=6, tau=0.5, causal=False, dtype="bf16"),
    # float32 inputs: CUDA-core kernels, ragged tail
    dict(N=1000, H=2, L=4, P=4, tau=0.5, causal=True, dtype="fp32"),
]


def test_scratch_limit_rejected_on_host():
    a = ra.race_args_init(1 << 24, 8, 64, 16, 8, 0.5, 1)
    assert ra.race_workspace_size(a) > ra.RACE_NOALLOC_SCRATCH_BYTES
    fake = 1 << 12  # never dereferenced: the size check comes first
    with pytest.raises(ra.RaceError) as e:
        ra.race_forward_noalloc(fake, fake, fake, fake, fake, a, stream=0)
    assert e.value.status == ra.RACE_ERR_SCRATCH_LIMIT
    assert "RACE_NOALLOC_SCRATCH_BYTES" in str(e.value)


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c['dtype']}_N{c['N']}_"
                         f"{'causal' if c['causal'] else 'noncausal'}")
def test_noalloc_matches_allocating_forward(case):
    wl = I.Workload("noalloc", H=case["H"], N=case["N"], d=64, L=case["L"], P=case["P"],
                    tau=case["tau"], causal=case["causal"], dtype=case["dtype"], seed=7)
    x = {k: t.to(DEV) for k, t in I.make_inputs(wl, "cpu").items()}
    q, k, v, W = x["q"], x["k"], x["v"], x["W"]
    args = ra.make_args(q, W, case["tau"], case["causal"], out_dtype=torch.float32)
    assert ra.race_workspace_size(args) <= ra.RACE_NOALLOC_SCRATCH_BYTES

    ref = torch.empty(case["H"], case["N"], 64, device=DEV, dtype=torch.float32)
    ra.race_forward_ex(q, k, v, W, ref, args)
    outs = []
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        ra.race_forward_noalloc(q, k, v, W, out, args)
        outs.append(out)
    torch.cuda.synchronize()
    assert ra.race_device_status() == 0

    vmax = v.abs().max().item()
    r = ref.double().cpu().numpy()
    assert np.isfinite(r).all()
    for i, out in enumerate(outs):
        o = out.double().cpu().numpy()
        assert np.isfinite(o).all(), i
        err = np.abs(o - r).max() / vmax
        assert err <= TOL, (i, err)
