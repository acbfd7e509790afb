"""Failure detection without a GPU fault.

A kernel's bounded wait that runs out must raise the device status flag, end the kernel
and leave the context usable.  race_selftest_wait_timeout runs one warp that waits, with a
short limit, on an mbarrier phase that nothing completes (no TMA copy or MMA is in
flight), through the same wait routine the tensor-core kernels use.  The status flag is
then reported once by race_device_status and cleared, and the next ordinary call works.
"""
import numpy as np
import pytest
import torch

from linear_lsh_sketch_race_b200 import inputs as I
from linear_lsh_sketch_race_b200 import race_attn as ra


@pytest.mark.parametrize("limit", [0, -5, 3_000_000_000])
def test_selftest_limit_checked_on_host(limit):
    with pytest.raises(ra.RaceError) as e:
        ra.race_selftest_wait_timeout(limit, stream=0)
    assert e.value.status == ra.RACE_ERR_INVALID_ARG


@pytest.mark.gpu
def test_bounded_wait_gives_up_and_the_library_recovers():
    import oracle

    ra.load()
    assert ra.race_device_status() == 0
    assert ra.race_selftest_wait_timeout(1_000_000) is True
    flags = ctypes_status()
    assert flags[0] == ra.RACE_ERR_DEVICE_STATUS and flags[1] & 1
    assert ctypes_status() == (ra.RACE_OK, 0)          # reported once, then cleared
    wl = I.Workload("after", H=2, N=300, d=64, L=2, P=8, tau=0.25, causal=True,
                    dtype="bf16", seed=1)
    x = I.make_inputs(wl, "cpu")
    g = {k: v.to("cuda") for k, v in x.items()}
    out = ra.forward(g["q"], g["k"], g["v"], g["W"], wl.tau, True, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ctypes_status() == (ra.RACE_OK, 0)
    f = lambda t: t.double().cpu().numpy()  # noqa: E731
    ref, _ = oracle.forward_heads(f(x["q"]), f(x["k"]), f(x["v"]), f(x["W"]), wl.tau, True)
    assert np.abs(f(out) - ref).max() / np.abs(f(x["v"])).max() <= 2e-3


def ctypes_status():
    import ctypes
    flags = ctypes.c_uint32(0)
    st = ra.load().race_device_status(None, ctypes.byref(flags))
    return st, flags.value
