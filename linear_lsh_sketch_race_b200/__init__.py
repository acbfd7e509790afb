"""RACE attention on one NVIDIA B200: a C-ABI CUDA library plus a thin binding.

The compute path lives in ``librace_attn.so`` (hand-written sm_100a kernels).  The
binding in :mod:`linear_lsh_sketch_race_b200.race_attn` only marshals pointers,
sizes and the CUDA stream; it loads the library on first use and raises if it is
missing.  :mod:`linear_lsh_sketch_race_b200.inputs` draws seeded workloads.
"""
