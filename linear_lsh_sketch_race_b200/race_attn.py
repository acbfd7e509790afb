"""ctypes binding of librace_attn.so (declarations in include/race_attn.h).

Argument marshalling only: tensors become device pointers, sizes become C integers
and the current torch CUDA stream becomes the cudaStream_t.  Every step of the
computation runs in the library's kernels.  A missing or unloadable library raises
immediately; there is no fallback.

The C entry points keep their names: ``race_forward``, ``race_backward``,
``race_forward_ex``, ``race_backward_ex``, ``race_forward_noalloc``,
``race_workspace_size``, ``race_hash``,
``race_device_status``, ``race_status_string``, ``race_version``, ``race_args_init``.
``forward``/``backward``/``hash`` are conveniences that allocate outputs.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librace_attn.so")

RACE_OK, RACE_ERR_INVALID_ARG, RACE_ERR_UNSUPPORTED, RACE_ERR_WORKSPACE, \
    RACE_ERR_CUDA, RACE_ERR_DEVICE_STATUS, RACE_ERR_SCRATCH_LIMIT = range(7)
RACE_NOALLOC_SCRATCH_BYTES = 64 << 20
RACE_BF16, RACE_FP32 = 0, 1
RACE_IMPL_AUTO, RACE_IMPL_SIMT, RACE_IMPL_TENSOR = 0, 1, 2
_IMPLS = {"auto": RACE_IMPL_AUTO, "simt": RACE_IMPL_SIMT, "tensor": RACE_IMPL_TENSOR}

EXPORTED = ("race_args_init", "race_forward", "race_backward", "race_forward_ex",
            "race_backward_ex", "race_workspace_size", "race_hash", "race_device_status",
            "race_status_string", "race_version", "race_timing_enable",
            "race_timing_report", "race_launch_count", "race_forward_noalloc",
            "race_selftest_wait_timeout", "race_forward_stream", "race_hard_forward",
            "race_hard_workspace_size", "race_hard_hash")


class RaceArgs(ctypes.Structure):
    """Mirror of race_args_t."""
    _fields_ = [
        ("N", ctypes.c_int64),
        ("H", ctypes.c_int),
        ("d", ctypes.c_int),
        ("L", ctypes.c_int),
        ("P", ctypes.c_int),
        ("tau", ctypes.c_float),
        ("causal", ctypes.c_int),
        ("dtype", ctypes.c_int),
        ("out_dtype", ctypes.c_int),
        ("chunk", ctypes.c_int),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("den", ctypes.c_void_p),
        ("impl", ctypes.c_int),
        ("grad_dtype", ctypes.c_int),
        ("w_per_head", ctypes.c_int),
    ]


class RaceError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {race_status_string(status)} ({status})")


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library once; raises OSError if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise OSError(f"{path} is not built; run `python -m linear_lsh_sketch_race_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    pargs = ctypes.POINTER(RaceArgs)
    lib.race_args_init.argtypes = [pargs, i64, i32, i32, i32, i32, f32, i32]
    lib.race_args_init.restype = None
    lib.race_forward.argtypes = [vp, vp, vp, vp, vp, i64, i32, i32, i32, i32, f32, i32, vp]
    lib.race_backward.argtypes = [vp] * 10 + [i64, i32, i32, i32, i32, f32, i32, vp]
    lib.race_forward_ex.argtypes = [vp, vp, vp, vp, vp, pargs, vp]
    lib.race_backward_ex.argtypes = [vp] * 10 + [pargs, vp]
    lib.race_forward_noalloc.argtypes = [vp, vp, vp, vp, vp, pargs, vp]
    lib.race_forward_stream.argtypes = [vp, vp, vp, vp, vp, vp, vp, pargs, vp]
    lib.race_hard_forward.argtypes = [vp, vp, vp, vp, vp, vp, pargs, vp]
    lib.race_hard_workspace_size.argtypes = [pargs, ctypes.POINTER(ctypes.c_size_t)]
    lib.race_hard_hash.argtypes = [vp, vp, vp, pargs, vp]
    lib.race_workspace_size.argtypes = [pargs, i32, ctypes.POINTER(ctypes.c_size_t)]
    lib.race_hash.argtypes = [vp, vp, vp, pargs, vp]
    lib.race_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.race_selftest_wait_timeout.argtypes = [i64, ctypes.POINTER(ctypes.c_int), vp]
    lib.race_status_string.argtypes = [i32]
    lib.race_status_string.restype = ctypes.c_char_p
    lib.race_version.argtypes = []
    lib.race_timing_enable.argtypes = [i32]
    lib.race_timing_report.argtypes = [i32, ctypes.POINTER(ctypes.c_char_p),
                                       ctypes.POINTER(ctypes.c_double),
                                       ctypes.POINTER(ctypes.c_int64)]
    lib.race_launch_count.argtypes = []
    lib.race_launch_count.restype = i64
    for name in ("race_forward", "race_backward", "race_forward_ex", "race_backward_ex",
                 "race_forward_noalloc", "race_workspace_size", "race_hash", "race_device_status",
                 "race_timing_enable", "race_timing_report", "race_selftest_wait_timeout",
                 "race_forward_stream", "race_hard_forward", "race_hard_workspace_size",
                 "race_hard_hash"):
        getattr(lib, name).restype = i32
    lib.race_version.restype = i32
    _lib = lib
    return lib


# ------------------------------------------------------------------ raw C entry points
def race_status_string(status: int) -> str:
    return load().race_status_string(int(status)).decode()


def race_version() -> int:
    return load().race_version()


def race_args_init(N, H, d, L, P, tau, causal) -> RaceArgs:
    a = RaceArgs()
    load().race_args_init(ctypes.byref(a), int(N), int(H), int(d), int(L), int(P),
                          float(tau), int(causal))
    return a


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != RACE_OK:
        raise RaceError(status, where)


def race_forward(q, k, v, W, out, N, H, d, L, P, tau, causal, stream=None):
    _check(load().race_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(W), _ptr(out), int(N),
                               int(H), int(d), int(L), int(P), float(tau), int(causal),
                               _stream(stream)), "race_forward")


def race_backward(q, k, v, W, out, dout, dq, dk, dv, dW, N, H, d, L, P, tau, causal,
                  stream=None):
    _check(load().race_backward(*(_ptr(t) for t in (q, k, v, W, out, dout, dq, dk, dv, dW)),
                                int(N), int(H), int(d), int(L), int(P), float(tau),
                                int(causal), _stream(stream)), "race_backward")


def race_forward_ex(q, k, v, W, out, args: RaceArgs, stream=None):
    _check(load().race_forward_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(W), _ptr(out),
                                  ctypes.byref(args), _stream(stream)), "race_forward_ex")


def race_forward_noalloc(q, k, v, W, out, args: RaceArgs, stream=None):
    _check(load().race_forward_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(W), _ptr(out),
                                       ctypes.byref(args), _stream(stream)),
           "race_forward_noalloc")


def race_forward_stream(q, k, v, W, out, state_in, state_out, args: RaceArgs, stream=None):
    _check(load().race_forward_stream(_ptr(q), _ptr(k), _ptr(v), _ptr(W), _ptr(out),
                                      _ptr(state_in), _ptr(state_out), ctypes.byref(args),
                                      _stream(stream)), "race_forward_stream")


def race_backward_ex(q, k, v, W, out, dout, dq, dk, dv, dW, args: RaceArgs, stream=None):
    _check(load().race_backward_ex(*(_ptr(t) for t in (q, k, v, W, out, dout, dq, dk, dv, dW)),
                                   ctypes.byref(args), _stream(stream)), "race_backward_ex")


def race_workspace_size(args: RaceArgs, backward: bool = False) -> int:
    n = ctypes.c_size_t(0)
    _check(load().race_workspace_size(ctypes.byref(args), int(bool(backward)),
                                      ctypes.byref(n)), "race_workspace_size")
    return n.value


def race_hash(x, W, phi, args: RaceArgs, stream=None):
    _check(load().race_hash(_ptr(x), _ptr(W), _ptr(phi), ctypes.byref(args),
                            _stream(stream)), "race_hash")


def race_device_status(stream=None) -> int:
    flags = ctypes.c_uint32(0)
    st = load().race_device_status(_stream(stream), ctypes.byref(flags))
    if st not in (RACE_OK, RACE_ERR_DEVICE_STATUS):
        raise RaceError(st, "race_device_status")
    return flags.value


def race_selftest_wait_timeout(limit_cycles: int, stream=None) -> bool:
    """Run the bounded-wait self-test kernel; True when its wait gave up (the device
    status flag is then raised for race_device_status to report)."""
    out = ctypes.c_int(0)
    _check(load().race_selftest_wait_timeout(int(limit_cycles), ctypes.byref(out),
                                             _stream(stream)), "race_selftest_wait_timeout")
    return bool(out.value)


def race_timing_enable(on: bool = True):
    _check(load().race_timing_enable(int(bool(on))), "race_timing_enable")


def race_timing_report():
    """{kernel name: (total device ms, launches)} recorded since race_timing_enable."""
    res = {}
    i = 0
    while True:
        name = ctypes.c_char_p()
        ms = ctypes.c_double()
        n = ctypes.c_int64()
        st = load().race_timing_report(i, ctypes.byref(name), ctypes.byref(ms),
                                       ctypes.byref(n))
        if st != RACE_OK:
            break
        res[name.value.decode()] = (ms.value, n.value)
        i += 1
    return res


def race_launch_count() -> int:
    return load().race_launch_count()


# ------------------------------------------------------------------ conveniences
def _dt(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return RACE_BF16
    if t == torch.float32:
        return RACE_FP32
    raise ValueError(f"unsupported dtype {t}")


def make_args(q, W, tau, causal, out_dtype=None, chunk=0, impl="auto", den=None,
              workspace=None, grad_dtype=None) -> RaceArgs:
    H, N, d = q.shape
    if W.dim() == 4:                     # one set of planes per head: [H, L, d, P]
        if W.shape[0] != H:
            raise ValueError(f"per-head planes {tuple(W.shape)} for {H} heads")
        _, L, dW_, P = W.shape
    else:                                # shared planes: [L, d, P]
        L, dW_, P = W.shape
    a = race_args_init(N, H, d, L, P, tau, int(bool(causal)))
    a.w_per_head = int(W.dim() == 4)
    a.dtype = _dt(q.dtype)
    a.out_dtype = _dt(out_dtype or q.dtype)
    a.grad_dtype = _dt(grad_dtype or q.dtype)
    a.chunk = int(chunk)
    a.impl = _IMPLS[impl]
    if den is not None:
        a.den = den.data_ptr()
    if workspace is not None:
        a.workspace = workspace.data_ptr()
        a.workspace_bytes = workspace.numel() * workspace.element_size()
    return a


def forward(q, k, v, W, tau, causal, out_dtype=None, chunk=0, impl="auto",
            return_den=False, out=None, den=None, workspace=None, stream=None):
    """RACE attention forward on [H, N, 64] tensors; returns out (and den)."""
    out_dtype = out_dtype or q.dtype
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
    if return_den and den is None:
        den = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device)
    a = make_args(q, W, tau, causal, out_dtype, chunk, impl, den, workspace)
    race_forward_ex(q, k, v, W, out, a, stream)
    return (out, den) if return_den else out


def backward(q, k, v, W, tau, causal, out, dout, den=None, chunk=0, impl="auto",
             workspace=None, stream=None, grads=None, grad_dtype=None):
    """Gradients (dq, dk, dv, dW) of sum(out * dout); dq, dk, dv in grad_dtype (default:
    the dtype of q), dW in float32."""
    gdt = grad_dtype or q.dtype
    if grads is None:
        grads = (torch.empty(q.shape, dtype=gdt, device=q.device),
                 torch.empty(k.shape, dtype=gdt, device=k.device),
                 torch.empty(v.shape, dtype=gdt, device=v.device), torch.empty_like(W))
    dq, dk, dv, dW = grads
    a = make_args(q, W, tau, causal, out.dtype, chunk, impl, den, workspace, gdt)
    race_backward_ex(q, k, v, W, out, dout, dq, dk, dv, dW, a, stream)
    return dq, dk, dv, dW


def race_hard_forward(q, k, v, W, out, counts, args: RaceArgs, stream=None):
    _check(load().race_hard_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(W), _ptr(out),
                                    _ptr(counts), ctypes.byref(args), _stream(stream)),
           "race_hard_forward")


def race_hard_workspace_size(args: RaceArgs) -> int:
    n = ctypes.c_size_t(0)
    _check(load().race_hard_workspace_size(ctypes.byref(args), ctypes.byref(n)),
           "race_hard_workspace_size")
    return n.value


def race_hard_hash(x, W, ids, args: RaceArgs, stream=None):
    _check(load().race_hard_hash(_ptr(x), _ptr(W), _ptr(ids), ctypes.byref(args),
                                 _stream(stream)), "race_hard_hash")


def hard_forward(q, k, v, W, causal, out_dtype=None, stream=None):
    """Classic RACE with hard hashes: returns (out, counts) with counts int32 [H, N]."""
    out_dtype = out_dtype or q.dtype
    out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
    counts = torch.empty(q.shape[:2], dtype=torch.int32, device=q.device)
    a = make_args(q, W, 1.0, causal, out_dtype)
    race_hard_forward(q, k, v, W, out, counts, a, stream)
    return out, counts


def hard_hash(x, W, stream=None):
    """Bucket ids uint8 [H, N, L] of the hard hash."""
    H, N, _ = x.shape
    ids = torch.empty((H, N, W.shape[-3]), dtype=torch.uint8, device=x.device)
    race_hard_hash(x, W, ids, make_args(x, W, 1.0, False), stream)
    return ids


def state_shape(H: int, L: int, P: int):
    """Shape of the carried sketch state of race_forward_stream: [H, L * 2^P, 65]."""
    return (H, L << P, 65)


def forward_stream(q, k, v, W, tau, causal=True, state=None, out_dtype=None, impl="auto",
                   inplace=False, stream=None):
    """RACE attention over a block of new tokens that continues earlier blocks: returns
    (out, new_state).  `state` is the carried [H, L*2^P, 65] float32 state (None: start of
    the sequences); with inplace=True it is updated in place and returned."""
    out_dtype = out_dtype or q.dtype
    out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
    H = q.shape[0]
    L, P = W.shape[-3], W.shape[-1]
    if inplace and state is not None:
        new_state = state
    else:
        new_state = torch.empty(state_shape(H, L, P), dtype=torch.float32, device=q.device)
    a = make_args(q, W, tau, causal, out_dtype, 0, impl)
    race_forward_stream(q, k, v, W, out, state, new_state, a, stream)
    return out, new_state


def hash(x, W, tau, out_dtype=torch.float32, stream=None):  # noqa: A001
    """phi(x) = concat_l softmax-over-corners / sqrt(L), shape [H, N, L*2^P]; W shared
    [L, d, P] or per head [H, L, d, P]."""
    H, N, d = x.shape
    L, P = W.shape[-3], W.shape[-1]
    phi = torch.empty((H, N, L << P), dtype=out_dtype, device=x.device)
    a = make_args(x, W, tau, False, out_dtype)
    race_hash(x, W, phi, a, stream)
    return phi
