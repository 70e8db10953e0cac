"""Thin Python binding of libdora.so (the C ABI in include/dora.h).

The functions keep the C names.  They only marshal arguments: check dtypes,
shapes and devices of torch tensors, take their data pointers and the current
CUDA stream, allocate outputs / workspaces with torch when the caller passes
none, and raise ``DoraError`` on a non-zero status.  Every step of the
computation runs in libdora.so's CUDA kernels; there is no fallback.
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdora.so")

DORA_BF16 = 0
DORA_F32 = 1

DORA_OK = 0
DORA_ERR_INVALID_ARG = 1
DORA_ERR_UNSUPPORTED = 2
DORA_ERR_WORKSPACE = 3
DORA_ERR_CUDA = 4
DORA_ERR_TIMEOUT = 5

_c_void_p, _i64, _f32, _size = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t


class NormProblem(ctypes.Structure):
    """dora_norm_problem of include/dora.h."""

    _fields_ = [("W", _c_void_p), ("A", _c_void_p), ("B", _c_void_p), ("d_out", _i64), ("d_in", _i64),
                ("r", _i64), ("s", _f32), ("n_out", _c_void_p)]


_problems_p = ctypes.POINTER(NormProblem)

# every symbol include/dora.h declares, with its ctypes signature
SIGNATURES = {
    "dora_factored_norm_workspace_size": (_size, [_i64, _i64, _i64, ctypes.c_int]),
    "dora_factored_norm": (
        ctypes.c_int,
        [_c_void_p, _c_void_p, _c_void_p, _i64, _i64, _i64, _f32, ctypes.c_int, _c_void_p, _c_void_p, _size, _c_void_p],
    ),
    "dora_compose_fwd": (
        ctypes.c_int,
        [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _f32, _i64, _i64, ctypes.c_int, _c_void_p, _c_void_p],
    ),
    "dora_compose_fwd_bias": (
        ctypes.c_int,
        [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _f32, _i64, _i64, ctypes.c_int, _c_void_p, _c_void_p],
    ),
    "dora_compose_bwd_workspace_size": (_size, [_i64, _i64]),
    "dora_compose_bwd": (
        ctypes.c_int,
        [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _f32, _i64, _i64, ctypes.c_int,
         _c_void_p, _c_void_p, _c_void_p, _c_void_p, _size, _c_void_p],
    ),
    "dora_compose_bwd_bias": (
        ctypes.c_int,
        [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _f32, _i64, _i64, ctypes.c_int,
         _c_void_p, _c_void_p, _c_void_p, _c_void_p, _size, _c_void_p],
    ),
    "dora_compose_bwd_noalloc": (
        ctypes.c_int,
        [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _f32, _i64, _i64, ctypes.c_int,
         _c_void_p, _c_void_p, _c_void_p, _c_void_p],
    ),
    "dora_compose_bwd_noalloc_bias": (
        ctypes.c_int,
        [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _f32, _i64, _i64, ctypes.c_int,
         _c_void_p, _c_void_p, _c_void_p, _c_void_p],
    ),
    "dora_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "dora_device_status": (ctypes.c_int, [_c_void_p]),
    "dora_num_sms": (ctypes.c_int, []),
    "dora_launch_count": (ctypes.c_uint64, []),
    "dora_selftest_timeout": (ctypes.c_int, [_i64, _c_void_p]),
    "dora_factored_norm_batched_workspace_size": (_size, [_problems_p, ctypes.c_int, ctypes.c_int]),
    "dora_factored_norm_batched": (ctypes.c_int, [_problems_p, ctypes.c_int, ctypes.c_int, _c_void_p, _size, _c_void_p]),
    "dora_factored_norm_bwd_workspace_size": (_size, [_i64, _i64, _i64]),
    "dora_factored_norm_bwd": (
        ctypes.c_int,
        [_c_void_p, _c_void_p, _c_void_p, _f32, _c_void_p, _c_void_p, _i64, _i64, _i64, ctypes.c_int, _c_void_p,
         _c_void_p, _c_void_p, _size, _c_void_p],
    ),
    "dora_factored_norm_sq": (
        ctypes.c_int,
        [_c_void_p, _c_void_p, _c_void_p, _i64, _i64, _i64, _f32, ctypes.c_int, _c_void_p, _c_void_p, _size, _c_void_p],
    ),
    "dora_norm_finish": (ctypes.c_int, [_c_void_p, _i64, _c_void_p]),
    "dora_fused_linear_fwd_workspace_size": (_size, [_i64, _i64]),
    "dora_fused_linear_fwd": (
        ctypes.c_int,
        [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _f32, _i64, _i64, _i64, _i64,
         ctypes.c_int, _c_void_p, _c_void_p, _size, _c_void_p],
    ),
}

_lib = None


class DoraError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """Loads libdora.so (built in-tree); raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m factored_weight_norm_b200.build` "
                "(nvcc, sm_100a). There is no CPU or PyTorch fallback."
            )
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def status_string(status: int) -> str:
    return lib().dora_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != DORA_OK:
        raise DoraError(status, where)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DORA_BF16
    if t.dtype == torch.float32:
        return DORA_F32
    raise TypeError(f"unsupported dtype {t.dtype}: bf16 or fp32 only")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dense_cuda(*ts):
    """Every tensor given is a contiguous CUDA tensor on the current device.

    Kernels launch on the current device's stream and read their operands
    there, so a tensor on another GPU (or the host) is refused before any
    launch rather than read through a pointer that belongs elsewhere."""
    cur = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")
        if cur is None:
            cur = torch.cuda.current_device()
        if t.device.index != cur:
            raise ValueError(f"tensor on {t.device} but the current device is cuda:{cur}")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous (row-major)")


def _like(ref, where: str, **named):
    """Each named tensor (None skipped) has ref's shape and dtype."""
    for name, t in named.items():
        if t is None:
            continue
        if tuple(t.shape) != tuple(ref.shape):
            raise ValueError(f"{where}: {name} has shape {tuple(t.shape)}, expected {tuple(ref.shape)}")
        if t.dtype != ref.dtype:
            raise TypeError(f"{where}: {name} is {t.dtype}, expected {ref.dtype}")


def _vec_f32(d: int, where: str, **named):
    """Each named tensor (None skipped) is fp32 of shape (d,)."""
    for name, t in named.items():
        if t is None:
            continue
        if tuple(t.shape) != (d,):
            raise ValueError(f"{where}: {name} has shape {tuple(t.shape)}, expected ({d},)")
        if t.dtype != torch.float32:
            raise TypeError(f"{where}: {name} must be fp32, got {t.dtype}")


def _acts2d(base_out, where: str):
    if base_out.dim() != 2:
        raise ValueError(f"{where}: activations must be 2-D [tokens, d_out], got {tuple(base_out.shape)}")
    _dt(base_out)


# ---------------------------------------------------------------- C names
def dora_factored_norm_workspace_size(d_out: int, d_in: int, r: int, dtype: torch.dtype = torch.bfloat16) -> int:
    return int(lib().dora_factored_norm_workspace_size(d_out, d_in, r, _dt(torch.empty(0, dtype=dtype))))


def dora_compose_bwd_workspace_size(tokens: int, d_out: int) -> int:
    return int(lib().dora_compose_bwd_workspace_size(tokens, d_out))


def dora_num_sms() -> int:
    return int(lib().dora_num_sms())


def dora_launch_count() -> int:
    """Kernels the library has launched in this process so far."""
    return int(lib().dora_launch_count())


def dora_device_status(stream=None) -> int:
    return int(lib().dora_device_status(_stream(stream)))


def dora_selftest_timeout(limit_cycles: int, stream=None) -> None:
    """Runs the bounded-wait failure path once (see include/dora.h)."""
    _check(lib().dora_selftest_timeout(int(limit_cycles), _stream(stream)), "dora_selftest_timeout")


def dora_status_string(status: int) -> str:
    return status_string(status)


def dora_factored_norm(W, A, B, s: float, n_out=None, workspace=None, stream=None):
    """n = ||W + s B A||_row as fp32 [d_out] (factored; no dense B A)."""
    return _factored_norm(W, A, B, s, n_out, workspace, stream, squared=False)


def dora_factored_norm_sq(W, A, B, s: float, n2_out=None, workspace=None, stream=None):
    """n^2 = ||W + s B A||_row^2 as summed (no sqrt, no clamp): a d_in shard's share."""
    return _factored_norm(W, A, B, s, n2_out, workspace, stream, squared=True)


def dora_norm_finish(n, stream=None):
    """n = sqrt(max(n, 0)) in place (after summing dora_factored_norm_sq shares)."""
    if n.dtype != torch.float32 or n.dim() != 1:
        raise TypeError("n must be a 1-D fp32 tensor")
    _dense_cuda(n)
    _check(lib().dora_norm_finish(_ptr(n), n.numel(), _stream(stream)), "dora_norm_finish")
    return n


def _factored_norm(W, A, B, s, n_out, workspace, stream, squared):
    where = "dora_factored_norm_sq" if squared else "dora_factored_norm"
    if W.dim() != 2 or A.dim() != 2 or B.dim() != 2:
        raise ValueError(f"{where}: W, A and B must be 2-D")
    d_out, d_in = W.shape
    r = A.shape[0]
    if A.shape != (r, d_in) or B.shape != (d_out, r):
        raise ValueError(f"shape mismatch: W {tuple(W.shape)}, A {tuple(A.shape)}, B {tuple(B.shape)}")
    if not (W.dtype == A.dtype == B.dtype):
        raise TypeError("W, A and B must share one dtype")
    _dt(W)
    _vec_f32(d_out, where, n_out=n_out)
    _dense_cuda(W, A, B, n_out, workspace)
    if n_out is None:
        n_out = torch.empty(d_out, dtype=torch.float32, device=W.device)
    need = dora_factored_norm_workspace_size(d_out, d_in, r, W.dtype)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    fn = lib().dora_factored_norm_sq if squared else lib().dora_factored_norm
    st = fn(
        _ptr(W), _ptr(A), _ptr(B), d_out, d_in, r, float(s), _dt(W), _ptr(n_out),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream),
    )
    _check(st, "dora_factored_norm_sq" if squared else "dora_factored_norm")
    return n_out


def _problem_array(modules, n_outs):
    arr = (NormProblem * len(modules))()
    dt0 = modules[0][0].dtype if modules else None
    for i, ((W, A, B, s), n) in enumerate(zip(modules, n_outs)):
        d_out, d_in = W.shape
        r = A.shape[0]
        if A.shape != (r, d_in) or B.shape != (d_out, r) or n.shape != (d_out,):
            raise ValueError(f"module {i}: shape mismatch: W {tuple(W.shape)}, A {tuple(A.shape)}, B {tuple(B.shape)}")
        if not (W.dtype == A.dtype == B.dtype == dt0) or n.dtype != torch.float32:
            raise TypeError(f"module {i}: W, A, B share the first module's dtype; n is fp32")
        _dense_cuda(W, A, B, n)
        arr[i] = NormProblem(W.data_ptr(), A.data_ptr(), B.data_ptr(), d_out, d_in, r, float(s), n.data_ptr())
    return arr


def dora_factored_norm_batched_workspace_size(modules, dtype: torch.dtype = torch.bfloat16) -> int:
    """modules: sequence of (W, A, B, s) with W [d_out, d_in], A [r, d_in], B [d_out, r]."""
    n_outs = [torch.empty(W.shape[0], dtype=torch.float32, device=W.device) for (W, _, _, _) in modules]
    arr = _problem_array(modules, n_outs)
    return int(lib().dora_factored_norm_batched_workspace_size(arr, len(modules), _dt(torch.empty(0, dtype=dtype))))


def dora_factored_norm_batched(modules, n_outs=None, workspace=None, stream=None):
    """The factored row norms of many modules at once; modules: sequence of
    (W, A, B, s).  Returns the list of fp32 n tensors."""
    modules = list(modules)
    if not modules:
        return []
    dev = modules[0][0].device
    if n_outs is None:
        n_outs = [torch.empty(W.shape[0], dtype=torch.float32, device=dev) for (W, _, _, _) in modules]
    arr = _problem_array(modules, n_outs)
    dt = _dt(modules[0][0])
    need = int(lib().dora_factored_norm_batched_workspace_size(arr, len(modules), dt))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _dense_cuda(workspace)
    st = lib().dora_factored_norm_batched(arr, len(modules), dt, _ptr(workspace),
                                          workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "dora_factored_norm_batched")
    return n_outs


def _check_bias(bias, base_out, name):
    if bias is None:
        return
    if bias.shape != (base_out.shape[1],):
        raise ValueError(f"bias must have shape (d_out,) in {name}")
    if bias.dtype != base_out.dtype:
        raise TypeError(f"bias must have the activations' dtype in {name}")


def dora_compose_fwd(base_out, lora_out, m, n, s: float, y=None, stream=None, bias=None):
    """y = b + (m / n) * ((base_out - b) + s * lora_out), single fused pass.

    base_out is the base layer's output including its bias b (``bias``,
    ``None`` for a layer without one)."""
    where = "dora_compose_fwd"
    _acts2d(base_out, where)
    tokens, d_out = base_out.shape
    _like(base_out, where, lora_out=lora_out, y=y)
    _vec_f32(d_out, where, m=m, n=n)
    _check_bias(bias, base_out, where)
    _dense_cuda(base_out, lora_out, m, n, y, bias)
    if y is None:
        y = torch.empty_like(base_out)
    head = (_ptr(base_out), _ptr(lora_out))
    tail = (_ptr(m), _ptr(n), float(s), tokens, d_out, _dt(base_out), _ptr(y), _stream(stream))
    if bias is None:
        st = lib().dora_compose_fwd(*head, *tail)
    else:
        st = lib().dora_compose_fwd_bias(*head, _ptr(bias), *tail)
    _check(st, "dora_compose_fwd")
    return y


def dora_compose_bwd(dy, base_out, lora_out, m, n, s: float, d_base=None, d_lora=None, d_m=None, workspace=None,
                     stream=None, bias=None):
    """(d_base, d_lora, d_m) of the compose with n held constant and the bias frozen."""
    where = "dora_compose_bwd"
    _acts2d(base_out, where)
    tokens, d_out = base_out.shape
    _like(base_out, where, dy=dy, lora_out=lora_out, d_base=d_base, d_lora=d_lora)
    _vec_f32(d_out, where, m=m, n=n, d_m=d_m)
    _check_bias(bias, base_out, where)
    _dense_cuda(dy, base_out, lora_out, m, n, d_base, d_lora, d_m, workspace, bias)
    if d_base is None:
        d_base = torch.empty_like(base_out)
    if d_lora is None:
        d_lora = torch.empty_like(base_out)
    if d_m is None:
        d_m = torch.empty(d_out, dtype=torch.float32, device=base_out.device)
    need = dora_compose_bwd_workspace_size(tokens, d_out)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=base_out.device)
    head = (_ptr(dy), _ptr(base_out), _ptr(lora_out))
    tail = (_ptr(m), _ptr(n), float(s), tokens, d_out, _dt(base_out), _ptr(d_base), _ptr(d_lora), _ptr(d_m),
            _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    if bias is None:
        st = lib().dora_compose_bwd(*head, *tail)
    else:
        st = lib().dora_compose_bwd_bias(*head, _ptr(bias), *tail)
    _check(st, "dora_compose_bwd")
    return d_base, d_lora, d_m


def dora_compose_bwd_noalloc(dy, base_out, lora_out, m, n, s: float, d_base, d_lora, d_m, stream=None, bias=None):
    """dora_compose_bwd into caller-provided outputs, with the library's own
    scratch instead of a workspace (nothing is allocated)."""
    where = "dora_compose_bwd_noalloc"
    if d_base is None or d_lora is None or d_m is None:
        raise ValueError(f"{where}: d_base, d_lora and d_m are required (nothing is allocated)")
    _acts2d(base_out, where)
    tokens, d_out = base_out.shape
    _like(base_out, where, dy=dy, lora_out=lora_out, d_base=d_base, d_lora=d_lora)
    _vec_f32(d_out, where, m=m, n=n, d_m=d_m)
    _check_bias(bias, base_out, where)
    _dense_cuda(dy, base_out, lora_out, m, n, d_base, d_lora, d_m, bias)
    head = (_ptr(dy), _ptr(base_out), _ptr(lora_out))
    tail = (_ptr(m), _ptr(n), float(s), tokens, d_out, _dt(base_out), _ptr(d_base), _ptr(d_lora), _ptr(d_m),
            _stream(stream))
    if bias is None:
        st = lib().dora_compose_bwd_noalloc(*head, *tail)
    else:
        st = lib().dora_compose_bwd_noalloc_bias(*head, _ptr(bias), *tail)
    _check(st, "dora_compose_bwd_noalloc")
    return d_base, d_lora, d_m


def dora_fused_linear_fwd_workspace_size(tokens: int, r: int) -> int:
    return int(lib().dora_fused_linear_fwd_workspace_size(tokens, r))


def dora_fused_linear_fwd(x, W, A, B, m, n, s: float, bias=None, y=None, workspace=None, stream=None):
    """y = b + (m / n) * (x W^T + s * (x A^T) B^T), the compose fused into the GEMMs (bf16)."""
    where = "dora_fused_linear_fwd"
    if x.dim() != 2 or W.dim() != 2 or A.dim() != 2 or B.dim() != 2:
        raise ValueError(f"{where}: x, W, A and B must be 2-D")
    T, d_in = x.shape
    d_out, r = W.shape[0], A.shape[0]
    if W.shape != (d_out, d_in) or A.shape != (r, d_in) or B.shape != (d_out, r):
        raise ValueError("shape mismatch in dora_fused_linear_fwd")
    _vec_f32(d_out, where, m=m, n=n)
    for t in (x, W, A, B):
        if t.dtype != torch.bfloat16:
            raise TypeError("x, W, A and B must be bf16")
    if bias is not None and (bias.shape != (d_out,) or bias.dtype != torch.bfloat16):
        raise ValueError("bias must be bf16 of shape (d_out,)")
    if y is not None and (tuple(y.shape) != (T, d_out) or y.dtype != torch.bfloat16):
        raise ValueError(f"{where}: y must be bf16 of shape ({T}, {d_out})")
    _dense_cuda(x, W, A, B, m, n, bias, y, workspace)
    if y is None:
        y = torch.empty(T, d_out, dtype=torch.bfloat16, device=x.device)
    need = dora_fused_linear_fwd_workspace_size(T, r)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    st = lib().dora_fused_linear_fwd(
        _ptr(x), _ptr(W), _ptr(A), _ptr(B), _ptr(bias), _ptr(m), _ptr(n), float(s), T, d_in, d_out, r, DORA_BF16,
        _ptr(y), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream),
    )
    _check(st, "dora_fused_linear_fwd")
    return y


def dora_factored_norm_bwd_workspace_size(d_out: int, d_in: int, r: int) -> int:
    return int(lib().dora_factored_norm_bwd_workspace_size(d_out, d_in, r))


def dora_factored_norm_bwd(W, A, B, s: float, n, d_n, dA=None, dB=None, workspace=None, stream=None):
    """(dA, dB): gradients of n_i = ||W_i + s B_i A|| into A and B (fp32), given d_n = dL/dn."""
    where = "dora_factored_norm_bwd"
    if W.dim() != 2 or A.dim() != 2 or B.dim() != 2:
        raise ValueError(f"{where}: W, A and B must be 2-D")
    d_out, d_in = W.shape
    r = A.shape[0]
    if A.shape != (r, d_in) or B.shape != (d_out, r) or n.shape != (d_out,) or d_n.shape != (d_out,):
        raise ValueError("shape mismatch in dora_factored_norm_bwd")
    for t in (W, A, B):
        if t.dtype != torch.bfloat16:
            raise TypeError("W, A and B must be bf16")
    _vec_f32(d_out, where, n=n, d_n=d_n)
    for name, t, shp in (("dA", dA, (r, d_in)), ("dB", dB, (d_out, r))):
        if t is not None and (tuple(t.shape) != shp or t.dtype != torch.float32):
            raise ValueError(f"{where}: {name} must be fp32 of shape {shp}")
    _dense_cuda(W, A, B, n, d_n, dA, dB, workspace)
    if dA is None:
        dA = torch.empty(r, d_in, dtype=torch.float32, device=W.device)
    if dB is None:
        dB = torch.empty(d_out, r, dtype=torch.float32, device=W.device)
    need = dora_factored_norm_bwd_workspace_size(d_out, d_in, r)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    st = lib().dora_factored_norm_bwd(
        _ptr(W), _ptr(A), _ptr(B), float(s), _ptr(n), _ptr(d_n), d_out, d_in, r, DORA_BF16, _ptr(dA), _ptr(dB),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream),
    )
    _check(st, "dora_factored_norm_bwd")
    return dA, dB
