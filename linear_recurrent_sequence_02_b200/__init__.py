"""Python binding of libretnet.so: RetNet multi-scale retention on B200.

Argument marshalling only.  Every function checks tensor dtypes, shapes,
devices and contiguity, then calls the C entry point of the same name with
raw device pointers and the current CUDA stream; all arithmetic runs in the
library's kernels.  There is no fallback: if libretnet.so is missing or
fails to load, importing the functions raises.

Tensors use the C ABI's layouts (see include/retnet.h):
    q, k [batch, seqlen, heads, dk]; v, out, gate [batch, seqlen, heads, dv];
    state [batch, heads, dk, dv] float32; decode-step tensors drop seqlen.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
from typing import Optional, Sequence

import torch

__all__ = [
    "RetnetError", "load_library", "retnet_status_string", "retnet_kernel_launch_count",
    "retnet_set_launch_overlap", "retnet_set_output_pairing",
    "retnet_default_gammas", "retnet_xpos_rotate", "retnet_chunkwise_workspace_size",
    "retnet_retention_chunkwise", "retnet_parallel_workspace_size", "retnet_retention_parallel",
    "retnet_workspace",
    "retnet_retention_step", "retnet_retention_recurrent", "retnet_groupnorm_swish",
    "retnet_backward_workspace_size", "retnet_retention_backward",
    "retnet_check_device_errors", "retnet_profiler_enable", "retnet_profiler_select",
    "retnet_profiler_reset",
    "retnet_profiler_read", "ALGO_AUTO", "ALGO_SIMT", "ALGO_TENSOR", "LIB_PATH",
    "DEBUG_LIB_PATH", "using_library", "retnet_test_set_hooks",
    "retnet_linear", "retnet_msr_workspace_size", "retnet_msr_layer",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libretnet.so")
# Same sources built with index checks and test hooks (build(variant="debug")).
DEBUG_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libretnet_debug.so")

RETNET_OK = 0
F32, BF16 = 0, 1
ALGO_AUTO, ALGO_SIMT, ALGO_TENSOR = 0, 1, 2
_ALGOS = {"auto": ALGO_AUTO, "simt": ALGO_SIMT, "tensor": ALGO_TENSOR,
          ALGO_AUTO: ALGO_AUTO, ALGO_SIMT: ALGO_SIMT, ALGO_TENSOR: ALGO_TENSOR}


class RetnetError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed: {msg} (status {status})")
        self.status = status


class _Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("heads", ctypes.c_int), ("seqlen", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("dtype", ctypes.c_int)]


class _Gate(ctypes.Structure):
    _fields_ = [("g", ctypes.c_void_p), ("weight", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("eps", ctypes.c_float)]


_libs = {}
_active = None           # path of the library the functions below call (None: LIB_PATH)


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Loads a build of the library once (default: the one the functions of
    this module currently call, libretnet.so unless `using_library` says
    otherwise); raises if it has not been built."""
    path = path or _active or LIB_PATH
    if path in _libs:
        return _libs[path]
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} not found: build it with `python -m linear_recurrent_sequence_02_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i, ll, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float, ctypes.c_size_t
    sigs = {
        "retnet_status_string": (ctypes.c_char_p, [i]),
        "retnet_kernel_launch_count": (ctypes.c_ulonglong, []),
        "retnet_set_launch_overlap": (i, [i]),
        "retnet_set_output_pairing": (i, [i]),
        "retnet_default_gammas": (i, [i, vp]),
        "retnet_xpos_rotate": (i, [vp, vp, i, i, i, i, i, ll, vp]),
        "retnet_chunkwise_workspace_size": (i, [ctypes.POINTER(_Shape), i, i, ctypes.POINTER(sz)]),
        "retnet_retention_chunkwise": (i, [vp, vp, vp, vp, i, vp, ctypes.POINTER(_Shape), ll, i,
                                           vp, vp, ctypes.POINTER(_Gate), i, vp, sz, vp]),
        "retnet_parallel_workspace_size": (i, [ctypes.POINTER(_Shape), ctypes.POINTER(sz)]),
        "retnet_retention_parallel": (i, [vp, vp, vp, vp, vp, ctypes.POINTER(_Shape), ll, i,
                                          ctypes.POINTER(_Gate), vp, sz, vp]),
        "retnet_retention_step": (i, [vp, vp, vp, vp, vp, vp, i, i, i, i, i, ll, i, vp]),
        "retnet_retention_recurrent": (i, [vp, vp, vp, vp, vp, vp, ctypes.POINTER(_Shape), ll, i,
                                           vp]),
        "retnet_backward_workspace_size": (i, [ctypes.POINTER(_Shape), i, i, ctypes.POINTER(sz)]),
        "retnet_retention_backward": (i, [vp, vp, vp, vp, vp, i, vp, vp, vp,
                                          ctypes.POINTER(_Shape), ll, i, i, vp, sz, vp]),
        "retnet_groupnorm_swish": (i, [vp, vp, vp, vp, f, ll, i, i, i, vp, vp]),
        "retnet_linear": (i, [vp, vp, vp, ll, i, i, vp]),
        "retnet_msr_workspace_size": (i, [ctypes.POINTER(_Shape), i, i, ctypes.POINTER(sz)]),
        "retnet_msr_layer": (i, [vp, vp, vp, vp, i, vp, ctypes.POINTER(_Shape), i, ll, vp, vp,
                                 f, vp, vp, vp, sz, vp]),
        "retnet_check_device_errors": (i, [vp]),
        "retnet_profiler_enable": (i, [i]),
        "retnet_profiler_select": (i, [ctypes.c_char_p]),
        "retnet_profiler_reset": (i, []),
        "retnet_profiler_read": (i, [i, ctypes.c_char_p, sz, ctypes.POINTER(ctypes.c_double),
                                     ctypes.POINTER(ctypes.c_ulonglong)]),
    }
    if hasattr(lib, "retnet_test_set_hooks"):            # debug build only
        sigs["retnet_test_set_hooks"] = (i, [ctypes.c_ulonglong, i])
    for name, (res, args) in sigs.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _libs[path] = lib
    return lib


@contextlib.contextmanager
def using_library(path: str):
    """Inside the with-block every function of this module calls the library
    at `path` (for example DEBUG_LIB_PATH) instead of libretnet.so."""
    global _active
    prev = _active
    lib = load_library(path)
    _active = path
    try:
        yield lib
    finally:
        _active = prev


def retnet_test_set_hooks(wait_limit_ns: int, skip_first_state_load: bool) -> None:
    """Debug build only: the pipeline waits' time limit and the state pass's
    skipped first load (see retnet_test_set_hooks in include/retnet.h)."""
    lib = load_library()
    if not hasattr(lib, "retnet_test_set_hooks"):
        raise RuntimeError("retnet_test_set_hooks exists only in the debug build")
    _check("retnet_test_set_hooks",
           lib.retnet_test_set_hooks(int(wait_limit_ns), int(bool(skip_first_state_load))))


def _check(fn: str, status: int):
    if status != RETNET_OK:
        raise RetnetError(fn, status, retnet_status_string(status))


def retnet_status_string(status: int) -> str:
    return load_library().retnet_status_string(int(status)).decode()


def retnet_kernel_launch_count() -> int:
    return int(load_library().retnet_kernel_launch_count())


def retnet_set_launch_overlap(enable: bool) -> None:
    """Programmatic launch overlap of the hot kernels (on by default)."""
    _check("retnet_set_launch_overlap", load_library().retnet_set_launch_overlap(int(bool(enable))))


def retnet_set_output_pairing(mode) -> None:
    """How the tensor-core output pass runs: 1 (or True) CTA pairs folding q
    themselves (default), 2 CTA pairs with q folded by the prep pass, 0 (or
    False) single CTAs."""
    _check("retnet_set_output_pairing", load_library().retnet_set_output_pairing(int(mode)))


def retnet_default_gammas(heads: int) -> list:
    buf = (ctypes.c_float * max(int(heads), 1))()
    _check("retnet_default_gammas", load_library().retnet_default_gammas(int(heads), buf))
    return [float(x) for x in buf[:heads]]


# ------------------------------------------------------------------ helpers
def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}: use torch.bfloat16 or torch.float32")


def _dev(t: Optional[torch.Tensor], name: str, dtype=None, shape=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _gammas(gammas: Sequence[float], heads: int):
    g = [float(x) for x in gammas]
    if len(g) != heads:
        raise ValueError(f"need {heads} gammas, got {len(g)}")
    return (ctypes.c_float * heads)(*g)


# ------------------------------------------------------------------ entry points
def retnet_xpos_rotate(x: torch.Tensor, pos0: int = 0, out: Optional[torch.Tensor] = None):
    """Rotation prologue on x [batch, seqlen, heads, d]; returns out (may be x)."""
    _dev(x, "x")
    if x.dim() != 4:
        raise ValueError("x must be [batch, seqlen, heads, d]")
    out = torch.empty_like(x) if out is None else _dev(out, "out", x.dtype, x.shape)
    B, n, H, d = x.shape
    with torch.cuda.device(x.device):
        st = load_library().retnet_xpos_rotate(_ptr(x), _ptr(out), B, n, H, d, _dtype_code(x),
                                               int(pos0), _stream(x))
    _check("retnet_xpos_rotate", st)
    return out


WORKSPACE_ALIGN = 1024


def retnet_workspace(nbytes: int, device) -> torch.Tensor:
    """A uint8 device buffer of at least `nbytes` whose first byte is
    1024-byte aligned, as the tensor-core path requires.  The caching
    allocator only guarantees 512-byte alignment for sub-allocations, so
    this over-allocates by one alignment unit and returns an aligned view."""
    buf = torch.empty(max(int(nbytes), 1) + WORKSPACE_ALIGN, dtype=torch.uint8, device=device)
    off = (-buf.data_ptr()) % WORKSPACE_ALIGN
    return buf[off:off + max(int(nbytes), 1)]


def retnet_chunkwise_workspace_size(batch: int, heads: int, seqlen: int, dk: int, dv: int,
                                    dtype: torch.dtype, chunk: int, algo="auto") -> int:
    shape = _Shape(batch, heads, seqlen, dk, dv, BF16 if dtype == torch.bfloat16 else F32)
    n = ctypes.c_size_t(0)
    _check("retnet_chunkwise_workspace_size",
           load_library().retnet_chunkwise_workspace_size(ctypes.byref(shape), int(chunk),
                                                          _ALGOS[algo], ctypes.byref(n)))
    return int(n.value)


def retnet_retention_chunkwise(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                               gammas: Sequence[float], chunk: int, *, pos0: int = 0,
                               rotate: bool = True, state_in: Optional[torch.Tensor] = None,
                               state_out: Optional[torch.Tensor] = None,
                               gate: Optional[torch.Tensor] = None,
                               weight: Optional[torch.Tensor] = None,
                               bias: Optional[torch.Tensor] = None, eps: float = 1e-5,
                               algo="auto", out: Optional[torch.Tensor] = None,
                               workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Chunkwise prefill.  Returns out: O, or swish(gate) * GroupNorm(O) if gate is given.

    state_out (float32 [batch, heads, dk, dv]) receives the state after the
    last token when given.  `workspace` (uint8 CUDA tensor) is allocated
    here when not supplied.
    """
    _dev(q, "q")
    if q.dim() != 4:
        raise ValueError("q must be [batch, seqlen, heads, dk]")
    B, n, H, dk = q.shape
    dv = v.shape[-1]
    _dev(k, "k", q.dtype, (B, n, H, dk))
    _dev(v, "v", q.dtype, (B, n, H, dv))
    sshape = (B, H, dk, dv)
    _dev(state_in, "state_in", torch.float32, sshape)
    _dev(state_out, "state_out", torch.float32, sshape)
    _dev(gate, "gate", q.dtype, (B, n, H, dv))
    _dev(weight, "weight", torch.float32, (H * dv,))
    _dev(bias, "bias", torch.float32, (H * dv,))
    out = torch.empty((B, n, H, dv), dtype=q.dtype, device=q.device) if out is None else \
        _dev(out, "out", q.dtype, (B, n, H, dv))
    a = _ALGOS[algo]
    need = retnet_chunkwise_workspace_size(B, H, n, dk, dv, q.dtype, chunk, a)
    if workspace is None:
        workspace = retnet_workspace(need, q.device)
    else:
        _dev(workspace, "workspace", torch.uint8)
    shape = _Shape(B, H, n, dk, dv, _dtype_code(q))
    g = None
    if gate is not None:
        g = _Gate(gate.data_ptr(), None if weight is None else weight.data_ptr(),
                  None if bias is None else bias.data_ptr(), float(eps))
    with torch.cuda.device(q.device):
        st = load_library().retnet_retention_chunkwise(
            _ptr(q), _ptr(k), _ptr(v), _gammas(gammas, H), int(chunk), _ptr(out),
            ctypes.byref(shape), int(pos0), int(bool(rotate)), _ptr(state_in), _ptr(state_out),
            None if g is None else ctypes.byref(g), a, _ptr(workspace),
            workspace.numel(), _stream(q))
    _check("retnet_retention_chunkwise", st)
    return out


def retnet_parallel_workspace_size(batch: int, heads: int, seqlen: int, dk: int, dv: int,
                                   dtype: torch.dtype) -> int:
    shape = _Shape(batch, heads, seqlen, dk, dv, BF16 if dtype == torch.bfloat16 else F32)
    n = ctypes.c_size_t(0)
    _check("retnet_parallel_workspace_size",
           load_library().retnet_parallel_workspace_size(ctypes.byref(shape), ctypes.byref(n)))
    return int(n.value)


def retnet_retention_parallel(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                              gammas: Sequence[float], *, pos0: int = 0, rotate: bool = True,
                              gate: Optional[torch.Tensor] = None,
                              weight: Optional[torch.Tensor] = None,
                              bias: Optional[torch.Tensor] = None, eps: float = 1e-5,
                              out: Optional[torch.Tensor] = None,
                              workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Parallel form over the whole sequence (zero initial state).  Returns
    out: O, or swish(gate) * GroupNorm(O) if gate is given."""
    _dev(q, "q")
    if q.dim() != 4:
        raise ValueError("q must be [batch, seqlen, heads, dk]")
    B, n, H, dk = q.shape
    dv = v.shape[-1]
    _dev(k, "k", q.dtype, (B, n, H, dk))
    _dev(v, "v", q.dtype, (B, n, H, dv))
    _dev(gate, "gate", q.dtype, (B, n, H, dv))
    _dev(weight, "weight", torch.float32, (H * dv,))
    _dev(bias, "bias", torch.float32, (H * dv,))
    out = torch.empty((B, n, H, dv), dtype=q.dtype, device=q.device) if out is None else \
        _dev(out, "out", q.dtype, (B, n, H, dv))
    need = retnet_parallel_workspace_size(B, H, n, dk, dv, q.dtype)
    if workspace is None:
        workspace = retnet_workspace(need, q.device)
    else:
        _dev(workspace, "workspace", torch.uint8)
    shape = _Shape(B, H, n, dk, dv, _dtype_code(q))
    g = None
    if gate is not None:
        g = _Gate(gate.data_ptr(), None if weight is None else weight.data_ptr(),
                  None if bias is None else bias.data_ptr(), float(eps))
    with torch.cuda.device(q.device):
        st = load_library().retnet_retention_parallel(
            _ptr(q), _ptr(k), _ptr(v), _gammas(gammas, H), _ptr(out), ctypes.byref(shape),
            int(pos0), int(bool(rotate)), None if g is None else ctypes.byref(g), _ptr(workspace),
            workspace.numel(), _stream(q))
    _check("retnet_retention_parallel", st)
    return out


def retnet_retention_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                          gammas: Sequence[float], state: torch.Tensor, pos: int, *,
                          rotate: bool = True, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One decode step: state <- gamma state + k^T v (in place); returns o = q state."""
    _dev(q, "q")
    if q.dim() != 3:
        raise ValueError("q must be [batch, heads, dk]")
    B, H, dk = q.shape
    dv = v.shape[-1]
    _dev(k, "k", q.dtype, (B, H, dk))
    _dev(v, "v", q.dtype, (B, H, dv))
    _dev(state, "state", torch.float32, (B, H, dk, dv))
    out = torch.empty((B, H, dv), dtype=q.dtype, device=q.device) if out is None else \
        _dev(out, "out", q.dtype, (B, H, dv))
    with torch.cuda.device(q.device):
        st = load_library().retnet_retention_step(
            _ptr(q), _ptr(k), _ptr(v), _gammas(gammas, H), _ptr(state), _ptr(out), B, H, dk, dv,
            _dtype_code(q), int(pos), int(bool(rotate)), _stream(q))
    _check("retnet_retention_step", st)
    return out


def retnet_retention_recurrent(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                               gammas: Sequence[float], state: torch.Tensor, pos0: int, *,
                               rotate: bool = True,
                               out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Recurrent form over a run of tokens, q, k, v [batch, seqlen, heads, d]:
    for each token, state <- gamma state + k^T v, o = q state (state updated
    in place).  Returns out [batch, seqlen, heads, dv]."""
    _dev(q, "q")
    if q.dim() != 4:
        raise ValueError("q must be [batch, seqlen, heads, dk]")
    B, n, H, dk = q.shape
    dv = v.shape[-1]
    _dev(k, "k", q.dtype, (B, n, H, dk))
    _dev(v, "v", q.dtype, (B, n, H, dv))
    _dev(state, "state", torch.float32, (B, H, dk, dv))
    out = torch.empty((B, n, H, dv), dtype=q.dtype, device=q.device) if out is None else \
        _dev(out, "out", q.dtype, (B, n, H, dv))
    shape = _Shape(B, H, n, dk, dv, _dtype_code(q))
    with torch.cuda.device(q.device):
        st = load_library().retnet_retention_recurrent(
            _ptr(q), _ptr(k), _ptr(v), _gammas(gammas, H), _ptr(state), _ptr(out),
            ctypes.byref(shape), int(pos0), int(bool(rotate)), _stream(q))
    _check("retnet_retention_recurrent", st)
    return out


def retnet_backward_workspace_size(batch: int, heads: int, seqlen: int, dk: int, dv: int,
                                   dtype: torch.dtype, chunk: int, algo="auto") -> int:
    shape = _Shape(batch, heads, seqlen, dk, dv, BF16 if dtype == torch.bfloat16 else F32)
    n = ctypes.c_size_t(0)
    _check("retnet_backward_workspace_size",
           load_library().retnet_backward_workspace_size(ctypes.byref(shape), int(chunk),
                                                         _ALGOS[algo], ctypes.byref(n)))
    return int(n.value)


def retnet_retention_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                              d_out: torch.Tensor, gammas: Sequence[float], chunk: int, *,
                              pos0: int = 0, rotate: bool = True, algo="auto",
                              dq: Optional[torch.Tensor] = None,
                              dk: Optional[torch.Tensor] = None,
                              dv: Optional[torch.Tensor] = None,
                              workspace: Optional[torch.Tensor] = None):
    """Gradients (dq, dk, dv) of O = retention(R q, R k, v) (no epilogue, zero
    initial state) given d_out = dL/dO; shapes as for the forward call."""
    _dev(q, "q")
    if q.dim() != 4:
        raise ValueError("q must be [batch, seqlen, heads, dk]")
    B, n, H, Dk = q.shape
    Dv = v.shape[-1]
    _dev(k, "k", q.dtype, (B, n, H, Dk))
    _dev(v, "v", q.dtype, (B, n, H, Dv))
    _dev(d_out, "d_out", q.dtype, (B, n, H, Dv))
    dq = torch.empty_like(q) if dq is None else _dev(dq, "dq", q.dtype, (B, n, H, Dk))
    dk = torch.empty_like(k) if dk is None else _dev(dk, "dk", q.dtype, (B, n, H, Dk))
    dv = torch.empty_like(v) if dv is None else _dev(dv, "dv", q.dtype, (B, n, H, Dv))
    need = retnet_backward_workspace_size(B, H, n, Dk, Dv, q.dtype, chunk, algo)
    if workspace is None:
        workspace = retnet_workspace(need, q.device)
    else:
        _dev(workspace, "workspace", torch.uint8)
    shape = _Shape(B, H, n, Dk, Dv, _dtype_code(q))
    with torch.cuda.device(q.device):
        st = load_library().retnet_retention_backward(
            _ptr(q), _ptr(k), _ptr(v), _ptr(d_out), _gammas(gammas, H), int(chunk), _ptr(dq),
            _ptr(dk), _ptr(dv), ctypes.byref(shape), int(pos0), int(bool(rotate)), _ALGOS[algo],
            _ptr(workspace), workspace.numel(), _stream(q))
    _check("retnet_retention_backward", st)
    return dq, dk, dv


def retnet_groupnorm_swish(o: torch.Tensor, g: torch.Tensor, weight: Optional[torch.Tensor] = None,
                           bias: Optional[torch.Tensor] = None, eps: float = 1e-5,
                           out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y = swish(g) * GroupNorm(o) for o, g [..., heads, dv]; returns Y (may be o)."""
    _dev(o, "o")
    if o.dim() < 2:
        raise ValueError("o must be [..., heads, dv]")
    H, dv = o.shape[-2], o.shape[-1]
    rows = o.numel() // (H * dv) if o.numel() else 0
    _dev(g, "g", o.dtype, o.shape)
    _dev(weight, "weight", torch.float32, (H * dv,))
    _dev(bias, "bias", torch.float32, (H * dv,))
    out = torch.empty_like(o) if out is None else _dev(out, "out", o.dtype, o.shape)
    with torch.cuda.device(o.device):
        st = load_library().retnet_groupnorm_swish(
            _ptr(o), _ptr(g), _ptr(weight), _ptr(bias), float(eps), rows, H, dv, _dtype_code(o),
            _ptr(out), _stream(o))
    _check("retnet_groupnorm_swish", st)
    return out


def retnet_linear(x: torch.Tensor, w: torch.Tensor,
                  out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y = x W^T on the tensor cores: x [..., in] bf16, w [out, in] bf16."""
    _dev(x, "x", torch.bfloat16)
    _dev(w, "w", torch.bfloat16)
    if w.dim() != 2 or x.shape[-1] != w.shape[1]:
        raise ValueError("need x [..., in] and w [out, in]")
    rows = x.numel() // x.shape[-1] if x.numel() else 0
    oshape = (*x.shape[:-1], w.shape[0])
    out = torch.empty(oshape, dtype=torch.bfloat16, device=x.device) if out is None else \
        _dev(out, "out", torch.bfloat16, oshape)
    with torch.cuda.device(x.device):
        st = load_library().retnet_linear(_ptr(x), _ptr(w), _ptr(out), rows, x.shape[-1],
                                          w.shape[0], _stream(x))
    _check("retnet_linear", st)
    return out


def retnet_msr_workspace_size(batch: int, heads: int, seqlen: int, d: int, hidden: int,
                              chunk: int) -> int:
    shape = _Shape(batch, heads, seqlen, d, d, BF16)
    n = ctypes.c_size_t(0)
    _check("retnet_msr_workspace_size",
           load_library().retnet_msr_workspace_size(ctypes.byref(shape), int(hidden), int(chunk),
                                                    ctypes.byref(n)))
    return int(n.value)


def retnet_msr_layer(x: torch.Tensor, w_qkvg: torch.Tensor, w_o: torch.Tensor,
                     gammas: Sequence[float], chunk: int, *, pos0: int = 0,
                     weight: Optional[torch.Tensor] = None, bias: Optional[torch.Tensor] = None,
                     eps: float = 1e-5, state_in: Optional[torch.Tensor] = None,
                     state_out: Optional[torch.Tensor] = None,
                     out: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The multi-scale retention layer on x [batch, seqlen, hidden] (bf16):
    projections by w_qkvg [4 H d, hidden] (rows of W_Q, W_K, W_V, W_G), the
    gated chunkwise retention, and the output projection w_o [hidden, H d].
    H = len(gammas).  Returns out [batch, seqlen, hidden]."""
    _dev(x, "x", torch.bfloat16)
    if x.dim() != 3:
        raise ValueError("x must be [batch, seqlen, hidden]")
    B, n, hidden = x.shape
    H = len(gammas)
    if w_qkvg.dim() != 2 or w_qkvg.shape[0] % (4 * H) or w_qkvg.shape[1] != hidden:
        raise ValueError("w_qkvg must be [4 * heads * d, hidden]")
    d = w_qkvg.shape[0] // (4 * H)
    _dev(w_qkvg, "w_qkvg", torch.bfloat16)
    _dev(w_o, "w_o", torch.bfloat16, (hidden, H * d))
    _dev(weight, "weight", torch.float32, (H * d,))
    _dev(bias, "bias", torch.float32, (H * d,))
    _dev(state_in, "state_in", torch.float32, (B, H, d, d))
    _dev(state_out, "state_out", torch.float32, (B, H, d, d))
    out = torch.empty_like(x) if out is None else _dev(out, "out", torch.bfloat16, x.shape)
    need = retnet_msr_workspace_size(B, H, n, d, hidden, chunk)
    if workspace is None:
        workspace = retnet_workspace(need, x.device)
    else:
        _dev(workspace, "workspace", torch.uint8)
    shape = _Shape(B, H, n, d, d, BF16)
    with torch.cuda.device(x.device):
        st = load_library().retnet_msr_layer(
            _ptr(x), _ptr(w_qkvg), _ptr(w_o), _gammas(gammas, H), int(chunk), _ptr(out),
            ctypes.byref(shape), int(hidden), int(pos0), _ptr(weight), _ptr(bias), float(eps),
            _ptr(state_in), _ptr(state_out), _ptr(workspace), workspace.numel(), _stream(x))
    _check("retnet_msr_layer", st)
    return out


def retnet_check_device_errors(device=None) -> None:
    """Synchronises the current stream and raises if a kernel reported an error."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    with torch.cuda.device(dev):
        s = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
        _check("retnet_check_device_errors", load_library().retnet_check_device_errors(s))


def retnet_profiler_enable(on: bool = True) -> None:
    """Start/stop bracketing every library kernel launch with CUDA events."""
    _check("retnet_profiler_enable", load_library().retnet_profiler_enable(int(bool(on))))


def retnet_profiler_select(name: Optional[str] = None) -> None:
    """Times only the kernel `name` (None: every kernel)."""
    _check("retnet_profiler_select",
           load_library().retnet_profiler_select(None if name is None else name.encode()))


def retnet_profiler_reset() -> None:
    _check("retnet_profiler_reset", load_library().retnet_profiler_reset())


def retnet_profiler_read() -> dict:
    """{kernel name: (total device ms, launches)} accumulated since the last reset."""
    lib = load_library()
    out = {}
    i = 0
    buf = ctypes.create_string_buffer(128)
    while True:
        ms = ctypes.c_double(0.0)
        n = ctypes.c_ulonglong(0)
        st = lib.retnet_profiler_read(i, buf, 128, ctypes.byref(ms), ctypes.byref(n))
        if st == 1:          # past the last kernel name
            break
        _check("retnet_profiler_read", st)
        out[buf.value.decode()] = (float(ms.value), int(n.value))
        i += 1
    return out
